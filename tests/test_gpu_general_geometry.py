"""The general path's two CTA geometries on the GPU against the oracle, bit for bit.

The integer-dot expert kernels stage weight rows in shared memory and fold
each row's blocks in ascending order ([HN] "Show HN: 느린 컴퓨터에서 GLM 5.2
실행하기", "구현된 주요 기능": the integer dot against Q8_0 activations), so
their outputs equal the oracle's exactly whichever geometry runs.  A batch
whose experts see at most two tokens on average (T K <= 2 min(E, T K)) takes
the wide geometry when H is a multiple of 256 and I of 128; the narrow one
otherwise.  Shapes below reach each geometry for every weight width, with
per-row and grouped scales, experts seeing more tokens than one pass holds
(two a pass wide, eight or sixteen narrow), and partial last chunks.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import oracle as O
from quantized_mixture_experts_sigmoid_b200 import moe
from synth.device import device_layer, to_dev_bf16
from tests.helpers import layer_inputs, oracle_experts

pytestmark = pytest.mark.gpu

SHAPES = {
    # wide: T K <= 2 min(E, T K), H % 256 == 0, I % 128 == 0
    "wide_int4": synth.LayerShape("wide_int4", T=6, H=512, I=256, E=64, n_group=4, topk_group=2, top_k=4),
    "wide_int8": synth.LayerShape("wide_int8", T=6, H=512, I=256, E=64, n_group=4, topk_group=2, top_k=4, qtype=8),
    "wide_int2": synth.LayerShape("wide_int2", T=6, H=512, I=256, E=64, n_group=4, topk_group=2, top_k=4, qtype=2),
    "wide_int4_g64": synth.LayerShape("wide_int4_g64", T=6, H=512, I=256, E=64, n_group=4, topk_group=2,
                                      top_k=4, group_size=64),
    # wide, with experts that see more than two tokens (several passes)
    "wide_int4_passes": synth.LayerShape("wide_int4_passes", T=20, H=768, I=384, E=48, n_group=4, topk_group=2,
                                         top_k=4),
    "wide_int2_passes": synth.LayerShape("wide_int2_passes", T=20, H=768, I=384, E=48, n_group=4, topk_group=2,
                                         top_k=4, qtype=2),
    # narrow: many tokens per expert, or H / I off the wide multiples (partial last chunks)
    "narrow_int4": synth.LayerShape("narrow_int4", T=24, H=512, I=256, E=16, n_group=4, topk_group=2, top_k=4),
    "narrow_int8_ragged": synth.LayerShape("narrow_int8_ragged", T=6, H=544, I=288, E=64, n_group=4,
                                           topk_group=2, top_k=4, qtype=8),
    "narrow_int2_ragged": synth.LayerShape("narrow_int2_ragged", T=6, H=544, I=288, E=64, n_group=4,
                                           topk_group=2, top_k=4, qtype=2),
}


def _wide(sh):
    pairs = sh.T * sh.top_k
    tpe = -(-pairs // min(sh.E, pairs))
    return tpe <= 2 and sh.H % 256 == 0 and sh.I % 128 == 0


def test_shapes_cover_both_geometries():
    assert {n for n, sh in SHAPES.items() if _wide(sh)} == {n for n in SHAPES if n.startswith("wide")}


@pytest.mark.parametrize("name", list(SHAPES))
def test_general_path_bit_exact(name):
    sh = SHAPES[name]
    dev = device_layer(sh)
    assert moe.moe_layer_path(sh.T, dev["cfg"], dev["routed"], dev["shared"]) == moe.PATH_GENERAL
    x, W, b = layer_inputs(sh)
    ws = moe.workspace(moe.moe_layer_workspace_bytes(sh.T, dev["cfg"], dev["routed"], dev["shared"]))
    of = torch.empty(sh.T, sh.H, dtype=torch.float32, device="cuda")
    idx = torch.empty(sh.T, sh.top_k, dtype=torch.int32, device="cuda")
    moe.moe_layer_forward(to_dev_bf16(x), dev["W"], dev["bias"], dev["cfg"], dev["routed"], dev["shared"], of, ws,
                          idx)
    assert moe.moe_workspace_status(ws) == 0
    idx_o, _, _, _ = O.route(x, W, b, sh.n_group, sh.topk_group, sh.top_k, sh.rsf)
    assert np.array_equal(idx.cpu().numpy(), idx_o)
    counts = np.bincount(idx_o.ravel(), minlength=sh.E)
    if name.endswith("_passes"):
        assert counts.max() > 2  # some expert needs more than one wide pass
    routed = oracle_experts(sh, np.unique(idx_o))
    shared = oracle_experts(sh, [0], shared=True)
    of_o, _, _, _ = O.layer_forward(x, W, b, sh.n_group, sh.topk_group, sh.top_k, sh.rsf, routed, shared)
    assert np.array_equal(of.cpu().numpy().view(np.uint32), of_o.view(np.uint32))
