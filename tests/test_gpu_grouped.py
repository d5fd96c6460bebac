"""Grouped weight scales ([MO] "int4 양자화 (Quantization)의 품질 비용": one
scale per row and group of codes along K) on the GPU against the oracle: the
fused single-launch path and the general path (routing bit-exact, outputs
within the parity bar; the general path equal to the oracle bit for bit), and
batches that would take the tensor cores report the general path.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import oracle as O
from quantized_mixture_experts_sigmoid_b200 import moe
from synth.device import bits, device_layer, to_dev_bf16
from tests.helpers import layer_inputs, oracle_experts, rel_err_rows

pytestmark = pytest.mark.gpu
TOL = 2e-3

SHAPES = {
    "fused_g32": (synth.LayerShape("fused_g32", T=3, H=544, I=288, E=64, n_group=2, topk_group=1, top_k=5,
                                   group_size=32), moe.PATH_FUSED),
    "fused_int8_g32": (synth.LayerShape("fused_int8_g32", T=4, H=544, I=288, E=96, n_group=3, topk_group=2,
                                        top_k=5, qtype=8, group_size=32), moe.PATH_FUSED),
    "decode_g128": (synth.CONFIGS["decode"].with_(name="decode_g128", group_size=128), moe.PATH_FUSED),
    "general_g64": (synth.LayerShape("general_g64", T=37, H=512, I=256, E=48, n_group=6, topk_group=3, top_k=5,
                                     group_size=64), moe.PATH_GENERAL),
    "general_int2_g32": (synth.LayerShape("general_int2_g32", T=20, H=256, I=128, E=16, n_group=4, topk_group=2,
                                          top_k=4, qtype=2, group_size=32), moe.PATH_GENERAL),
    "tc_shape_g128": (synth.LayerShape("tc_shape_g128", T=40, H=256, I=128, E=16, n_group=4, topk_group=2,
                                       top_k=4, group_size=128), moe.PATH_GENERAL),
}


@pytest.mark.parametrize("name", list(SHAPES))
def test_layer_grouped_scales(name):
    sh, want_path = SHAPES[name]
    dev = device_layer(sh)
    assert moe.moe_layer_path(sh.T, dev["cfg"], dev["routed"], dev["shared"]) == want_path
    x, W, b = layer_inputs(sh)
    ws = moe.workspace(moe.moe_layer_workspace_bytes(sh.T, dev["cfg"], dev["routed"], dev["shared"]))
    of = torch.empty(sh.T, sh.H, dtype=torch.float32, device="cuda")
    ob = torch.empty(sh.T, sh.H, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(sh.T, sh.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(sh.T, sh.top_k, dtype=torch.float32, device="cuda")
    xd = to_dev_bf16(x)
    moe.moe_layer_forward(xd, dev["W"], dev["bias"], dev["cfg"], dev["routed"], dev["shared"], of, ws, idx, w)
    moe.moe_layer_forward(xd, dev["W"], dev["bias"], dev["cfg"], dev["routed"], dev["shared"], ob, ws)
    assert moe.moe_workspace_status(ws) == 0
    idx_o, w_o, _, _ = O.route(x, W, b, sh.n_group, sh.topk_group, sh.top_k, sh.rsf)
    assert np.array_equal(idx.cpu().numpy(), idx_o)
    assert np.array_equal(w.cpu().numpy().view(np.uint32), w_o.view(np.uint32))
    routed = oracle_experts(sh, np.unique(idx_o))
    shared = oracle_experts(sh, [0], shared=True)
    of_o, _, _, _ = O.layer_forward(x, W, b, sh.n_group, sh.topk_group, sh.top_k, sh.rsf, routed, shared)
    of_g = of.cpu().numpy()
    assert rel_err_rows(of_g, of_o) <= TOL
    assert np.array_equal(bits(ob), synth.bf16_bits(of_g))
    if want_path == moe.PATH_GENERAL:  # lane-per-row folds in the definition's order
        assert np.array_equal(of_g.view(np.uint32), of_o.view(np.uint32))


def test_grouped_scales_change_the_result():
    # the same codes with per-row scales give a different layer: the grouped scales are used
    sh, _ = SHAPES["general_g64"]
    flat = sh.with_(group_size=0)
    x, W, b = layer_inputs(sh)
    outs = []
    for s in (sh, flat):
        dev = device_layer(s)
        ws = moe.workspace(moe.moe_layer_workspace_bytes(s.T, dev["cfg"], dev["routed"], dev["shared"]))
        o = torch.empty(s.T, s.H, dtype=torch.float32, device="cuda")
        moe.moe_layer_forward(to_dev_bf16(x), dev["W"], dev["bias"], dev["cfg"], dev["routed"], dev["shared"], o, ws)
        outs.append(o.cpu().numpy())
    assert rel_err_rows(outs[0], outs[1]) > 0.05
