"""Adaptive expert top-p on the GPU against the oracle ([HN] options list,
"--topp 0.7"): routing bit-exact through moe_route and moe_route_noalloc,
empty slots in the union, and the whole layer on the fused, tensor-core and
general paths (indices and weights bit-exact, outputs within the parity bar).
"""
import numpy as np
import pytest
import torch

import synth
from oracle import oracle as O
from quantized_mixture_experts_sigmoid_b200 import moe
from synth.device import bits, to_dev_bf16
from tests.helpers import layer_inputs, oracle_experts, rel_err_rows
from tests.test_gpu_parity import TOL, gpu_union, layer

pytestmark = pytest.mark.gpu


def cfg_p(c, p):
    return moe.RouterCfg(c.n_expert, c.n_group, c.topk_group, c.top_k, c.routed_scaling_factor, p)


def _inputs(sh, name):
    # decode and verify get more tokens than their T: routing is per token
    if name in ("decode", "verify"):
        return (synth.hidden_states(sh, tokens=range(64)), synth.router_weight(sh), synth.router_bias(sh))
    return layer_inputs(sh)


@pytest.mark.parametrize("p", [0.5, 0.7, 0.9])
@pytest.mark.parametrize("name", ["tiny", "ragged", "decode", "verify", "crowded"])
def test_route_topp_bit_exact(name, p):
    sh, dev = layer(name)
    x, W, b = _inputs(sh, name)
    cfg = cfg_p(dev["cfg"], p)
    T, K = x.shape[0], sh.top_k
    xd = to_dev_bf16(x)
    idx_o, w_o, _, _ = O.route(x, W, b, sh.n_group, sh.topk_group, K, sh.rsf, top_p=p)
    for noalloc in (False, True):
        idx = torch.empty(T, K, dtype=torch.int32, device="cuda")
        w = torch.empty(T, K, dtype=torch.float32, device="cuda")
        if noalloc:
            moe.moe_route_noalloc(xd, dev["W"], dev["bias"], cfg, idx, w)
        else:
            ws = moe.workspace(moe.moe_route_workspace_bytes(T, cfg))
            moe.moe_route(xd, dev["W"], dev["bias"], cfg, idx, w, ws)
            assert moe.moe_workspace_status(ws) == 0
        assert np.array_equal(idx.cpu().numpy(), idx_o)
        assert np.array_equal(w.cpu().numpy().view(np.uint32), w_o.view(np.uint32))
    if p == 0.5:
        assert (idx_o < 0).any()  # the shape really drops some slots


def test_union_leaves_out_empty_slots_on_gpu():
    rng = np.random.default_rng(21)
    for T, E, K in [(1, 256, 8), (4, 256, 8), (37, 48, 5), (300, 64, 6)]:
        idx = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
        idx[rng.random((T, K)) < 0.35] = -1
        g = gpu_union(idx, E)
        o = O.union(idx, E)
        n = int(o["offsets"][o["n_unique"]])
        assert g["status"] == 0
        assert g["n_unique"] == o["n_unique"]
        assert np.array_equal(g["uniq"], o["uniq"][:o["n_unique"]])
        assert np.array_equal(g["offsets"], o["offsets"][:o["n_unique"] + 1])
        assert np.array_equal(g["counts"], o["counts"])
        assert np.array_equal(g["pair_tok"][:n], o["pair_tok"][:n])
        assert np.array_equal(g["pair_slot"][:n], o["pair_slot"][:n])
        assert np.all(g["pair_tok"][n:] == 0) and np.all(g["pair_slot"][n:] == -1)


LAYERS = {"tiny": moe.PATH_GENERAL, "crowded_int8": moe.PATH_GENERAL, "fused_ragged": moe.PATH_FUSED,
          "fused_ragged_int8": moe.PATH_FUSED, "decode": moe.PATH_FUSED, "verify": moe.PATH_FUSED,
          "tc_small": moe.PATH_TENSOR_CORE, "tc_ragged": moe.PATH_TENSOR_CORE}


@pytest.mark.parametrize("name", list(LAYERS))
def test_layer_topp_within_tolerance(name):
    p = 0.7
    sh, dev = layer(name)
    x, W, b = layer_inputs(sh)
    cfg = cfg_p(dev["cfg"], p)
    T, K = sh.T, sh.top_k
    assert moe.moe_layer_path(T, cfg, dev["routed"], dev["shared"]) == LAYERS[name]
    xd = to_dev_bf16(x)
    ws = moe.workspace(moe.moe_layer_workspace_bytes(T, cfg, dev["routed"], dev["shared"]))
    of = torch.empty(T, sh.H, dtype=torch.float32, device="cuda")
    ob = torch.empty(T, sh.H, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(T, K, dtype=torch.int32, device="cuda")
    w = torch.empty(T, K, dtype=torch.float32, device="cuda")
    moe.moe_layer_forward(xd, dev["W"], dev["bias"], cfg, dev["routed"], dev["shared"], of, ws, idx, w)
    moe.moe_layer_forward(xd, dev["W"], dev["bias"], cfg, dev["routed"], dev["shared"], ob, ws)
    assert moe.moe_workspace_status(ws) == 0
    idx_o, w_o, _, _ = O.route(x, W, b, sh.n_group, sh.topk_group, K, sh.rsf, top_p=p)
    assert np.array_equal(idx.cpu().numpy(), idx_o)
    assert np.array_equal(w.cpu().numpy().view(np.uint32), w_o.view(np.uint32))
    routed = oracle_experts(sh, np.unique(idx_o[idx_o >= 0]))
    shared_ex = oracle_experts(sh, [0], shared=True)
    of_o, _, _, _ = O.layer_forward(x, W, b, sh.n_group, sh.topk_group, K, sh.rsf, routed, shared_ex, top_p=p)
    of_g = of.cpu().numpy()
    assert rel_err_rows(of_g, of_o) <= TOL
    assert np.array_equal(bits(ob), synth.bf16_bits(of_g))
    # the same call without top-p reads at least as many distinct experts
    idx_full, _, _, _ = O.route(x, W, b, sh.n_group, sh.topk_group, K, sh.rsf)
    assert len(np.unique(idx_o[idx_o >= 0])) <= len(np.unique(idx_full))
