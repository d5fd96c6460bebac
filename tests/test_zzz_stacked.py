"""Stacked decode on the GPU against the oracle: 16 consecutive layers of the
GLM-5.2 shape with all 4096 routed experts resident (about 78 GB int4), run as
one sequence of 16 layer calls with fresh seeded hidden states per layer, at
T = 1 and T = 8, then the int2 variant of the stack at T = 1.

Routing of every layer and token is checked bit-exactly; the outputs of three
sampled layers (first, middle, last) for up to two tokens each are checked
within the parity bar.  The oracle regenerates only the experts those tokens
touch.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import oracle as O
from quantized_mixture_experts_sigmoid_b200 import moe
from synth.device import device_layer, to_dev_bf16
from tests.helpers import layer_inputs, oracle_experts, rel_err_rows

pytestmark = pytest.mark.gpu

TOL = 2e-3
SAMPLE_LAYERS = (0, 7, 15)


def _run_sequence(sh, layers, T):
    """16 layer calls on one stream, one workspace; returns per-layer (x, out fp32, idx, w)."""
    shT = sh.with_(T=T)
    xs = [synth.hidden_states(shT, layer=l) for l in range(sh.n_layers)]
    d0 = layers[0]
    ws = moe.workspace(moe.moe_layer_workspace_bytes(T, d0["cfg"], d0["routed"], d0["shared"]))
    outs, idxs, ws_ = [], [], []
    xd = [to_dev_bf16(x) for x in xs]
    for l in range(sh.n_layers):
        d = layers[l]
        out = torch.empty(T, sh.H, dtype=torch.float32, device="cuda")
        idx = torch.empty(T, sh.top_k, dtype=torch.int32, device="cuda")
        w = torch.empty(T, sh.top_k, dtype=torch.float32, device="cuda")
        moe.moe_layer_forward(xd[l], d["W"], d["bias"], d["cfg"], d["routed"], d["shared"], out, ws, idx, w)
        outs.append(out)
        idxs.append(idx)
        ws_.append(w)
    torch.cuda.synchronize()
    assert moe.moe_workspace_status(ws) == 0
    return [(xs[l], outs[l].cpu().numpy(), idxs[l].cpu().numpy(), ws_[l].cpu().numpy())
            for l in range(sh.n_layers)]


def _check(sh, results, T):
    for l, (x, out, idx, w) in enumerate(results):
        _, W, b = layer_inputs(sh, layer=l, tokens=range(T))
        idx_o, w_o, _, _ = O.route(x, W, b, sh.n_group, sh.topk_group, sh.top_k, sh.rsf)
        assert np.array_equal(idx, idx_o), l
        assert np.array_equal(w.view(np.uint32), w_o.view(np.uint32)), l
        if l not in SAMPLE_LAYERS:
            continue
        toks = sorted({0, T - 1})
        routed = oracle_experts(sh, np.unique(idx_o[toks]), layer=l)
        shared = oracle_experts(sh, [0], layer=l, shared=True)
        ref, _, _, _ = O.layer_forward(x[toks], W, b, sh.n_group, sh.topk_group, sh.top_k, sh.rsf, routed, shared)
        err = rel_err_rows(out[toks], ref)
        assert err <= TOL, (l, err)


def _stack(sh):
    return [device_layer(sh, layer=l) for l in range(sh.n_layers)]


def test_stacked_int4_t1_and_t8():
    sh = synth.CONFIGS["stacked"]
    layers = _stack(sh)
    res1 = _run_sequence(sh, layers, 1)
    res8 = _run_sequence(sh, layers, synth.CONFIGS["stacked_t8"].T)
    del layers
    torch.cuda.empty_cache()
    _check(sh, res1, 1)
    _check(sh, res8, synth.CONFIGS["stacked_t8"].T)


def test_stacked_int2_t1():
    sh = synth.CONFIGS["stacked_int2"]
    layers = _stack(sh)
    res = _run_sequence(sh, layers, 1)
    del layers
    torch.cuda.empty_cache()
    _check(sh, res, 1)
