"""moe_route_noalloc: the router entry point that allocates nothing.

It exists for callers that cannot allocate device memory when they route (work
captured into a CUDA graph, engine plugins that must not allocate at enqueue
time, latency-critical loops that cannot pay for cudaMalloc's device
synchronisation); its logits live in a fixed array inside the library.  This
file is collected last on purpose: it must pass alone in a fresh process and
after every other test, when earlier calls have left their data in the array.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from quantized_mixture_experts_sigmoid_b200 import moe
from synth.device import to_dev_bf16


def _route_both(sh, tokens):
    x = to_dev_bf16(synth.hidden_states(sh, tokens=tokens))
    W = torch.from_numpy(synth.router_weight(sh)).cuda()
    b = torch.from_numpy(synth.router_bias(sh)).cuda()
    cfg = moe.RouterCfg(sh.E, sh.n_group, sh.topk_group, sh.top_k, sh.rsf)
    T = len(tokens)
    idx_ws = torch.empty(T, sh.top_k, dtype=torch.int32, device="cuda")
    w_ws = torch.empty(T, sh.top_k, dtype=torch.float32, device="cuda")
    ws = moe.workspace(moe.moe_route_workspace_bytes(T, cfg))
    moe.moe_route(x, W, b, cfg, idx_ws, w_ws, ws)
    idx_na = torch.full((T, sh.top_k), -1, dtype=torch.int32, device="cuda")
    w_na = torch.full((T, sh.top_k), -1.0, dtype=torch.float32, device="cuda")
    moe.moe_route_noalloc(x, W, b, cfg, idx_na, w_na)
    torch.cuda.synchronize()
    return idx_ws.cpu().numpy(), w_ws.cpu().numpy(), idx_na.cpu().numpy(), w_na.cpu().numpy()


@pytest.mark.gpu
def test_noalloc_route_matches_workspace_route_twice():
    sh = synth.CONFIGS["decode"]
    # two calls in a row with different batches: the second reuses the array
    # the first one filled (and whatever earlier tests left in it)
    for tokens in (list(range(64, 320)), [7, 3, 11]):
        idx_ws, w_ws, idx_na, w_na = _route_both(sh, tokens)
        assert np.array_equal(idx_na, idx_ws)  # indices: bit-exact, as every routing test
        assert np.array_equal(w_na.view(np.uint32), w_ws.view(np.uint32))


@pytest.mark.gpu
def test_noalloc_route_rejects_batches_over_capacity():
    sh = synth.CONFIGS["decode"]
    cfg = moe.RouterCfg(sh.E, sh.n_group, sh.topk_group, sh.top_k, sh.rsf)
    T = moe.MOE_ROUTE_NOALLOC_MAX_LOGITS // sh.E + 1
    x = torch.zeros(T, sh.H, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(sh.E, sh.H, dtype=torch.float32, device="cuda")
    b = torch.zeros(sh.E, dtype=torch.float32, device="cuda")
    idx = torch.empty(T, sh.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, sh.top_k, dtype=torch.float32, device="cuda")
    rc = moe.lib().moe_route_noalloc(x.data_ptr(), T, sh.H, W.data_ptr(), b.data_ptr(), ctypes.byref(cfg),
                                     idx.data_ptr(), w.data_ptr(), None)
    assert rc == moe.MOE_ETOO_LARGE
