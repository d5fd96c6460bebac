"""Expert parallelism on the GPU: the layer's CUDA compute steps under the
expert-parallel exchange (one rank: the all-to-alls are local copies), and a
rank's share of the experts (rank 1 of 2, a contiguous slice or dealt by
usage), against the oracle bit for bit (the integer-dot expert kernels fold
in the definition's order)."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import synth
from oracle import oracle as O
from quantized_mixture_experts_sigmoid_b200 import moe
from quantized_mixture_experts_sigmoid_b200.expert_parallel import ep_cuda_compute, ep_forward
from synth.device import device_layer, to_dev_bf16
from tests.helpers import layer_inputs, oracle_experts

pytestmark = pytest.mark.gpu

SHAPES = {
    "ep_decode": synth.LayerShape("ep_decode", T=6, H=512, I=256, E=64, n_group=4, topk_group=2, top_k=4),
    "ep_int8_topp": synth.LayerShape("ep_int8_topp", T=9, H=544, I=288, E=32, n_group=4, topk_group=2, top_k=5,
                                     qtype=8),
}


@pytest.fixture(scope="module")
def one_rank_group():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True, timeout=datetime.timedelta(seconds=30))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("name", list(SHAPES))
def test_ep_one_rank_equals_oracle(name, one_rank_group):
    sh = SHAPES[name]
    top_p = 0.7 if name.endswith("topp") else 0.0
    dev = device_layer(sh)
    cfg = dev["cfg"]
    cfg.top_p = top_p
    x, W, b = layer_inputs(sh)
    compute = ep_cuda_compute(dev["W"], dev["bias"], cfg, dev["routed"], dev["shared"], out_dtype=torch.float32)
    out = ep_forward(to_dev_bf16(x), sh.E, compute)
    assert compute.status() == moe.MOE_OK  # no device-side error recorded by the rank's steps
    routed = oracle_experts(sh, range(sh.E))
    shared = oracle_experts(sh, [0], shared=True)
    of, _, idx, _ = O.layer_forward(x, W, b, sh.n_group, sh.topk_group, sh.top_k, sh.rsf, routed, shared, top_p)
    if top_p:
        assert (idx < 0).any()
    assert np.array_equal(out.cpu().numpy().view(np.uint32), of.view(np.uint32))


def test_ep_rank_slice_experts():
    # rank 1 of 2 holds experts E/2 .. E-1 and computes them from local indices
    sh = SHAPES["ep_decode"]
    dev = device_layer(sh)
    compute = ep_cuda_compute(dev["W"], dev["bias"], dev["cfg"], dev["routed"], dev["shared"], rank=1, n_ranks=2)
    x, _, _ = layer_inputs(sh)
    per = sh.E // 2
    local = (np.arange(sh.T) * 7 % per).astype(np.int32)
    y = compute.experts(to_dev_bf16(x), torch.from_numpy(local).cuda()).cpu().numpy()
    routed = oracle_experts(sh, np.unique(local) + per)
    y_o = O.expert_ffn_per_token(routed, x, (local + per).reshape(-1, 1))[:, 0, :]
    assert np.array_equal(y.view(np.uint32), y_o.view(np.uint32))


def test_ep_rank_experts_under_usage_placement():
    # experts dealt to 2 ranks in a most-used-first order: rank 1 gathers its own stack
    from quantized_mixture_experts_sigmoid_b200.expert_parallel import experts_of_rank, placement_by_usage
    sh = SHAPES["ep_decode"]
    dev = device_layer(sh)
    x, W, b = layer_inputs(sh)
    idx, _, _, _ = O.route(x, W, b, sh.n_group, sh.topk_group, sh.top_k, sh.rsf)
    order = O.usage_rank(O.usage_accumulate(idx, sh.E))
    placement = placement_by_usage(torch.from_numpy(np.asarray(order)), 2)
    compute = ep_cuda_compute(dev["W"], dev["bias"], dev["cfg"], dev["routed"], dev["shared"], rank=1, n_ranks=2,
                              placement=placement)
    mine = experts_of_rank(*placement, 1).numpy()
    local = (np.arange(sh.T) * 5 % len(mine)).astype(np.int32)
    y = compute.experts(to_dev_bf16(x), torch.from_numpy(local).cuda()).cpu().numpy()
    routed = oracle_experts(sh, np.unique(mine[local]))
    y_o = O.expert_ffn_per_token(routed, x, mine[local].astype(np.int32).reshape(-1, 1))[:, 0, :]
    assert np.array_equal(y.view(np.uint32), y_o.view(np.uint32))
