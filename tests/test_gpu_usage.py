"""Expert-usage record and pin order on the GPU against their plain definitions
([HN] "Learning cache와 하드웨어별 기대치": routed experts recorded, the most
used pinned first)."""
import numpy as np
import pytest
import torch

import synth
from oracle import oracle as O
from quantized_mixture_experts_sigmoid_b200 import moe
from synth.device import to_dev_bf16

pytestmark = pytest.mark.gpu


def test_usage_record_and_rank_match_the_definition():
    rng = np.random.default_rng(41)
    E = 256
    usage = torch.zeros(E, dtype=torch.int32, device="cuda")
    ref = np.zeros(E, np.int64)
    for T, K in [(1, 8), (4, 8), (2048, 8), (37, 5)]:
        idx = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
        idx[rng.random((T, K)) < 0.2] = -1
        moe.moe_usage_accumulate(torch.from_numpy(idx).cuda(), E, usage)
        ref = O.usage_accumulate(idx, E, ref)
    assert np.array_equal(usage.cpu().numpy().astype(np.int64), ref)
    order = torch.empty(E, dtype=torch.int32, device="cuda")
    moe.moe_usage_rank(usage, order)
    assert np.array_equal(order.cpu().numpy(), O.usage_rank(ref))


def test_usage_rank_ties_and_sizes():
    for E in (1, 16, 100, 1024):
        u = np.random.default_rng(E).integers(0, 3, E).astype(np.int32)
        order = torch.empty(E, dtype=torch.int32, device="cuda")
        moe.moe_usage_rank(torch.from_numpy(u).cuda(), order)
        assert np.array_equal(order.cpu().numpy(), O.usage_rank(u))


def test_prefill_routing_record_finds_the_popular_experts():
    # the Zipf-skewed prefill workload: the record ranks experts by how many tokens chose them
    sh = synth.CONFIGS["prefill"]
    W = torch.from_numpy(synth.router_weight(sh)).cuda()
    b = torch.from_numpy(synth.router_bias(sh)).cuda()
    cfg = moe.RouterCfg(sh.E, sh.n_group, sh.topk_group, sh.top_k, sh.rsf)
    x = to_dev_bf16(synth.hidden_states(sh))
    idx = torch.empty(sh.T, sh.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(sh.T, sh.top_k, dtype=torch.float32, device="cuda")
    ws = moe.workspace(moe.moe_route_workspace_bytes(sh.T, cfg))
    moe.moe_route(x, W, b, cfg, idx, w, ws)
    usage = torch.zeros(sh.E, dtype=torch.int32, device="cuda")
    moe.moe_usage_accumulate(idx, sh.E, usage)
    order = torch.empty(sh.E, dtype=torch.int32, device="cuda")
    moe.moe_usage_rank(usage, order)
    ref = O.usage_accumulate(idx.cpu().numpy(), sh.E)
    assert np.array_equal(order.cpu().numpy(), O.usage_rank(ref))
    top = ref[order.cpu().numpy()[:16]].sum() / ref.sum()
    assert top > 16 / sh.E  # skewed: the 16 hottest carry more than their share
