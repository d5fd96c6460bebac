"""Expert parallelism across ranks (the routed experts split by expert; after
the counts, one all-to-all each way): two or four gloo ranks on the CPU, each
with its own tokens (a rank may have none) and its share of the experts, the
compute steps given by the oracle; every rank's output rows equal the
single-process oracle layer's bit for bit, with and without adaptive top-p
(empty slots are not sent), under contiguous and usage-dealt placements.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synth

SHAPE = synth.LayerShape("ep_small", T=7, H=256, I=128, E=16, n_group=4, topk_group=2, top_k=4)


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_compute(sh, top_p, rank, n_ranks, placement=None):
    from oracle import oracle as O
    from oracle.synth_inputs import oracle_experts
    from quantized_mixture_experts_sigmoid_b200.expert_parallel import EPCompute, experts_of_rank

    W, b = synth.router_weight(sh), synth.router_bias(sh)
    per = sh.E // n_ranks
    if placement is None:
        mine = np.arange(rank * per, (rank + 1) * per)
    else:
        mine = experts_of_rank(*placement, rank).numpy()
    routed = oracle_experts(sh, mine)  # this rank's experts only
    shared = oracle_experts(sh, [0], shared=True)

    def bits(t):
        return t.view(torch.int16).numpy().view(np.uint16)

    def route(x):
        idx, w, _, _ = O.route(bits(x), W, b, sh.n_group, sh.topk_group, sh.top_k, sh.rsf, top_p)
        return torch.from_numpy(idx.astype(np.int32)), torch.from_numpy(w.astype(np.float32))

    def experts(rows, local_idx):
        gidx = mine[local_idx.numpy()].astype(np.int32).reshape(-1, 1)
        return torch.from_numpy(O.expert_ffn_per_token(routed, bits(rows), gidx)[:, 0, :].copy())

    def shared_fn(x):
        zero = np.zeros((x.shape[0], 1), dtype=np.int32)
        return torch.from_numpy(O.expert_ffn_per_token(shared, bits(x), zero)[:, 0, :].copy())

    def combine(y_pairs, w, shared_y):
        of, _ = O.combine(y_pairs.numpy(), w.numpy(), None if shared_y is None else shared_y.numpy())
        return torch.from_numpy(of)

    return EPCompute(route, experts, shared_fn, combine)


def _rank_main(rank, n_ranks, port, top_p, splits, q, usage_placement=False):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=n_ranks, timeout=datetime.timedelta(seconds=60))
    try:
        from quantized_mixture_experts_sigmoid_b200.expert_parallel import ep_forward
        x = synth.hidden_states(SHAPE)
        t0, t1 = splits[rank], splits[rank + 1]
        xr = torch.from_numpy(x[t0:t1].view(np.int16).copy()).view(torch.bfloat16)
        placement = _usage_placement(n_ranks) if usage_placement else None
        out = ep_forward(xr, SHAPE.E, _oracle_compute(SHAPE, top_p, rank, n_ranks, placement), placement=placement)
        q.put((rank, out.numpy().copy()))
    finally:
        dist.destroy_process_group()


def _usage_placement(n_ranks):
    # the usage record of the batch's own routing, then its most-used-first order
    from oracle import oracle as O
    from quantized_mixture_experts_sigmoid_b200.expert_parallel import placement_by_usage
    x = synth.hidden_states(SHAPE)
    idx, _, _, _ = O.route(x, synth.router_weight(SHAPE), synth.router_bias(SHAPE), SHAPE.n_group,
                           SHAPE.topk_group, SHAPE.top_k, SHAPE.rsf)
    order = O.usage_rank(O.usage_accumulate(idx, SHAPE.E))
    return placement_by_usage(torch.from_numpy(np.asarray(order)), n_ranks)


def test_four_ranks_equal_one_process():
    # every rank sends to and receives from several others; ranks of 2, 1, 0 and 4 tokens
    splits = [0, 2, 3, 3, SHAPE.T]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _port()
    procs = [ctx.Process(target=_rank_main, args=(r, 4, port, 0.0, splits, q, True)) for r in range(4)]
    for p in procs:
        p.start()
    try:
        got = dict(q.get(timeout=90) for _ in procs)
        for p in procs:
            p.join(timeout=60)
            assert p.exitcode == 0
    finally:
        for p in procs:
            if p.is_alive():
                p.kill()
    ref, _ = _reference(0.0)
    for r in range(4):
        assert np.array_equal(got[r].view(np.uint32), ref[splits[r]:splits[r + 1]].view(np.uint32))


def _reference(top_p):
    from oracle import oracle as O
    from oracle.synth_inputs import oracle_experts
    x = synth.hidden_states(SHAPE)
    W, b = synth.router_weight(SHAPE), synth.router_bias(SHAPE)
    routed = oracle_experts(SHAPE, range(SHAPE.E))
    shared = oracle_experts(SHAPE, [0], shared=True)
    of, _, idx, _ = O.layer_forward(x, W, b, SHAPE.n_group, SHAPE.topk_group, SHAPE.top_k, SHAPE.rsf,
                                    routed, shared, top_p)
    return of, idx


@pytest.mark.parametrize("top_p,usage_placement,split", [(0.0, False, 4), (0.6, False, 4), (0.0, True, 4),
                                                         (0.0, False, SHAPE.T)])
def test_two_ranks_equal_one_process(top_p, usage_placement, split):
    # ragged: 4 and 3 tokens; or rank 1 without tokens (it still serves its experts)
    splits = [0, split, SHAPE.T]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, top_p, splits, q, usage_placement))
             for r in range(2)]
    for p in procs:
        p.start()
    try:
        got = dict(q.get(timeout=60) for _ in procs)
        for p in procs:
            p.join(timeout=60)
            assert p.exitcode == 0
    finally:
        for p in procs:  # a rank that failed leaves the other waiting in a collective
            if p.is_alive():
                p.kill()
    ref, idx = _reference(top_p)
    if top_p:
        assert (idx < 0).any()  # some slots are empty and go nowhere
    owner = _usage_placement(2)[0].numpy() if usage_placement else np.arange(SHAPE.E) // (SHAPE.E // 2)
    own = np.where(idx >= 0, owner[np.maximum(idx, 0)], -1)
    assert ((own == 1) & (np.arange(SHAPE.T)[:, None] < split)).any()  # rank 0 sends to rank 1
    if split < SHAPE.T:
        assert ((own == 0) & (np.arange(SHAPE.T)[:, None] >= split)).any()  # and back
    for r in range(2):
        assert np.array_equal(got[r].view(np.uint32), ref[splits[r]:splits[r + 1]].view(np.uint32))


def test_placement_by_usage_deals_hot_experts_evenly():
    from quantized_mixture_experts_sigmoid_b200.expert_parallel import experts_of_rank, placement_by_usage
    rng = np.random.default_rng(3)
    E, N = 64, 4
    usage = (1000 * rng.zipf(1.3, E).clip(max=50)).astype(np.int64)
    order = torch.from_numpy(np.lexsort((np.arange(E), -usage)))  # most used first, ties to the lower index
    owner, local = placement_by_usage(order, N)
    held = [experts_of_rank(owner, local, r).numpy() for r in range(N)]
    assert sorted(np.concatenate(held).tolist()) == list(range(E))  # every expert exactly once
    assert all(len(h) == E // N for h in held)
    for r in range(N):  # local indices number each rank's experts in dealing order
        assert np.array_equal(local.numpy()[held[r]], np.arange(E // N))
    top = order[:N].numpy()  # the N hottest experts land on N different ranks
    assert len(set(owner.numpy()[top].tolist())) == N
    loads = np.array([usage[h].sum() for h in held])
    contiguous = np.array([usage[r * E // N:(r + 1) * E // N].sum() for r in range(N)])
    assert loads.max() - loads.min() <= usage.max()  # within one expert's load of even
    assert loads.max() <= contiguous.max()


def test_placement_by_usage_properties_hold_for_any_usage():
    # for any usage record and rank count: each rank holds E / N experts numbered 0 .. E/N - 1 in
    # dealing order, the N hottest sit on N different ranks, and two ranks' loads differ by at most
    # the largest single expert's usage (snake dealing of a sorted list)
    from hypothesis import given, settings
    from hypothesis import strategies as st

    from quantized_mixture_experts_sigmoid_b200.expert_parallel import experts_of_rank, placement_by_usage

    @settings(max_examples=200, deadline=None)
    @given(st.integers(1, 8).flatmap(lambda n: st.tuples(
        st.just(n), st.lists(st.integers(0, 10**6), min_size=n, max_size=16 * n).map(lambda u: u[:len(u) // n * n]))))
    def check(case):
        N, usage = case
        usage = np.array(usage, dtype=np.int64)
        E = len(usage)
        order = torch.from_numpy(np.lexsort((np.arange(E), -usage)))
        owner, local = placement_by_usage(order, N)
        held = [experts_of_rank(owner, local, r).numpy() for r in range(N)]
        assert sorted(np.concatenate(held).tolist()) == list(range(E))
        for r in range(N):
            assert len(held[r]) == E // N
            assert np.array_equal(local.numpy()[held[r]], np.arange(E // N))
        assert len(set(owner.numpy()[order[:N].numpy()].tolist())) == N
        loads = np.array([usage[h].sum() for h in held])
        assert loads.max() - loads.min() <= usage.max()

    check()
