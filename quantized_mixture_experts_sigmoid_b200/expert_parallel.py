"""Expert-parallel routed-MoE layer over a torch.distributed process group.

The layer of [HN] "Show HN: 느린 컴퓨터에서 GLM 5.2 실행하기", section "구현된
주요 기능" (sigmoid noaux_tc router, routed experts, shared expert), split by
expert across the ranks of a group: rank r of N holds routed experts
[r E/N, (r+1) E/N) (a contiguous slice of the stacked matrices), a replica of
the router and of the shared expert, and its own tokens.  One call:

1. routes the rank's tokens (every rank routes over all E experts);
2. sends each (token, slot) pair's token row to the rank holding the pair's
   expert with the expert's local index (one all-to-all of 32-bit words: the
   row's raw bf16 bits, then the index);
3. runs the rank's experts over the rows it received (a batch union over the
   local experts, then the quantised SwiGLU experts);
4. returns every pair's expert output to the token's rank (all-to-all);
5. combines them with the shared expert in slot order.

Empty slots (index -1: adaptive top-p) are not sent and add nothing.  Each
pair's output is the same expert function of the same token row on any rank,
and step 5 sums in slot order, so the result equals the single-GPU layer's.

Which rank holds which expert is a placement: contiguous slices by default,
or `placement_by_usage`, which deals the experts out in the usage record's
most-used-first order ([HN] "Learning cache와 하드웨어별 기대치": the hottest
experts are the ones worth placing) so every rank gets an even share of the
hot ones and of the routed pairs.

The exchange is plain collectives (NCCL between GPUs); the compute steps are
this library's C-ABI calls (`ep_cuda_compute`) or, in tests, any functions of
the same signatures.  Device-side errors that the kernels record (a bounded
wait that gave up, an index out of range) are read after a call with the
compute's `status()`.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Optional

import torch
import torch.distributed as dist


@dataclass
class EPCompute:
    """The per-rank compute steps of an expert-parallel call.

    route(x) -> (idx [T, K] int32, w [T, K] float32), over all E experts;
    experts(rows, local_idx) -> y [R, H] float32: the rank's experts (local index) on bf16 rows [R, H];
    shared(x) -> y [T, H] float32, or None without a shared expert;
    combine(y_pairs [T, K, H], w [T, K], shared_y or None) -> out [T, H] of out_dtype.
    A rank without tokens calls only `experts` (for the rows other ranks send it).
    status() -> the first device-side error code (MOE_E*) the latest calls recorded, MOE_OK if
    none, clearing them (synchronises); None when the steps record none.
    """
    route: Callable
    experts: Callable
    shared: Optional[Callable]
    combine: Callable
    out_dtype: torch.dtype = torch.float32
    status: Optional[Callable] = None


def placement_by_usage(order: torch.Tensor, n_ranks: int) -> tuple[torch.Tensor, torch.Tensor]:
    """Expert placement from a most-used-first order (moe_usage_rank's output).

    Deals the experts to the ranks in that order, turning at the ends (0, 1, .., N-1, N-1, .., 0,
    0, 1, ..), so each rank holds E / N experts and a near-even share of the usage.  Returns
    (owner [E]: the rank holding each expert, local [E]: its index among that rank's experts,
    which are numbered in dealing order).
    """
    order = order.to(torch.int64).cpu()
    E = order.numel()
    if E % n_ranks:
        raise ValueError(f"{E} experts do not split evenly over {n_ranks} ranks")
    owner = torch.empty(E, dtype=torch.int64)
    local = torch.empty(E, dtype=torch.int64)
    filled = [0] * n_ranks
    for i, e in enumerate(order.tolist()):
        lap, pos = divmod(i, n_ranks)
        r = pos if lap % 2 == 0 else n_ranks - 1 - pos
        owner[e] = r
        local[e] = filled[r]
        filled[r] += 1
    return owner, local


def experts_of_rank(owner: torch.Tensor, local: torch.Tensor, rank: int) -> torch.Tensor:
    """The global indices of the experts `rank` holds, in local-index order."""
    mine = torch.nonzero(owner.cpu() == rank).flatten()
    return mine[torch.argsort(local.cpu()[mine])]


def _a2a(out: torch.Tensor, inp: torch.Tensor, out_splits, in_splits, group) -> torch.Tensor:
    dist.all_to_all_single(out, inp, output_split_sizes=out_splits, input_split_sizes=in_splits, group=group)
    return out


def ep_forward(x: torch.Tensor, n_expert: int, compute: EPCompute, group=None,
               placement: tuple[torch.Tensor, torch.Tensor] | None = None) -> torch.Tensor:
    """One expert-parallel layer call on this rank's tokens x [T, H] (bf16).

    placement: (owner [E], local [E]) as from placement_by_usage, the same on every rank; None for
    contiguous slices (rank r holds experts r E/N .. (r+1) E/N - 1).
    """
    n = dist.get_world_size(group)
    if n_expert % n:
        raise ValueError(f"{n_expert} experts do not split evenly over {n} ranks")
    per = n_expert // n
    T, H = x.shape
    if T:
        idx, w = compute.route(x)
        K = idx.shape[1]
        flat = idx.reshape(-1).to(torch.int64)
    else:  # no tokens here this call: nothing to send, but this rank's experts still serve the others
        w, K = None, 1
        flat = torch.empty(0, dtype=torch.int64, device=x.device)
    valid = flat >= 0
    if placement is None:
        owner_of = torch.where(valid, flat // per, torch.full_like(flat, n))
        local_of = flat - owner_of * per
    else:
        owner, loc = (t.to(device=x.device, dtype=torch.int64) for t in placement)
        safe = torch.where(valid, flat, torch.zeros_like(flat))
        owner_of = torch.where(valid, owner[safe], torch.full_like(flat, n))
        local_of = loc[safe]
    dest = owner_of  # empty slots (rank n) sort last and go nowhere
    order = torch.argsort(dest, stable=True)  # pairs by destination rank, (token, slot) ascending within
    n_send = int(valid.sum())
    order = order[:n_send]
    send_counts = torch.bincount(dest[order], minlength=n).to(torch.int64)
    recv_counts = torch.empty_like(send_counts)
    _a2a(recv_counts, send_counts, None, None, group)
    sc, rc = send_counts.tolist(), recv_counts.tolist()
    n_recv = sum(rc)

    # one message per pair: the token row as raw bf16 bits, two to a 32-bit word (H is even), then
    # the expert's index on the destination rank
    W = H // 2
    send = torch.empty(n_send, W + 1, dtype=torch.int32, device=x.device)
    if n_send:
        send[:, :W] = x.contiguous().view(torch.int32).index_select(0, order // K)
        send[:, W] = local_of[order].to(torch.int32)
    recv = _a2a(torch.empty(n_recv, W + 1, dtype=torch.int32, device=x.device), send, rc, sc, group)

    y_recv = compute.experts(recv[:, :W].contiguous().view(torch.bfloat16), recv[:, W].contiguous()) if n_recv \
        else torch.empty(0, H, dtype=torch.float32, device=x.device)
    y_back = _a2a(torch.empty(n_send, H, dtype=torch.float32, device=x.device), y_recv.contiguous(), sc, rc, group)
    if not T:
        return torch.empty(0, H, dtype=compute.out_dtype, device=x.device)

    y_pairs = torch.zeros(T * K, H, dtype=torch.float32, device=x.device)
    y_pairs.index_copy_(0, order, y_back)
    shared_y = compute.shared(x) if compute.shared is not None else None
    return compute.combine(y_pairs.view(T, K, H), w, shared_y)


def ep_cuda_compute(w_router: torch.Tensor, bias: torch.Tensor, cfg, routed, shared=None,
                    rank: int = 0, n_ranks: int = 1, out_dtype=torch.bfloat16,
                    placement: tuple[torch.Tensor, torch.Tensor] | None = None) -> EPCompute:
    """EPCompute on this library's kernels for rank `rank` of `n_ranks`.

    routed: the full stacked ExpertSet (all E experts; this rank uses its share), or an ExpertSet
    already holding only the rank's E / n_ranks experts in local-index order.  shared: ExpertSet
    of one expert or None.  placement: as for ep_forward (the rank's experts are gathered into a
    stack of their own when it is given with the full set).
    """
    from . import moe

    E = cfg.n_expert
    per = E // n_ranks
    if placement is not None and routed.n_expert == E:
        mine = experts_of_rank(*placement, rank).to(routed.w_gate.device)
        pick = lambda t: t.index_select(0, mine).contiguous()  # noqa: E731
        local = moe.ExpertSet(routed.qtype, per, routed.hidden, routed.inter, pick(routed.w_gate),
                              pick(routed.w_up), pick(routed.w_down), pick(routed.s_gate), pick(routed.s_up),
                              pick(routed.s_down), routed.group_size)
    elif routed.n_expert == E:
        e0, e1 = rank * per, (rank + 1) * per
        local = moe.ExpertSet(routed.qtype, per, routed.hidden, routed.inter, routed.w_gate[e0:e1],
                              routed.w_up[e0:e1], routed.w_down[e0:e1], routed.s_gate[e0:e1],
                              routed.s_up[e0:e1], routed.s_down[e0:e1], routed.group_size)
    elif routed.n_expert == per:
        local = routed
    else:
        raise ValueError("routed experts: all E, or this rank's E / n_ranks")

    last = {}  # each step's latest workspace: the kernels record device-side errors there

    def route(x):
        T = x.shape[0]
        idx = torch.empty(T, cfg.top_k, dtype=torch.int32, device=x.device)
        w = torch.empty(T, cfg.top_k, dtype=torch.float32, device=x.device)
        ws = last["route"] = moe.workspace(moe.moe_route_workspace_bytes(T, cfg))
        moe.moe_route(x, w_router, bias, cfg, idx, w, ws)
        return idx, w

    def experts(rows, local_idx):
        R = rows.shape[0]
        dev = rows.device
        n_unique = torch.empty(4, dtype=torch.int32, device=dev)
        uniq = torch.empty(per, dtype=torch.int32, device=dev)
        offsets = torch.empty(per + 1, dtype=torch.int32, device=dev)
        pair_tok = torch.empty(R, dtype=torch.int32, device=dev)
        pair_slot = torch.empty(R, dtype=torch.int32, device=dev)
        moe.moe_union(local_idx.view(R, 1), per, n_unique, uniq, offsets, pair_tok, pair_slot)
        y = torch.empty(R, 1, local.hidden, dtype=torch.float32, device=dev)
        ws = last["experts"] = moe.workspace(moe.moe_expert_ffn_workspace_bytes(local, R, 1))
        moe.moe_expert_ffn_q(local, rows, 1, (n_unique, uniq, offsets, pair_tok, pair_slot), y, ws)
        return y.view(R, local.hidden)

    def shared_fn(x):
        T = x.shape[0]
        y = torch.empty(T, 1, shared.hidden, dtype=torch.float32, device=x.device)
        ws = last["shared"] = moe.workspace(moe.moe_expert_ffn_workspace_bytes(shared, T, 1))
        moe.moe_expert_ffn_q(shared, x, 1, None, y, ws)
        return y.view(T, shared.hidden)

    def combine(y_pairs, w, shared_y):
        T, _, H = y_pairs.shape
        out = torch.empty(T, H, dtype=out_dtype, device=y_pairs.device)
        moe.moe_combine(y_pairs, w, shared_y, out)
        return out

    def status():
        codes = [moe.moe_workspace_status(ws) for ws in last.values()]
        return next((c for c in codes if c != moe.MOE_OK), moe.MOE_OK)

    return EPCompute(route, experts, shared_fn if shared is not None else None, combine, out_dtype, status)
