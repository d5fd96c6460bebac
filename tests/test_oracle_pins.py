"""Pins of the CPU oracle against facts other than itself (no GPU).

Each test compares the oracle with something independent: hand-worked values
from the golden fixtures, a brute-force full sort, a textbook special case,
exact integer arithmetic, an fp64 dense reformulation in numpy, torch's own
bf16 rounding, or the size figures the pages print.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import synth
from oracle import oracle as O
from tests.helpers import oracle_experts, rel_err_rows, unpack_ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ bf16
def test_bf16_widen_narrow_against_torch():
    rng = np.random.default_rng(1)
    f = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 10.0 ** rng.integers(-6, 6, 20000),
                        np.float32([0.0, -0.0, 1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8])])
    f = f.astype(np.float32)
    want = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([O.f32_to_bf16(float(v)) for v in f], dtype=np.uint16)
    assert np.array_equal(got, want)
    back = np.array([O.bf16_to_f32(int(b)) for b in want[:2000]], dtype=np.float32)
    assert np.array_equal(back, torch.from_numpy(want[:2000].view(np.int16)).view(torch.bfloat16).float().numpy())


# ---------------------------------------------------------------- logits
def test_router_logits_equal_exact_rational_rounded_once():
    rng = np.random.default_rng(2)
    T, H, E = 3, 96, 5
    x = synth.bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    W = (0.02 * rng.standard_normal((E, H))).astype(np.float32)
    got = O.router_logits(x, W)
    xf = synth.bf16_to_f32(x)
    for t in range(T):
        for e in range(E):
            exact = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(xf[t], W[e]))
            assert got[t, e] == np.float32(float(exact))


# -------------------------------------------------------------- routing
_SYM = {"Z": 0.0, "P": float(np.float32(math.log(3.0))), "M": float(np.float32(-math.log(3.0)))}


def _hand_cases():
    out = []
    with open(os.path.join(GOLDEN, "router_hand_cases.txt")) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, cfg, lg, bias, idx, w = [s.strip() for s in line.split("|")]
            E, G, TG, K, rsf = cfg.split()
            out.append(dict(name=name, E=int(E), G=int(G), TG=int(TG), K=int(K), rsf=float(rsf),
                            logits=np.float32([_SYM[s] for s in lg.split()]),
                            bias=np.float32([float(b) for b in bias.split()]),
                            idx=[int(i) for i in idx.split()], w=np.float32([float(v) for v in w.split()])))
    return out


@pytest.mark.parametrize("case", _hand_cases(), ids=lambda c: c["name"])
def test_select_hand_worked(case):
    idx, w, _, _ = O.select(case["logits"][None, :], case["bias"], case["G"], case["TG"], case["K"], case["rsf"])
    assert idx[0].tolist() == case["idx"]
    assert np.array_equal(w[0], case["w"])


@pytest.mark.parametrize("case", _hand_cases()[:3], ids=lambda c: c["name"])
def test_route_hand_worked_through_logits(case):
    # x = e_0, so the logit of expert e is W[e][0] exactly
    E, H = case["E"], 32
    x = np.zeros((1, H), np.float32)
    x[0, 0] = 1.0
    W = np.zeros((E, H), np.float32)
    W[:, 0] = case["logits"]
    idx, w, _, _ = O.route(synth.bf16_bits(x), W, case["bias"], case["G"], case["TG"], case["K"], case["rsf"])
    assert idx[0].tolist() == case["idx"] and np.array_equal(w[0], case["w"])


def _brute_select(logits, bias, G, TG, K):
    """Full sorts with explicit (value desc, index asc) keys."""
    T, E = logits.shape
    gsz = E // G
    out = np.empty((T, K), np.int32)
    for t in range(T):
        s = np.float32(1.0 / (1.0 + np.exp(-logits[t].astype(np.float64))))
        b = (s + bias).astype(np.float32)
        gs = []
        for g in range(G):
            vals = sorted(b[g * gsz:(g + 1) * gsz].tolist(), reverse=True)
            gs.append(np.float32(np.float32(vals[0]) + np.float32(vals[1])))
        gorder = sorted(range(G), key=lambda g: (-gs[g], g))[:TG]
        cand = [e for e in range(E) if e // gsz in gorder]
        out[t] = sorted(cand, key=lambda e: (-b[e], e))[:K]
    return out


@pytest.mark.parametrize("E,G,TG,K", [(256, 8, 4, 8), (16, 4, 2, 2), (64, 8, 3, 6), (32, 1, 1, 4)])
def test_select_matches_brute_force_sort(E, G, TG, K):
    rng = np.random.default_rng(E * 100 + K)
    T = 2500 if E == 256 else 1500
    logits = (1.57 * rng.standard_normal((T, E))).astype(np.float32)
    # quantise some logits to force ties
    logits[: T // 4] = np.round(logits[: T // 4] * 4) / 4
    bias = (0.1 * rng.standard_normal(E)).astype(np.float32)
    idx, w, _, _ = O.select(logits, bias, G, TG, K, 2.5)
    assert np.array_equal(idx, _brute_select(logits, bias, G, TG, K))


def _brute_margins(logits, bias, G, TG, K):
    """Margins at the two selection boundaries from full sorts (fp32 differences):
    the K-th chosen b minus the best b left among kept groups' experts, and the
    TG-th kept group score minus the best dropped group score (inf where none is left)."""
    T, E = logits.shape
    gsz = E // G
    ge, gg = np.empty(T, np.float32), np.empty(T, np.float32)
    for t in range(T):
        s = np.float32(1.0 / (1.0 + np.exp(-logits[t].astype(np.float64))))
        b = (s + bias).astype(np.float32)
        gs = []
        for g in range(G):
            vals = sorted(b[g * gsz:(g + 1) * gsz].tolist(), reverse=True)
            gs.append(np.float32(np.float32(vals[0]) + np.float32(vals[1])))
        order = sorted(range(G), key=lambda g: (-gs[g], g))
        gg[t] = np.float32(gs[order[TG - 1]] - gs[order[TG]]) if TG < G else np.float32(np.inf)
        cand = sorted([e for e in range(E) if e // gsz in order[:TG]], key=lambda e: (-b[e], e))
        ge[t] = np.float32(b[cand[K - 1]] - b[cand[K]]) if K < len(cand) else np.float32(np.inf)
    return ge, gg


@pytest.mark.parametrize("E,G,TG,K", [(256, 8, 4, 8), (16, 4, 2, 2), (64, 8, 8, 6), (32, 1, 1, 4),
                                      (8, 2, 1, 4)])
def test_select_margins_match_brute_force(E, G, TG, K):
    # the margin diagnostics back the claim that no seeded token sits on a
    # selection tie; pinned here against full sorts, ties and exhausted
    # candidate lists included (TG = G: no dropped group; K = group size: no expert left)
    rng = np.random.default_rng(E * 10 + K + TG)
    T = 600
    logits = (1.57 * rng.standard_normal((T, E))).astype(np.float32)
    logits[: T // 3] = np.round(logits[: T // 3] * 4) / 4
    for bias in ((0.1 * rng.standard_normal(E)).astype(np.float32), np.zeros(E, np.float32)):
        _, _, ge, gg = O.select(logits, bias, G, TG, K, 2.5)
        be, bg = _brute_margins(logits, bias, G, TG, K)
        assert np.array_equal(ge.view(np.uint32), be.view(np.uint32))
        assert np.array_equal(gg.view(np.uint32), bg.view(np.uint32))
        assert np.all(ge >= 0) and np.all(gg >= 0)
    if K < TG * (E // G):
        assert np.any(ge[: T // 3] == 0)  # zero bias, quantised logits: exact ties occur


def test_select_special_case_is_textbook_topk():
    # one group, no bias: sigmoid is monotone, so the choice is the top-k of the logits
    rng = np.random.default_rng(5)
    T, E, K = 400, 64, 8
    grid = (np.arange(E) - E / 2) * 0.05
    logits = np.stack([rng.permutation(grid) for _ in range(T)]).astype(np.float32)
    idx, _, _, _ = O.select(logits, np.zeros(E, np.float32), 1, 1, K, 1.0)
    assert np.array_equal(idx, np.argsort(-logits, axis=1, kind="stable")[:, :K])


def test_gate_weights_sum_to_rsf():
    rng = np.random.default_rng(6)
    T, E = 3000, 256
    logits = (1.57 * rng.standard_normal((T, E))).astype(np.float32)
    bias = (0.1 * rng.standard_normal(E)).astype(np.float32)
    for rsf in (2.5, 1.0, 1.8):
        _, w, _, _ = O.select(logits, bias, 8, 4, 8, rsf)
        ulp = np.spacing(np.float32(rsf))
        assert np.all(np.abs(w.astype(np.float64).sum(1) - rsf) <= 8 * ulp)
        assert np.all(w > 0)


def test_select_weights_use_unbiased_scores():
    rng = np.random.default_rng(7)
    T, E = 200, 32
    logits = (1.57 * rng.standard_normal((T, E))).astype(np.float32)
    bias = (0.3 * rng.standard_normal(E)).astype(np.float32)
    idx, w, _, _ = O.select(logits, bias, 4, 2, 4, 2.5)
    s = 1.0 / (1.0 + np.exp(-logits.astype(np.float64)))
    for t in range(T):
        ref = s[t, idx[t]] / s[t, idx[t]].sum() * 2.5
        assert np.allclose(w[t], ref, rtol=1e-6)


def test_select_rejects_bad_configs():
    lg = np.zeros((1, 16), np.float32)
    b = np.zeros(16, np.float32)
    for G, TG, K in [(3, 1, 1), (16, 1, 1), (4, 5, 1), (4, 2, 9), (4, 0, 1), (4, 2, 0)]:
        with pytest.raises(ValueError):
            O.select(lg, b, G, TG, K, 2.5)


# -------------------------------------------------------- adaptive top-p
def _topp_cases():
    out = []
    with open(os.path.join(GOLDEN, "topp_hand_cases.txt")) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, cfg, lg, bias, idx, w = [s.strip() for s in line.split("|")]
            E, G, TG, K, rsf, pp = cfg.split()
            out.append(dict(name=name, E=int(E), G=int(G), TG=int(TG), K=int(K), rsf=float(rsf), p=float(pp),
                            logits=np.float32([_SYM[s] for s in lg.split()]),
                            bias=np.float32([float(b) for b in bias.split()]),
                            idx=[int(i) for i in idx.split()], w=np.float32([float(v) for v in w.split()])))
    return out


@pytest.mark.parametrize("case", _topp_cases(), ids=lambda c: c["name"])
def test_topp_hand_worked(case):
    idx, w, _, _ = O.select(case["logits"][None, :], case["bias"], case["G"], case["TG"], case["K"], case["rsf"],
                            top_p=case["p"])
    assert idx[0].tolist() == case["idx"]
    assert np.array_equal(w[0], case["w"])


def _brute_topp(logits, bias, G, TG, K, rsf, p):
    """The top-p reading written out from its definition over the brute-force selection."""
    T = logits.shape[0]
    sel = _brute_select(logits, bias, G, TG, K)
    idx = np.full((T, K), -1, np.int32)
    w = np.zeros((T, K), np.float32)
    pf = float(np.float32(p))
    for t in range(T):
        s_all = np.float32(1.0 / (1.0 + np.exp(-logits[t].astype(np.float64))))
        s = [s_all[e] for e in sel[t]]
        keep = set(range(K))
        if 0.0 < pf < 1.0:
            order = sorted(range(K), key=lambda k: (-float(s[k]), k))
            total = 0.0
            for k in range(K):
                total += float(s[k])
            run = 0.0
            for m, k in enumerate(order):
                run += float(s[k])
                if run >= pf * total:
                    keep = set(order[:m + 1])
                    break
        kept = [k for k in range(K) if k in keep]
        den = np.float32(0.0)
        for k in kept:
            den = np.float32(den + s[k])
        for j, k in enumerate(kept):
            idx[t, j] = sel[t][k]
            w[t, j] = np.float32(np.float32(s[k] / den) * np.float32(rsf))
    return idx, w


@pytest.mark.parametrize("E,G,TG,K", [(256, 8, 4, 8), (16, 4, 2, 2), (64, 8, 3, 6)])
@pytest.mark.parametrize("p", [0.3, 0.5, 0.7, 0.9, 0.97])
def test_topp_matches_brute_force(E, G, TG, K, p):
    rng = np.random.default_rng(E + K + int(p * 100))
    logits = (1.57 * rng.standard_normal((400, E))).astype(np.float32)
    logits[:100] = np.round(logits[:100] * 4) / 4  # ties in s
    bias = (0.1 * rng.standard_normal(E)).astype(np.float32)
    idx, w, _, _ = O.select(logits, bias, G, TG, K, 2.5, top_p=p)
    bi, bw = _brute_topp(logits, bias, G, TG, K, 2.5, p)
    assert np.array_equal(idx, bi)
    assert np.array_equal(w.view(np.uint32), bw.view(np.uint32))


def test_topp_invariants():
    rng = np.random.default_rng(31)
    E, G, TG, K, rsf = 256, 8, 4, 8, 2.5
    logits = (1.57 * rng.standard_normal((500, E))).astype(np.float32)
    bias = (0.1 * rng.standard_normal(E)).astype(np.float32)
    base_i, base_w, _, _ = O.select(logits, bias, G, TG, K, rsf)
    # outside (0, 1) the routing is untouched, bit for bit
    for p in (0.0, 1.0, -0.5, 1.5, float("nan")):
        i, w, _, _ = O.select(logits, bias, G, TG, K, rsf, top_p=p)
        assert np.array_equal(i, base_i) and np.array_equal(w.view(np.uint32), base_w.view(np.uint32))
    prev = np.ones(len(logits), int)
    s = np.float32(1.0 / (1.0 + np.exp(-logits.astype(np.float64))))
    for p in (1e-6, 0.2, 0.5, 0.7, 0.9, 0.999):
        i, w, _, _ = O.select(logits, bias, G, TG, K, rsf, top_p=p)
        kept = (i >= 0).sum(1)
        assert kept.min() >= 1
        assert np.all(kept >= prev)  # more mass kept, never fewer experts
        prev = kept
        for t in range(len(logits)):
            n = kept[t]
            assert np.all(i[t, n:] == -1) and np.all(w[t, n:] == 0.0)
            # kept experts are a subsequence of the full slot list (slot order kept)
            pos = [base_i[t].tolist().index(e) for e in i[t, :n]]
            assert pos == sorted(pos)
            # the kept mass reaches p, and dropping the smallest kept score would not
            sk = s[t, i[t, :n]].astype(np.float64)
            S = s[t, base_i[t]].astype(np.float64).sum()
            assert sk.sum() >= np.float32(p) * S * (1 - 1e-12)
            assert sk.sum() - sk.min() < np.float32(p) * S
            assert abs(float(w[t, :n].astype(np.float64).sum()) - rsf) < 1e-5
        if p == 1e-6:
            assert np.all(kept == 1) and np.array_equal(i[:, 0], base_i[np.arange(len(logits)),
                                                                          np.argmax(s[np.arange(len(logits))[:, None], base_i], 1)])


# ----------------------------------------------------------------- union
def test_union_against_bitmap_brute_force_and_invariants():
    rng = np.random.default_rng(8)
    for T, E, K in [(1, 256, 8), (4, 16, 2), (37, 64, 6), (300, 256, 8)]:
        idx = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
        un = O.union(idx, E)
        bitmap = np.zeros((E, T), bool)
        for t in range(T):
            bitmap[idx[t], t] = True
        present = np.nonzero(bitmap.any(1))[0]
        assert un["n_unique"] == len(present)
        assert np.array_equal(un["uniq"], present)
        assert np.array_equal(un["counts"], bitmap.sum(1))
        flat = idx.reshape(-1)
        order = np.argsort(flat, kind="stable")  # (expert asc, flat index asc) = (expert, token)
        assert np.array_equal(un["pair_tok"], order // K)
        assert np.array_equal(un["pair_slot"], order % K)
        assert np.array_equal(un["offsets"], np.concatenate([[0], np.cumsum(bitmap.sum(1)[present])]))
        assert np.all(idx[un["pair_tok"], un["pair_slot"]] == np.repeat(present, np.diff(un["offsets"])))


def test_union_leaves_out_empty_slots():
    # -1 marks an empty slot (top-p drop or an unroutable token): no pair, no count
    rng = np.random.default_rng(12)
    T, E, K = 50, 64, 6
    idx = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    drop = rng.random((T, K)) < 0.3
    idx2 = np.where(drop, -1, idx).astype(np.int32)
    un = O.union(idx2, E)
    flat = idx2.reshape(-1)
    valid = np.nonzero(flat >= 0)[0]
    order = valid[np.argsort(flat[valid], kind="stable")]
    assert un["offsets"][un["n_unique"]] == len(valid)
    assert np.array_equal(un["pair_tok"][:len(valid)], order // K)
    assert np.array_equal(un["pair_slot"][:len(valid)], order % K)
    assert np.array_equal(un["counts"], np.bincount(flat[valid], minlength=E))
    with pytest.raises(ValueError):
        O.union(np.where(drop, -2, idx).astype(np.int32), E)


def test_combine_skips_zero_weight_slots():
    # a zero-weight slot adds nothing and its y is not read (NaN there changes nothing)
    rng = np.random.default_rng(13)
    T, K, H = 3, 4, 64
    y = rng.standard_normal((T, K, H)).astype(np.float32)
    w = rng.random((T, K)).astype(np.float32)
    w[:, 2] = 0.0
    ys = rng.standard_normal((T, H)).astype(np.float32)
    of, _ = O.combine(y, w, ys)
    y2 = y.copy()
    y2[:, 2] = np.nan
    of2, _ = O.combine(y2, w, ys)
    assert np.array_equal(of.view(np.uint32), of2.view(np.uint32))
    ref = ys.copy()
    for k in (0, 1, 3):
        ref = (ref + w[:, k:k + 1] * y[:, k]).astype(np.float32)
    assert np.array_equal(of.view(np.uint32), ref.view(np.uint32))


def test_usage_record_and_rank_hand_worked():
    # two batches: experts 1 and 2 used 5 times, 0 three times, 3 never; -1 slots ignored
    u = O.usage_accumulate(np.array([[1, 2], [0, 1], [2, -1]]), 4)
    u = O.usage_accumulate(np.array([[1, 2, 0], [2, 1, 0], [1, 2, -1]]), 4, u)
    assert u.tolist() == [3, 5, 5, 0]
    assert O.usage_rank(u).tolist() == [1, 2, 0, 3]  # the tie 1 / 2 goes to the lower index
    assert O.usage_rank(np.zeros(5)).tolist() == [0, 1, 2, 3, 4]


def test_usage_rank_is_a_permutation_sorted_by_count():
    rng = np.random.default_rng(14)
    u = rng.integers(0, 6, 300)
    order = O.usage_rank(u)
    assert sorted(order.tolist()) == list(range(300))
    keys = [(-int(u[e]), int(e)) for e in order]
    assert keys == sorted(keys)


# ------------------------------------------------------------------ Q8_0
def test_q8_0_grid_values_round_trip_exactly():
    rng = np.random.default_rng(9)
    for k in range(-12, 6):
        d = np.float32(2.0 ** k)
        q = rng.integers(-127, 128, (8, 32)).astype(np.int8)
        q[:, 3] = rng.choice([-127, 127], 8)  # make max|q| = 127 in every block
        v = (q.astype(np.float32) * d).reshape(-1)
        gq, gd = O.q8_0(v)
        assert np.array_equal(gq, q.reshape(-1)) and np.all(gd == d)


def test_q8_0_error_bound_zero_block_and_ties():
    rng = np.random.default_rng(10)
    v = (rng.standard_normal(32 * 500) * 3).astype(np.float32)
    v[32:64] = 0.0
    q, d = O.q8_0(v)
    assert np.all(q[32:64] == 0) and d[1] == 0.0
    vb = v.reshape(-1, 32).astype(np.float64)
    err = np.abs(vb - q.reshape(-1, 32).astype(np.float64) * d[:, None])
    assert np.all(err <= d[:, None].astype(np.float64) * (0.5 + 1e-6))
    assert np.all(np.abs(q) <= 127)
    assert np.all(np.abs(q.reshape(-1, 32)).max(1)[d > 0] == 127)
    # half-way values round away from zero (block with max 127 -> d = 1)
    blk = np.zeros(32, np.float32)
    blk[:5] = [127.0, 2.5, -2.5, 0.5, -0.5]
    q, d = O.q8_0(blk)
    assert d[0] == 1.0 and q[:5].tolist() == [127, 3, -3, 1, -1]


# -------------------------------------------------------------- packing
def _pack_ref(codes, qtype):
    """Independent packer (the opposite direction of the oracle's unpacker)."""
    c = codes.astype(np.int16)
    if qtype == 4:
        u = (c + 8).reshape(-1, 2)
        return (u[:, 0] | (u[:, 1] << 4)).astype(np.uint8)
    if qtype == 2:
        u = (c + 2).reshape(-1, 4)
        return (u[:, 0] | (u[:, 1] << 2) | (u[:, 2] << 4) | (u[:, 3] << 6)).astype(np.uint8)
    return codes.astype(np.int8).view(np.uint8)


@pytest.mark.parametrize("qtype,lo,hi", [(4, -8, 7), (2, -2, 1), (8, -127, 127)])
def test_unpack_inverts_independent_packer(qtype, lo, hi):
    rng = np.random.default_rng(qtype)
    codes = rng.integers(lo, hi + 1, 4096).astype(np.int8)
    assert np.array_equal(O.unpack(_pack_ref(codes, qtype), qtype, 4096), codes)


# ------------------------------------------------------------- quant dot
@pytest.mark.parametrize("qtype,lo,hi", [(4, -8, 7), (2, -2, 1), (8, -127, 127)])
def test_qdot_exact_integer_case(qtype, lo, hi):
    # weight scale 1, integer activations with max|x| = 127 in every block ->
    # d = 1 and the result is the integer dot product exactly (partial sums < 2^24)
    rng = np.random.default_rng(20 + qtype)
    n = 6144
    for _ in range(20):
        codes = rng.integers(lo, hi + 1, n).astype(np.int8)
        x = rng.integers(-127, 128, n).astype(np.float32)
        x[::32] = 127.0
        qa, da = O.q8_0(x)
        assert np.all(da == 1.0)
        wc = O.unpack(_pack_ref(codes, qtype), qtype, n)
        want = int(np.dot(codes.astype(np.int64), x.astype(np.int64)))
        partial = np.cumsum((codes.astype(np.int64) * x.astype(np.int64)).reshape(-1, 32).sum(1))
        assert np.all(np.abs(partial) < 2 ** 24)
        assert O.qdot(wc, 1.0, qa, da) == float(want)


def test_qdot_against_fp64_dequantised_dot():
    rng = np.random.default_rng(30)
    n = 2048
    for _ in range(50):
        codes = rng.integers(-8, 8, n).astype(np.int8)
        x = rng.standard_normal(n).astype(np.float32)
        s = np.float32(rng.uniform(0.01, 0.05))
        qa, da = O.q8_0(x)
        ref = float(np.dot(codes.astype(np.float64), qa.astype(np.float64) * np.repeat(da.astype(np.float64), 32))) * float(s)
        got = O.qdot(codes, s, qa, da)
        scale = float(np.sum(np.abs(codes * qa.astype(np.float64) * np.repeat(da, 32)))) * float(s)
        assert abs(got - ref) <= 1e-5 * scale


@pytest.mark.parametrize("group", [32, 128])
def test_qdot_grouped_exact_integer_case(group):
    # every weight scale 1 and activation scales 1: the integer dot exactly
    rng = np.random.default_rng(40 + group)
    n = 2048
    for _ in range(10):
        codes = rng.integers(-8, 8, n).astype(np.int8)
        x = rng.integers(-127, 128, n).astype(np.float32)
        x[::32] = 127.0
        qa, da = O.q8_0(x)
        want = int(np.dot(codes.astype(np.int64), x.astype(np.int64)))
        assert O.qdot_grouped(codes, np.ones(n // group, np.float32), group, qa, da) == float(want)


@pytest.mark.parametrize("group", [32, 64, 128, 2048])
def test_qdot_grouped_against_fp64_dequantised_dot(group):
    # sum_k s_w[g(k)] q_w[k] d_a[b(k)] q_a[k] in fp64; each group's scale applies to its codes only
    rng = np.random.default_rng(50 + group)
    n = 2048
    for _ in range(30):
        codes = rng.integers(-8, 8, n).astype(np.int8)
        x = rng.standard_normal(n).astype(np.float32)
        sw = rng.uniform(0.01, 0.05, n // group).astype(np.float32)
        qa, da = O.q8_0(x)
        terms = (codes.astype(np.float64) * np.repeat(sw.astype(np.float64), group)
                 * qa.astype(np.float64) * np.repeat(da.astype(np.float64), 32))
        got = O.qdot_grouped(codes, sw, group, qa, da)
        assert abs(got - terms.sum()) <= 1e-5 * np.abs(terms).sum()
        if group < n:  # doubling one group's scale moves only that group's share
            sw2 = sw.copy()
            sw2[1] *= 2
            d = O.qdot_grouped(codes, sw2, group, qa, da) - got
            share = terms[group:2 * group].sum()
            assert abs(d - share) <= 1e-5 * np.abs(terms).sum()


@pytest.mark.parametrize("qtype,group", [(4, 32), (4, 128), (8, 64), (2, 32)])
def test_expert_grouped_against_fp64_dense(qtype, group):
    sh = synth.CONFIGS["tiny"].with_(qtype=qtype, H=512, I=256, group_size=group)
    x = synth.bf16_to_f32(synth.hidden_states(sh)[0])
    ex = oracle_experts(sh, [3])
    y, h = O.expert_token(ex, 3, x, want_h=True)
    g, sg = synth.expert_matrix(sh, 0, 3, synth.GATE)
    u, su = synth.expert_matrix(sh, 0, 3, synth.UP)
    d, sd = synth.expert_matrix(sh, 0, 3, synth.DOWN)
    assert sg.shape == (sh.I, sh.H // group) and sd.shape == (sh.H, sh.I // group)
    Wg = unpack_ref(g, qtype) * np.repeat(sg.astype(np.float64), group, axis=1)
    Wu = unpack_ref(u, qtype) * np.repeat(su.astype(np.float64), group, axis=1)
    Wd = unpack_ref(d, qtype) * np.repeat(sd.astype(np.float64), group, axis=1)
    qa, da = O.q8_0(x)
    xa = qa.astype(np.float64) * np.repeat(da.astype(np.float64), 32)
    gg, uu = Wg @ xa, Wu @ xa
    h64 = gg / (1.0 + np.exp(-gg)) * uu
    assert np.allclose(h, h64, rtol=1e-5, atol=1e-6 * np.abs(h64).max())
    qh, dh = O.q8_0(h.astype(np.float32))
    ha = qh.astype(np.float64) * np.repeat(dh.astype(np.float64), 32)
    y64, mag = Wd @ ha, np.abs(Wd) @ np.abs(ha)
    assert np.all(np.abs(y - y64) <= 1e-5 * mag + 1e-30)


def _round_f32(q):
    """The fp32 value nearest the rational q (ties to even), found exactly."""
    from fractions import Fraction
    c = np.float32(float(q))
    best = None
    for v in (np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf))):
        err = abs(Fraction(float(v)) - q)
        even = (int(np.float32(v).view(np.uint32)) & 1) == 0
        key = (err, not even)
        if best is None or key < best[0]:
            best = (key, v)
    return np.float32(best[1])


def test_qdot_fold_rounds_once_per_block():
    # reading of the quantised dot: each block step is the fp32 value nearest
    # isum_b * d_b + acc (one rounding), blocks ascending, then one rounding of
    # acc * s.  The steps are computed here with exact rationals; the same data
    # folded with two roundings per step (multiply, then add) must differ
    # somewhere, so this pin can tell the two apart.
    from fractions import Fraction
    rng = np.random.default_rng(31)
    n = 1024
    differs = 0
    for _ in range(40):
        codes = rng.integers(-8, 8, n).astype(np.int8)
        x = rng.standard_normal(n).astype(np.float32)
        s = np.float32(rng.uniform(0.01, 0.05))
        qa, da = O.q8_0(x)
        acc = np.float32(0.0)
        acc2 = np.float32(0.0)
        for b in range(n // 32):
            isum = int(np.dot(codes[32 * b:32 * b + 32].astype(np.int64), qa[32 * b:32 * b + 32].astype(np.int64)))
            acc = _round_f32(Fraction(isum) * Fraction(float(da[b])) + Fraction(float(acc)))
            acc2 = np.float32(np.float32(np.float32(isum) * da[b]) + acc2)
        want = _round_f32(Fraction(float(acc)) * Fraction(float(s)))
        got = np.float32(O.qdot(codes, s, qa, da))
        assert got.view(np.uint32) == want.view(np.uint32)
        differs += int(np.float32(acc2 * s).view(np.uint32) != want.view(np.uint32))
    assert differs > 0


# --------------------------------------------------------------- expert
def _expert_fp64(sh, layer, eid, x_f32, h_oracle=None):
    """Dense fp64 reformulation: dequantise everything, multiply, SwiGLU, requantise h."""
    g, sg = synth.expert_matrix(sh, layer, eid, synth.GATE)
    u, su = synth.expert_matrix(sh, layer, eid, synth.UP)
    d, sd = synth.expert_matrix(sh, layer, eid, synth.DOWN)
    Wg = unpack_ref(g, sh.qtype) * sg[:, None].astype(np.float64)
    Wu = unpack_ref(u, sh.qtype) * su[:, None].astype(np.float64)
    Wd = unpack_ref(d, sh.qtype) * sd[:, None].astype(np.float64)
    qa, da = O.q8_0(x_f32)
    xa = qa.astype(np.float64) * np.repeat(da.astype(np.float64), 32)
    gg, uu = Wg @ xa, Wu @ xa
    h = gg / (1.0 + np.exp(-gg)) * uu
    hq_src = h if h_oracle is None else h_oracle
    qh, dh = O.q8_0(hq_src.astype(np.float32))
    ha = qh.astype(np.float64) * np.repeat(dh.astype(np.float64), 32)
    return Wd @ ha, h, np.abs(Wd) @ np.abs(ha)


def test_expert_h_is_fp64_silu_rounded_once_times_u():
    # reading of SwiGLU: silu(g) = g / (1 + e^-g) evaluated in fp64 and rounded
    # once to fp32, then times u in fp32.  Here silu is computed to 40 digits
    # (decimal), rounded to fp64 and then to fp32; g and u come from the pinned
    # quantised dot.  The expert's h must match for every row.
    from decimal import Decimal, getcontext
    getcontext().prec = 40
    sh = synth.CONFIGS["tiny"]
    for eid in (0, 5, 11):
        ex = oracle_experts(sh, [eid])
        x = synth.hidden_states(sh, tokens=[eid])[0]
        xf = synth.bf16_to_f32(x).astype(np.float32)
        _, h = O.expert_token(ex, eid, xf, want_h=True)
        g_pk, sg = synth.expert_matrix(sh, 0, eid, synth.GATE)
        u_pk, su = synth.expert_matrix(sh, 0, eid, synth.UP)
        qa, da = O.q8_0(xf)
        for r in range(sh.I):  # packed rows [I, row bytes]
            g = np.float32(O.qdot(O.unpack(g_pk[r], sh.qtype, sh.H), sg[r], qa, da))
            u = np.float32(O.qdot(O.unpack(u_pk[r], sh.qtype, sh.H), su[r], qa, da))
            gd = Decimal(float(g))
            silu = gd / (1 + (-gd).exp())
            want = np.float32(np.float32(float(silu)) * u)
            assert np.float32(h[r]).view(np.uint32) == want.view(np.uint32), (eid, r)


@pytest.mark.parametrize("qtype", [4, 8, 2])
def test_expert_against_fp64_dense(qtype):
    sh = synth.CONFIGS["tiny"].with_(qtype=qtype, H=512, I=256)
    x = synth.bf16_to_f32(synth.hidden_states(sh)[0])
    ex = oracle_experts(sh, [3])
    y, h = O.expert_token(ex, 3, x, want_h=True)
    y64, h64, mag = _expert_fp64(sh, 0, 3, x, h_oracle=h)
    assert np.allclose(h, h64, rtol=1e-5, atol=1e-6 * np.abs(h64).max())
    assert np.all(np.abs(y - y64) <= 1e-5 * mag + 1e-30)
    assert np.all(np.sign(y[np.abs(y64) > 1e-3 * mag]) == np.sign(y64[np.abs(y64) > 1e-3 * mag]))


def test_expert_zero_gate_gives_zero_output():
    sh = synth.CONFIGS["tiny"]
    ex = oracle_experts(sh, [0])
    ex.gate[0] = np.full_like(ex.gate[0], 0x88)  # every int4 code 0 -> g = 0 -> silu(0) = 0
    x = synth.bf16_to_f32(synth.hidden_states(sh)[1])
    y, h = O.expert_token(ex, 0, x, want_h=True)
    assert np.all(h == 0.0) and np.all(y == 0.0)


# ------------------------------------------------------ union == per-token
@pytest.mark.parametrize("cfg", ["tiny", "verify_small", "tiny_grouped", "tiny_topp"])
def test_union_path_equals_per_token_path_bitwise(cfg):
    top_p = 0.0
    if cfg == "tiny":
        sh = synth.CONFIGS["tiny"]
    elif cfg == "tiny_grouped":
        sh = synth.CONFIGS["tiny"].with_(group_size=64)
    elif cfg == "tiny_topp":
        sh, top_p = synth.CONFIGS["tiny"].with_(T=12, top_k=4), 0.6
    else:
        sh = synth.CONFIGS["verify"].with_(H=512, I=256, E=32, n_group=4, topk_group=2, top_k=4, T=6)
    x, W, b = synth.hidden_states(sh), synth.router_weight(sh), synth.router_bias(sh)
    idx, w, _, _ = O.route(x, W, b, sh.n_group, sh.topk_group, sh.top_k, sh.rsf, top_p=top_p)
    ex = oracle_experts(sh, np.unique(idx[idx >= 0]))
    un = O.union(idx, sh.E)
    y_union = O.expert_ffn(ex, x, sh.top_k, un)
    y_tok = O.expert_ffn_per_token(ex, x, idx)
    assert np.array_equal(y_union.view(np.uint32), y_tok.view(np.uint32))


# ---------------------------------------------------------------- combine
def test_combine_k1_and_fp64():
    rng = np.random.default_rng(40)
    T, H = 5, 64
    y = rng.standard_normal((T, 1, H)).astype(np.float32)
    sh_y = rng.standard_normal((T, H)).astype(np.float32)
    # K = 1: the renormalised weight is s/s * rsf = rsf exactly
    idx, w, _, _ = O.select(rng.standard_normal((T, 8)).astype(np.float32), np.zeros(8, np.float32), 4, 1, 1, 2.5)
    assert np.all(w == 2.5)
    of, ob = O.combine(y, w, sh_y)
    assert np.array_equal(of, sh_y + np.float32(2.5) * y[:, 0])
    # zero shared output isolates the routed terms; general K against fp64
    K = 8
    y = rng.standard_normal((T, K, H)).astype(np.float32)
    w = rng.uniform(0.1, 0.5, (T, K)).astype(np.float32)
    of, ob = O.combine(y, w, None)
    ref = np.einsum("tk,tkh->th", w.astype(np.float64), y.astype(np.float64))
    assert np.allclose(of, ref, rtol=1e-5, atol=1e-6)
    assert np.array_equal(ob, synth.bf16_bits(of))


# ---------------------------------------------------------------- layer
def test_layer_forward_against_fp64_composition():
    sh = synth.CONFIGS["tiny"]
    x, W, b = synth.hidden_states(sh), synth.router_weight(sh), synth.router_bias(sh)
    routed = oracle_experts(sh, range(sh.E))
    shared = oracle_experts(sh, [0], shared=True)
    of, ob, idx, w = O.layer_forward(x, W, b, sh.n_group, sh.topk_group, sh.top_k, sh.rsf, routed, shared)
    assert np.array_equal(idx, _brute_select(
        (synth.bf16_to_f32(x).astype(np.float64) @ W.T.astype(np.float64)).astype(np.float32), b,
        sh.n_group, sh.topk_group, sh.top_k))
    xf = synth.bf16_to_f32(x)
    ref = np.zeros((sh.T, sh.H))
    for t in range(sh.T):
        ref[t] = _expert_fp64(sh, 0, synth.SHARED, xf[t])[0]
        for k in range(sh.top_k):
            ref[t] += float(w[t, k]) * _expert_fp64(sh, 0, int(idx[t, k]), xf[t])[0]
    assert rel_err_rows(of, ref) < 2e-3
    assert np.array_equal(ob, synth.bf16_bits(of))


# ------------------------------------------------------------------ sizes
def test_page_size_figures():
    rows = {}
    with open(os.path.join(GOLDEN, "page_sizes.txt")) as fh:
        for line in fh:
            if line.strip() and not line.startswith("#"):
                k, v, tol = [s.strip() for s in line.split("|")]
                rows[k] = (float(v), float(tol))
    sh = synth.CONFIGS["decode"]
    per = sh.expert_bytes()
    assert per == 18_915_328
    assert sh.E == rows["experts_per_layer"][0] and sh.top_k == rows["top_k"][0]
    layers = rows["moe_layers"][0]
    total = rows["experts_total"][0]
    assert layers * sh.E + sh.E == total  # 75 MoE layers plus the MTP layer's 256
    for key, val in [("int4_expert_bytes", per), ("routed_bytes_per_token", layers * sh.top_k * per),
                     ("total_routed_bytes", total * per)]:
        want, tol = rows[key]
        assert abs(val - want) <= tol * want, key
