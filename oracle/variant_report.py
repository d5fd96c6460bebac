"""How much the layer output depends on roundings the pages leave open -- TEST INFRASTRUCTURE.

The pages fix neither how silu is evaluated nor in which order the per-block
integer dots are folded into fp32.  The oracle takes one reading of each
(silu in fp64 rounded once; one fused multiply-add per block, ascending);
moe_oracle.c's compile-time switches build the three other combinations:

  ""              default: fp64 silu, fma fold
  "silu32"        silu = g / (1 + expf(-g)) in fp32
  "muladd"        fold acc = acc + isum * d (two roundings)
  "silu32_muladd" both

For seeded inputs of the measured workloads this script routes every token
with the default oracle (routing uses neither rounding), evaluates every
(token, expert) pair under all four variants and reports, against the
default: h elements that differ, Q8_0(h) codes that flip, and the layer
output's difference under the parity metric
max_i |g_i - r_i| / max(|r_i|, rms(row of r)).

Run:  python -m oracle.variant_report [--out oracle/variant_report.md]
      [--decode-tokens 64] [--verify-batches 8]
It calls only oracle/ (for every value) and synth/ (for the inputs).
"""
from __future__ import annotations

import argparse
import os
import sys
import time
from collections import defaultdict

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402
from oracle import oracle as O  # noqa: E402
from oracle.synth_inputs import oracle_experts  # noqa: E402

VARIANTS = ("", "silu32", "muladd", "silu32_muladd")


def _experts(sh, ids, shared=False):
    return oracle_experts(sh, ids, shared=shared)


def layer_outputs(sh, batches, variant: str = ""):
    """Oracle layer outputs of each batch (a list of token ids, one layer call
    each): [(x_bits, idx, w, out_f32)], with each touched expert generated once
    and evaluated for all its tokens (so no more than one expert is held)."""
    W, b = synth.router_weight(sh), synth.router_bias(sh)
    xbits, xs, routes = [], [], []
    for tok in batches:
        x = synth.hidden_states(sh, tokens=tok)
        idx, w, _, _ = O.route(x, W, b, sh.n_group, sh.topk_group, sh.top_k, sh.rsf)
        xbits.append(x)
        xs.append(synth.bf16_to_f32(x).astype(np.float32))
        routes.append((idx, w))
    by_expert = defaultdict(list)
    for bi, (idx, _) in enumerate(routes):
        for t in range(idx.shape[0]):
            for k in range(idx.shape[1]):
                by_expert[int(idx[t, k])].append((bi, t, k))
    y = {}
    units = [(e, by_expert[e]) for e in sorted(by_expert)]
    units.append((-1, [(bi, t, -1) for bi, x in enumerate(xs) for t in range(x.shape[0])]))
    for e, uses in units:
        ex = _experts(sh, [0], shared=True) if e < 0 else _experts(sh, [e])
        for bi, t, k in uses:
            y[(bi, t, k)] = O.expert_token(ex, 0 if e < 0 else e, xs[bi][t], variant=variant)
    out = []
    for bi, (idx, w) in enumerate(routes):
        T, K = idx.shape
        yp = np.stack([np.stack([y[(bi, t, k)] for k in range(K)]) for t in range(T)])
        ys = np.stack([y[(bi, t, -1)] for t in range(T)])
        of, _ = O.combine(yp, w, ys)
        out.append((xbits[bi], idx, w, of))
    return out


def rel_metric(got, ref):
    got = np.asarray(got, np.float64).reshape(-1, ref.shape[-1])
    ref = np.asarray(ref, np.float64).reshape(-1, ref.shape[-1])
    rms = np.sqrt(np.mean(ref * ref, axis=1, keepdims=True))
    den = np.maximum(np.abs(ref), np.maximum(rms, 1e-30))
    return np.max(np.abs(got - ref) / den, axis=1)  # per row (token)


def evaluate(sh, batches, variants=VARIANTS):
    """batches: lists of token ids, each one layer call of len(batch) positions."""
    W, b = synth.router_weight(sh), synth.router_bias(sh)
    xs, routes = [], []
    for tok in batches:
        x = synth.hidden_states(sh, tokens=tok)
        idx, w, _, _ = O.route(x, W, b, sh.n_group, sh.topk_group, sh.top_k, sh.rsf)
        xs.append(synth.bf16_to_f32(x).astype(np.float32))
        routes.append((idx, w))
    by_expert = defaultdict(list)  # expert -> [(batch, t, k)]
    for bi, (idx, _) in enumerate(routes):
        for t in range(idx.shape[0]):
            for k in range(idx.shape[1]):
                by_expert[int(idx[t, k])].append((bi, t, k))
    # results[v][(bi, t, k)] = (y, h); k = -1 is the shared expert
    res = {v: {} for v in variants}
    units = [(e, by_expert[e]) for e in sorted(by_expert)]
    units.append((-1, [(bi, t, -1) for bi, x in enumerate(xs) for t in range(x.shape[0])]))
    for e, uses in units:
        ex = _experts(sh, [0], shared=True) if e < 0 else _experts(sh, [e])
        eid = 0 if e < 0 else e
        for v in variants:
            for bi, t, k in uses:
                res[v][(bi, t, k)] = O.expert_token(ex, eid, xs[bi][t], want_h=True, variant=v)
    stats = {}
    base = res[""]
    for v in variants:
        if v == "":
            continue
        h_diff = flips = max_code = 0
        n_h = 0
        per_token = []
        for key, (y0, h0) in base.items():
            y1, h1 = res[v][key]
            n_h += h0.size
            h_diff += int(np.count_nonzero(h0.view(np.uint32) != h1.view(np.uint32)))
            q0, _ = O.q8_0(h0)
            q1, _ = O.q8_0(h1)
            dq = np.abs(q0.astype(np.int16) - q1.astype(np.int16))
            flips += int(np.count_nonzero(dq))
            max_code = max(max_code, int(dq.max()) if dq.size else 0)
        for bi, (idx, w) in enumerate(routes):
            T, K = idx.shape
            outs = []
            for var in ("", v):
                yp = np.stack([np.stack([res[var][(bi, t, k)][0] for k in range(K)]) for t in range(T)])
                ys = np.stack([res[var][(bi, t, -1)][0] for t in range(T)])
                of, _ = O.combine(yp, w, ys)
                outs.append(of)
            per_token.extend(rel_metric(outs[1], outs[0]).tolist())
        per_token = np.array(per_token)
        stats[v] = dict(h_elements=n_h, h_diff=h_diff, flips=flips, max_code_step=max_code,
                        tokens=per_token.size, max_rel=float(per_token.max()),
                        tokens_over_2e3=int(np.count_nonzero(per_token > 2e-3)),
                        median_rel=float(np.median(per_token)))
    n_pairs = sum(len(u) for _, u in units)
    return stats, n_pairs


def workloads(decode_tokens, verify_batches):
    C = synth.CONFIGS
    yield "tiny (T=4, 4 calls)", C["tiny"], [list(range(4 * i, 4 * i + 4)) for i in range(4)]
    yield (f"decode (T=1, {decode_tokens} calls)", C["decode"],
           [[t] for t in range(decode_tokens)])
    yield (f"verify int4 (T=4, {verify_batches} calls)", C["verify"],
           [list(range(4 * i, 4 * i + 4)) for i in range(verify_batches)])
    yield (f"verify int8 (T=4, {verify_batches} calls)", C["verify_int8"],
           [list(range(4 * i, 4 * i + 4)) for i in range(verify_batches)])


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--out", default=None)
    ap.add_argument("--decode-tokens", type=int, default=64)
    ap.add_argument("--verify-batches", type=int, default=8)
    a = ap.parse_args()
    lines = ["# Oracle rounding variants against the default oracle", "",
             "Generated by `python -m oracle.variant_report` (oracle/ and synth/ only; seed 0).",
             "Per variant: h elements that differ bitwise from the default oracle's, Q8_0(h) codes",
             "that flip, the largest code step, and the layer output's difference from the default",
             "under the parity metric max_i |g_i - r_i| / max(|r_i|, rms(row)), per token.", "",
             "| workload | (token, expert) pairs | variant | h differing | Q8_0(h) flips | max step "
             "| median rel | max rel | tokens > 2e-3 |",
             "|---|---|---|---|---|---|---|---|---|"]
    t0 = time.time()
    for name, sh, batches in workloads(a.decode_tokens, a.verify_batches):
        stats, n_pairs = evaluate(sh, batches)
        for v, st in stats.items():
            lines.append(f"| {name} | {n_pairs} | {v} | {st['h_diff']} of {st['h_elements']} | "
                         f"{st['flips']} | {st['max_code_step']} | {st['median_rel']:.2e} | "
                         f"{st['max_rel']:.2e} | {st['tokens_over_2e3']} of {st['tokens']} |")
        print(lines[-3:], flush=True)
    lines += ["", f"({time.time() - t0:.0f} s on {os.cpu_count()} host cores)"]
    text = "\n".join(lines) + "\n"
    if a.out:
        with open(a.out, "w") as fh:
            fh.write(text)
    print(text)


if __name__ == "__main__":
    main()
