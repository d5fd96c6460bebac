"""Calibrate the Zipf strength of the prefill workload's router bias (oracle only).

The prefill workload skews expert popularity through the noaux_tc correction
bias: bias_e = N(0, 0.1^2) + alpha * ln(p_e / p_max), p_e proportional to
rank_e^-1.1 over a seeded permutation.  This script routes the workload's
2048 tokens with the CPU oracle for a grid of alpha values and reports the
log-log slope of the realised per-expert token counts against their rank, so
that alpha can be fixed where the slope is near -1.1.  It calls only the
oracle and the input generator.

usage: python -m oracle.calibrate_zipf [alpha ...]
"""
from __future__ import annotations

import sys

import numpy as np

import synth
from oracle import oracle as O


def slope(counts: np.ndarray, top: int = 128) -> float:
    c = np.sort(counts)[::-1][:top].astype(np.float64)
    c = c[c > 0]
    r = np.arange(1, c.size + 1, dtype=np.float64)
    return float(np.polyfit(np.log(r), np.log(c), 1)[0])


def main(alphas):
    sh = synth.CONFIGS["prefill"]
    x = synth.hidden_states(sh)
    W = synth.router_weight(sh)
    logits = O.router_logits(x, W)
    for a in alphas:
        b = synth.router_bias(sh.with_(zipf_alpha=a))
        idx, _, ge, gg = O.select(logits, b, sh.n_group, sh.topk_group, sh.top_k, sh.rsf)
        counts = np.bincount(idx.reshape(-1), minlength=sh.E)
        srt = np.sort(counts)[::-1]
        print(f"alpha={a:.4f} slope(top128)={slope(counts):+.3f} slope(top64)={slope(counts, 64):+.3f} "
              f"unique={int((counts > 0).sum())} >=64 tokens: {int((counts >= 64).sum())} "
              f"top10={srt[:10].tolist()} rank64={int(srt[63])} rank128={int(srt[127])} "
              f"min_gap_expert={float(ge.min()):.3g} min_gap_group={float(gg.min()):.3g}")


if __name__ == "__main__":
    main([float(a) for a in sys.argv[1:]] or [0.0, 0.02, 0.04, 0.06, 0.08, 0.1, 0.12, 0.15])
