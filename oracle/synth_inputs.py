"""Oracle expert sets built from the seeded generator -- TEST INFRASTRUCTURE ONLY.

Marshalling only: regenerates the listed experts' packed codes and scales with
synth (which holds no arithmetic of the layer) and hands them to the oracle's
host expert table.  Used by the tests, the variant report and the benchmark's
CPU-baseline leg.
"""
from __future__ import annotations

import synth
from oracle import oracle as O


def oracle_experts(sh: synth.LayerShape, experts, layer: int = 0, shared: bool = False) -> O.Experts:
    """Oracle expert set holding only the listed experts (regenerated from the seed)."""
    ex = O.Experts(sh.qtype, sh.H, sh.I, 1 if shared else sh.E, group=sh.group_size)
    for e in experts:
        sid = synth.SHARED if shared else int(e)
        g, sg = synth.expert_matrix(sh, layer, sid, synth.GATE)
        u, su = synth.expert_matrix(sh, layer, sid, synth.UP)
        d, sd = synth.expert_matrix(sh, layer, sid, synth.DOWN)
        ex.set(0 if shared else int(e), g, sg, u, su, d, sd)
    return ex
