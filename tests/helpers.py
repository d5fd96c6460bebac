"""Test-side glue: synthetic inputs -> oracle structures, and the parity tolerance.

Test infrastructure only (may use the oracle).
"""
from __future__ import annotations

import numpy as np

import synth
from oracle import oracle as O  # noqa: F401
from oracle.synth_inputs import oracle_experts  # noqa: F401


def layer_inputs(sh: synth.LayerShape, layer: int = 0, tokens=None):
    return (synth.hidden_states(sh, layer, tokens), synth.router_weight(sh, layer),
            synth.router_bias(sh, layer))


def rel_err_rows(got: np.ndarray, ref: np.ndarray) -> float:
    """max_i |g_i - r_i| / max(|r_i|, rms(r_row)): the output check of the parity bar.

    The per-row rms floor keeps near-zero outputs from dominating a relative error.
    """
    got = np.asarray(got, dtype=np.float64).reshape(-1, ref.shape[-1])
    ref = np.asarray(ref, dtype=np.float64).reshape(-1, ref.shape[-1])
    rms = np.sqrt(np.mean(ref * ref, axis=1, keepdims=True))
    den = np.maximum(np.abs(ref), np.maximum(rms, 1e-30))
    return float(np.max(np.abs(got - ref) / den)) if got.size else 0.0


def bf16_ulps(got_bits: np.ndarray, ref_f32: np.ndarray) -> int:
    """Largest distance, in bf16 ulps, between a bf16 output and RNE(reference)."""
    ref_bits = synth.bf16_bits(np.asarray(ref_f32, dtype=np.float32))

    def ordered(b):
        b = b.astype(np.int64)
        return np.where(b & 0x8000, -(b & 0x7FFF), b)

    if got_bits.size == 0:
        return 0
    return int(np.max(np.abs(ordered(got_bits.reshape(-1)) - ordered(ref_bits.reshape(-1)))))


def unpack_ref(packed_rows: np.ndarray, qtype: int) -> np.ndarray:
    """numpy unpacking used by the fp64 dense reference (independent of the oracle's C)."""
    p = packed_rows.astype(np.int16)
    if qtype == 4:
        lo = (p & 0x0F) - 8
        hi = (p >> 4) - 8
        return np.stack([lo, hi], axis=-1).reshape(p.shape[0], -1)
    if qtype == 2:
        parts = [((p >> (2 * m)) & 3) - 2 for m in range(4)]
        return np.stack(parts, axis=-1).reshape(p.shape[0], -1)
    return packed_rows.view(np.int8).astype(np.int16)
