"""Seeded synthetic inputs for the routed-MoE layer (test/bench infrastructure).

Every value comes from a counter hash (splitmix64 mixer, see synth_host.c),
keyed by (seed, stream id, counter), so any expert of any layer can be
regenerated on its own, on the host (C, for the oracle) or on the device
(CUDA twin, for multi-GB resident weight sets).  Normals are drawn on the host
only (Box-Muller in float64) and copied, so no transcendental function is
evaluated on the device.

Input recipe (shapes from the GLM-5.2 layer: H=6144, I=2048, E=256 routed
experts in 8 groups, top-8, one shared expert):
  * expert weights: packed int4 / int2 codes are uniform random bytes (every
    nibble / 2-bit field of a uniform byte is uniform over its code range,
    [-8,7] / [-2,1] after the offset); int8 codes are uniform on [-127,127];
  * per-row scales: U(0.01, 0.05) in fp32 (grouped scales, group_size != 0: one
    per row and group, the same stream read at index row * groups + group);
  * router weight: fp32 N(0, 0.02^2); correction bias: fp32 N(0, 0.1^2),
    plus, for the Zipf-skewed prefill workload, alpha * ln(p_e / p_max) with
    p_e proportional to rank_e^-s over a seeded permutation of the experts;
  * hidden states: bf16 (round-to-nearest-even of fp32) N(0,1); the MTP-verify
    workload adds a shared N(0,1) component to per-position N(0, 0.5^2) noise.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, replace

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
BUILD = os.path.join(HERE, "_build")
HOST_SO = os.path.join(BUILD, "libsynth_host.so")
GPU_SO = os.path.join(BUILD, "libsynth_gpu.so")

# ----------------------------------------------------------------- streams
SHARED = 0xFFF  # expert id used for the shared expert's streams
GATE, UP, DOWN = 0, 1, 2
_CODES = {GATE: 0x01, UP: 0x02, DOWN: 0x03}
_SCALES = {GATE: 0x11, UP: 0x12, DOWN: 0x13}
W_ROUTER, W_BIAS, W_ZIPF, W_X, W_XC = 0x21, 0x22, 0x23, 0x31, 0x32


def stream_id(layer: int, expert: int, what: int, qtype: int = 0) -> int:
    return (int(layer) << 32) | (int(expert) << 16) | (int(qtype) << 8) | int(what)


# ----------------------------------------------------------------- shapes
@dataclass(frozen=True)
class LayerShape:
    name: str
    T: int
    H: int
    I: int
    E: int
    n_group: int
    topk_group: int
    top_k: int
    qtype: int = 4
    rsf: float = 2.5
    n_layers: int = 1
    x_mode: str = "iid"  # "iid" or "correlated" (MTP verify)
    zipf_s: float = 0.0  # popularity exponent realised through the bias (0: none)
    zipf_alpha: float = 0.0
    seed: int = 0
    group_size: int = 0  # 0: one weight scale per row; else one per row and group of this many codes

    def row_bytes(self, matrix: int) -> int:
        k = self.H if matrix in (GATE, UP) else self.I
        return k * self.qtype // 8

    def rows(self, matrix: int) -> int:
        return self.I if matrix in (GATE, UP) else self.H

    def matrix_bytes(self, matrix: int) -> int:
        return self.rows(matrix) * self.row_bytes(matrix)

    def scales_per_row(self, matrix: int) -> int:
        k = self.H if matrix in (GATE, UP) else self.I
        return k // self.group_size if self.group_size else 1

    def expert_bytes(self) -> int:
        """Packed codes plus fp32 scales of one expert (gate, up, down)."""
        return sum(self.matrix_bytes(m) + 4 * self.rows(m) * self.scales_per_row(m) for m in (GATE, UP, DOWN))

    def router_bytes(self) -> int:
        return 4 * self.E * self.H

    def with_(self, **kw) -> "LayerShape":
        return replace(self, **kw)


GLM = dict(H=6144, I=2048, E=256, n_group=8, topk_group=4, top_k=8, rsf=2.5)

# Zipf calibration for the prefill workload: alpha fixed once at seed 0 so that
# the realised per-expert token counts of the 128 most popular experts have a
# log-log slope against rank of -1.10 (oracle/calibrate_zipf.py prints the
# sweep).  At alpha = 0.074: 164 distinct experts, 73 of them with >= 64
# tokens, most popular counts 735, 627, 608, 528, ...
PREFILL_ZIPF_ALPHA = 0.074

CONFIGS = {
    "tiny": LayerShape("tiny", T=4, H=256, I=128, E=16, n_group=4, topk_group=2, top_k=2),
    "decode": LayerShape("decode", T=1, **GLM),
    "verify": LayerShape("verify", T=4, x_mode="correlated", **GLM),
    "verify_int8": LayerShape("verify_int8", T=4, x_mode="correlated", qtype=8, **GLM),
    "prefill": LayerShape("prefill", T=2048, zipf_s=1.1, zipf_alpha=PREFILL_ZIPF_ALPHA, **GLM),
    "stacked": LayerShape("stacked", T=1, n_layers=16, **GLM),
    "stacked_t8": LayerShape("stacked_t8", T=8, n_layers=16, **GLM),
    "stacked_int2": LayerShape("stacked_int2", T=1, n_layers=16, qtype=2, **GLM),
}


# ----------------------------------------------------------------- builds
def _newer(target: str, *sources: str) -> bool:
    return os.path.exists(target) and all(
        os.path.getmtime(target) >= os.path.getmtime(s) for s in sources)


def build_host(force: bool = False) -> str:
    src = os.path.join(HERE, "synth_host.c")
    if force or not _newer(HOST_SO, src):
        os.makedirs(BUILD, exist_ok=True)
        tmp = f"{HOST_SO}.{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", src, "-o", tmp])
        os.replace(tmp, HOST_SO)
    return HOST_SO


def build_gpu(force: bool = False) -> str:
    src = os.path.join(HERE, "synth_gpu.cu")
    if force or not _newer(GPU_SO, src):
        os.makedirs(BUILD, exist_ok=True)
        tmp = f"{GPU_SO}.{os.getpid()}.tmp"
        subprocess.check_call([
            "nvcc", "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
            "-Xcompiler", "-fPIC", "-shared", src, "-o", tmp])
        os.replace(tmp, GPU_SO)
    return GPU_SO


_host_lib = None
_gpu_lib = None


def _host() -> ctypes.CDLL:
    global _host_lib
    if _host_lib is None:
        lib = ctypes.CDLL(build_host())
        u64, sz, vp = ctypes.c_uint64, ctypes.c_size_t, ctypes.c_void_p
        lib.synth_words.argtypes = [u64, u64, u64, sz, vp]
        lib.synth_bytes.argtypes = [u64, u64, u64, sz, vp]
        lib.synth_codes_i8.argtypes = [u64, u64, u64, sz, vp]
        lib.synth_scales.argtypes = [u64, u64, u64, sz, ctypes.c_float, ctypes.c_float, vp]
        lib.synth_key.argtypes = [u64, u64]
        lib.synth_key.restype = u64
        _host_lib = lib
    return _host_lib


def _gpu() -> ctypes.CDLL:
    global _gpu_lib
    if _gpu_lib is None:
        lib = ctypes.CDLL(build_gpu())
        u64, sz, vp = ctypes.c_uint64, ctypes.c_size_t, ctypes.c_void_p
        lib.synth_gpu_bytes.argtypes = [u64, u64, u64, sz, vp, vp]
        lib.synth_gpu_codes_i8.argtypes = [u64, u64, u64, sz, vp, vp]
        lib.synth_gpu_scales.argtypes = [u64, u64, u64, sz, ctypes.c_float, ctypes.c_float, vp, vp]
        _gpu_lib = lib
    return _gpu_lib


# ----------------------------------------------------------------- host draws
def words(seed: int, stream: int, start: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    _host().synth_words(seed, stream, start, n, out.ctypes.data)
    return out


def uniform_bytes(seed: int, stream: int, start: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint8)
    _host().synth_bytes(seed, stream, start, n, out.ctypes.data)
    return out


def codes_i8(seed: int, stream: int, start: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int8)
    _host().synth_codes_i8(seed, stream, start, n, out.ctypes.data)
    return out


SCALE_LO, SCALE_SPAN = 0.01, 0.04


def scales(seed: int, stream: int, start: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    _host().synth_scales(seed, stream, start, n, SCALE_LO, SCALE_SPAN, out.ctypes.data)
    return out


def normals(seed: int, stream: int, start: int, n: int) -> np.ndarray:
    """n standard normals; normal j uses words 2j and 2j+1 (Box-Muller, float64)."""
    w = words(seed, stream, 2 * start, 2 * n)
    u1 = ((w[0::2] >> np.uint64(11)).astype(np.float64) + 1.0) * 2.0 ** -53  # (0, 1]
    u2 = (w[1::2] >> np.uint64(11)).astype(np.float64) * 2.0 ** -53  # [0, 1)
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16, returned as uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------- layer inputs
def router_weight(sh: LayerShape, layer: int = 0) -> np.ndarray:
    z = normals(sh.seed, stream_id(layer, 0, W_ROUTER), 0, sh.E * sh.H)
    return (0.02 * z).astype(np.float32).reshape(sh.E, sh.H)


def zipf_ranks(sh: LayerShape, layer: int = 0) -> np.ndarray:
    """rank (1-based) of each expert under a seeded permutation."""
    keys = words(sh.seed, stream_id(layer, 0, W_ZIPF), 0, sh.E)
    order = np.argsort(keys, kind="stable")
    rank = np.empty(sh.E, dtype=np.int64)
    rank[order] = np.arange(1, sh.E + 1)
    return rank


def router_bias(sh: LayerShape, layer: int = 0) -> np.ndarray:
    b = 0.1 * normals(sh.seed, stream_id(layer, 0, W_BIAS), 0, sh.E)
    if sh.zipf_s > 0.0:
        b = b + sh.zipf_alpha * (-sh.zipf_s * np.log(zipf_ranks(sh, layer).astype(np.float64)))
    return b.astype(np.float32)


def hidden_states(sh: LayerShape, layer: int = 0, tokens=None) -> np.ndarray:
    """bf16 bit patterns [len(tokens), H]; token t's row does not depend on T."""
    tokens = np.arange(sh.T) if tokens is None else np.asarray(tokens)
    rows = []
    c = None
    if sh.x_mode == "correlated":
        c = normals(sh.seed, stream_id(layer, 0, W_XC), 0, sh.H)
    for t in tokens:
        z = normals(sh.seed, stream_id(layer, 0, W_X), int(t) * sh.H, sh.H)
        if c is not None:
            z = c + 0.5 * z
        rows.append(z)
    if not rows:
        return np.zeros((0, sh.H), dtype=np.uint16)
    return bf16_bits(np.stack(rows).astype(np.float32))


def expert_matrix(sh: LayerShape, layer: int, expert: int, matrix: int):
    """(packed codes uint8 [rows, row_bytes], scales fp32 [rows] or, grouped, [rows, groups]) of one matrix.

    expert == SHARED selects the shared expert.
    """
    rows, rb = sh.rows(matrix), sh.row_bytes(matrix)
    sid = stream_id(layer, expert, _CODES[matrix], sh.qtype)
    if sh.qtype == 8:
        codes = codes_i8(sh.seed, sid, 0, rows * rb).view(np.uint8)
    else:
        codes = uniform_bytes(sh.seed, sid, 0, rows * rb)
    spr = sh.scales_per_row(matrix)
    sc = scales(sh.seed, stream_id(layer, expert, _SCALES[matrix], sh.qtype), 0, rows * spr)
    return codes.reshape(rows, rb), (sc.reshape(rows, spr) if sh.group_size else sc)


def fill_matrix_gpu(sh: LayerShape, layer: int, expert: int, matrix: int,
                    codes_ptr: int, scales_ptr: int, cuda_stream: int = 0) -> None:
    """Device twin of expert_matrix: writes the same codes and scales to device memory."""
    lib = _gpu()
    rows, rb = sh.rows(matrix), sh.row_bytes(matrix)
    sid = stream_id(layer, expert, _CODES[matrix], sh.qtype)
    if sh.qtype == 8:
        rc = lib.synth_gpu_codes_i8(sh.seed, sid, 0, rows * rb, codes_ptr, cuda_stream)
    else:
        rc = lib.synth_gpu_bytes(sh.seed, sid, 0, rows * rb, codes_ptr, cuda_stream)
    if rc != 0:
        raise RuntimeError(f"synth_gpu codes launch failed: cudaError {rc}")
    rc = lib.synth_gpu_scales(sh.seed, stream_id(layer, expert, _SCALES[matrix], sh.qtype), 0,
                              rows * sh.scales_per_row(matrix), SCALE_LO, SCALE_SPAN, scales_ptr, cuda_stream)
    if rc != 0:
        raise RuntimeError(f"synth_gpu scales launch failed: cudaError {rc}")
