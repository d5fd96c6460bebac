"""Python marshalling for the CPU oracle (liboracle.so) -- TEST INFRASTRUCTURE ONLY.

Only tests/, the package smoke check and bench.py's CPU-baseline leg may
import this module.  The GPU library never loads it.  This file contains no
arithmetic of the layer: it builds the C library, converts numpy arrays into
pointers and calls the C functions of moe_oracle.c.  The one exception is the
expert-usage record at the end: two plain definitions (count the routed
entries per expert; order the experts by count), written in Python because
they involve no floating point.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
BUILD = os.path.join(HERE, "_build")
SO = os.path.join(BUILD, "liboracle.so")
SRC = os.path.join(HERE, "moe_oracle.c")
HDR = os.path.join(HERE, "moe_oracle.h")


# Rounding variants of the oracle (compile-time switches of moe_oracle.c), used
# only to measure how much the output depends on roundings the pages leave
# open.  The default oracle is variant "".
VARIANTS = {
    "": [],
    "silu32": ["-DORACLE_SILU_F32"],
    "muladd": ["-DORACLE_FOLD_MULADD"],
    "silu32_muladd": ["-DORACLE_SILU_F32", "-DORACLE_FOLD_MULADD"],
}


def so_path(variant: str = "") -> str:
    return SO if not variant else os.path.join(BUILD, f"liboracle_{variant}.so")


def build(force: bool = False, variant: str = "") -> str:
    so = so_path(variant)
    fresh = os.path.exists(so) and all(
        os.path.getmtime(so) >= os.path.getmtime(s) for s in (SRC, HDR))
    if force or not fresh:
        os.makedirs(BUILD, exist_ok=True)
        tmp = f"{so}.{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math",
                               "-fopenmp", "-fPIC", "-shared", *VARIANTS[variant], SRC, "-o", tmp,
                               "-lm"])
        os.replace(tmp, so)
    return so


class _Experts(ctypes.Structure):
    _fields_ = [("qtype", ctypes.c_int), ("n_expert", ctypes.c_int), ("H", ctypes.c_int),
                ("I", ctypes.c_int), ("w_gate", ctypes.c_void_p), ("w_up", ctypes.c_void_p),
                ("w_down", ctypes.c_void_p), ("s_gate", ctypes.c_void_p),
                ("s_up", ctypes.c_void_p), ("s_down", ctypes.c_void_p), ("group", ctypes.c_int)]


_libs = {}


def lib(variant: str = "") -> ctypes.CDLL:
    if variant not in _libs:
        L = ctypes.CDLL(build(variant=variant))
        vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        L.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_f32.restype = f
        L.oracle_f32_to_bf16.argtypes = [f]
        L.oracle_f32_to_bf16.restype = ctypes.c_uint16
        L.oracle_router_logits.argtypes = [vp, i, i, vp, i, vp]
        L.oracle_router_logits.restype = None
        L.oracle_select.argtypes = [vp, i, vp, i, i, i, i, f, vp, vp, vp, vp]
        L.oracle_select_topp.argtypes = [vp, i, vp, i, i, i, i, f, f, vp, vp, vp, vp]
        L.oracle_route.argtypes = [vp, i, i, vp, vp, i, i, i, i, f, vp, vp, vp, vp]
        L.oracle_route_topp.argtypes = [vp, i, i, vp, vp, i, i, i, i, f, f, vp, vp, vp, vp]
        L.oracle_union.argtypes = [vp, i, i, i, vp, vp, vp, vp, vp, vp]
        L.oracle_q8_0.argtypes = [vp, i, vp, vp]
        L.oracle_q8_0.restype = None
        L.oracle_unpack.argtypes = [vp, i, i, vp]
        L.oracle_qdot.argtypes = [vp, f, vp, vp, i]
        L.oracle_qdot.restype = f
        L.oracle_qdot_grouped.argtypes = [vp, vp, i, vp, vp, i]
        L.oracle_qdot_grouped.restype = f
        L.oracle_expert_token.argtypes = [vp, i, vp, vp, vp]
        L.oracle_expert_ffn.argtypes = [vp, vp, i, i, i, vp, vp, vp, vp, vp]
        L.oracle_expert_ffn_per_token.argtypes = [vp, vp, i, i, vp, vp]
        L.oracle_combine.argtypes = [vp, vp, vp, i, i, i, vp, vp]
        L.oracle_combine.restype = None
        L.oracle_layer_forward.argtypes = [vp, i, vp, vp, i, i, i, i, f, vp, vp, vp, vp, vp, vp]
        L.oracle_layer_forward_topp.argtypes = [vp, i, vp, vp, i, i, i, i, f, f, vp, vp, vp, vp, vp, vp]
        _libs[variant] = L
    return _libs[variant]


def _p(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"{what}: oracle returned {rc}")


class Experts:
    """Host expert set: per-expert arrays (None where not needed).

    gate/up[e]: uint8 [I, H*q/8]; down[e]: uint8 [H, I*q/8];
    s_gate/s_up[e]: fp32 [I]; s_down[e]: fp32 [H]; with grouped scales (group != 0)
    s_gate/s_up[e]: fp32 [I, H/group]; s_down[e]: fp32 [H, I/group].
    """

    def __init__(self, qtype, H, I, n_expert, group=0):
        self.qtype, self.H, self.I, self.n, self.group = qtype, H, I, n_expert, group
        self.gate = [None] * n_expert
        self.up = [None] * n_expert
        self.down = [None] * n_expert
        self.s_gate = [None] * n_expert
        self.s_up = [None] * n_expert
        self.s_down = [None] * n_expert

    def set(self, e, gate, s_gate, up, s_up, down, s_down):
        self.gate[e] = _c(gate, np.uint8)
        self.up[e] = _c(up, np.uint8)
        self.down[e] = _c(down, np.uint8)
        self.s_gate[e] = _c(s_gate, np.float32)
        self.s_up[e] = _c(s_up, np.float32)
        self.s_down[e] = _c(s_down, np.float32)

    def struct(self):
        tabs = []
        for lst in (self.gate, self.up, self.down, self.s_gate, self.s_up, self.s_down):
            arr = (ctypes.c_void_p * self.n)(*[(_p(a) or 0) for a in lst])
            tabs.append(arr)
        self._tabs = tabs  # keep alive
        s = _Experts(self.qtype, self.n, self.H, self.I,
                     *[ctypes.cast(t, ctypes.c_void_p) for t in tabs], self.group)
        self._struct = s
        return s


def bf16_to_f32(v: int) -> float:
    return lib().oracle_bf16_to_f32(int(v))


def f32_to_bf16(f: float) -> int:
    return lib().oracle_f32_to_bf16(float(f))


def router_logits(x_bf16, W):
    x = _c(x_bf16, np.uint16)
    W = _c(W, np.float32)
    T, H = x.shape
    E = W.shape[0]
    out = np.empty((T, E), dtype=np.float32)
    lib().oracle_router_logits(_p(x), T, H, _p(W), E, _p(out))
    return out


def select(logits, bias, n_group, topk_group, top_k, rsf, top_p=0.0):
    """-> (idx, w, gap_expert, gap_group); 0 < top_p < 1 applies adaptive top-p (empty slots: -1, 0)."""
    lg = _c(logits, np.float32)
    T, E = lg.shape
    b = _c(bias, np.float32)
    idx = np.empty((T, top_k), dtype=np.int32)
    w = np.empty((T, top_k), dtype=np.float32)
    ge = np.empty(T, dtype=np.float32)
    gg = np.empty(T, dtype=np.float32)
    _check(lib().oracle_select_topp(_p(lg), T, _p(b), E, n_group, topk_group, top_k, rsf, top_p,
                                    _p(idx), _p(w), _p(ge), _p(gg)), "oracle_select")
    return idx, w, ge, gg


def route(x_bf16, W, bias, n_group, topk_group, top_k, rsf, top_p=0.0):
    """-> (idx [T,K] int32, w [T,K] fp32, gap_expert [T], gap_group [T]); see select for top_p."""
    x = _c(x_bf16, np.uint16)
    W = _c(W, np.float32)
    b = _c(bias, np.float32)
    T, H = x.shape
    E = W.shape[0]
    idx = np.empty((T, top_k), dtype=np.int32)
    w = np.empty((T, top_k), dtype=np.float32)
    ge = np.empty(T, dtype=np.float32)
    gg = np.empty(T, dtype=np.float32)
    _check(lib().oracle_route_topp(_p(x), T, H, _p(W), _p(b), E, n_group, topk_group, top_k, rsf,
                                   top_p, _p(idx), _p(w), _p(ge), _p(gg)), "oracle_route")
    return idx, w, ge, gg


def union(idx, E):
    """-> dict(n_unique, uniq, offsets, pair_tok, pair_slot, counts)."""
    idx = _c(idx, np.int32)
    T, K = idx.shape
    nu = np.zeros(1, dtype=np.int32)
    uniq = np.full(E, -1, dtype=np.int32)
    offs = np.full(E + 1, -1, dtype=np.int32)
    ptok = np.full(max(T * K, 1), -1, dtype=np.int32)
    pslot = np.full(max(T * K, 1), -1, dtype=np.int32)
    counts = np.zeros(E, dtype=np.int32)
    _check(lib().oracle_union(_p(idx), T, K, E, _p(nu), _p(uniq), _p(offs), _p(ptok), _p(pslot),
                              _p(counts)), "oracle_union")
    U = int(nu[0])
    return dict(n_unique=U, uniq=uniq[:U], offsets=offs[:U + 1], pair_tok=ptok[:T * K],
                pair_slot=pslot[:T * K], counts=counts)


def q8_0(v):
    v = _c(v, np.float32).reshape(-1)
    n = v.size
    q = np.empty(n, dtype=np.int8)
    d = np.empty(n // 32, dtype=np.float32)
    lib().oracle_q8_0(_p(v), n, _p(q), _p(d))
    return q, d


def unpack(packed, qtype, n):
    p = _c(packed, np.uint8)
    out = np.empty(n, dtype=np.int8)
    _check(lib().oracle_unpack(_p(p), qtype, n, _p(out)), "oracle_unpack")
    return out


def qdot(wcodes, w_scale, qa, da, variant: str = ""):
    wc = _c(wcodes, np.int8)
    qa = _c(qa, np.int8)
    da = _c(da, np.float32)
    return lib(variant).oracle_qdot(_p(wc), float(w_scale), _p(qa), _p(da), wc.size)


def qdot_grouped(wcodes, w_scales, group, qa, da, variant: str = ""):
    wc = _c(wcodes, np.int8)
    ws = _c(w_scales, np.float32)
    qa = _c(qa, np.int8)
    da = _c(da, np.float32)
    return lib(variant).oracle_qdot_grouped(_p(wc), _p(ws), int(group), _p(qa), _p(da), wc.size)


def expert_token(ex: Experts, e, x_f32, want_h=False, variant: str = ""):
    x = _c(x_f32, np.float32)
    y = np.empty(ex.H, dtype=np.float32)
    h = np.empty(ex.I, dtype=np.float32) if want_h else None
    _check(lib(variant).oracle_expert_token(ctypes.byref(ex.struct()), e, _p(x), _p(y), _p(h)),
           "oracle_expert_token")
    return (y, h) if want_h else y


def expert_ffn(ex: Experts, x_bf16, top_k, un):
    x = _c(x_bf16, np.uint16)
    T = x.shape[0]
    y = np.zeros((T, top_k, ex.H), dtype=np.float32)
    _check(lib().oracle_expert_ffn(ctypes.byref(ex.struct()), _p(x), T, top_k, un["n_unique"],
                                   _p(_c(un["uniq"], np.int32)), _p(_c(un["offsets"], np.int32)),
                                   _p(_c(un["pair_tok"], np.int32)),
                                   _p(_c(un["pair_slot"], np.int32)), _p(y)), "oracle_expert_ffn")
    return y


def expert_ffn_per_token(ex: Experts, x_bf16, idx):
    x = _c(x_bf16, np.uint16)
    idx = _c(idx, np.int32)
    T, K = idx.shape
    y = np.zeros((T, K, ex.H), dtype=np.float32)
    _check(lib().oracle_expert_ffn_per_token(ctypes.byref(ex.struct()), _p(x), T, K, _p(idx),
                                             _p(y)), "oracle_expert_ffn_per_token")
    return y


def combine(y_pairs, w, shared_y):
    y = _c(y_pairs, np.float32)
    T, K, H = y.shape
    w = _c(w, np.float32)
    sy = None if shared_y is None else _c(shared_y, np.float32)
    of = np.empty((T, H), dtype=np.float32)
    ob = np.empty((T, H), dtype=np.uint16)
    lib().oracle_combine(_p(y), _p(w), _p(sy), T, K, H, _p(of), _p(ob))
    return of, ob


def layer_forward(x_bf16, W, bias, n_group, topk_group, top_k, rsf, routed: Experts,
                  shared: Experts | None, top_p=0.0):
    """-> (out_f32 [T,H], out_bf16 [T,H] uint16, idx [T,K], w [T,K])."""
    x = _c(x_bf16, np.uint16)
    W = _c(W, np.float32)
    b = _c(bias, np.float32)
    T = x.shape[0]
    E = W.shape[0]
    of = np.empty((T, routed.H), dtype=np.float32)
    ob = np.empty((T, routed.H), dtype=np.uint16)
    idx = np.empty((T, top_k), dtype=np.int32)
    w = np.empty((T, top_k), dtype=np.float32)
    rs = routed.struct()
    ss = shared.struct() if shared is not None else None
    _check(lib().oracle_layer_forward_topp(_p(x), T, _p(W), _p(b), E, n_group, topk_group, top_k, rsf,
                                           top_p, ctypes.byref(rs),
                                           ctypes.byref(ss) if ss is not None else None,
                                           _p(of), _p(ob), _p(idx), _p(w)), "oracle_layer_forward")
    return of, ob, idx, w


# ------------------------------------------------------------- expert usage
# [HN] "Learning cache와 하드웨어별 기대치": routed experts are recorded and the
# most used ones pinned first.  Plain definitions of the record and its order.
def usage_accumulate(idx, E, usage=None):
    """usage[e] + number of entries of idx equal to e (entries outside [0, E), such as the
    empty slot -1, count for nothing)."""
    u = np.zeros(E, dtype=np.int64) if usage is None else np.array(usage, dtype=np.int64)
    for e in np.asarray(idx).reshape(-1).tolist():
        if 0 <= e < E:
            u[e] += 1
    return u


def usage_rank(usage):
    """The experts, most used first, ties to the lower index."""
    u = [int(v) for v in np.asarray(usage).reshape(-1)]
    return np.array(sorted(range(len(u)), key=lambda e: (-u[e], e)), dtype=np.int32)
