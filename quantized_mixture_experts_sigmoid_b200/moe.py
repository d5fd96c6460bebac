"""Python binding of libmoe.so (include/moe.h): argument marshalling only.

Every step of the layer runs in the library's CUDA kernels.  Tensors are
passed as device pointers (``tensor.data_ptr()``) together with the current
torch CUDA stream; torch supplies device memory and streams, nothing else.
There is no CPU fallback: if the library cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

from . import build as _build

MOE_OK = 0
MOE_EINVAL = -1
MOE_EWORKSPACE = -2
MOE_EUNSUPPORTED = -3
MOE_ECUDA = -4
MOE_EDEVICE_TIMEOUT = -5
MOE_EDEVICE_INDEX = -6
MOE_ETOO_LARGE = -7
MOE_ROUTE_NOALLOC_MAX_LOGITS = 65536
MOE_Q_INT2, MOE_Q_INT4, MOE_Q_INT8 = 2, 4, 8
MOE_OUT_BF16, MOE_OUT_F32 = 0, 1


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int):
        extra = f": {lib().moe_cuda_error_string().decode()}" if code == MOE_ECUDA else ""
        super().__init__(f"{fn} failed: {code} ({strerror(code)}{extra})")
        self.code = code


class RouterCfg(ctypes.Structure):
    _fields_ = [("n_expert", ctypes.c_int), ("n_group", ctypes.c_int),
                ("topk_group", ctypes.c_int), ("top_k", ctypes.c_int),
                ("routed_scaling_factor", ctypes.c_float), ("top_p", ctypes.c_float)]


class _Experts(ctypes.Structure):
    _fields_ = [("qtype", ctypes.c_int), ("n_expert", ctypes.c_int), ("hidden", ctypes.c_int),
                ("inter", ctypes.c_int), ("w_gate", ctypes.c_void_p), ("w_up", ctypes.c_void_p),
                ("w_down", ctypes.c_void_p), ("s_gate", ctypes.c_void_p),
                ("s_up", ctypes.c_void_p), ("s_down", ctypes.c_void_p), ("group_size", ctypes.c_int)]


@dataclass
class ExpertSet:
    """A stack of experts resident on the device (tensors owned by the caller).

    w_gate, w_up: uint8 [n, inter, hidden*q/8]; w_down: uint8 [n, hidden, inter*q/8];
    s_gate, s_up: fp32 [n, inter]; s_down: fp32 [n, hidden]; with grouped scales (group_size G)
    s_gate, s_up: fp32 [n, inter, hidden/G]; s_down: fp32 [n, hidden, inter/G].
    """
    qtype: int
    n_expert: int
    hidden: int
    inter: int
    w_gate: torch.Tensor
    w_up: torch.Tensor
    w_down: torch.Tensor
    s_gate: torch.Tensor
    s_up: torch.Tensor
    s_down: torch.Tensor
    group_size: int = 0

    def struct(self) -> _Experts:
        return _Experts(self.qtype, self.n_expert, self.hidden, self.inter, self.w_gate.data_ptr(),
                        self.w_up.data_ptr(), self.w_down.data_ptr(), self.s_gate.data_ptr(),
                        self.s_up.data_ptr(), self.s_down.data_ptr(), self.group_size)

    @staticmethod
    def empty(qtype: int, n_expert: int, hidden: int, inter: int, device="cuda", group_size: int = 0) -> "ExpertSet":
        u8 = dict(dtype=torch.uint8, device=device)
        f32 = dict(dtype=torch.float32, device=device)
        gh = (hidden // group_size,) if group_size else ()
        gi = (inter // group_size,) if group_size else ()
        return ExpertSet(qtype, n_expert, hidden, inter,
                         torch.empty(n_expert, inter, hidden * qtype // 8, **u8),
                         torch.empty(n_expert, inter, hidden * qtype // 8, **u8),
                         torch.empty(n_expert, hidden, inter * qtype // 8, **u8),
                         torch.empty(n_expert, inter, *gh, **f32), torch.empty(n_expert, inter, *gh, **f32),
                         torch.empty(n_expert, hidden, *gi, **f32), group_size)


_lib = None

EXPORTS = ["moe_strerror", "moe_route_workspace_bytes", "moe_route", "moe_union",
           "moe_quantize_q8_0", "moe_expert_ffn_workspace_bytes", "moe_expert_ffn_q",
           "moe_combine", "moe_layer_workspace_bytes", "moe_layer_forward",
           "moe_workspace_status", "moe_profile_enable", "moe_profile_read", "moe_launch_count",
           "moe_route_noalloc", "moe_layer_path", "moe_cuda_error_string", "moe_workspace_set_wait_limit",
           "moe_usage_accumulate", "moe_usage_rank"]


def lib() -> ctypes.CDLL:
    """Load (building in-tree first if stale) libmoe.so; raises if that fails."""
    global _lib
    if _lib is not None:
        return _lib
    path = _build.build()
    if not os.path.exists(path):
        raise RuntimeError(f"libmoe.so missing at {path}")
    L = ctypes.CDLL(path)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.moe_strerror.argtypes = [i]
    L.moe_strerror.restype = ctypes.c_char_p
    L.moe_cuda_error_string.argtypes = []
    L.moe_cuda_error_string.restype = ctypes.c_char_p
    L.moe_route_workspace_bytes.argtypes = [i, vp]
    L.moe_route_workspace_bytes.restype = sz
    L.moe_route.argtypes = [vp, i, i, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_route_noalloc.argtypes = [vp, i, i, vp, vp, vp, vp, vp, vp]
    L.moe_union.argtypes = [vp, i, i, i, vp, vp, vp, vp, vp, vp, vp, vp]
    L.moe_quantize_q8_0.argtypes = [vp, i, i, i, vp, vp, vp]
    L.moe_expert_ffn_workspace_bytes.argtypes = [vp, i, i]
    L.moe_expert_ffn_workspace_bytes.restype = sz
    L.moe_expert_ffn_q.argtypes = [vp, vp, i, i, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_combine.argtypes = [vp, vp, vp, i, i, i, vp, i, vp]
    L.moe_layer_workspace_bytes.argtypes = [i, vp, vp, vp]
    L.moe_layer_workspace_bytes.restype = sz
    L.moe_layer_path.argtypes = [i, vp, vp, vp]
    L.moe_layer_path.restype = i
    L.moe_layer_forward.argtypes = [vp, i, vp, vp, vp, vp, vp, vp, i, vp, vp, vp, sz, vp]
    L.moe_workspace_status.argtypes = [vp, i, vp, vp]
    L.moe_workspace_set_wait_limit.argtypes = [vp, i, vp]
    L.moe_usage_accumulate.argtypes = [vp, i, i, i, vp, vp]
    L.moe_usage_rank.argtypes = [vp, i, vp, vp]
    L.moe_profile_enable.argtypes = [i]
    L.moe_profile_read.argtypes = [vp, vp]
    L.moe_launch_count.argtypes = []
    L.moe_launch_count.restype = ctypes.c_longlong
    _lib = L
    return L


def strerror(code: int) -> str:
    return lib().moe_strerror(int(code)).decode()


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ok(fn, rc):
    if rc != MOE_OK:
        raise MoeError(fn, rc)


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A zeroed, 256-byte aligned workspace (torch allocations are aligned)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def moe_route_workspace_bytes(T: int, cfg: RouterCfg) -> int:
    return lib().moe_route_workspace_bytes(T, ctypes.byref(cfg))


def moe_route(x, w_router, bias, cfg: RouterCfg, topk_idx, topk_w, ws, stream=None):
    T, H = x.shape
    _ok("moe_route", lib().moe_route(_ptr(x), T, H, _ptr(w_router), _ptr(bias), ctypes.byref(cfg),
                                     _ptr(topk_idx), _ptr(topk_w), _ptr(ws), ws.numel(),
                                     _stream(stream)))


def moe_route_noalloc(x, w_router, bias, cfg: RouterCfg, topk_idx, topk_w, stream=None):
    """moe_route with the library's built-in logits scratch (no workspace, allocates nothing)."""
    T, H = x.shape
    _ok("moe_route_noalloc", lib().moe_route_noalloc(_ptr(x), T, H, _ptr(w_router), _ptr(bias),
                                                     ctypes.byref(cfg), _ptr(topk_idx),
                                                     _ptr(topk_w), _stream(stream)))


def moe_union(topk_idx, E, n_unique, uniq, offsets, pair_tok, pair_slot, counts=None,
              status=None, stream=None):
    T, K = topk_idx.shape
    _ok("moe_union", lib().moe_union(_ptr(topk_idx), T, K, E, _ptr(n_unique), _ptr(uniq),
                                     _ptr(offsets), _ptr(pair_tok), _ptr(pair_slot), _ptr(counts),
                                     _ptr(status), _stream(stream)))


def moe_quantize_q8_0(v, q, d, stream=None):
    rows, n = v.shape
    dt = MOE_OUT_BF16 if v.dtype in (torch.bfloat16, torch.int16, torch.uint16) else MOE_OUT_F32
    _ok("moe_quantize_q8_0", lib().moe_quantize_q8_0(_ptr(v), dt, rows, n, _ptr(q), _ptr(d),
                                                     _stream(stream)))


def moe_expert_ffn_workspace_bytes(ex: ExpertSet, T: int, top_k: int) -> int:
    s = ex.struct()
    return lib().moe_expert_ffn_workspace_bytes(ctypes.byref(s), T, top_k)


def moe_expert_ffn_q(ex: ExpertSet, x, top_k, union, y_pairs, ws, stream=None):
    """union: (n_unique, uniq, offsets, pair_tok, pair_slot) device tensors, or None (dense)."""
    T = x.shape[0]
    s = ex.struct()
    u = (None,) * 5 if union is None else union
    _ok("moe_expert_ffn_q", lib().moe_expert_ffn_q(ctypes.byref(s), _ptr(x), T, top_k,
                                                   *[_ptr(a) for a in u], _ptr(y_pairs), _ptr(ws),
                                                   ws.numel(), _stream(stream)))


def moe_combine(y_pairs, topk_w, shared_y, out, stream=None):
    T, K, H = y_pairs.shape
    dt = MOE_OUT_F32 if out.dtype == torch.float32 else MOE_OUT_BF16
    _ok("moe_combine", lib().moe_combine(_ptr(y_pairs), _ptr(topk_w), _ptr(shared_y), T, K, H,
                                         _ptr(out), dt, _stream(stream)))


def moe_layer_workspace_bytes(T: int, cfg: RouterCfg, routed: ExpertSet, shared: ExpertSet | None):
    rs = routed.struct()
    ss = shared.struct() if shared is not None else None
    return lib().moe_layer_workspace_bytes(T, ctypes.byref(cfg), ctypes.byref(rs),
                                           ctypes.byref(ss) if ss is not None else None)


PATH_FUSED, PATH_TENSOR_CORE, PATH_GENERAL = 1, 2, 3


def moe_layer_path(T: int, cfg: RouterCfg, routed: ExpertSet, shared: ExpertSet | None) -> int:
    """Which kernels moe_layer_forward runs for these shapes (PATH_*)."""
    rs = routed.struct()
    ss = shared.struct() if shared is not None else None
    rc = lib().moe_layer_path(T, ctypes.byref(cfg), ctypes.byref(rs), ctypes.byref(ss) if ss is not None else None)
    if rc < 0:
        raise MoeError("moe_layer_path", rc)
    return rc


def moe_layer_forward(x, w_router, bias, cfg: RouterCfg, routed: ExpertSet,
                      shared: ExpertSet | None, out, ws, topk_idx=None, topk_w=None, stream=None):
    T = x.shape[0]
    rs = routed.struct()
    ss = shared.struct() if shared is not None else None
    dt = MOE_OUT_F32 if out.dtype == torch.float32 else MOE_OUT_BF16
    _ok("moe_layer_forward", lib().moe_layer_forward(
        _ptr(x), T, _ptr(w_router), _ptr(bias), ctypes.byref(cfg), ctypes.byref(rs),
        ctypes.byref(ss) if ss is not None else None, _ptr(out), dt, _ptr(topk_idx), _ptr(topk_w),
        _ptr(ws), ws.numel(), _stream(stream)))


def moe_usage_accumulate(topk_idx, E: int, usage, stream=None) -> None:
    """usage[e] += entries of topk_idx [T][K] routed to e (empty slots add nothing)."""
    T, K = topk_idx.shape
    _ok("moe_usage_accumulate", lib().moe_usage_accumulate(_ptr(topk_idx), T, K, int(E), _ptr(usage), _stream(stream)))


def moe_usage_rank(usage, order, stream=None) -> None:
    """order[r] = the expert of rank r in the usage record (most used first, ties to the lower index)."""
    _ok("moe_usage_rank", lib().moe_usage_rank(_ptr(usage), usage.numel(), _ptr(order), _stream(stream)))


def moe_workspace_set_wait_limit(ws, polls: int, stream=None) -> None:
    """Test knob: cap every bounded device wait of later calls on `ws` at `polls` polls (0: defaults)."""
    _ok("moe_workspace_set_wait_limit", lib().moe_workspace_set_wait_limit(_ptr(ws), int(polls), _stream(stream)))


def moe_workspace_status(ws, clear: bool = True, stream=None) -> int:
    st = ctypes.c_int(0)
    _ok("moe_workspace_status", lib().moe_workspace_status(_ptr(ws), int(clear), ctypes.byref(st),
                                                           _stream(stream)))
    return st.value
