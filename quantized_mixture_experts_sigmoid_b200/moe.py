"""Python binding of libmoe.so (include/moe.h): argument marshalling only.

Every step of the layer runs in the library's CUDA kernels.  Tensors are
passed as device pointers (``tensor.data_ptr()``) together with the current
torch CUDA stream; torch supplies device memory and streams, nothing else.
There is no CPU fallback: if the library cannot be loaded, every call raises.

The library sees only addresses and sizes, so the binding checks what it
cannot before passing a tensor: that it lives on a CUDA device, is
contiguous, has elements of the width the C signature reads, and holds at
least the elements the call will touch (a host tensor or a short buffer would
otherwise be read or written out of bounds on the device).
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


@dataclass(frozen=True, eq=False)  # compared and hashed by identity: the fields are device tensors
class ExpertSet:
    """A stack of experts resident on the device (tensors owned by the caller).

    Checked once when made (device, contiguity, element widths, sizes); its C struct is built
    then too, so a layer call only passes it.  Fields cannot be reassigned (the tensors' contents
    can change in place).

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

    def __post_init__(self):
        q, n, H, I, G = self.qtype, self.n_expert, self.hidden, self.inter, self.group_size
        per_h = H // G if G > 0 else 1
        per_i = I // G if G > 0 else 1
        for name, width, count in (("w_gate", 1, n * I * H * q // 8), ("w_up", 1, n * I * H * q // 8),
                                   ("w_down", 1, n * H * I * q // 8), ("s_gate", 4, n * I * per_h),
                                   ("s_up", 4, n * I * per_h), ("s_down", 4, n * H * per_i)):
            _dev(getattr(self, name), width, count, name)
        object.__setattr__(self, "_struct", _Experts(
            q, n, H, I, self.w_gate.data_ptr(), self.w_up.data_ptr(), self.w_down.data_ptr(),
            self.s_gate.data_ptr(), self.s_up.data_ptr(), self.s_down.data_ptr(), G))

    def struct(self) -> _Experts:
        return self._struct

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


def _dev(t, width: int, count: int, name: str):
    """t's device address once t is a contiguous CUDA tensor of `width`-byte elements holding at
    least `count` of them; None (an optional argument) stays None."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name}: a CUDA tensor is required, got one on {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if t.element_size() != width:
        raise TypeError(f"{name}: elements of {width} bytes expected, got {t.dtype}")
    if t.numel() < count:
        raise ValueError(f"{name}: {count} elements needed, {t.numel()} given")
    return t.data_ptr()


def _ws(ws):
    """A workspace's address and size in bytes."""
    _dev(ws, ws.element_size(), 0, "ws")
    return ws.data_ptr(), ws.numel() * ws.element_size()


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


def _route_args(x, w_router, bias, cfg, topk_idx, topk_w):
    T, H = x.shape
    E, K = cfg.n_expert, cfg.top_k
    return (_dev(x, 2, T * H, "x"), T, H, _dev(w_router, 4, E * H, "w_router"), _dev(bias, 4, E, "bias"),
            ctypes.byref(cfg), _dev(topk_idx, 4, T * K, "topk_idx"), _dev(topk_w, 4, T * K, "topk_w"))


def moe_route(x, w_router, bias, cfg: RouterCfg, topk_idx, topk_w, ws, stream=None):
    _ok("moe_route", lib().moe_route(*_route_args(x, w_router, bias, cfg, topk_idx, topk_w), *_ws(ws),
                                     _stream(stream)))


def moe_route_noalloc(x, w_router, bias, cfg: RouterCfg, topk_idx, topk_w, stream=None):
    """moe_route with the library's built-in logits scratch (no workspace, allocates nothing)."""
    _ok("moe_route_noalloc", lib().moe_route_noalloc(*_route_args(x, w_router, bias, cfg, topk_idx, topk_w),
                                                     _stream(stream)))


def moe_union(topk_idx, E, n_unique, uniq, offsets, pair_tok, pair_slot, counts=None,
              status=None, stream=None):
    T, K = topk_idx.shape
    _ok("moe_union", lib().moe_union(_dev(topk_idx, 4, T * K, "topk_idx"), T, K, E, _dev(n_unique, 4, 1, "n_unique"),
                                     _dev(uniq, 4, E, "uniq"), _dev(offsets, 4, E + 1, "offsets"),
                                     _dev(pair_tok, 4, T * K, "pair_tok"), _dev(pair_slot, 4, T * K, "pair_slot"),
                                     _dev(counts, 4, E, "counts"), _dev(status, 4, 1, "status"), _stream(stream)))


def moe_quantize_q8_0(v, q, d, stream=None):
    rows, n = v.shape
    dt = MOE_OUT_BF16 if v.dtype in (torch.bfloat16, torch.int16, torch.uint16) else MOE_OUT_F32
    _ok("moe_quantize_q8_0", lib().moe_quantize_q8_0(_dev(v, 2 if dt == MOE_OUT_BF16 else 4, rows * n, "v"), dt,
                                                     rows, n, _dev(q, 1, rows * n, "q"),
                                                     _dev(d, 4, rows * (n // 32), "d"), _stream(stream)))


def moe_expert_ffn_workspace_bytes(ex: ExpertSet, T: int, top_k: int) -> int:
    s = ex.struct()
    return lib().moe_expert_ffn_workspace_bytes(ctypes.byref(s), T, top_k)


def moe_expert_ffn_q(ex: ExpertSet, x, top_k, union, y_pairs, ws, stream=None):
    """union: (n_unique, uniq, offsets, pair_tok, pair_slot) device tensors, or None (dense)."""
    T = x.shape[0]
    s = ex.struct()
    if union is None:
        u = (None,) * 5
    else:
        nu, uq, of, pt, ps = union
        u = (_dev(nu, 4, 1, "n_unique"), _dev(uq, 4, 0, "uniq"), _dev(of, 4, 1, "offsets"),
             _dev(pt, 4, T * top_k, "pair_tok"), _dev(ps, 4, T * top_k, "pair_slot"))
    _ok("moe_expert_ffn_q", lib().moe_expert_ffn_q(ctypes.byref(s), _dev(x, 2, T * ex.hidden, "x"), T, top_k, *u,
                                                   _dev(y_pairs, 4, T * top_k * ex.hidden, "y_pairs"), *_ws(ws),
                                                   _stream(stream)))


def moe_combine(y_pairs, topk_w, shared_y, out, stream=None):
    T, K, H = y_pairs.shape
    dt = MOE_OUT_F32 if out.dtype == torch.float32 else MOE_OUT_BF16
    _ok("moe_combine", lib().moe_combine(_dev(y_pairs, 4, T * K * H, "y_pairs"), _dev(topk_w, 4, T * K, "topk_w"),
                                         _dev(shared_y, 4, T * H, "shared_y"), T, K, H,
                                         _dev(out, 4 if dt == MOE_OUT_F32 else 2, T * H, "out"), dt, _stream(stream)))


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
    H, E, K = routed.hidden, cfg.n_expert, cfg.top_k
    rs = routed.struct()
    ss = shared.struct() if shared is not None else None
    dt = MOE_OUT_F32 if out.dtype == torch.float32 else MOE_OUT_BF16
    _ok("moe_layer_forward", lib().moe_layer_forward(
        _dev(x, 2, T * H, "x"), T, _dev(w_router, 4, E * H, "w_router"), _dev(bias, 4, E, "bias"), ctypes.byref(cfg),
        ctypes.byref(rs), ctypes.byref(ss) if ss is not None else None,
        _dev(out, 4 if dt == MOE_OUT_F32 else 2, T * H, "out"), dt, _dev(topk_idx, 4, T * K, "topk_idx"),
        _dev(topk_w, 4, T * K, "topk_w"), *_ws(ws), _stream(stream)))


def moe_usage_accumulate(topk_idx, E: int, usage, stream=None) -> None:
    """usage[e] += entries of topk_idx [T][K] routed to e (empty slots add nothing)."""
    T, K = topk_idx.shape
    _ok("moe_usage_accumulate", lib().moe_usage_accumulate(_dev(topk_idx, 4, T * K, "topk_idx"), T, K, int(E),
                                                           _dev(usage, 4, int(E), "usage"), _stream(stream)))


def moe_usage_rank(usage, order, stream=None) -> None:
    """order[r] = the expert of rank r in the usage record (most used first, ties to the lower index)."""
    E = usage.numel()
    _ok("moe_usage_rank", lib().moe_usage_rank(_dev(usage, 4, E, "usage"), E, _dev(order, 4, E, "order"),
                                               _stream(stream)))


def moe_workspace_set_wait_limit(ws, polls: int, stream=None) -> None:
    """Test knob: cap every bounded device wait of later calls on `ws` at `polls` polls (0: defaults)."""
    _ok("moe_workspace_set_wait_limit", lib().moe_workspace_set_wait_limit(_ws(ws)[0], int(polls), _stream(stream)))


def moe_workspace_status(ws, clear: bool = True, stream=None) -> int:
    st = ctypes.c_int(0)
    _ok("moe_workspace_status", lib().moe_workspace_status(_ws(ws)[0], int(clear), ctypes.byref(st),
                                                           _stream(stream)))
    return st.value
