"""The C ABI library without a GPU: it loads, exports every declared entry
point, and rejects bad arguments before launching anything."""
import ctypes
import os
import re

import pytest

from quantized_mixture_experts_sigmoid_b200 import moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^\s*(?:\w+\s*\**\s+)+\**\s*(moe_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    L = moe.lib()
    names = declared()
    assert len(names) >= 11
    for n in names:
        assert hasattr(L, n), n
    assert set(moe.EXPORTS) <= set(names)


def test_error_strings():
    for code in (0, -1, -2, -3, -4, -5, -6, -7, -99):
        assert isinstance(moe.strerror(code), str) and moe.strerror(code)
    # no call on this thread has returned MOE_ECUDA: the CUDA error text says so
    assert moe.lib().moe_cuda_error_string().decode() == "no CUDA error"


P = 1 << 20  # a fake, 16-byte aligned "device" address: never dereferenced on these paths


def _cfg(E=256, G=8, TG=4, K=8, rsf=2.5):
    return moe.RouterCfg(E, G, TG, K, rsf)


def _ex(q=4, n=256, H=6144, I=2048, ptr=P, group=0):
    return moe._Experts(q, n, H, I, ptr, ptr, ptr, ptr, ptr, ptr, group)


@pytest.mark.parametrize("cfg", [_cfg(E=0), _cfg(G=3), _cfg(G=64, E=64), _cfg(TG=9), _cfg(K=0),
                                 _cfg(K=33), _cfg(E=8, G=8), _cfg(E=16, G=4, TG=1, K=5),
                                 _cfg(rsf=float("nan")), _cfg(E=2048, G=8)])
def test_route_rejects_bad_config(cfg):
    L = moe.lib()
    rc = L.moe_route(P, 4, 6144, P, P, ctypes.byref(cfg), P, P, P, 1 << 30, None)
    assert rc == moe.MOE_EINVAL
    assert L.moe_route_workspace_bytes(4, ctypes.byref(cfg)) == 0


def test_route_rejects_bad_pointers_sizes_workspace():
    L = moe.lib()
    c = ctypes.byref(_cfg())
    assert L.moe_route(P, 4, 6000, P, P, c, P, P, P, 1 << 30, None) == moe.MOE_EINVAL  # H % 32
    assert L.moe_route(P + 2, 4, 6144, P, P, c, P, P, P, 1 << 30, None) == moe.MOE_EINVAL  # misaligned x
    assert L.moe_route(None, 4, 6144, P, P, c, P, P, P, 1 << 30, None) == moe.MOE_EINVAL
    assert L.moe_route(P, -1, 6144, P, P, c, P, P, P, 1 << 30, None) == moe.MOE_EINVAL
    need = L.moe_route_workspace_bytes(4, c)
    assert need >= 256 + 4 * 256 * 4
    assert L.moe_route(P, 4, 6144, P, P, c, P, P, P, need - 1, None) == moe.MOE_EWORKSPACE
    assert L.moe_route(P, 4, 6144, P, P, c, P, P, P + 16, need, None) == moe.MOE_EWORKSPACE
    assert L.moe_route(P, 0, 6144, P, P, c, P, P, None, 0, None) == moe.MOE_OK  # empty batch


def test_expert_and_layer_argument_checks():
    L = moe.lib()
    c = ctypes.byref(_cfg())
    for bad, code in [(_ex(q=3), moe.MOE_EUNSUPPORTED), (_ex(H=100), moe.MOE_EINVAL),
                      (_ex(I=2047), moe.MOE_EINVAL), (_ex(ptr=P + 4), moe.MOE_EINVAL),
                      (_ex(H=32768), moe.MOE_EUNSUPPORTED), (_ex(n=0), moe.MOE_EINVAL)]:
        rc = L.moe_expert_ffn_q(ctypes.byref(bad), P, 4, 1, None, None, None, None, None, P, P, 1 << 40, None)
        assert rc == code
        rc = L.moe_layer_forward(P, 4, P, P, c, ctypes.byref(bad), None, P, 0, None, None, P, 1 << 40, None)
        assert rc == code
    good = ctypes.byref(_ex())
    # dense mode needs top_k == 1 and no partial union lists
    assert L.moe_expert_ffn_q(good, P, 4, 2, None, None, None, None, None, P, P, 1 << 40, None) == moe.MOE_EINVAL
    assert L.moe_expert_ffn_q(good, P, 4, 1, P, None, None, None, None, P, P, 1 << 40, None) == moe.MOE_EINVAL
    need = L.moe_expert_ffn_workspace_bytes(good, 4, 8)
    assert L.moe_expert_ffn_q(good, P, 4, 8, P, P, P, P, P, P, P, need - 256, None) == moe.MOE_EWORKSPACE
    # layer: routed count must match the router, shared hidden must match, dtype must be known
    assert L.moe_layer_forward(P, 1, P, P, ctypes.byref(_cfg(E=128, G=8)), good, None, P, 0, None, None, P,
                               1 << 40, None) == moe.MOE_EINVAL
    assert L.moe_layer_forward(P, 1, P, P, c, good, ctypes.byref(_ex(n=1, H=4096)), P, 0, None, None, P,
                               1 << 40, None) == moe.MOE_EINVAL
    assert L.moe_layer_forward(P, 1, P, P, c, good, None, P, 7, None, None, P, 1 << 40, None) == moe.MOE_EINVAL
    need = L.moe_layer_workspace_bytes(1, c, good, ctypes.byref(_ex(n=1)))
    assert L.moe_layer_forward(P, 1, P, P, c, good, ctypes.byref(_ex(n=1)), P, 0, None, None, P, need - 1,
                               None) == moe.MOE_EWORKSPACE


def test_other_argument_checks():
    L = moe.lib()
    assert L.moe_union(P, 4, 0, 16, P, P, P, P, P, None, None, None) == moe.MOE_EINVAL
    assert L.moe_union(P, 4, 2, 2000, P, P, P, P, P, None, None, None) == moe.MOE_EINVAL
    assert L.moe_union(P, 4, 2, 16, None, P, P, P, P, None, None, None) == moe.MOE_EINVAL
    assert L.moe_quantize_q8_0(P, 0, 4, 33, P, P, None) == moe.MOE_EINVAL
    assert L.moe_quantize_q8_0(P, 5, 4, 64, P, P, None) == moe.MOE_EINVAL
    assert L.moe_quantize_q8_0(P, 0, 0, 64, P, P, None) == moe.MOE_OK
    assert L.moe_combine(P, P, None, 4, 8, 6, P, 0, None) == moe.MOE_EINVAL
    assert L.moe_combine(P, P, P + 8, 4, 8, 64, P, 0, None) == moe.MOE_EINVAL
    assert L.moe_workspace_status(None, 1, None, None) == moe.MOE_EINVAL


def test_workspace_sizes_cover_the_buffers():
    L = moe.lib()
    c = ctypes.byref(_cfg())
    r, s = ctypes.byref(_ex()), ctypes.byref(_ex(n=1))
    b1 = L.moe_layer_workspace_bytes(1, c, r, s)
    b2048 = L.moe_layer_workspace_bytes(2048, c, r, s)
    assert b1 % 256 == 0 and b2048 > b1
    # at least the per-pair fp32 outputs, the routed and shared h codes and the logits
    assert b2048 >= 2048 * 8 * 6144 * 4 + 2048 * 9 * 2048 + 2048 * 256 * 4


def test_layer_path_query():
    # host-only: which kernels a call would run (nothing is launched)
    L = moe.lib()
    glm = _cfg()
    r, s = _ex(), _ex(n=1)
    path = lambda T, cfg=glm, rr=r, ss=s: L.moe_layer_path(T, ctypes.byref(cfg), ctypes.byref(rr),
                                                          ctypes.byref(ss) if ss is not None else None)
    assert path(1) == moe.PATH_FUSED
    assert path(4) == moe.PATH_FUSED
    assert path(5) == moe.PATH_GENERAL        # a few tokens per expert: lane-per-row kernels
    assert path(32) == moe.PATH_GENERAL
    assert path(33) == moe.PATH_TENSOR_CORE
    assert path(2048) == moe.PATH_TENSOR_CORE
    assert path(2048, rr=_ex(q=8)) == moe.PATH_GENERAL           # int8 experts: integer-dot kernels
    assert path(2048, rr=_ex(H=544, I=288), ss=_ex(n=1, H=544, I=288)) == moe.PATH_GENERAL  # K not a multiple of 64
    small = _cfg(E=16, G=4, TG=2, K=2)
    assert path(4, cfg=small, rr=_ex(n=16)) == moe.PATH_GENERAL  # groups of 4 experts: no fused kernel
    assert path(0) == moe.MOE_EINVAL


def test_wait_limit_knob_rejects_bad_arguments_without_a_gpu():
    # host-side argument checks: nothing is written or launched
    L = moe.lib()
    assert L.moe_workspace_set_wait_limit(None, 1, None) == moe.MOE_EINVAL
    assert L.moe_workspace_set_wait_limit(ctypes.c_void_p(1 << 20), -1, None) == moe.MOE_EINVAL


def test_usage_calls_reject_bad_arguments_without_a_gpu():
    L = moe.lib()
    P = ctypes.c_void_p(1 << 20)
    assert L.moe_usage_accumulate(None, 4, 8, 256, P, None) == moe.MOE_EINVAL
    assert L.moe_usage_accumulate(P, 4, 8, 2048, P, None) == moe.MOE_EINVAL
    assert L.moe_usage_accumulate(P, 0, 8, 256, P, None) == moe.MOE_OK  # empty batch: nothing to add
    assert L.moe_usage_rank(P, 0, P, None) == moe.MOE_EINVAL
    assert L.moe_usage_rank(None, 256, P, None) == moe.MOE_EINVAL


def test_grouped_scales_geometry_and_paths_on_the_host():
    # group sizes: a multiple of 32 dividing hidden and inter; the fused kernel takes
    # grouped scales, the tensor-core GEMMs do not (those batches report the general path)
    L = moe.lib()
    c = _cfg()
    path = lambda T, r, s: L.moe_layer_path(T, ctypes.byref(c), ctypes.byref(r), ctypes.byref(s))
    assert path(1, _ex(group=48), _ex(n=1, group=48)) == moe.MOE_EINVAL
    assert path(1, _ex(group=96), _ex(n=1, group=96)) == moe.MOE_EINVAL  # 2048 % 96 != 0
    assert path(1, _ex(group=-32), _ex(n=1, group=-32)) == moe.MOE_EINVAL
    assert path(1, _ex(group=128), _ex(n=1, group=128)) == moe.PATH_FUSED
    assert path(40, _ex(group=128), _ex(n=1, group=128)) == moe.PATH_GENERAL
    assert path(40, _ex(), _ex(n=1)) == moe.PATH_TENSOR_CORE
    assert path(1, _ex(group=128), _ex(n=1, group=32)) == moe.PATH_GENERAL  # mixed sizes: not fused
