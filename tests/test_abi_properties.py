"""The layer's host-side decisions over random shapes, without a GPU.

For any router configuration, expert shape, weight width, scale grouping,
shared expert and batch size, moe_layer_path answers one of the three paths
exactly under the rules include/moe.h states (the fused kernel only for small
batches of shapes it can hold; the tensor cores exactly for int4 batches of
more than 32 tokens with per-row scales and hidden, inter multiples of 64),
the workspace size is a positive multiple of 256 bytes, and moe_layer_forward
refuses a workspace one byte short or misaligned before it launches anything.
"""
import ctypes

from hypothesis import given, settings
from hypothesis import strategies as st

from quantized_mixture_experts_sigmoid_b200 import moe

P = 1 << 20  # a fake, aligned "device" address: never dereferenced on these paths


@st.composite
def layer_shapes(draw):
    E = draw(st.sampled_from([16, 32, 64, 96, 128, 256, 512, 1024]))
    G = draw(st.sampled_from([g for g in (1, 2, 4, 8, 16, 32) if E % g == 0 and E // g >= 2]))
    TG = draw(st.integers(1, G))
    K = draw(st.integers(1, min(32, TG * (E // G))))
    H = 32 * draw(st.integers(1, 256))
    I = 32 * draw(st.integers(1, 128))
    q = draw(st.sampled_from([2, 4, 8]))
    gs = draw(st.sampled_from([0, 0, 32, 64, 128]))
    shared = draw(st.sampled_from(["none", "same", "other_inter"]))
    T = draw(st.one_of(st.integers(1, 40), st.integers(1, 4096)))
    return E, G, TG, K, H, I, q, gs, shared, T


def _experts(q, n, H, I, gs):
    return moe._Experts(q, n, H, I, P, P, P, P, P, P, gs)


@settings(max_examples=200, deadline=None)
@given(layer_shapes())
def test_path_and_workspace_follow_the_documented_rules(shape):
    E, G, TG, K, H, I, q, gs, shared_kind, T = shape
    L = moe.lib()
    cfg = moe.RouterCfg(E, G, TG, K, 2.5)
    routed = _experts(q, E, H, I, gs)
    shared = None
    if shared_kind == "same":
        shared = _experts(q, 1, H, I, gs)
    elif shared_kind == "other_inter":
        shared = _experts(q, 1, H, I + 32 if I < 4096 else I - 32, gs)
    sref = ctypes.byref(shared) if shared is not None else None
    path = L.moe_layer_path(T, ctypes.byref(cfg), ctypes.byref(routed), sref)
    ws = L.moe_layer_workspace_bytes(T, ctypes.byref(cfg), ctypes.byref(routed), sref)

    grouping_ok = gs == 0 or (H % gs == 0 and I % gs == 0)
    if not grouping_ok or (shared is not None and not (gs == 0 or shared.inter % gs == 0)):
        # the size query reads only the sizes; the path query and the call reject the grouping
        assert path == moe.MOE_EINVAL
        assert L.moe_layer_forward(P, T, P, P, ctypes.byref(cfg), ctypes.byref(routed), sref, P, moe.MOE_OUT_BF16,
                                   None, None, P, 1 << 40, None) == moe.MOE_EINVAL
        return
    assert path in (moe.PATH_FUSED, moe.PATH_TENSOR_CORE, moe.PATH_GENERAL)
    assert ws > 0 and ws % 256 == 0

    same_shared = shared is None or (shared.inter == I and shared.hidden == H)
    if path == moe.PATH_FUSED:
        assert T <= 4 and T * K <= 32 and K <= 8 and T * E <= 1024
        assert E <= 256 and E % 32 == 0 and (E // G) % 32 == 0 and same_shared
    tc = T > 32 and q == 4 and gs == 0 and H % 64 == 0 and I % 64 == 0 and same_shared
    assert (path == moe.PATH_TENSOR_CORE) == tc

    # the workspace checks come before any launch: one byte short, or off a 256-byte boundary
    fwd = lambda ptr, nbytes: L.moe_layer_forward(P, T, P, P, ctypes.byref(cfg), ctypes.byref(routed), sref, P,  # noqa: E731
                                                  moe.MOE_OUT_BF16, None, None, ptr, nbytes, None)
    assert fwd(P, ws - 1) == moe.MOE_EWORKSPACE
    assert fwd(P + 128, ws) == moe.MOE_EWORKSPACE
