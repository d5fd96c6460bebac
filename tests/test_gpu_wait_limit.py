"""Bounded device waits that run out, in the allowed form: the workspace's test
knob caps every bounded wait at one poll, so the kernels give up at once,
record MOE_EDEVICE_TIMEOUT, drain and exit; no GPU fault, trap or hang is
involved.  After a status clear the same workspace computes bitwise the same
result as before.  One shape per path with waits: the fused single-launch
kernel and the tensor-core GEMMs.
"""
import time

import pytest
import torch

import synth
from quantized_mixture_experts_sigmoid_b200 import moe
from synth.device import bits, device_layer, to_dev_bf16
from tests.helpers import layer_inputs

pytestmark = pytest.mark.gpu

SHAPES = {
    "fused_ragged": (synth.LayerShape("fused_ragged", T=3, H=544, I=288, E=64, n_group=2, topk_group=1, top_k=5),
                     moe.PATH_FUSED),
    "tc_small": (synth.LayerShape("tc_small", T=40, H=256, I=128, E=16, n_group=4, topk_group=2, top_k=4),
                 moe.PATH_TENSOR_CORE),
}


@pytest.mark.parametrize("name", list(SHAPES))
def test_bounded_waits_expire_and_the_workspace_recovers(name):
    sh, want_path = SHAPES[name]
    dev = device_layer(sh)
    assert moe.moe_layer_path(sh.T, dev["cfg"], dev["routed"], dev["shared"]) == want_path
    x, _, _ = layer_inputs(sh)
    xd = to_dev_bf16(x)
    ws = moe.workspace(moe.moe_layer_workspace_bytes(sh.T, dev["cfg"], dev["routed"], dev["shared"]))

    def forward():
        out = torch.empty(sh.T, sh.H, dtype=torch.bfloat16, device="cuda")
        moe.moe_layer_forward(xd, dev["W"], dev["bias"], dev["cfg"], dev["routed"], dev["shared"], out, ws)
        return out

    ref = bits(forward())
    assert moe.moe_workspace_status(ws) == moe.MOE_OK

    moe.moe_workspace_set_wait_limit(ws, 1)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    forward()
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    # the timeout is recorded, and promptly: the default limits would take seconds
    assert moe.moe_workspace_status(ws, clear=True) == moe.MOE_EDEVICE_TIMEOUT
    assert elapsed < 1.0, elapsed

    # the clear restored the default limits and the counters: the same call, the same bits
    again = bits(forward())
    assert moe.moe_workspace_status(ws) == moe.MOE_OK
    assert (again == ref).all()
    # and so does a call after that (the fused kernel's counters reset themselves)
    assert (bits(forward()) == ref).all()
    assert moe.moe_workspace_status(ws) == moe.MOE_OK
