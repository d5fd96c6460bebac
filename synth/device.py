"""Device-resident copies of the synthetic layer inputs (test and benchmark input setup).

Holds no arithmetic of the layer: it asks synth's CUDA twin to generate expert
weights directly in device memory and copies the host-generated router weight,
bias and hidden states to the device.
"""
from __future__ import annotations

import numpy as np
import torch

import synth
from quantized_mixture_experts_sigmoid_b200 import moe

_MATS = ((synth.GATE, "w_gate", "s_gate"), (synth.UP, "w_up", "s_up"), (synth.DOWN, "w_down", "s_down"))


def fill_experts(sh: synth.LayerShape, layer: int, ids, dst: moe.ExpertSet, slot_of=None) -> None:
    """Generate experts `ids` of `layer` on the device (synth's CUDA twin) into dst."""
    stream = torch.cuda.current_stream().cuda_stream
    for j, eid in enumerate(ids):
        slot = j if slot_of is None else slot_of(eid)
        for m, wn, sn in _MATS:
            w, s = getattr(dst, wn), getattr(dst, sn)
            synth.fill_matrix_gpu(sh, layer, eid, m, w[slot].data_ptr(), s[slot].data_ptr(), stream)


def device_layer(sh: synth.LayerShape, layer: int = 0, routed: moe.ExpertSet | None = None,
                 with_shared: bool = True):
    """routed + shared ExpertSets, router weight and bias on the device, router cfg."""
    if routed is None:
        routed = moe.ExpertSet.empty(sh.qtype, sh.E, sh.H, sh.I, group_size=sh.group_size)
    fill_experts(sh, layer, range(sh.E), routed)
    shared = None
    if with_shared:
        shared = moe.ExpertSet.empty(sh.qtype, 1, sh.H, sh.I, group_size=sh.group_size)
        fill_experts(sh, layer, [synth.SHARED], shared, slot_of=lambda e: 0)
    W = torch.from_numpy(synth.router_weight(sh, layer)).cuda()
    b = torch.from_numpy(synth.router_bias(sh, layer)).cuda()
    cfg = moe.RouterCfg(sh.E, sh.n_group, sh.topk_group, sh.top_k, sh.rsf)
    return dict(routed=routed, shared=shared, W=W, bias=b, cfg=cfg)


def to_dev_bf16(x_bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).cuda().view(torch.bfloat16)


def bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)
