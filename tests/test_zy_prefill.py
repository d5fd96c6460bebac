"""Full-size prefill (T = 2048, GLM-5.2 shape, Zipf-skewed routing) on the GPU
against the oracle: routing of every token bit-exact, the layer output of a
seeded sample of tokens within the parity bar.

The layer runs the tensor-core batch-union path (every unique expert applied
to its tokens in 128-row tiles).  The oracle routes all 2048 tokens and
computes the output of the sampled tokens only, regenerating just the experts
they touch.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import oracle as O
from quantized_mixture_experts_sigmoid_b200 import moe
from synth.device import device_layer, to_dev_bf16
from tests.helpers import layer_inputs, oracle_experts, rel_err_rows

pytestmark = pytest.mark.gpu

TOL = 2e-3
SAMPLE = 64


def test_prefill_full_size_sampled():
    sh = synth.CONFIGS["prefill"]
    dev = device_layer(sh)
    assert moe.moe_layer_path(sh.T, dev["cfg"], dev["routed"], dev["shared"]) == moe.PATH_TENSOR_CORE
    x, W, b = layer_inputs(sh)
    ws = moe.workspace(moe.moe_layer_workspace_bytes(sh.T, dev["cfg"], dev["routed"], dev["shared"]))
    out = torch.empty(sh.T, sh.H, dtype=torch.float32, device="cuda")
    idx = torch.empty(sh.T, sh.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(sh.T, sh.top_k, dtype=torch.float32, device="cuda")
    moe.moe_layer_forward(to_dev_bf16(x), dev["W"], dev["bias"], dev["cfg"], dev["routed"], dev["shared"], out,
                          ws, idx, w)
    torch.cuda.synchronize()
    assert moe.moe_workspace_status(ws) == 0
    idx_g, w_g, out_g = idx.cpu().numpy(), w.cpu().numpy(), out.cpu().numpy()
    del dev, ws
    torch.cuda.empty_cache()

    idx_o, w_o, _, _ = O.route(x, W, b, sh.n_group, sh.topk_group, sh.top_k, sh.rsf)
    assert np.array_equal(idx_g, idx_o)
    assert np.array_equal(w_g.view(np.uint32), w_o.view(np.uint32))

    rng = np.random.default_rng(7)
    toks = np.sort(rng.choice(sh.T, size=SAMPLE, replace=False))
    toks[0], toks[-1] = 0, sh.T - 1  # include both ends of the batch
    routed = oracle_experts(sh, np.unique(idx_o[toks]))
    shared = oracle_experts(sh, [0], shared=True)
    ref, _, _, _ = O.layer_forward(x[toks], W, b, sh.n_group, sh.topk_group, sh.top_k, sh.rsf, routed, shared)
    err = rel_err_rows(out_g[toks], ref)
    assert err <= TOL, err
