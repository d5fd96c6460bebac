"""The device twin of the input generator produces the host generator's bytes."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("qtype", [4, 8, 2])
def test_gpu_generator_matches_host(qtype):
    sh = synth.CONFIGS["decode"].with_(qtype=qtype)
    for layer, expert in [(0, 0), (0, 255), (3, synth.SHARED)]:
        for m in (synth.GATE, synth.UP, synth.DOWN):
            rows, rb = sh.rows(m), sh.row_bytes(m)
            codes = torch.empty(rows, rb, dtype=torch.uint8, device="cuda")
            sc = torch.empty(rows, dtype=torch.float32, device="cuda")
            synth.fill_matrix_gpu(sh, layer, expert, m, codes.data_ptr(), sc.data_ptr(),
                                  torch.cuda.current_stream().cuda_stream)
            hc, hs = synth.expert_matrix(sh, layer, expert, m)
            assert np.array_equal(codes.cpu().numpy(), hc)
            assert np.array_equal(sc.cpu().numpy().view(np.uint32), hs.view(np.uint32))


def test_gpu_generator_unaligned_ranges():
    lib = synth.synth._gpu()
    out = torch.zeros(1000, dtype=torch.uint8, device="cuda")
    for start, n in [(3, 997), (8, 992), (13, 77)]:
        assert lib.synth_gpu_bytes(7, 99, start, n, out.data_ptr(), 0) == 0
        torch.cuda.synchronize()
        assert np.array_equal(out[:n].cpu().numpy(), synth.uniform_bytes(7, 99, start, n))
