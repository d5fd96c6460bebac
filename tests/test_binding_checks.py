"""The Python binding's checks, on the host: tensors the library would read or
write out of bounds (host memory, strided views, the wrong element width, too
few elements) are refused before any call reaches the library."""
import pytest
import torch

from quantized_mixture_experts_sigmoid_b200 import moe


def test_host_tensors_are_refused():
    cfg = moe.RouterCfg(16, 4, 2, 4, 2.5)
    x = torch.zeros(2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="x: a CUDA tensor"):
        moe.moe_route(x, torch.zeros(16, 64), torch.zeros(16), cfg, torch.zeros(2, 4, dtype=torch.int32),
                      torch.zeros(2, 4), torch.zeros(256, dtype=torch.uint8))
    with pytest.raises(ValueError, match="CUDA tensor"):
        moe.moe_combine(torch.zeros(2, 4, 64), torch.zeros(2, 4), None, torch.zeros(2, 64))
    with pytest.raises(ValueError, match="ws: a CUDA tensor"):
        moe.moe_workspace_status(torch.zeros(256, dtype=torch.uint8))
    with pytest.raises(ValueError, match="w_gate: a CUDA tensor"):
        moe.ExpertSet.empty(4, 2, 64, 32, device="cpu")


def test_checks_in_order(monkeypatch):
    # pretend every tensor is on the device so the later checks are reached (the library is not called)
    monkeypatch.setattr(torch.Tensor, "is_cuda", property(lambda self: True))
    x = torch.zeros(4, 64)
    with pytest.raises(ValueError, match="t: must be contiguous"):
        moe._dev(x.t(), 4, 0, "t")
    with pytest.raises(TypeError, match="elements of 2 bytes"):
        moe._dev(x, 2, 0, "t")
    with pytest.raises(ValueError, match="257 elements needed, 256 given"):
        moe._dev(x, 4, 257, "t")
    assert moe._dev(x, 4, 256, "t") == x.data_ptr()
    assert moe._dev(None, 4, 256, "t") is None


def test_expert_set_sizes(monkeypatch):
    monkeypatch.setattr(torch.Tensor, "is_cuda", property(lambda self: True))
    for q in (2, 4, 8):
        for G in (0, 32):
            es = moe.ExpertSet.empty(q, 3, 128, 64, device="cpu", group_size=G)
            assert es.w_gate.numel() == 3 * 64 * 128 * q // 8
    es = moe.ExpertSet.empty(4, 3, 128, 64, device="cpu")
    with pytest.raises(ValueError, match="w_down: 12288 elements needed"):
        moe.ExpertSet(4, 3, 128, 64, es.w_gate, es.w_up, es.w_down[:2], es.s_gate, es.s_up, es.s_down)
    with pytest.raises(TypeError, match="s_up: elements of 4 bytes"):
        moe.ExpertSet(4, 3, 128, 64, es.w_gate, es.w_up, es.w_down, es.s_gate, es.s_up.half(), es.s_down)
    with pytest.raises(ValueError, match="s_gate: 384 elements needed, 192 given"):  # grouped scales need H / G per row
        moe.ExpertSet(4, 3, 128, 64, es.w_gate, es.w_up, es.w_down, es.s_gate, es.s_up, es.s_down, 64)


def test_workspace_size_counts_bytes(monkeypatch):
    monkeypatch.setattr(torch.Tensor, "is_cuda", property(lambda self: True))
    ws = torch.zeros(64, dtype=torch.int32)
    assert moe._ws(ws) == (ws.data_ptr(), 256)
