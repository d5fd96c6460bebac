"""bench.py's multi-rank plumbing on CPU (gloo, world size 2): the max-over-ranks
device time, the whole-job throughput of replicas, and the reference arm under
torchrun (rank 0 alone runs the oracle and prints one line)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, _ = bench.rank_env()
        # rank r reports a device time of 10 + r ms: every rank must see the slowest one
        out[r] = bench.max_over_ranks(10.0 + r, w, "cpu")
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world_2():
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    assert dict(out) == {0: 11.0, 1: 11.0}


def test_replicas_throughput_counts_every_rank():
    # 2 replicas x 1 token x 1000 steps in 50 ms (the slowest rank) = 40k tokens/s
    assert bench.replicas_tokens_per_s(2, 1, 1000, 50.0) == pytest.approx(40000.0)
    assert bench.replicas_tokens_per_s(1, 1, 1000, 50.0) == pytest.approx(20000.0)


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "0"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["value"] > 0
    # the line carries the contract's keys, on the CUDA arm's metric and workload
    for key in ("metric", "unit", "higher_is_better", "steps", "warmup", "ms_per_step", "config", "cpu_baseline", "e2e"):
        assert key in rec, key
    assert rec["unit"] == "tokens/s" and rec["higher_is_better"] is True and "workload" in rec["config"]
    cb = rec["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == rec["value"]
    e2e = rec["e2e"]
    assert e2e["value"] == rec["value"] and e2e["unit"] == rec["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_layer_roofline_takes_the_slower_of_stream_and_contraction():
    # 18.9 MB at 6550 GB/s = 2.89 us; 64 rows x 75.5 MFLOP at 1670.9 TFLOP/s = 2.89 us
    eb, fr = 18_915_328, 2.0 * 3 * 6144 * 2048
    t_stream = eb / 6550.1e9 * 1e3
    t_row = fr / 1670.9e12 * 1e3
    assert bench.layer_roofline_ms([1], eb, fr, 6550.1, 1670.9) == pytest.approx(t_stream)
    assert bench.layer_roofline_ms([2048], eb, fr, 6550.1, 1670.9) == pytest.approx(2048 * t_row)
    assert bench.layer_roofline_ms([0, 1, 2048], eb, fr, 6550.1, 1670.9) == pytest.approx(t_stream + 2048 * t_row)
