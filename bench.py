#!/usr/bin/env python3
"""Benchmark of the routed-MoE layer on B200: GLM-5.2-shaped single-layer decode.

Workload (one "step" = one pass of the whole layer over one batch):
  T = 1 token, hidden 6144, 256 routed experts in 8 groups (topk_group 4),
  top-8, expert intermediate 2048, packed int4 weights with fp32 per-row
  scales (18,915,328 B per expert), one shared expert of the same shape,
  fp32 router N(0, 0.02^2), bias N(0, 0.1^2), rsf 2.5; all 257 experts
  resident in HBM (4.86 GB per layer).  Inputs are larger than L2: --layers
  independent layer replicas (default 8, 39 GB) stay resident and step i runs
  layer i mod --layers on a different seeded bf16 N(0,1) token, so every step
  reads weights last touched (layers - 1) steps (over 1 GB of traffic) before.

Arms:
  default           the CUDA path through the C ABI (moe_layer_forward)
  --impl reference  the CPU oracle (plain C, OpenMP) on the host cores, on a
                    bounded sample of the same workload

Prints ONE JSON line (rank 0).  Multi-GPU (torchrun): replicas only, each rank
runs its own copy of the layer; the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "routed-MoE layer tokens/s; int4 expert-weight GB/s vs ~8 TB/s HBM peak"
WORKLOAD = ("GLM-5.2-shaped single-layer decode: T=1, hidden 6144, 256 routed experts "
            "(8 groups, topk_group 4), top-8, intermediate 2048, packed int4 + fp32 row scales, "
            "1 shared expert, rsf 2.5")
NOMINAL_HBM_GBS = 8000.0


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            p = json.load(fh)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def tensor_peak():
    """Dense fp16/bf16 tensor TFLOP/s (same nominal rate): the measured cuBLAS bf16 burst figure."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            return float(json.load(fh)["bf16_tflops"]), "measured (cuBLAS bf16 burst)"
    except Exception:
        return 1590.0, "fallback"


KERNEL_SOURCES = ("decode_fused.cu", "common.cuh", "quant.cuh", "sm100_async.cuh")


def profiled_traffic():
    """DRAM bytes per launch of the fused kernel from the committed ncu capture
    (profiles/k_decode_fused_decode.json), or None when the kernel sources have
    changed since that capture."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "k_decode_fused_decode.json")) as fh:
            rec = json.load(fh)
        traffic, sha = int(rec["traffic_bytes_per_launch"]), rec["source_sha256"]
    except (OSError, KeyError, ValueError):
        return None
    return traffic if kernel_sources_sha256() == sha else None


def kernel_sources_sha256() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "quantized_mixture_experts_sigmoid_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=15000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--layers", type=int, default=8, help="resident layer replicas rotated per step")
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--pool", type=int, default=512, help="distinct seeded tokens cycled through")
    ap.add_argument("--prefill", type=int, default=10,
                    help="prefill layers (T = 2048) timed for the extra 'prefill' entry; 0 skips it")
    ap.add_argument("--prefill-tokens", type=int, default=2048, help="prefill batch size (profiling: smaller)")
    ap.add_argument("--prefill-experts", type=int, default=256,
                    help="routed experts of the prefill layer (profiling: 32, in 4 groups)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the verify and stacked entries (measured only on one GPU)")
    ap.add_argument("--clock-window", type=float, default=1.5,
                    help="seconds of the same decode loop, right after the timed steps, during which "
                         "clocks are sampled")
    ap.add_argument("--prefill-only", action="store_true",
                    help="run only the prefill measurement and print its entry (for profiler captures)")
    ap.add_argument("--layer-calls", default=None, metavar="CONFIG",
                    help="run only a few layer calls of a named workload (synth.CONFIGS; for profiler "
                         "captures) and print the path taken and the time per call")
    ap.add_argument("--layer-tokens", type=int, default=0, help="--layer-calls: tokens per call (0: the config's)")
    ap.add_argument("--layer-experts", type=int, default=0,
                    help="--layer-calls: routed experts (0: the config's; otherwise in 8 groups, top-4 groups)")
    ap.add_argument("--layer-reps", type=int, default=8, help="--layer-calls: calls made")
    return ap.parse_args()


# ---------------------------------------------------------------- CPU oracle
def oracle_sample(sh, seconds: float, first_token: int = 0, max_tokens: int | None = None):
    """Time the CPU oracle's full layer on successive seeded tokens for ~`seconds`."""
    from oracle import oracle as O
    from oracle.synth_inputs import oracle_experts

    W = synth.router_weight(sh)
    b = synth.router_bias(sh)
    shared = oracle_experts(sh, [0], shared=True)
    total, n, t = 0.0, 0, first_token
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    while (total < seconds or n == 0) and (max_tokens is None or n < max_tokens):
        x = synth.hidden_states(sh, tokens=[t])
        idx, _, _, _ = O.route(x, W, b, sh.n_group, sh.topk_group, sh.top_k, sh.rsf)
        routed = oracle_experts(sh, np.unique(idx))
        t0 = time.perf_counter()
        O.layer_forward(x, W, b, sh.n_group, sh.topk_group, sh.top_k, sh.rsf, routed, shared)
        total += time.perf_counter() - t0
        n += 1
        t += 1
    return dict(value=n * sh.T / total, unit="tokens/s", cores=threads, kind="oracle",
                sample=f"{n} decode tokens (T=1 layer calls, each routed afresh), "
                       f"{total:.1f} s of oracle time; weight generation excluded"), n, total


def layer_calls(args, moe, device_layer, to_dev_bf16):
    """A few back-to-back layer calls of one workload, one resident layer (profiler captures; the
    time per call includes the first call's one-time setup)."""
    import torch
    sh = synth.CONFIGS[args.layer_calls].with_(n_layers=1)
    if args.layer_tokens:
        sh = sh.with_(T=args.layer_tokens)
    if args.layer_experts:
        sh = sh.with_(E=args.layer_experts, n_group=8, topk_group=4)
    dev = device_layer(sh)
    x = to_dev_bf16(synth.hidden_states(sh, tokens=range(sh.T)))
    out = torch.empty(sh.T, sh.H, dtype=torch.bfloat16, device="cuda")
    ws = moe.workspace(moe.moe_layer_workspace_bytes(sh.T, dev["cfg"], dev["routed"], dev["shared"]))
    path = moe.moe_layer_path(sh.T, dev["cfg"], dev["routed"], dev["shared"])
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.layer_reps):
        moe.moe_layer_forward(x, dev["W"], dev["bias"], dev["cfg"], dev["routed"], dev["shared"], out, ws)
    e1.record()
    torch.cuda.synchronize()
    if moe.moe_workspace_status(ws) != 0:
        raise RuntimeError("device status error during the layer calls")
    return {"workload": f"{sh.name}: T={sh.T}, {sh.E} routed experts, {sh.qtype}-bit, one resident layer",
            "path": {moe.PATH_FUSED: "fused", moe.PATH_TENSOR_CORE: "tensor_core", moe.PATH_GENERAL: "general"}[path],
            "calls": args.layer_reps, "ms_per_call": e0.elapsed_time(e1) / max(args.layer_reps, 1),
            "device_GB": torch.cuda.max_memory_allocated() / 1e9}


def run_reference(args):
    _, rank, _ = rank_env()
    if rank != 0:  # the oracle runs once, on rank 0; the other ranks exit without work
        return
    sh = synth.CONFIGS["decode"]
    # one step = one token's full layer on the CPU oracle; warm-up and timed
    # tokens are capped so that the whole run stays within a few minutes
    if args.warmup > 0:
        oracle_sample(sh, 0.0, first_token=10_000, max_tokens=min(args.warmup, 3))
    cb, n, total = oracle_sample(sh, 120.0, first_token=0, max_tokens=args.steps)
    value = cb["value"]
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / max(n, 1), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int4xint8", "data": "synthetic",
            "config": {"workload": WORKLOAD, "T": sh.T, "cpu": "host cores"},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- clocks
# NVML clock-event reason bits (nvmlClocksEventReason*)
_REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
            0x80: "hw_power_brake_slowdown"}


class ClockSampler:
    """SM clock and clock-event reasons sampled every `period` seconds in a thread
    (NVML, in process); mark() labels the samples taken from then on."""

    def __init__(self, gpu: int, period: float = 0.002):
        self.gpu, self.period = gpu, period
        self.samples = []  # (label, sm_mhz, max_mhz, reasons bitmask)
        self.label = None
        self._stop = None

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:
            return self
        self._stop = threading.Event()

        def run():
            while not self._stop.is_set():
                try:
                    sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                    rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    if self.label is not None:
                        self.samples.append((self.label, sm, mx, rs))
                except Exception:
                    pass
                self._stop.wait(self.period)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()
        return self

    def mark(self, label):
        self.label = label

    def __exit__(self, *a):
        if self._stop is not None:
            self._stop.set()
            self._thread.join(timeout=2)

    def summary(self, labels):
        sel = [x for x in self.samples if x[0] in labels]
        reasons = set()
        for _, _, _, rs in sel:
            for bit, nm in _REASONS.items():
                if rs & bit:
                    reasons.add(nm)
        out = {"sm_mhz": statistics.median([x[1] for x in sel]) if sel else None,
               "sm_max_mhz": sel[0][2] if sel else None, "reasons": sorted(reasons),
               "samples": len(sel), "period_ms": self.period * 1e3}
        for lb in labels:
            out[f"samples_{lb}"] = sum(1 for x in sel if x[0] == lb)
        return out


# ---------------------------------------------------------------- CUDA arm
def rank_env():
    """(world size, rank, local rank) from the torchrun environment; (1, 0, 0) without it."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(value: float, world: int, device) -> float:
    """The largest of every rank's value (a device time): all ranks call it in the same order."""
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replicas_tokens_per_s(world: int, tokens_per_step: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput of `world` replicas, each running `steps` steps, timed by the slowest."""
    return world * tokens_per_step * steps / (max_ms / 1e3)


def layer_roofline_ms(rows_per_expert, expert_bytes: int, flops_per_row: float, hbm_gbs: float,
                      tensor_tflops: float) -> float:
    """Roofline time of a batch-union layer: every distinct expert (shared included) is read once
    and applied to its rows; each takes the longer of its weight stream at the HBM peak and its
    contractions at the tensor peak (experts with few rows are bandwidth-bound)."""
    t = 0.0
    for n in rows_per_expert:
        if n > 0:
            t += max(expert_bytes / (hbm_gbs * 1e9), n * flops_per_row / (tensor_tflops * 1e12))
    return t * 1e3


def prefill_measurement(args, moe, L, device_layer, to_dev_bf16):
    """The batch-union prefill layer (T = 2048, Zipf-skewed routing) on the tensor-core path:
    whole-layer tokens/s and the two expert GEMMs' share of the dense tensor roofline."""
    import ctypes

    import torch
    sh = synth.CONFIGS["prefill"]
    if args.prefill_tokens != sh.T or args.prefill_experts != sh.E:
        groups = 8 if args.prefill_experts >= 256 else 4
        sh = sh.with_(T=args.prefill_tokens, E=args.prefill_experts, n_group=groups, topk_group=groups // 2)
    dev = device_layer(sh)
    x = to_dev_bf16(synth.hidden_states(sh))
    out = torch.empty(sh.T, sh.H, dtype=torch.bfloat16, device="cuda")
    ws = moe.workspace(moe.moe_layer_workspace_bytes(sh.T, dev["cfg"], dev["routed"], dev["shared"]))
    path = moe.moe_layer_path(sh.T, dev["cfg"], dev["routed"], dev["shared"])
    stream = torch.cuda.current_stream()

    idx = torch.empty(sh.T, sh.top_k, dtype=torch.int32, device="cuda")

    def fwd():
        moe.moe_layer_forward(x, dev["W"], dev["bias"], dev["cfg"], dev["routed"], dev["shared"], out, ws, idx)

    for _ in range(3):
        fwd()
    torch.cuda.synchronize()
    reps = max(3, args.prefill)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        fwd()
    e1.record(stream)
    torch.cuda.synchronize()
    layer_ms = e0.elapsed_time(e1) / reps
    L.moe_profile_enable(1)
    for _ in range(reps):
        fwd()
    torch.cuda.synchronize()
    kms, kn = ctypes.c_double(0), ctypes.c_int(0)
    L.moe_profile_read(ctypes.byref(kms), ctypes.byref(kn))
    L.moe_profile_enable(0)
    if moe.moe_workspace_status(ws) != 0:
        raise RuntimeError("device status error during the prefill measurement")
    gemm_ms = kms.value / max(kn.value, 1)
    rows = sh.T * sh.top_k + sh.T  # (token, expert) pairs plus the shared expert's rows
    flops = 2.0 * rows * 3 * sh.H * sh.I  # up, gate and down contractions actually needed
    peak, kind = tensor_peak()
    achieved = flops / (gemm_ms / 1e3) / 1e12 if gemm_ms > 0 else None
    counts = np.bincount(idx.cpu().numpy().ravel(), minlength=sh.E).tolist() + [sh.T]  # routed experts + shared
    hbm, _ = peaks()
    roof_ms = layer_roofline_ms(counts, sh.expert_bytes(), 2.0 * 3 * sh.H * sh.I, hbm, peak)
    del ws, dev
    torch.cuda.empty_cache()
    return {
        "workload": f"prefill batch-union: T={sh.T}, GLM-5.2 layer shape ({sh.E} routed experts), "
                    "Zipf(1.1) expert popularity",
        "path": {moe.PATH_FUSED: "fused", moe.PATH_TENSOR_CORE: "tensor_core", moe.PATH_GENERAL: "general"}[path],
        "tokens_per_s": sh.T / (layer_ms / 1e3), "ms_per_layer": layer_ms, "layers_timed": reps,
        "distinct_experts": int(sum(1 for c in counts[:-1] if c > 0)),
        "layer_roofline": {"ms": roof_ms, "frac": roof_ms / layer_ms,
                           "definition": "sum over distinct experts (shared included) of max(expert bytes / "
                                         "measured HBM GB/s, rows x 2*3*H*I FLOP / measured dense TFLOP/s)"},
        "roofline": {"bound": "tensor", "kernel": "k_moe_gemm up/gate + down (both launches)",
                     "achieved": achieved, "peak": peak, "peak_kind": kind, "unit": "TFLOP/s",
                     "frac": achieved / peak if achieved else None, "flops_per_layer": flops,
                     "ms_per_layer_gemms": gemm_ms,
                     "flops_note": "2 x (T*top_k + T) x 3 x H x I: only the rows the layer needs; "
                                   "tile padding is not counted"},
    }


def call_roofline(path: str, call_bytes: float, call_ms: float, kernel_ms: float, hbm: float, kind: str) -> dict:
    """HBM roofline of one layer call's weight bytes.  On the fused path it is timed per launch of
    k_decode_fused (the whole layer); on the other paths the profiled region covers only some of
    the call's launches, so the whole call's time is used."""
    if path == "fused":
        ms, kernel, key = kernel_ms, "k_decode_fused", "ms_per_launch"
    else:
        ms, kernel, key = call_ms, f"whole layer call ({path} path, several launches)", "ms_per_call"
    achieved = call_bytes / (ms / 1e3) / 1e9
    return {"bound": "hbm", "kernel": kernel, "achieved": achieved, "peak": hbm, "peak_kind": kind,
            "unit": "GB/s", "frac": achieved / hbm, key: ms}


def verify_measurement(moe, L, device_layer, to_dev_bf16, name: str, n_layers: int = 4, steps: int = 200):
    """MTP verify (T = 4 correlated positions; int4 takes the fused kernel, int8 the general path):
    tokens/s, the realised batch unions, and the call's weight bytes against the HBM roofline."""
    import ctypes

    import torch
    sh = synth.CONFIGS[name]
    devs = [device_layer(sh, layer=l) for l in range(n_layers)]
    T, K = sh.T, sh.top_k
    n_calls = 64
    pool = to_dev_bf16(synth.hidden_states(sh, tokens=range(T * n_calls)))
    out = torch.empty(T, sh.H, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(steps, T, K, dtype=torch.int32, device="cuda")
    ws = moe.workspace(moe.moe_layer_workspace_bytes(T, devs[0]["cfg"], devs[0]["routed"], devs[0]["shared"]))
    path = moe.moe_layer_path(T, devs[0]["cfg"], devs[0]["routed"], devs[0]["shared"])

    def step(i):
        d = devs[i % n_layers]
        j = (i % n_calls) * T
        moe.moe_layer_forward(pool[j:j + T], d["W"], d["bias"], d["cfg"], d["routed"], d["shared"], out, ws,
                              idx[i % steps])

    for i in range(5):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(steps):
        step(i)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    L.moe_profile_enable(1)
    for i in range(steps):
        step(i)
    torch.cuda.synchronize()
    kms, kn = ctypes.c_double(0), ctypes.c_int(0)
    L.moe_profile_read(ctypes.byref(kms), ctypes.byref(kn))
    L.moe_profile_enable(0)
    if moe.moe_workspace_status(ws) != 0:
        raise RuntimeError(f"device status error during the {name} measurement")
    ids = idx.cpu().numpy()
    U = np.array([len(np.unique(ids[i])) for i in range(steps)])
    call_bytes = (U.mean() + 1) * sh.expert_bytes() + sh.router_bytes()
    k_ms = kms.value / max(kn.value, 1)
    hbm, kind = peaks()
    del devs, ws
    torch.cuda.empty_cache()
    return {
        "workload": f"MTP verify batch union: T={T} correlated positions, GLM-5.2 layer shape, "
                    f"{'int8' if sh.qtype == 8 else 'int4'} experts, {n_layers} resident layers rotated",
        "path": {moe.PATH_FUSED: "fused", moe.PATH_TENSOR_CORE: "tensor_core", moe.PATH_GENERAL: "general"}[path],
        "tokens_per_s": T / (ms / 1e3), "ms_per_call": ms,
        "distinct_experts": {"mean": float(U.mean()), "min": int(U.min()), "max": int(U.max())},
        "bytes_per_call": call_bytes, "GBps": call_bytes / (ms / 1e3) / 1e9,
        "roofline": call_roofline({moe.PATH_FUSED: "fused", moe.PATH_TENSOR_CORE: "tensor_core",
                                   moe.PATH_GENERAL: "general"}[path], call_bytes, ms, k_ms, hbm, kind),
    }


def topp_measurement(moe, L, device_layer, to_dev_bf16, top_p: float, n_layers: int = 4, steps: int = 2000):
    """Decode (T = 1) with adaptive expert top-p next to the same loop without it: tokens/s, the
    realised experts per token and the bytes the layer streams per token."""
    import ctypes

    import torch
    sh = synth.CONFIGS["decode"]
    devs = [device_layer(sh, layer=l) for l in range(n_layers)]
    pool = to_dev_bf16(synth.hidden_states(sh, tokens=range(512)))
    out = torch.empty(1, sh.H, dtype=torch.bfloat16, device="cuda")
    d0 = devs[0]
    ws = moe.workspace(moe.moe_layer_workspace_bytes(1, d0["cfg"], d0["routed"], d0["shared"]))
    res = {}
    for p in (1.0, top_p):
        cfgs = [moe.RouterCfg(d["cfg"].n_expert, d["cfg"].n_group, d["cfg"].topk_group, d["cfg"].top_k,
                              d["cfg"].routed_scaling_factor, p) for d in devs]
        idx = torch.empty(steps, sh.top_k, dtype=torch.int32, device="cuda")

        def step(i):
            d = devs[i % n_layers]
            moe.moe_layer_forward(pool[i % 512:i % 512 + 1], d["W"], d["bias"], cfgs[i % n_layers], d["routed"],
                                  d["shared"], out, ws, idx[i % steps])

        for i in range(5):
            step(i)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(steps):
            step(i)
        e1.record()
        torch.cuda.synchronize()
        if moe.moe_workspace_status(ws) != 0:
            raise RuntimeError("device status error during the top-p measurement")
        ms = e0.elapsed_time(e1) / steps
        kept = (idx.cpu().numpy() >= 0).sum(1)
        tok_bytes = float((kept.mean() + 1) * sh.expert_bytes() + sh.router_bytes())
        hbm, kind = peaks()
        res["p1" if p == 1.0 else "topp"] = {
            "top_p": p, "tokens_per_s": 1.0 / (ms / 1e3), "us_per_token": ms * 1e3,
            "experts_per_token": float(kept.mean()), "bytes_per_token": tok_bytes,
            "GBps": tok_bytes / (ms / 1e3) / 1e9, "frac_of_hbm_peak": tok_bytes / (ms / 1e3) / 1e9 / hbm,
            "peak_kind": kind}
    del devs, ws
    torch.cuda.empty_cache()
    res["workload"] = (f"GLM-5.2 decode (T=1), {n_layers} resident layers rotated, adaptive expert top-p "
                       f"{top_p} next to the same loop without it")
    res["bytes_saved"] = 1.0 - res["topp"]["bytes_per_token"] / res["p1"]["bytes_per_token"]
    res["speedup"] = res["topp"]["tokens_per_s"] / res["p1"]["tokens_per_s"]
    return res


def stacked_measurement(moe, device_layer, to_dev_bf16, name: str, Ts, reps: int = 10):
    """Stacked decode: all 16 layers resident, timed as one sequence of 16 layer calls (a token
    through the stack), fresh seeded hidden states per layer."""
    import torch
    sh = synth.CONFIGS[name]
    layers = [device_layer(sh, layer=l) for l in range(sh.n_layers)]
    entries = []
    for T in Ts:
        shT = sh.with_(T=T)
        xs = [to_dev_bf16(synth.hidden_states(shT, layer=l)) for l in range(sh.n_layers)]
        d0 = layers[0]
        ws = moe.workspace(moe.moe_layer_workspace_bytes(T, d0["cfg"], d0["routed"], d0["shared"]))
        out = torch.empty(T, sh.H, dtype=torch.bfloat16, device="cuda")
        idx = torch.empty(sh.n_layers, T, sh.top_k, dtype=torch.int32, device="cuda")
        path = moe.moe_layer_path(T, d0["cfg"], d0["routed"], d0["shared"])

        def sequence():
            for l in range(sh.n_layers):
                d = layers[l]
                moe.moe_layer_forward(xs[l], d["W"], d["bias"], d["cfg"], d["routed"], d["shared"], out, ws,
                                      idx[l])

        sequence()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            sequence()
        e1.record()
        torch.cuda.synchronize()
        if moe.moe_workspace_status(ws) != 0:
            raise RuntimeError(f"device status error during the {name} T={T} measurement")
        ms = e0.elapsed_time(e1) / reps
        ids = idx.cpu().numpy()
        U = np.array([len(np.unique(ids[l])) for l in range(sh.n_layers)])
        seq_bytes = float(((U + 1) * sh.expert_bytes() + sh.router_bytes()).sum())
        hbm, kind = peaks()
        entries.append({
            "workload": f"stacked decode: {sh.n_layers} resident GLM-5.2 layers "
                        f"({sh.n_layers * (sh.E + 1) * sh.expert_bytes() / 1e9:.1f} GB "
                        f"{'int2' if sh.qtype == 2 else 'int4'}), T={T}, one sequence of {sh.n_layers} layer calls",
            "path": {moe.PATH_FUSED: "fused", moe.PATH_TENSOR_CORE: "tensor_core", moe.PATH_GENERAL: "general"}[path],
            "tokens_per_s": T / (ms / 1e3), "ms_per_sequence": ms, "layer_calls_per_s": sh.n_layers / (ms / 1e3),
            "distinct_experts_per_layer": float(U.mean()), "bytes_per_sequence": seq_bytes,
            "GBps": seq_bytes / (ms / 1e3) / 1e9, "frac_of_hbm_peak": seq_bytes / (ms / 1e3) / 1e9 / hbm,
            "peak_kind": kind,
        })
        del ws, xs
    del layers
    torch.cuda.empty_cache()
    return entries


def run_cuda(args):
    import torch
    import torch.distributed as dist

    from quantized_mixture_experts_sigmoid_b200 import moe
    from synth.device import device_layer, to_dev_bf16

    if args.prefill_only:
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        print(json.dumps(prefill_measurement(args, moe, moe.lib(), device_layer, to_dev_bf16)), flush=True)
        return
    if args.layer_calls:
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        print(json.dumps(layer_calls(args, moe, device_layer, to_dev_bf16)), flush=True)
        return

    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    sh = synth.CONFIGS["decode"]
    NL = max(1, args.layers)
    devs = [device_layer(sh, layer=l) for l in range(NL)]
    T, H = sh.T, sh.H
    pool = synth.hidden_states(sh, tokens=range(rank * args.pool, (rank + 1) * args.pool))
    xs = to_dev_bf16(pool)  # [pool, H]: one distinct token per step, cycled
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(T, sh.top_k, dtype=torch.int32, device="cuda")
    wts = torch.empty(T, sh.top_k, dtype=torch.float32, device="cuda")
    ws = moe.workspace(moe.moe_layer_workspace_bytes(T, devs[0]["cfg"], devs[0]["routed"], devs[0]["shared"]))
    stream = torch.cuda.current_stream()

    def step(i):
        d = devs[i % NL]
        j = i % args.pool
        moe.moe_layer_forward(xs[j:j + 1], d["W"], d["bias"], d["cfg"], d["routed"], d["shared"], out, ws,
                              idx, wts)

    clk = ClockSampler(local).__enter__()
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if moe.moe_workspace_status(ws) != 0:
        raise RuntimeError("device status error during warm-up")

    # ---- device-resident timing: K back-to-back layer calls between two events
    L = moe.lib()
    import ctypes
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = L.moe_launch_count()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk.mark("timed")
    wall0 = time.perf_counter()
    ev0.record(stream)
    for i in range(args.steps):
        step(args.warmup + i)
    ev1.record(stream)
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    clk.mark(None)
    launches = L.moe_launch_count() - launches0
    dev_ms = ev0.elapsed_time(ev1)
    dev_ms = max_over_ranks(dev_ms, world, "cuda")
    if moe.moe_workspace_status(ws) != 0:
        raise RuntimeError("device status error during timing")

    # ---- clock window: the same back-to-back loop for at least `clock_window` seconds
    # right after the timed steps (which last about a millisecond at the driver's K, too
    # short to sample); its own tokens/s is reported next to the timed value
    clk.mark("window")
    cw_steps, cw_wall0 = 0, time.perf_counter()
    cw0, cw1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cw0.record(stream)
    while time.perf_counter() - cw_wall0 < args.clock_window:
        for i in range(500):
            step(args.warmup + args.steps + cw_steps + i)
        cw_steps += 500
        torch.cuda.synchronize()
    cw1.record(stream)
    torch.cuda.synchronize()
    clk.mark(None)
    cw_ms = cw0.elapsed_time(cw1)
    clk.__exit__(None, None, None)

    # ---- the dominant kernel's own duration: events around each launch (they also keep
    # consecutive launches from overlapping, so this is the standalone kernel time)
    prof_steps = min(args.steps, 2000) if args.steps >= 200 else 2000
    torch.cuda.synchronize()
    L.moe_profile_enable(1)
    for i in range(prof_steps):
        step(args.warmup + i)
    torch.cuda.synchronize()
    kms, kn = ctypes.c_double(0), ctypes.c_int(0)
    L.moe_profile_read(ctypes.byref(kms), ctypes.byref(kn))
    L.moe_profile_enable(0)

    # ---- end to end through the C ABI with host buffers (pinned), copies inside the timed region.
    # Each step copies its own token host -> device and its output row device -> host (one
    # copy each way per step).  The copies run on two side streams, in chunks of C steps
    # through rings of 2 C buffers: chunk j + 1's inputs cross while chunk j computes, and
    # the compute stream waits on the side streams once per chunk, so the layer kernels
    # otherwise run back to back.
    x_host = torch.from_numpy(pool.view(np.int16)).view(torch.bfloat16).pin_memory()
    C = 8
    e2e_steps = max(min(args.steps, 3000), 1000) // C * C
    out_host = torch.empty(e2e_steps, T, H, dtype=torch.bfloat16).pin_memory()
    x_ring = [torch.empty(T, H, dtype=torch.bfloat16, device="cuda") for _ in range(2 * C)]
    o_ring = [torch.empty(T, H, dtype=torch.bfloat16, device="cuda") for _ in range(2 * C)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]    # chunk's inputs are on the device
    ev_done = [torch.cuda.Event() for _ in range(2)]  # chunk's layers have run
    ev_out = [torch.cuda.Event() for _ in range(2)]   # chunk's outputs have left the device

    def h2d_chunk(j):
        b = j % 2
        with torch.cuda.stream(s_in):
            if j >= 2:
                s_in.wait_event(ev_done[b])  # chunk j - 2 has read these buffers
            for i in range(j * C, (j + 1) * C):
                r = (args.warmup + i) % args.pool
                x_ring[i % (2 * C)].copy_(x_host[r:r + 1], non_blocking=True)
            ev_in[b].record(s_in)

    n_chunks = e2e_steps // C
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h2d_chunk(0)
    for j in range(n_chunks):
        b = j % 2
        stream.wait_event(ev_in[b])
        if j >= 2:
            stream.wait_event(ev_out[b])  # chunk j - 2's outputs have left these buffers
        for i in range(j * C, (j + 1) * C):
            d = devs[i % NL]
            moe.moe_layer_forward(x_ring[i % (2 * C)], d["W"], d["bias"], d["cfg"], d["routed"], d["shared"],
                                  o_ring[i % (2 * C)], ws)
        ev_done[b].record(stream)
        if j + 1 < n_chunks:
            h2d_chunk(j + 1)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[b])
            for i in range(j * C, (j + 1) * C):
                out_host[i].copy_(o_ring[i % (2 * C)], non_blocking=True)
            ev_out[b].record(s_out)
    stream.wait_event(ev_out[(n_chunks - 1) % 2])
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_ms, world, "cuda")
    del devs, ws
    torch.cuda.empty_cache()

    extras = {}
    if world == 1 and not args.no_extras:
        extras["verify"] = verify_measurement(moe, L, device_layer, to_dev_bf16, "verify")
        extras["verify_int8"] = verify_measurement(moe, L, device_layer, to_dev_bf16, "verify_int8")
        extras["decode_topp"] = topp_measurement(moe, L, device_layer, to_dev_bf16, 0.7)
        extras["stacked"] = stacked_measurement(moe, device_layer, to_dev_bf16, "stacked", (1, 8))
        extras["stacked_int2"] = stacked_measurement(moe, device_layer, to_dev_bf16, "stacked_int2", (1,))
    prefill = prefill_measurement(args, moe, L, device_layer, to_dev_bf16) if args.prefill else None

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    ms_step = dev_ms / args.steps
    tok_s = replicas_tokens_per_s(world, T, args.steps, dev_ms)
    U = sh.top_k  # T = 1: every step touches top_k distinct routed experts
    expert_bytes = (U + 1) * sh.expert_bytes()
    layer_bytes = expert_bytes + sh.router_bytes()
    hbm_peak, peak_kind = peaks()
    # dominant kernel: the fused layer kernel, which streams every byte of the
    # step (router rows + the shared and top_k routed experts, scales included)
    dom_bytes = layer_bytes
    dom_ms = kms.value / max(kn.value, 1)
    dom_gbs = dom_bytes / (dom_ms / 1e3) / 1e9 if dom_ms > 0 else None
    clocks = clk.summary(("timed", "window"))
    clocks["window_s"] = cw_ms / 1e3
    clocks["window_tokens_per_s"] = T * cw_steps / (cw_ms / 1e3)
    line = {
        "metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int4xint8", "data": "synthetic",
        "config": {"workload": WORKLOAD, "T": T, "H": H, "I": sh.I, "E": sh.E, "top_k": sh.top_k,
                   "parallelism": f"replicas x{world}",
                   "l2": f"no flush; inputs larger than L2: {NL} resident layer replicas "
                         f"({NL * 257 * sh.expert_bytes() / 1e9:.0f} GB) rotated, a layer's weights "
                         f"are re-read after {NL - 1} other layers",
                   "tokens_cycled": args.pool, "layers_rotated": NL},
        "expert_weight_GBps": expert_bytes / (ms_step / 1e3) / 1e9,
        "layer_GBps": layer_bytes / (ms_step / 1e3) / 1e9,
        "layer_bytes_per_step": layer_bytes,
        "frac_of_8TBps": layer_bytes / (ms_step / 1e3) / 1e9 / NOMINAL_HBM_GBS,
        "roofline": {"bound": "hbm", "kernel": "k_decode_fused (whole layer, one launch)",
                     "achieved": dom_gbs, "peak": hbm_peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": (dom_gbs / hbm_peak) if dom_gbs else None, "traffic": profiled_traffic(),
                     "bytes_per_launch": dom_bytes, "ms_per_launch": dom_ms},
        "e2e": {"value": replicas_tokens_per_s(world, T, e2e_steps, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": T * H * 2, "d2h_bytes_per_step": T * H * 2, "steps": e2e_steps,
                "copies": "one per step each way, on side streams in chunks of 8 steps, rings of 16 buffers"},
        "gpu_launches": int(launches),
        "clocks": clocks,
        "wall_s_timed_region": wall,
    }
    line.update(extras)
    if prefill is not None:
        line["prefill"] = prefill
    if not args.no_cpu_baseline and world == 1:
        cb, _, _ = oracle_sample(sh, args.cpu_seconds)
        line["cpu_baseline"] = cb
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_cuda(args)


if __name__ == "__main__":
    main()
