#!/usr/bin/env python
"""Throughput of the LLM.int8() linear-layer forward on B200, one process per GPU.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one int8_linear_forward over one batch of synthetic inputs already resident in
HBM: outlier-column detection, per-row activation quantization, the fp16 outlier
operands, the int8 and fp16 tensor-core products and the fused epilogue.  The weights are
quantized once before timing (the layer's one-time load step).  Each rank runs its own
replica of the layer on its own batch (no collective on the data path), so the work per
GPU is fixed as N grows ("weak" scaling) and the reported value is the whole job's rate:
all ranks' operations divided by the slowest rank's device time.

Rank 0 prints one JSON line.  `--impl reference` times the CPU oracle instead (rank 0
only), on a bounded sample of the same workload per step.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "int8_linear_forward effective TOPS (2·M·N·K/s) and GB/s vs B200 roofline"
UNIT = "TOPS"
DEFAULT_WORKLOAD = "decode_q_proj"
INT8_OVER_BF16 = 2.0  # nominal dense int8 : bf16 tensor throughput on B200 (4.5 : 2.25 PFLOP/s)
CSRC = os.path.join(ROOT, "int8_mixed_precision_absmax_b200", "csrc")


# ----------------------------------------------------------------------------- helpers

def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: enough for about 2 s of device time)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-graph", action="store_true", help="launch every step from Python")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=12.0)
    return ap.parse_args(argv)


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world: int, backend: str):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def max_over_ranks(value: float, device) -> float:
    """The maximum of `value` over all ranks (the value itself without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def whole_job_rate(units_per_rank_step: float, steps: int, world: int, max_seconds: float) -> float:
    """Units processed by all ranks per second of the slowest rank."""
    return units_per_rank_step * steps * world / max_seconds


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# the sources each timed kernel is built from (its own file and the shared headers)
KERNEL_SOURCES = {"decode_kernel": "decode.cu", "gemm_kernel": "gemm.cu",
                  "rowquant_kernel": "quant.cu", "colmask_kernel": "quant.cu",
                  "gemv_kernel": "gemv.cu", "small_fused_kernel": "small.cu"}


def kernel_source_hash(kernel: str | None = None) -> str:
    """Hash of the sources of `kernel` (of every kernel source when None)."""
    h = hashlib.sha256()
    names = sorted(n for n in os.listdir(CSRC) if n.endswith((".cu", ".cuh")))
    if kernel in KERNEL_SOURCES:
        names = sorted([KERNEL_SOURCES[kernel], "kernels.cuh", "ptx.cuh"])
    for name in names:
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if taken on the current kernels."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    e = rec.get(workload, {}).get(kernel)
    if not e or e.get("kernel_source_hash") != kernel_source_hash(kernel):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi sampling (every 200 ms) of the SM clock and throttle reasons."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_uuid: str | None):
        self.uuid = gpu_uuid
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "200"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.25)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"],
                    "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        smax = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(rows)}


# ----------------------------------------------------------------------------- oracle timing

def oracle_sample_rate(w, X, W_q, sw, bias, budget_s: float):
    """Time the CPU oracle on a bounded sample of the workload.

    The sample is a set of rows of X against a contiguous slice of the output channels,
    grown until one evaluation takes about `budget_s`.  Returns (TOPS, seconds, sample
    description, threads)."""
    import numpy as np
    import oracle
    rows_all = np.arange(w.M, dtype=np.int64)
    n_cols = min(w.N, 256)
    n_rows = 1
    t = 0.0
    while True:
        rows = rows_all[np.linspace(0, w.M - 1, n_rows).astype(np.int64)] if n_rows < w.M else rows_all
        t0 = time.perf_counter()
        oracle.linear_forward_rows(X, W_q[:n_cols], sw[:n_cols], None if bias is None else bias[:n_cols],
                                   w.threshold, rows)
        t = time.perf_counter() - t0
        if t >= budget_s / 4 or (n_rows == w.M and n_cols == w.N):
            break
        grow = max(2.0, min(8.0, (budget_s / 4) / max(t, 1e-4)))
        if n_cols < w.N:
            n_cols = min(w.N, int(n_cols * grow))
        else:
            n_rows = min(w.M, int(n_rows * grow))
    # one final evaluation sized to the budget; a problem the oracle finishes well inside it
    # is evaluated repeatedly
    scale = max(1.0, budget_s / max(t, 1e-6))
    if n_cols < w.N:
        n_cols = min(w.N, int(n_cols * scale))
    elif n_rows < w.M:
        n_rows = min(w.M, int(n_rows * scale))
    rows = rows_all[np.linspace(0, w.M - 1, n_rows).astype(np.int64)] if n_rows < w.M else rows_all
    passes = 0
    t0 = time.perf_counter()
    while True:
        oracle.linear_forward_rows(X, W_q[:n_cols], sw[:n_cols],
                                   None if bias is None else bias[:n_cols], w.threshold, rows)
        passes += 1
        t = time.perf_counter() - t0
        if t >= budget_s * 0.8 or n_rows < w.M or n_cols < w.N:
            break
    ops = 2.0 * len(rows) * n_cols * w.K * passes
    threads = min(os.cpu_count() or 1, len(rows))
    desc = (f"{len(rows)} of {w.M} rows x {n_cols} of {w.N} output channels "
            f"(K={w.K}, outlier set over all rows), {passes} pass(es)")
    return ops / t / 1e12, t, desc, threads, (len(rows), n_cols)


# ----------------------------------------------------------------------------- reference arm

def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import numpy as np
    import oracle
    import synth
    w = synth.WORKLOADS[args.workload]
    X, W, bias, _ = synth.make_inputs(w, seed=w.seed)
    Wq, sw = oracle.quant_weight(W)
    steps = args.steps if args.steps is not None else 5
    warm = max(args.warmup, 0)
    per_step_budget = max(0.05, min(10.0, 150.0 / max(1, steps + warm)))
    rate, t, desc, threads, (nr, nc) = oracle_sample_rate(w, X, Wq, sw, bias, per_step_budget)
    rows = np.linspace(0, w.M - 1, nr).astype(np.int64) if nr < w.M else np.arange(w.M)
    b = None if bias is None else bias[:nc]

    def one():
        oracle.linear_forward_rows(X, Wq[:nc], sw[:nc], b, w.threshold, rows)
    for _ in range(warm):
        one()
    t0 = time.perf_counter()
    for _ in range(steps):
        one()
    el = time.perf_counter() - t0
    ops = 2.0 * len(rows) * nc * w.K
    value = ops * steps / el / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": steps, "warmup": warm, "ms_per_step": el / steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64",
        "data": "synthetic",
        "config": {"workload": w.name, "M": w.M, "K": w.K, "N": w.N, "threshold": w.threshold,
                   "parallelism": "rank 0 only (CPU oracle)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": desc + f" per step, {steps} steps"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- our arm

def forward_path(M: int, N: int, K: int):
    """Which kernels one int8_linear_forward launches for this shape (the library's dispatch:
    api.cu with the plan functions of decode.cu, gemv.cu and small.cu)."""
    if M <= 8 and K % 128 == 0 and K <= 8192:
        return {"name": "decode", "launches": 1, "quantize": [],
                "matmul": "decode_kernel (one launch: one CTA per 32 channels over all of K, X "
                          "statistics in every CTA, mma.sync int8 + fp16 outlier term)"}
    if M <= 16:
        if K % 128 == 0 and K <= 8192:
            return {"name": "few_tokens", "launches": 2, "quantize": ["few_quant_kernel"],
                    "matmul": "gemv_kernel (mma.sync int8 + fp16 outlier term)"}
        return {"name": "cluster", "launches": 1, "quantize": [],
                "matmul": "small_fused_kernel (tcgen05, one cluster per channel tile)"}
    return {"name": "tiled", "launches": 3, "quantize": ["colmask_kernel", "rowquant_kernel"],
            "matmul": "gemm_kernel (int8 + fp16 tcgen05, fused epilogue)"}


def graph_time_ms(fn, n: int, device) -> float:
    """Average device time of fn() replayed back to back from one CUDA graph of n calls."""
    import torch
    side = torch.cuda.Stream(device)
    side.wait_stream(torch.cuda.current_stream(device))
    with torch.cuda.stream(side):
        for i in range(n):
            fn(i)
    torch.cuda.current_stream(device).wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(n):
            fn(i)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 10
    a.record()
    for _ in range(reps):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / (reps * n)
    del g
    return ms


def run_ours(args):
    import numpy as np
    import torch

    import int8_mixed_precision_absmax_b200 as i8
    import synth

    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the product path has no CPU fallback)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl")
    i8.load_library()

    w = synth.WORKLOADS[args.workload]
    X_h, W_h, b_h, _ = synth.make_inputs(w, seed=w.seed + rank)
    props = torch.cuda.get_device_properties(device)
    l2 = int(getattr(props, "L2_cache_size", 0) or 126 * 2**20)

    # inputs resident in HBM; enough rotating copies that each step's operands left L2
    step_bytes = w.algorithmic_bytes
    copies = max(1, math.ceil(2 * l2 / step_bytes))
    X0 = torch.from_numpy(X_h).to(device)
    Wq0, sw0 = i8.int8_quant_weight(torch.from_numpy(W_h).to(device))
    b0 = None if b_h is None else torch.from_numpy(b_h).to(device)
    Xs = [X0] + [X0.clone() for _ in range(copies - 1)]
    Wqs = [Wq0] + [Wq0.clone() for _ in range(copies - 1)]
    sws = [sw0] + [sw0.clone() for _ in range(copies - 1)]
    bs = [b0] + [None if b0 is None else b0.clone() for _ in range(copies - 1)]
    Ys = [torch.empty((w.M, w.N), dtype=torch.float16, device=device) for _ in range(copies)]
    wss = [i8.new_workspace(w.M, w.N, w.K, device) for _ in range(copies)]
    del W_h

    def step(i):
        c = i % copies
        i8.int8_linear_forward(Xs[c], Wqs[c], sws[c], bs[c], w.threshold, Y=Ys[c],
                               workspace=wss[c])

    warm = max(args.warmup, 0)
    for i in range(max(warm, 1)):
        step(i)
    torch.cuda.synchronize()

    # estimate the step time to size the default step count (about 2 s of device time)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    probe = max(copies, 8)
    e0.record()
    for i in range(probe):
        step(i)
    e1.record()
    torch.cuda.synchronize()
    est_ms = e0.elapsed_time(e1) / probe
    steps = args.steps if args.steps is not None else max(20, int(2000.0 / max(est_ms, 1e-3)))
    steps = int(max_over_ranks(float(steps), device))

    # CUDA graphs: one replay = `copies` consecutive steps, plus one for the remainder
    use_graph = not args.no_graph
    graphs = []
    if use_graph:
        try:
            chunk = copies if steps >= copies else steps
            sizes = [chunk] + ([steps % chunk] if steps % chunk else [])
            side = torch.cuda.Stream(device)
            side.wait_stream(torch.cuda.current_stream(device))
            with torch.cuda.stream(side):
                for i in range(copies):
                    step(i)
            torch.cuda.current_stream(device).wait_stream(side)
            torch.cuda.synchronize()
            for n in sizes:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    for i in range(n):
                        step(i)
                graphs.append((g, n))
        except Exception as exc:  # capture unsupported: fall back to direct launches
            print(f"[bench] graph capture failed ({exc}); launching directly", file=sys.stderr)
            graphs, use_graph = [], False

    def run_steps(n):
        if use_graph:
            g, chunk = graphs[0]
            for _ in range(n // chunk):
                g.replay()
            r = n % chunk
            if r:
                graphs[1][0].replay()
        else:
            for i in range(n):
                step(i)

    for _ in range(2):  # graph warm-up (the untimed warm-up steps above ran direct launches)
        run_steps(min(steps, copies))
    torch.cuda.synchronize()

    uuid = None
    try:
        uuid = "GPU-" + str(props.uuid)
    except Exception:
        uuid = None
    sampler = ClockSampler(uuid) if rank == 0 else None
    if sampler:
        sampler.start()
    barrier(device)
    torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_start.record()
    run_steps(steps)
    t_end.record()
    torch.cuda.synchronize()
    barrier(device)
    clocks = sampler.stop() if sampler else None
    elapsed_s = t_start.elapsed_time(t_end) / 1e3
    max_s = max_over_ranks(elapsed_s, device)

    for ws in wss:
        st = i8.int8_read_device_status(ws[:4].view(torch.int32))
        if st != 0:
            raise SystemExit(f"device status {st}: {i8.int8_status_string(st)}")

    value = whole_job_rate(w.ops, steps, world, max_s) / 1e12
    gbs = whole_job_rate(step_bytes, steps, world, max_s) / 1e9

    # ---- per-kernel durations, live: the activation side and the product, each replayed
    # back to back from its own CUDA graph over the rotating copies (CUDA events around the
    # replays, on the launching stream); the product reads what earlier steps left in each
    # copy's workspace
    path = forward_path(w.M, w.N, w.K)
    if path["quantize"]:
        q_ms = graph_time_ms(lambda i: i8.int8_linear_quantize(
            Xs[i % copies], Wqs[i % copies], sws[i % copies], w.threshold, wss[i % copies]),
            max(copies, 32), device)
    else:
        q_ms = 0.0
    g_ms = graph_time_ms(lambda i: i8.int8_linear_matmul(
        Xs[i % copies], Wqs[i % copies], sws[i % copies], bs[i % copies], w.threshold,
        Ys[i % copies], wss[i % copies]), max(copies, 32), device)
    for c in range(copies):  # leave every copy's Y from a complete forward
        step(c)
    torch.cuda.synchronize()

    peaks = load_peaks()
    tensor_bound = w.ops / step_bytes > (peaks["bf16_tflops"] * INT8_OVER_BF16 * 1e12) / (peaks["hbm_gbs"] * 1e9)
    # algorithmic bytes of the matmul kernel: its operands and output, each once
    n_out = int(i8.int8_quantize_rows(Xs[0], w.threshold)[3].item())
    pad = (n_out + 63) // 64 * 64 if n_out else 0
    few_tokens = w.M <= 16
    kernel = path["matmul"]
    if few_tokens:  # reads X (fp16) and Wq, writes Y
        gemm_bytes = (2 * w.M * w.K + w.N * w.K + 4 * w.N + 2 * w.M * w.N
                      + (2 * w.N if b_h is not None else 0))
    else:           # reads Xq, Wq and the fp16 outlier operands, writes Y
        gemm_bytes = (w.M * w.K + w.N * w.K + 4 * (w.M + w.N) + 2 * w.M * w.N
                      + 2 * pad * (w.M + w.N) + (2 * w.N if b_h is not None else 0))
    if tensor_bound:
        achieved = w.ops / (g_ms / 1e3) / 1e12
        peak = peaks["bf16_tflops"] * INT8_OVER_BF16
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "kernel": kernel,
                "kernel_ms": g_ms, "quantize_ms": q_ms,
                "peak_source": f"{peaks['source']} bf16 x {INT8_OVER_BF16:g} (int8:bf16 nominal)"}
    else:
        achieved = gemm_bytes / (g_ms / 1e3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "kernel": kernel,
                "kernel_ms": g_ms, "quantize_ms": q_ms, "algorithmic_bytes": gemm_bytes,
                "peak_source": f"{peaks['source']} HBM copy"}
    roof["traffic"] = recorded_traffic(w.name, kernel.split()[0])

    # ---- end to end through the public API: pinned H2D of X, forward, D2H of Y
    Xh = torch.from_numpy(X_h).pin_memory()
    Yh = torch.empty((w.M, w.N), dtype=torch.float16).pin_memory()
    n_e = max(10, min(steps, 2000))
    for i in range(3):
        Xs[0].copy_(Xh, non_blocking=True)
        step(0)
        Yh.copy_(Ys[0], non_blocking=True)
    torch.cuda.synchronize()
    barrier(device)
    e_a, e_b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_a.record()
    for i in range(n_e):
        c = i % copies
        Xs[c].copy_(Xh, non_blocking=True)
        step(c)
        Yh.copy_(Ys[c], non_blocking=True)
    e_b.record()
    torch.cuda.synchronize()
    e2e_s = max_over_ranks(e_a.elapsed_time(e_b) / 1e3, device)
    e2e = {"value": whole_job_rate(w.ops, n_e, world, e2e_s) / 1e12, "unit": UNIT,
           "h2d_bytes_per_step": int(Xh.numel() * Xh.element_size()),
           "d2h_bytes_per_step": int(Yh.numel() * Yh.element_size()), "steps": n_e}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        Wq_h = Wqs[0].cpu().numpy()
        sw_h = sws[0].cpu().numpy()
        rate, t, desc, threads, _ = oracle_sample_rate(w, X_h, Wq_h, sw_h, b_h, args.cpu_budget_s)
        cpu = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": desc + f", {t:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps,
            "warmup": warm, "ms_per_step": max_s / steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "gbs": gbs,
            "config": {"workload": w.name, "M": w.M, "K": w.K, "N": w.N,
                       "threshold": w.threshold, "bias": b_h is not None,
                       "outlier_cols": n_out,
                       "l2": f"{copies} rotating copies of X, Wq, w_scale, Y and workspace "
                             f"({copies * step_bytes / 2**20:.0f} MiB of operands > 2 x L2)",
                       "launch": "CUDA graph replay" if use_graph else "direct launches",
                       "path": path["name"],
                       "parallelism": f"{world} independent replica(s), one per GPU"},
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": path["launches"] * steps,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)

    graphs.clear()
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
