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
DEFAULT_WORKLOAD = "ffn_175b_f0.001_t6"
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
    ap.add_argument("--no-per-config", action="store_true",
                    help="time only the headline workload")
    ap.add_argument("--cpu-budget-s", type=float, default=12.0)
    ap.add_argument("--quick", action="store_true",
                    help="few launches (for profilers): no clock sampling, short end-to-end "
                         "and per-kernel timings; the line's numbers are indicative only")
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
KERNEL_SOURCES = {"decode_kernel": ["decode.cu", "codes.cuh"], "gemm_kernel": ["gemm.cu"],
                  "rowquant_kernel": ["quant.cu", "codes.cuh"], "colmask_kernel": ["quant.cu", "codes.cuh"],
                  "gemv_kernel": ["gemv.cu", "codes.cuh"], "small_fused_kernel": ["small.cu", "codes.cuh"]}


def kernel_source_hash(kernel: str | None = None) -> str:
    """Hash of the sources of `kernel` (of every kernel source when None)."""
    h = hashlib.sha256()
    names = sorted(n for n in os.listdir(CSRC) if n.endswith((".cu", ".cuh")))
    if kernel in KERNEL_SOURCES:
        names = sorted(KERNEL_SOURCES[kernel] + ["kernels.cuh", "ptx.cuh"])
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
        # samples under load: power within half of the highest seen in the window (the window
        # opens and closes with a quarter second of idle GPU)
        pw = [num(r[3]) for r in rows]
        top = max([p for p in pw if p is not None], default=None)
        loaded = [r for r, p in zip(rows, pw) if top is None or (p is not None and p >= 0.5 * top)]
        if len(loaded) >= 3:
            rows = loaded
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
                         "host_cores": os.cpu_count(), "cpu_model": cpu_model(),
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
        return {"name": "decode", "launches": 1, "quantize": [], "kernel": "decode_kernel",
                "matmul": "decode_kernel (one launch: one CTA per 32 channels over all of K, X "
                          "statistics in every CTA, mma.sync int8 + fp16 outlier term)"}
    if M <= 16:
        if K % 128 == 0 and K <= 8192:
            return {"name": "few_tokens", "launches": 2, "quantize": ["few_quant_kernel"],
                    "kernel": "gemv_kernel",
                    "matmul": "gemv_kernel (mma.sync int8 + fp16 outlier term)"}
        return {"name": "cluster", "launches": 1, "quantize": [], "kernel": "small_fused_kernel",
                "matmul": "small_fused_kernel (tcgen05, one cluster per channel tile)"}
    return {"name": "tiled", "launches": 3, "quantize": ["colmask_kernel", "rowquant_kernel"],
            "kernel": "gemm_kernel",
            "matmul": "gemm_kernel (int8 + fp16 tcgen05, fused epilogue)"}


GRAPH_MIN_MS = 200.0  # replays per per-kernel timing (lowered by --quick)


def graph_time_ms(fn, n: int, device, min_ms: float | None = None) -> float:
    """Average device time of fn() replayed back to back from one CUDA graph of n calls, over
    at least `min_ms` of replays (CUDA events on the launching stream)."""
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
    a.record()
    g.replay()
    b.record()
    torch.cuda.synchronize()
    min_ms = GRAPH_MIN_MS if min_ms is None else min_ms
    reps = max(3, min(10000, int(min_ms / max(a.elapsed_time(b), 1e-3))))
    a.record()
    for _ in range(reps):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / (reps * n)
    del g
    return ms


def op_counts(w, n_out: int):
    """The method's own work: 2 M N (K - |O|) int8 operations and 2 M N |O| fp16 flops."""
    return 2.0 * w.M * w.N * (w.K - n_out), 2.0 * w.M * w.N * n_out


def tensor_roof_s(int8_ops: float, f16_flops: float, peaks) -> float:
    """Seconds the work takes at the tensor peaks: int8 at the int8 peak, fp16 at the fp16 one."""
    return int8_ops / (peaks["int8_tops"] * 1e12) + f16_flops / (peaks["f16_tflops"] * 1e12)


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


class Layer:
    """One workload resident in HBM: rotating copies of X, Wq, w_scale, bias, Y and workspace,
    enough that every step's operands have left L2 before they are read again."""

    def __init__(self, w, rank: int, device, l2: int):
        import torch
        import int8_mixed_precision_absmax_b200 as i8
        import synth
        self.w = w
        X_h, W_h, b_h, _ = synth.make_inputs(w, seed=w.seed + rank)
        self.X_h, self.b_h = X_h, b_h
        self.copies = max(1, math.ceil(2 * l2 / w.algorithmic_bytes))
        X0 = torch.from_numpy(X_h).to(device)
        Wq0, sw0 = i8.int8_quant_weight(torch.from_numpy(W_h).to(device))
        del W_h
        b0 = None if b_h is None else torch.from_numpy(b_h).to(device)
        c = self.copies
        self.Xs = [X0] + [X0.clone() for _ in range(c - 1)]
        self.Wqs = [Wq0] + [Wq0.clone() for _ in range(c - 1)]
        self.sws = [sw0] + [sw0.clone() for _ in range(c - 1)]
        self.bs = [b0] + [None if b0 is None else b0.clone() for _ in range(c - 1)]
        self.Ys = [torch.empty((w.M, w.N), dtype=torch.float16, device=device) for _ in range(c)]
        self.wss = [i8.new_workspace(w.M, w.N, w.K, device) for _ in range(c)]
        self.device = device
        self.path = forward_path(w.M, w.N, w.K)

    def step(self, i: int):
        import int8_mixed_precision_absmax_b200 as i8
        c = i % self.copies
        i8.int8_linear_forward(self.Xs[c], self.Wqs[c], self.sws[c], self.bs[c],
                               self.w.threshold, Y=self.Ys[c], workspace=self.wss[c])

    def estimate_ms(self) -> float:
        import torch
        for i in range(max(self.copies, 3)):
            self.step(i)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n = max(self.copies, 8)
        e0.record()
        for i in range(n):
            self.step(i)
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    def make_runner(self, steps: int, use_graph: bool):
        """run(n) launches n steps (n <= steps) from CUDA graphs of `copies` steps each."""
        import torch
        graphs = []
        if use_graph:
            try:
                chunk = self.copies if steps >= self.copies else steps
                sizes = [chunk] + ([steps % chunk] if steps % chunk else [])
                side = torch.cuda.Stream(self.device)
                side.wait_stream(torch.cuda.current_stream(self.device))
                with torch.cuda.stream(side):
                    for i in range(self.copies):
                        self.step(i)
                torch.cuda.current_stream(self.device).wait_stream(side)
                torch.cuda.synchronize()
                for n in sizes:
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g):
                        for i in range(n):
                            self.step(i)
                    graphs.append((g, n))
            except Exception as exc:  # capture unsupported: launch directly
                print(f"[bench] graph capture failed ({exc}); launching directly",
                      file=sys.stderr)
                graphs = []

        def run(n):
            if graphs:
                g, chunk = graphs[0]
                for _ in range(n // chunk):
                    g.replay()
                if n % chunk:
                    graphs[1][0].replay()
            else:
                for i in range(n):
                    self.step(i)
        run.graphs = graphs
        run.chunk = graphs[0][1] if graphs else 1
        return run

    def check_status(self):
        import torch
        import int8_mixed_precision_absmax_b200 as i8
        for ws in self.wss:
            st = i8.int8_read_device_status(ws[:4].view(torch.int32))
            if st != 0:
                raise SystemExit(f"device status {st}: {i8.int8_status_string(st)}")

    def outlier_count(self) -> int:
        import int8_mixed_precision_absmax_b200 as i8
        return int(i8.int8_quantize_rows(self.Xs[0], self.w.threshold)[3].item())

    def kernel_times(self):
        """(activation-side ms, product ms) per step, each replayed alone from its own graph."""
        import int8_mixed_precision_absmax_b200 as i8
        c = self.copies
        n = max(c, 32)
        if self.path["quantize"]:
            q_ms = graph_time_ms(lambda i: i8.int8_linear_quantize(
                self.Xs[i % c], self.Wqs[i % c], self.sws[i % c], self.w.threshold,
                self.wss[i % c]), n, self.device)
        else:
            q_ms = 0.0
        g_ms = graph_time_ms(lambda i: i8.int8_linear_matmul(
            self.Xs[i % c], self.Wqs[i % c], self.sws[i % c], self.bs[i % c], self.w.threshold,
            self.Ys[i % c], self.wss[i % c]), n, self.device)
        for i in range(c):  # leave every copy's Y from a complete forward
            self.step(i)
        return q_ms, g_ms

    def e2e(self, world: int, budget_s: float):
        """The same metric through the public call, with a pinned host->device copy of X and a
        device->host copy of Y inside every step.  The copies of neighbouring steps overlap the
        forward on their own streams (X and Y double-buffered on the device, two pinned Y
        buffers on the host), as a serving loop would run them: step i's Y goes back while
        step i+1 computes and step i+2's X comes in."""
        import torch
        w = self.w
        dev = self.device
        Xh = torch.from_numpy(self.X_h).pin_memory()
        Yh = [torch.empty((w.M, w.N), dtype=torch.float16).pin_memory() for _ in range(2)]
        Xd = [self.Xs[0], self.Xs[1] if self.copies > 1 else torch.empty_like(self.Xs[0])]
        Yd = [self.Ys[0], self.Ys[1] if self.copies > 1 else torch.empty_like(self.Ys[0])]
        s_in, s_run, s_out = (torch.cuda.Stream(dev) for _ in range(3))
        ev = lambda: torch.cuda.Event()
        import int8_mixed_precision_absmax_b200 as i8

        def run(n):
            x_free = [None, None]   # forward done with Xd[b]
            y_free = [None, None]   # Yd[b] copied out
            for i in range(n):
                b = i % 2
                with torch.cuda.stream(s_in):
                    if x_free[b] is not None:
                        s_in.wait_event(x_free[b])
                    Xd[b].copy_(Xh, non_blocking=True)
                    x_in = ev(); x_in.record(s_in)
                with torch.cuda.stream(s_run):
                    s_run.wait_event(x_in)
                    if y_free[b] is not None:
                        s_run.wait_event(y_free[b])
                    c = i % self.copies
                    i8.int8_linear_forward(Xd[b], self.Wqs[c], self.sws[c], self.bs[c],
                                           w.threshold, Y=Yd[b], workspace=self.wss[c],
                                           stream=s_run)
                    done = ev(); done.record(s_run)
                    x_free[b] = done
                with torch.cuda.stream(s_out):
                    s_out.wait_event(done)
                    Yh[b].copy_(Yd[b], non_blocking=True)
                    out = ev(); out.record(s_out)
                    y_free[b] = out
            for s_ in (s_in, s_run, s_out):
                torch.cuda.current_stream(dev).wait_stream(s_)
        def run_serial(n):  # one stream: copy in, forward, copy out, step after step
            for i in range(n):
                c = i % self.copies
                self.Xs[c].copy_(Xh, non_blocking=True)
                self.step(i)
                Yh[0].copy_(self.Ys[c], non_blocking=True)

        run(3)
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record()
        for s_ in (s_in, s_run, s_out):
            s_.wait_stream(torch.cuda.current_stream(dev))
        run(3)
        t1.record()
        torch.cuda.synchronize()
        est = t0.elapsed_time(t1) / 3
        n_e = int(max(5, min(20000, budget_s * 1e3 / max(est, 1e-3))))
        n_e = int(max_over_ranks(float(n_e), dev))
        barrier(dev)
        t0.record()
        for s_ in (s_in, s_run, s_out):  # no copy starts before t0
            s_.wait_stream(torch.cuda.current_stream(dev))
        run(n_e)
        t1.record()
        torch.cuda.synchronize()
        overlapped_s = max_over_ranks(t0.elapsed_time(t1) / 1e3, dev)
        # the one-stream schedule as well: for steps of a few microseconds the per-step host
        # work of three streams costs more than the overlap saves; report the faster schedule
        run_serial(3)
        torch.cuda.synchronize()
        barrier(dev)
        t0.record()
        run_serial(n_e)
        t1.record()
        torch.cuda.synchronize()
        serial_s = max_over_ranks(t0.elapsed_time(t1) / 1e3, dev)
        e2e_s = min(overlapped_s, serial_s)
        schedule = ("H2D of X, forward and D2H of Y on three streams, double-buffered"
                    if overlapped_s <= serial_s else
                    "H2D of X, forward and D2H of Y in turn on one stream")
        return {"value": whole_job_rate(w.ops, n_e, world, e2e_s) / 1e12, "unit": UNIT,
                "h2d_bytes_per_step": int(Xh.numel() * Xh.element_size()),
                "d2h_bytes_per_step": int(Yh[0].numel() * Yh[0].element_size()), "steps": n_e,
                "ms_per_step": e2e_s / n_e * 1e3, "schedule": schedule,
                "ms_per_step_overlapped": overlapped_s / n_e * 1e3,
                "ms_per_step_one_stream": serial_s / n_e * 1e3}

    def roofline(self, n_out: int, q_ms: float, g_ms: float, step_ms: float, peaks):
        """The product kernel against its roofline, and the whole step against the same."""
        w = self.w
        path = self.path
        few_tokens = path["name"] != "tiled"
        if few_tokens:
            # weight streaming: X (fp16) and Wq in, Y out -- the whole step is one kernel pair
            nbytes = w.algorithmic_bytes
            achieved = nbytes / (g_ms / 1e3) / 1e9
            peak = peaks["hbm_gbs"]
            return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                    "frac": achieved / peak, "frac_end_to_end": nbytes / (step_ms / 1e3) / 1e9 / peak,
                    "kernel": path["kernel"], "kernel_ms": g_ms, "quantize_ms": q_ms,
                    "algorithmic_bytes": nbytes,
                    "peak_source": f"{peaks['source']} HBM copy (burst)"}
        i8_ops, f16_flops = op_counts(w, n_out)
        t_roof = tensor_roof_s(i8_ops, f16_flops, peaks)
        work = i8_ops + f16_flops
        peak = work / t_roof / 1e12  # the int8/fp16 mix at the two peaks
        achieved = work / (g_ms / 1e3) / 1e12
        return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "frac_end_to_end": t_roof / (step_ms / 1e3),
                "kernel": path["kernel"], "kernel_ms": g_ms, "quantize_ms": q_ms,
                "int8_ops": i8_ops, "fp16_flops": f16_flops,
                "peak_source": (f"{peaks['source']}: int8 = bf16 burst x {INT8_OVER_BF16:g} "
                                f"({peaks['int8_tops']:.0f} TOPS), fp16 = bf16 burst "
                                f"({peaks['f16_tflops']:.0f} TFLOP/s); peak = the work's mix")}


def measure(layer, world: int, steps: int, warm: int, use_graph: bool, peaks, sampler=None,
            e2e_budget_s: float = 2.0):
    """Time exactly `steps` steps (after `warm` untimed ones and graph warm-up), the kernels
    apart, and the end-to-end variant; returns the numbers of one JSON entry."""
    import torch
    w = layer.w
    for i in range(max(warm, 1)):
        layer.step(i)
    torch.cuda.synchronize()
    run = layer.make_runner(steps, use_graph)
    for _ in range(2):
        run(min(steps, layer.copies))
    torch.cuda.synchronize()
    if sampler:
        # keep the GPU busy while the sampler starts, so the clocks it sees are those under load
        sampler.start()
        lead = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        lead[0].record()
        run(min(steps, layer.copies))
        lead[1].record()
        torch.cuda.synchronize()
        per = lead[0].elapsed_time(lead[1]) / min(steps, layer.copies)
        n_lead = int(max(1, min(1e6, 1000.0 / max(per, 1e-3))))  # about 1 s of steps
        for _ in range(max(1, n_lead // run.chunk)):
            run(run.chunk)
    barrier(layer.device)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    run(steps)
    t1.record()
    torch.cuda.synchronize()
    barrier(layer.device)
    clocks = sampler.stop() if sampler else None
    max_s = max_over_ranks(t0.elapsed_time(t1) / 1e3, layer.device)
    layer.check_status()
    run.graphs.clear()
    q_ms, g_ms = layer.kernel_times()
    n_out = layer.outlier_count()
    step_ms = max_s / steps * 1e3
    return {
        "value": whole_job_rate(w.ops, steps, world, max_s) / 1e12,
        "gbs": whole_job_rate(w.algorithmic_bytes, steps, world, max_s) / 1e9,
        "ms_per_step": step_ms, "steps": steps, "outlier_cols": n_out,
        "roofline": layer.roofline(n_out, q_ms, g_ms, step_ms, peaks),
        "e2e": layer.e2e(world, e2e_budget_s),
        "gpu_launches": layer.path["launches"] * steps,
        "clocks": clocks,
        "config": {"workload": w.name, "M": w.M, "K": w.K, "N": w.N, "threshold": w.threshold,
                   "bias": layer.b_h is not None, "outlier_cols": n_out,
                   "path": layer.path["name"],
                   "l2": f"{layer.copies} rotating copies of X, Wq, w_scale, Y and workspace "
                         f"({layer.copies * w.algorithmic_bytes / 2**20:.0f} MiB of operands, "
                         f"> 2 x L2)" if layer.copies > 1 else
                         f"operands ({w.algorithmic_bytes / 2**20:.0f} MiB) larger than 2 x L2"},
    }


# configurations reported beside the headline, each timed for at least this long
PER_CONFIG = ("decode_q_proj", "prefill_up_proj", "down_proj_13b")
PER_CONFIG_MIN_S = 1.0


def run_ours(args):
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
    props = torch.cuda.get_device_properties(device)
    l2 = int(getattr(props, "L2_cache_size", 0) or 126 * 2**20)
    peaks = load_peaks()
    peaks["int8_tops"] = peaks["bf16_tflops"] * INT8_OVER_BF16
    peaks["f16_tflops"] = peaks["bf16_tflops"]
    use_graph = not args.no_graph
    warm = max(args.warmup, 0)
    global GRAPH_MIN_MS
    if args.quick:
        GRAPH_MIN_MS = 5.0
    e2e_budget = 0.02 if args.quick else 2.0
    uuid = None
    try:
        uuid = "GPU-" + str(props.uuid)
    except Exception:
        uuid = None

    # ---- the headline: exactly --steps steps (default: about 2 s of device time)
    w = synth.WORKLOADS[args.workload]
    layer = Layer(w, rank, device, l2)
    est_ms = layer.estimate_ms()
    steps = args.steps if args.steps is not None else max(20, int(2000.0 / max(est_ms, 1e-3)))
    steps = int(max_over_ranks(float(steps), device))
    sampler = ClockSampler(uuid) if rank == 0 and not args.quick else None
    head = measure(layer, world, steps, warm, use_graph, peaks, sampler, e2e_budget_s=e2e_budget)
    head["roofline"]["traffic"] = recorded_traffic(w.name, layer.path["kernel"])

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        Wq_h = layer.Wqs[0].cpu().numpy()
        sw_h = layer.sws[0].cpu().numpy()
        rate, t, desc, threads, _ = oracle_sample_rate(w, layer.X_h, Wq_h, sw_h, layer.b_h,
                                                       args.cpu_budget_s)
        cpu = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
               "host_cores": os.cpu_count(), "cpu_model": cpu_model(),
               "sample": desc + f", {t:.1f} s; OpenMP over the sampled rows"}
    del layer
    torch.cuda.empty_cache()

    # ---- the other configurations: each timed for at least PER_CONFIG_MIN_S
    per_config = {}
    if not args.no_per_config:
        for name in PER_CONFIG:
            if name == w.name:
                continue
            pw = synth.WORKLOADS[name]
            pl = Layer(pw, rank, device, l2)
            p_est = pl.estimate_ms()
            p_steps = int(max_over_ranks(float(max(20, int(PER_CONFIG_MIN_S * 1e3 / max(p_est, 1e-3)))),
                                         device))
            r = measure(pl, world, p_steps, warm, use_graph, peaks, None,
                        e2e_budget_s=min(1.0, e2e_budget))
            r["roofline"]["traffic"] = recorded_traffic(pw.name, pl.path["kernel"])
            r.pop("clocks", None)
            per_config[name] = r
            del pl
            torch.cuda.empty_cache()

    if rank == 0:
        cfg = dict(head["config"])
        cfg["launch"] = "CUDA graph replay" if use_graph else "direct launches"
        cfg["parallelism"] = f"{world} independent replica(s), one per GPU"
        cfg["clocks_window"] = ("nvidia-smi every 200 ms over about 1 s of the same steps run "
                                "back to back just before the timed ones, and over the timed ones")
        if args.quick:
            cfg["quick"] = "profiling run: no clock sampling, short timings"
        line = {
            "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world,
            "steps": steps, "warmup": warm, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
            "data": "synthetic", "gbs": head["gbs"], "config": cfg,
            "roofline": head["roofline"], "cpu_baseline": cpu, "e2e": head["e2e"],
            "gpu_launches": head["gpu_launches"], "clocks": head["clocks"],
            "per_config": per_config,
        }
        print(json.dumps(line), flush=True)

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
