#!/usr/bin/env python3
"""Benchmark of C = ReLU(A . B) (fp16 in, fp32 accumulate, fp16 out) on B200.

One step = one full GEMM+ReLU over one problem whose operands are already
resident in HBM.  Prints ONE JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload square8192]
    python bench.py --impl reference ...     # the CPU oracle, timed on host cores

At N=1 the line also carries one record per other configuration of the
metric's workloads ("configs"), a back-to-back "sustained" run of the headline
kernel, and the measured host-link rates beside the end-to-end number.

Multi-GPU (torchrun, one process per GPU): by default one problem's M rows are
split over the ranks, rank r taking rows [floor(rM/G), floor((r+1)M/G)) with B
replicated, each rank running the unchanged kernel on its row block (strong
scaling, no collective in the timed step; C is stitched afterwards by an NCCL
all-gather, which --gather-c also times).  --parallel cols splits N instead:
rank r keeps the column block [c_r, c_{r+1}) of B (boundaries floor(rN/G)
rounded down to a multiple of 8) with A replicated, and C's column blocks are
stitched the same way.  --parallel replicas gives every rank its own
independent problem instead (weak scaling).  The timed region is
bracketed by barriers and the slowest rank's time is reported.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from tiled_dense_gemm_fp16_b200 import inputs  # noqa: E402

METRIC = "GEMM+ReLU TFLOP/s at 8192³ fp16 (1×B200) and % of dense FP16 tensor peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Sources of each kernel path; a committed ncu traffic figure is only
# reported while these are unchanged.
_CSRC = "tiled_dense_gemm_fp16_b200/csrc/"
KERNEL_SOURCES = {
    "tc": [_CSRC + "gemm_tc.cuh", _CSRC + "ptx.cuh"],
    "tc_edge": [_CSRC + "gemm_tc.cuh", _CSRC + "ptx.cuh"],
    "tc_pair": [_CSRC + "gemm_tc.cuh", _CSRC + "gemm_tc_pair.cuh", _CSRC + "ptx.cuh"],
    "tc_pair512": [_CSRC + "gemm_tc.cuh", _CSRC + "gemm_tc_pair.cuh", _CSRC + "ptx.cuh"],
    "skinny": [_CSRC + "gemm_skinny.cuh", _CSRC + "ptx.cuh"],
    "mxf8": [_CSRC + "gemm_mx.cuh", _CSRC + "ptx.cuh"],
    "nvf4": [_CSRC + "gemm_mx.cuh", _CSRC + "ptx.cuh"],
    "w4a16": [_CSRC + "gemm_w4a16.cuh", _CSRC + "ptx.cuh"],
    "rc": [_CSRC + "gemm_rc.cuh", _CSRC + "gemm_tc.cuh", _CSRC + "ptx.cuh"],
    "rc_ws": [_CSRC + "gemm_rc.cuh", _CSRC + "gemm_tc.cuh", _CSRC + "repack.cuh", _CSRC + "ptx.cuh"],
    "repack": [_CSRC + "repack.cuh", _CSRC + "gemm_tc.cuh", _CSRC + "gemm_tc_pair.cuh", _CSRC + "gemm_skinny.cuh",
               _CSRC + "ptx.cuh"],
}
E2E_MODE = "every step uploads its inputs and downloads its result; two buffer sets overlap the copies with the GEMM"
MX_METRIC = "MXFP8 block-scaled grouped GEMM TFLOP/s (1×B200) and % of dense FP8 tensor peak"
NVF4_METRIC = "NVF4 block-scaled grouped GEMM TFLOP/s (1×B200) and % of dense FP4 tensor peak"
W4_METRIC = "W4A16 GEMM+ReLU TFLOP/s (1×B200) and % of its roofline (HBM for decode, tensor for large M)"
PROFILES = os.path.join(ROOT, "profiles")
L2_BYTES = 126 * 1024 * 1024


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="square8192",
                    help="square8192 (the metric's workload), square4096, square256, skinny:<M>, ragged:<i>, "
                         "linear8192, mxf8_moe, mxf8_8192, nvf4_8192, nvf4_moe, w4a16_decode, w4a16_8192")
    ap.add_argument("--path", default="auto",
                    help="force a kernel path: auto, tc, tc_edge, skinny, tc_pair, tc_pair512, rc")
    ap.add_argument("--workspace", choices=["auto", "none"], default="auto",
                    help="auto: give the library the scratch bytes it asks for (repack path for "
                         "operands TMA cannot describe), allocated by torch outside the timed region")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU work of the oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--configs", default="all",
                    help="all: at N=1 also measure every other configuration of the metric's workloads "
                         "(square256 float and integer, square4096, skinny M=1/16/64, the three ragged shapes "
                         "with and without a workspace), one record each in the line's 'configs'; none: skip; "
                         "or a comma-separated list of their labels")
    ap.add_argument("--config-cpu-seconds", type=float, default=1.0,
                    help="target CPU work of each configuration's oracle sample")
    ap.add_argument("--sustained-seconds", type=float, default=2.0,
                    help="at N=1, also run the headline kernel back to back this long (0: skip)")
    ap.add_argument("--parallel", choices=["rows", "cols", "replicas"], default="rows",
                    help="N>1: rows = split one problem's M rows over the ranks with B replicated "
                         "(strong scaling); cols = split its N columns with A replicated (strong scaling); "
                         "replicas = every rank runs its own problem (weak scaling)")
    ap.add_argument("--gather-c", action="store_true",
                    help="rows or cols mode: also time the NCCL all-gather that stitches C on every rank")
    ap.add_argument("--cublas", action="store_true",
                    help="also time torch.relu(torch.matmul(A, B)) (cuBLAS) on the same operands, as context")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# Workload
# ---------------------------------------------------------------------------

def workload_problem(spec: str, rank: int = 0):
    """(name, M, N, K, A, B) for a workload spec; ranks > 0 draw their own problem."""
    name, _, sub = spec.partition(":")
    wl = inputs.WORKLOADS[name]
    problems = list(wl.shapes)
    idx = 0
    if name == "skinny":
        ms = [s[0] for s in problems]
        idx = ms.index(int(sub)) if sub else len(ms) - 1
    elif name == "ragged":
        idx = int(sub) if sub else 0
    M, N, K = problems[idx]
    if name == "linear8192":
        x, W, b = inputs.linear_operands(M, N, K, seed=wl.seed if rank == 0 else rank_seed(wl.seed, rank))
        return name, M, N, K, x, (W, b)
    if rank == 0:
        # Exactly the workload's own draw (the generator is advanced over earlier shapes).
        for i, ((m, n, k), A, B) in enumerate(wl.problems()):
            if i == idx:
                return f"{name}" + (f":{sub}" if sub else ""), m, n, k, A, B
    A, B = inputs.operands(M, N, K, wl.dist, seed=rank_seed(wl.seed, rank))
    return f"{name}" + (f":{sub}" if sub else ""), M, N, K, A, B


def describe(name, M, N, K):
    wl = inputs.WORKLOADS[name.partition(":")[0]]
    layout = ("x (M x K) row-major, weight stored N x K, fp16 bias, C row-major" if name == "linear8192"
              else "row-major A, B, C")
    return {"workload": name, "M": M, "N": N, "K": K, "dtype_in": "fp16", "accumulate": "fp32",
            "dtype_out": "fp16", "layout": layout, "values": wl.dist, "seed": wl.seed}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# Clock sampling (NVML) during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int, period_s: float = 0.001):
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: report that instead of clocks
            self.nvml = None
            self.error = str(e)

    def _run(self):
        nv = self.nvml
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append((mhz, reasons))
                self.reasons |= reasons & ~self.REASONS["gpu_idle"]
            except Exception:
                pass
            self._stop.wait(self.period)

    def start(self):
        if self.nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()

    def summary(self):
        if self.nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "error", "")}
        names = [k for k, bit in self.REASONS.items() if self.reasons & bit and k != "gpu_idle"]
        busy = [mhz for mhz, r in self.samples if not (r & self.REASONS["gpu_idle"])]
        return {"sm_mhz": statistics.median(busy) if busy else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples),
                "samples_under_load": len(busy), "period_ms": self.period * 1e3}


# ---------------------------------------------------------------------------
# ncu traffic figure (committed summary), valid only for unchanged sources
# ---------------------------------------------------------------------------

def _code_only(text: str) -> str:
    """Source text without comments and blank lines, so that a comment edit leaves the hash alone."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*$", "", line).rstrip() for line in text.splitlines())
    return "\n".join(line for line in lines if line.strip())


def kernel_source_sha(path_name: str):
    """Hash of the code (comments and blank lines dropped) of the sources a path's kernels come from."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES.get(path_name, []):
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def committed_traffic(path_name: str, workload: str):
    """DRAM bytes per launch from profiles/gemm_relu_<path>_<workload>.md, if still valid."""
    summary = os.path.join(PROFILES, f"gemm_relu_{path_name}_{workload.replace(':', '_m')}.md")
    if not os.path.exists(summary) or path_name not in KERNEL_SOURCES:
        return None
    text = open(summary).read()
    m_sha = re.search(r"kernel_source_sha:\s*([0-9a-f]+)", text)
    m_wl = re.search(r"traffic_workload:\s*(\S+)", text)
    m_b = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not (m_sha and m_b and m_wl) or m_sha.group(1) != kernel_source_sha(path_name) or m_wl.group(1) != workload:
        return None
    return float(m_b.group(1))


# ---------------------------------------------------------------------------
# CPU baseline: the oracle as it stands, on a bounded sample of rows
# ---------------------------------------------------------------------------

def _oracle_rows_time(oracle, A, B, rows, cores):
    t0 = time.perf_counter()
    oracle.gemm_relu_f16_rows(A, B, np.arange(rows), nthreads=cores)
    return time.perf_counter() - t0


def _rows_for_budget(oracle, A, B, cores, budget_s):
    """Rows of C the oracle computes in about budget_s seconds.

    Doubles a probe sample until it takes a quarter of the budget (so the
    fixed cost of widening B is a small share), then scales linearly.
    """
    M = A.shape[0]
    rows = max(1, min(M, cores))
    t = _oracle_rows_time(oracle, A, B, rows, cores)
    while t < budget_s / 4 and rows < M:
        rows = min(M, rows * 2)
        t = _oracle_rows_time(oracle, A, B, rows, cores)
    rows = int(rows * budget_s / max(t, 1e-6))
    if rows >= cores:
        rows = (rows // cores) * cores
    return max(1, min(M, rows))


def pipelined_e2e(dev, compute_stream, hosts, make_inputs, out_shape, out_dtype, call, steps):
    """End-to-end time per step through the library call, with every step's inputs copied from
    pinned host memory and its result copied back.  Two device buffer sets let step i+1's
    uploads (copy stream) and step i-1's download (second copy stream) overlap step i's GEMM;
    events order each set's reuse.  Returns milliseconds per step (steps after one untimed step)."""
    import torch
    sets = [make_inputs() for _ in range(2)]
    outs = [torch.empty(out_shape, dtype=out_dtype, device=dev) for _ in range(2)]
    houts = [torch.empty(out_shape, dtype=out_dtype).pin_memory() for _ in range(2)]
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event(enable_timing=False)
    freed = [None, None]          # set k may be overwritten once its GEMM and download are done
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for i in range(steps + 1):
        k = i % 2
        if i == 1:
            start.record(up)
        if freed[k] is not None:
            up.wait_event(freed[k])
        with torch.cuda.stream(up):
            for d_, h_ in zip(sets[k], hosts):
                d_.copy_(h_, non_blocking=True)
        loaded = ev()
        loaded.record(up)
        compute_stream.wait_event(loaded)
        with torch.cuda.stream(compute_stream):
            call(*sets[k], outs[k])
        done = ev()
        done.record(compute_stream)
        down.wait_event(done)
        with torch.cuda.stream(down):
            houts[k].copy_(outs[k], non_blocking=True)
        fin = ev()
        fin.record(down)
        freed[k] = fin
    end.record(down)
    torch.cuda.synchronize(dev)
    return start.elapsed_time(end) / steps


def cpu_baseline(A, B, target_s: float):
    import oracle
    cores = os.cpu_count() or 1
    N = B.shape[1]
    K = A.shape[1]
    rows = _rows_for_budget(oracle, A, B, cores, target_s)
    dt = _oracle_rows_time(oracle, A, B, rows, cores)
    flops = inputs.flops(rows, N, K)
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"rows 0..{rows - 1} of C ({rows} x {N} x {K}), {dt:.1f} s on {cores} threads",
            "seconds": dt}


# ---------------------------------------------------------------------------
# Reference arm: the oracle on host cores, per step a bounded row sample
# ---------------------------------------------------------------------------

def run_reference_variant(args):
    """The oracle on a bounded sample of a block-scaled or W4A16 workload (rank 0 only)."""
    import oracle
    cores = os.cpu_count() or 1
    budget = 120.0 / max(1, args.steps + args.warmup)
    if args.workload in inputs.W4_WORKLOADS:
        M, N, K, group, seed = inputs.W4_WORKLOADS[args.workload]
        A, Wq, S = inputs.w4_operands(M, N, K, group, seed, "uniform")
        metric, shape = W4_METRIC, (M, N, K)
        run = lambda rows: oracle.gemm_relu_w4a16(A[:rows], Wq, S, group, nthreads=cores)
        limit = M
        config = {"workload": args.workload, "M": M, "N": N, "K": K, "group": group, "seed": seed}
    else:
        kind = "mxf8" if args.workload in inputs.MX_WORKLOADS else "nvf4"
        m_sizes, N, K, seed = (inputs.MX_WORKLOADS if kind == "mxf8" else inputs.NVF4_WORKLOADS)[args.workload]
        ops = (inputs.mx_operands(list(m_sizes), N, K, seed, "normal") if kind == "mxf8"
               else inputs.nvf4_operands(list(m_sizes), N, K, seed, "codes"))
        A, SFA, B, SFB = ops
        fn = oracle.gemm_mxf8_grouped if kind == "mxf8" else oracle.gemm_nvf4_grouped
        metric, shape = (MX_METRIC if kind == "mxf8" else NVF4_METRIC), (sum(m_sizes), N, K)
        run = lambda rows: fn(A[:rows], SFA[:rows], B[:1], SFB[:1], [rows], [0], N, K, nthreads=cores)
        limit = m_sizes[0]
        config = {"workload": args.workload, "groups": len(m_sizes), "m_sizes": list(m_sizes), "N": N, "K": K,
                  "seed": seed}
    rows = 1
    while True:
        t0 = time.perf_counter()
        run(rows)
        dt = time.perf_counter() - t0
        if dt >= budget or rows >= limit:
            break
        rows = min(limit, max(rows * 2, int(rows * budget / max(dt, 1e-3) * 0.9)))
    for _ in range(args.warmup):
        run(rows)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        run(rows)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = inputs.flops(rows, shape[1], shape[2]) * args.steps / total / 1e12
    sample = f"each step computes {rows} rows of group 0 ({rows} x {shape[1]} x {shape[2]}) with the CPU oracle"
    line = {
        "impl": "reference", "metric": metric, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 sum (oracle)",
        "data": "synthetic", "config": config,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    if (args.workload in inputs.MX_WORKLOADS or args.workload in inputs.NVF4_WORKLOADS
            or args.workload in inputs.W4_WORKLOADS):
        return run_reference_variant(args)
    import oracle
    name, M, N, K, A, B = workload_problem(args.workload)
    cores = os.cpu_count() or 1
    # Each step computes `rows` rows of C; sized so that warmup + steps fit a few minutes.
    budget = 120.0 / max(1, args.steps + args.warmup)
    rows = _rows_for_budget(oracle, A, B, cores, budget)
    sel = np.arange(rows)
    for _ in range(args.warmup):
        oracle.gemm_relu_f16_rows(A, B, sel, nthreads=cores)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.gemm_relu_f16_rows(A, B, sel, nthreads=cores)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = inputs.flops(rows, N, K) * args.steps / total / 1e12
    sample = f"each step computes rows 0..{rows - 1} of C ({rows} x {N} x {K}) with the CPU oracle"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32-accumulate f16",
        "data": "synthetic", "config": describe(name, M, N, K),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# Multi-rank plumbing (also exercised by CPU tests with the gloo backend)
# ---------------------------------------------------------------------------

def max_over_ranks(dist, value: float, device) -> float:
    """The largest of every rank's `value` (all ranks take part)."""
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t[0])


def aggregate_throughput(world: int, flops_per_rank: int, slowest_ms: float) -> float:
    """Whole-job TFLOP/s: every rank's independent problem over the slowest rank's step time."""
    return world * flops_per_rank / (slowest_ms * 1e-3) / 1e12


def rank_seed(workload_seed: int, rank: int) -> int:
    """Seed of rank `rank`'s own problem (rank 0 draws the workload itself)."""
    return workload_seed * 1000 + rank


# ---------------------------------------------------------------------------
# Our arm
# ---------------------------------------------------------------------------

# ---------------------------------------------------------------------------
# Row partition of one problem over ranks (also exercised by CPU gloo tests)
# ---------------------------------------------------------------------------

def row_range(M: int, world: int, rank: int):
    """Rows [r0, r1) of C (and of A) that rank `rank` of `world` computes: floor(r*M/G) .. floor((r+1)*M/G)."""
    return (rank * M) // world, ((rank + 1) * M) // world


def col_range(N: int, world: int, rank: int):
    """Columns [c0, c1) of C (and of B) that rank `rank` of `world` computes: the boundaries
    floor(r*N/G) rounded down to a multiple of 8 (so every block of a row-major B or C starts on a
    16-byte boundary), the last one N."""
    def bound(r):
        return N if r >= world else ((r * N // world) // 8) * 8
    return bound(rank), bound(rank + 1)


def gather_cols(dist, block, N: int, world: int, rank: int):
    """All-gather every rank's column block of C (M x (c1 - c0), row-major) into the full M x N C.
    Blocks are padded to the widest so the collective moves equal sizes; the padding is dropped
    when stitching.  Works on CPU tensors (gloo) and CUDA tensors (NCCL)."""
    import torch
    cols = [col_range(N, world, r) for r in range(world)]
    widest = max(c1 - c0 for c0, c1 in cols)
    M = block.shape[0]
    padded = torch.zeros((M, widest), dtype=block.dtype, device=block.device)
    padded[:, : block.shape[1]].copy_(block)
    parts = [torch.empty_like(padded) for _ in range(world)]
    dist.all_gather(parts, padded)
    return torch.cat([parts[r][:, : c1 - c0] for r, (c0, c1) in enumerate(cols)], dim=1)


def gather_rows(dist, block, M: int, world: int, rank: int):
    """All-gather every rank's row block of C into the full M x N C (row-major, rank order).

    Blocks differ by at most one row; each is padded to the largest so that the
    collective moves equal sizes, and the padding is dropped when stitching.
    Works on CPU tensors (gloo) and CUDA tensors (NCCL)."""
    import torch
    rows = [row_range(M, world, r) for r in range(world)]
    most = max(r1 - r0 for r0, r1 in rows)
    N = block.shape[1]
    padded = torch.zeros((most, N), dtype=block.dtype, device=block.device)
    padded[: block.shape[0]].copy_(block)
    parts = [torch.empty_like(padded) for _ in range(world)]
    dist.all_gather(parts, padded)
    return torch.cat([parts[r][: r1 - r0] for r, (r0, r1) in enumerate(rows)], dim=0)


# ---------------------------------------------------------------------------
# Roofline, host link, L2 hygiene
# ---------------------------------------------------------------------------

def roofline_for(M, N, K, kernel_ms, peaks, peak_src, sustained=False):
    """Roofline record of one fp16 GEMM: the bound is whichever roof its arithmetic
    intensity (2MNK flops over the compulsory 2(MK+KN+MN) bytes) meets first."""
    flops = inputs.flops(M, N, K)
    nbytes = inputs.min_bytes(M, N, K)
    tkey = "bf16_tflops_sustained" if sustained and "bf16_tflops_sustained" in peaks else "bf16_tflops"
    t_peak, h_peak = float(peaks[tkey]), float(peaks["hbm_gbs"])
    ridge = t_peak * 1e12 / (h_peak * 1e9)
    intensity = flops / nbytes
    if intensity >= ridge:
        achieved = flops / (kernel_ms * 1e-3) / 1e12
        rec = {"bound": "tensor", "achieved": achieved, "peak": t_peak, "unit": "TFLOP/s",
               "peak_source": f"{peak_src} cuBLAS bf16 {'sustained' if 'sustained' in tkey else 'burst'} peak "
                              f"(fp16 kind::f16 runs at the bf16 rate)"}
    else:
        achieved = nbytes / (kernel_ms * 1e-3) / 1e9
        rec = {"bound": "hbm", "achieved": achieved, "peak": h_peak, "unit": "GB/s",
               "peak_source": f"{peak_src} STREAM-copy HBM bandwidth"}
    rec["frac"] = rec["achieved"] / rec["peak"]
    rec["intensity_flop_per_byte"] = intensity
    rec["ridge_flop_per_byte"] = ridge
    rec["kernel_ms"] = kernel_ms
    return rec


def host_link(dev, h2d_bytes: int, d2h_bytes: int, reps: int = 5):
    """Measured pinned-host <-> device copy bandwidth (GB/s) for copies of the e2e leg's sizes: the
    best of `reps` timed copies after one untimed copy (the first touch of fresh pinned pages)."""
    import torch
    out = {}
    for name, nbytes in (("h2d", h2d_bytes), ("d2h", d2h_bytes)):
        n = max(1, nbytes)
        host = torch.empty(n, dtype=torch.uint8).pin_memory()
        devb = torch.empty(n, dtype=torch.uint8, device=dev)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        best = None
        for _ in range(reps + 1):
            torch.cuda.synchronize(dev)
            ev0.record()
            if name == "h2d":
                devb.copy_(host, non_blocking=True)
            else:
                host.copy_(devb, non_blocking=True)
            ev1.record()
            torch.cuda.synchronize(dev)
            ms = ev0.elapsed_time(ev1)
            if _ > 0:
                best = ms if best is None else min(best, ms)
        out[name + "_gbs"] = n / (best * 1e-3) / 1e9
        del host, devb
    # Both directions at once, as an e2e step runs them (upload on one copy
    # engine, download on the other): their shared link can be slower than
    # either alone.
    hin = torch.empty(max(1, h2d_bytes), dtype=torch.uint8).pin_memory()
    hout = torch.empty(max(1, d2h_bytes), dtype=torch.uint8).pin_memory()
    din = torch.empty(max(1, h2d_bytes), dtype=torch.uint8, device=dev)
    dout = torch.empty(max(1, d2h_bytes), dtype=torch.uint8, device=dev)
    s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    best = None
    for i in range(reps + 1):
        torch.cuda.synchronize(dev)
        ev0 = torch.cuda.Event(enable_timing=True)
        e_up, e_down = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record()
        s_up.wait_event(ev0)
        s_down.wait_event(ev0)
        with torch.cuda.stream(s_up):
            din.copy_(hin, non_blocking=True)
            e_up.record(s_up)
        with torch.cuda.stream(s_down):
            hout.copy_(dout, non_blocking=True)
            e_down.record(s_down)
        torch.cuda.synchronize(dev)
        ms = max(ev0.elapsed_time(e_up), ev0.elapsed_time(e_down))
        if i > 0:
            best = ms if best is None else min(best, ms)
    out["both_ms"] = best
    del hin, hout, din, dout
    return out


def operand_sets(torch, dev, tensors, work_bytes: int):
    """Device operand sets for timing: operands well beyond L2 are used as they are; mid-size ones
    rotate over R identical copies (R x working set >= 3 x L2) so every step reads cold operands;
    tiny ones get an L2 flush buffer (a write of twice the L2 size between timed steps)."""
    sets = [tuple(tensors)]
    flush = None
    if work_bytes <= 2 * L2_BYTES:
        R = -(-3 * L2_BYTES // max(1, work_bytes))
        if R <= 64:
            for _ in range(R - 1):
                sets.append(tuple(t.clone() for t in tensors))
        else:
            flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.int32, device=dev)
    note = ("inputs larger than L2" if work_bytes > 2 * L2_BYTES else
            f"rotating {len(sets)} operand copies ({len(sets) * work_bytes / 2**20:.0f} MiB > 3x L2)"
            if flush is None else "L2 flushed between timed steps")
    return sets, flush, note


def repack_launches(tg, M, N, K, a_ptr, b_ptr, c_ptr, chosen, ws_bytes=0) -> int:
    """Kernels one call launches: the GEMM, plus on the repack path one row-padding copy per operand TMA
    cannot describe and, when the GEMM writes a padded C (rows of C not 16-byte aligned, M > 256), the
    copy that moves it into C; on the residue-class path with a workspace, the copy of B when TMA cannot
    describe B."""
    n = 1
    b_unaligned = N % 8 != 0 or b_ptr % 16 != 0
    if chosen == tg.Path.REPACK:
        n += int(K % 8 != 0 or a_ptr % 16 != 0) + int(b_unaligned)
        n += int((N % 8 != 0 or c_ptr % 16 != 0) and M > 256)
    elif chosen == tg.Path.RC and ws_bytes > 0:
        n += int(b_unaligned)
    return n


def timed_region(torch, dev, stream, step, steps, flush, dist=None, clock_period_s=0.001):
    """Mean device time per step (ms) of `steps` calls of step() on `stream`, bracketed by a barrier and a
    synchronize on both sides, with NVML clocks sampled during the region.  With an L2 flush buffer, each
    step gets its own event pair so the flush stays outside the timed steps; otherwise one pair around
    the region (tiny kernels are not charged for event records)."""
    per_step = flush is not None
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps if per_step else 0)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps if per_step else 0)]
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index if dev.index is not None else 0, clock_period_s)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    with torch.cuda.stream(stream):
        r0.record(stream)
        for i in range(steps):
            if per_step:
                flush.fill_(1)
                starts[i].record(stream)
            step()
            if per_step:
                ends[i].record(stream)
        r1.record(stream)
    torch.cuda.synchronize(dev)
    sampler.stop()
    if dist is not None:
        dist.barrier()
    if per_step:
        ms = sum(a.elapsed_time(b) for a, b in zip(starts, ends)) / steps
    else:
        ms = r0.elapsed_time(r1) / steps
    return ms, sampler.summary()


class Fp16Case:
    """One fp16 GEMM+ReLU problem resident in HBM, called through the C ABI.

    mode "auto": tg_gemm_relu_f16_ws with the scratch bytes the library asks for (allocated by torch
    outside the timed region); "none": tg_gemm_relu_f16, no workspace; "linear": tg_gemm_relu_f16_ex with
    the weight stored N x K and a bias."""

    def __init__(self, tg, torch, dev, stream, M, N, K, A, B, mode="auto", path=None, bias=None):
        self.tg, self.torch, self.dev, self.stream = tg, torch, dev, stream
        self.M, self.N, self.K, self.mode = M, N, K, mode
        self.A_host, self.B_host = A, B
        Ad, Bd = torch.from_numpy(A).to(dev), torch.from_numpy(B).to(dev)
        Cd = torch.empty((M, N), dtype=torch.float16, device=dev)
        self.bias_d = torch.from_numpy(bias).to(dev) if bias is not None else None
        self.sets, self.flush, self.l2_note = operand_sets(torch, dev, (Ad, Bd, Cd), inputs.min_bytes(M, N, K))
        self.path = tg.Path.AUTO if path is None else path
        self.ws_bytes = 0
        if mode == "auto" and self.path == tg.Path.AUTO:
            self.ws_bytes = max(tg.workspace_size(a.data_ptr(), b.data_ptr(), c.data_ptr(), M, N, K)
                                for a, b, c in self.sets)
        self.ws = torch.empty(max(self.ws_bytes, 1), dtype=torch.uint8, device=dev)
        self.opts = (tg.options(b_layout=tg.B_NK, bias=self.bias_d.data_ptr()) if mode == "linear" else None)
        a, b, c = self.sets[0]
        if mode == "linear":
            self.chosen = tg.select_path_ex(a.data_ptr(), b.data_ptr(), c.data_ptr(), M, N, K, self.opts, 0)
        elif self.path != tg.Path.AUTO:
            self.chosen = self.path
        else:
            self.chosen = tg.select_path_ws(a.data_ptr(), b.data_ptr(), c.data_ptr(), M, N, K, self.ws_bytes)
        self.launches_per_step = repack_launches(tg, M, N, K, a.data_ptr(), b.data_ptr(), c.data_ptr(), self.chosen,
                                                 self.ws_bytes)
        self.cur = 0

    def call(self, a, b, c):
        tg, sh = self.tg, self.stream.cuda_stream
        M, N, K = self.M, self.N, self.K
        if self.mode == "linear":
            st = tg.gemm_relu_f16_ex_raw(a.data_ptr(), b.data_ptr(), c.data_ptr(), M, N, K, self.opts, sh)
        elif self.ws_bytes > 0:
            st = tg.gemm_relu_f16_ws_raw(a.data_ptr(), b.data_ptr(), c.data_ptr(), M, N, K, sh,
                                         self.ws.data_ptr(), self.ws_bytes)
        else:
            st = tg.gemm_relu_f16_raw(a.data_ptr(), b.data_ptr(), c.data_ptr(), M, N, K, sh, self.path)
        if st != tg.Status.OK:
            raise tg.TGError(st, "tg_gemm_relu_f16")

    def step(self):
        self.call(*self.sets[self.cur % len(self.sets)])
        self.cur += 1

    def warm(self, warmup):
        torch, tg = self.torch, self.tg
        with torch.cuda.stream(self.stream):
            for _ in range(warmup):
                if self.flush is not None:
                    self.flush.fill_(1)
                self.step()
        torch.cuda.synchronize(self.dev)
        st, word = tg.device_status()
        if st != tg.Status.OK:
            raise SystemExit(f"device error after warm-up: {tg.status_string(st)} 0x{word:x}")

    def time(self, steps, dist=None):
        ms, clocks = timed_region(self.torch, self.dev, self.stream, self.step, steps, self.flush, dist)
        st, word = self.tg.device_status()
        if st != self.tg.Status.OK:
            raise SystemExit(f"device error in timed region: {self.tg.status_string(st)} 0x{word:x}")
        return ms, clocks

    def release(self):
        self.sets = self.ws = self.flush = None


def sustained_record(case, seconds, peaks, peak_src):
    """The headline kernel back to back for about `seconds` (one event pair around the loop, clocks
    sampled every millisecond), against the sustained (power-capped) tensor peak."""
    # Estimate the step time from a short burst, then size the loop.
    ms, _ = case.time(5)
    est_ms = max(ms, 1e-3)
    steps = max(10, int(seconds * 1e3 / est_ms))
    ms, clocks = case.time(steps)
    rec = roofline_for(case.M, case.N, case.K, ms, peaks, peak_src, sustained=True)
    rec.update({"steps": steps, "seconds": steps * ms * 1e-3, "ms_per_step": ms, "clocks": clocks})
    if clocks.get("sm_mhz"):
        rec["ms_x_sm_mhz"] = ms * clocks["sm_mhz"]
    return rec


# The configurations the metric's workloads are quoted on (besides the headline square8192), each
# measured as its own record: (label, workload, sub-index, value distribution or None, workspace mode).
CONFIG_RECORDS = [
    ("square256", "square256", None, None, "auto"),
    ("square256_int", "square256", None, "int", "auto"),
    ("square4096", "square4096", None, None, "auto"),
    ("skinny_m1", "skinny", 0, None, "auto"),
    ("skinny_m16", "skinny", 1, None, "auto"),
    ("skinny_m64", "skinny", 2, None, "auto"),
    ("ragged0_no_ws", "ragged", 0, None, "none"),
    ("ragged0_ws", "ragged", 0, None, "auto"),
    ("ragged1_no_ws", "ragged", 1, None, "none"),
    ("ragged1_ws", "ragged", 1, None, "auto"),
    ("ragged2_no_ws", "ragged", 2, None, "none"),
    ("ragged2_ws", "ragged", 2, None, "auto"),
]


def config_problem(workload, idx, dist):
    """(M, N, K, A, B) of one shape of a workload, exactly as the workload draws it (the generator is
    advanced over the workload's earlier shapes); `dist` overrides the value distribution."""
    wl = inputs.WORKLOADS[workload]
    for i, ((m, n, k), A, B) in enumerate(wl.problems(dist)):
        if i == (idx or 0):
            return m, n, k, A, B
    raise KeyError((workload, idx))


def measure_configs(tg, torch, dev, stream, args, peaks, peak_src):
    """One record per configuration: time, roofline against the roof its intensity meets, clocks, and the
    oracle timed on a short row sample on the host cores."""
    records = []
    wanted = None if args.configs == "all" else set(args.configs.split(","))
    for label, workload, idx, dist, mode in CONFIG_RECORDS:
        if wanted is not None and label not in wanted:
            continue
        M, N, K, A, B = config_problem(workload, idx, dist)
        case = Fp16Case(tg, torch, dev, stream, M, N, K, A, B, mode=mode)
        # Short kernels get more steps than the headline: at least 20 ms of
        # warm-up (clocks settle after the set-up between records) and 10 ms
        # of timed steps, so a record is not one launch's jitter.
        case.warm(args.warmup)
        est_ms, _ = case.time(max(3, args.warmup))
        steps = min(4000, max(args.steps, math.ceil(10.0 / max(est_ms, 1e-3))))
        case.warm(min(4000, max(args.warmup, math.ceil(20.0 / max(est_ms, 1e-3)))))
        ms, clocks = case.time(steps)
        spec = f"skinny:{M}" if workload == "skinny" else workload + (f":{idx}" if idx is not None else "")
        rec = {"config": label, "workload": spec,
               "M": M, "N": N, "K": K, "values": dist or inputs.WORKLOADS[workload].dist,
               "seed": inputs.WORKLOADS[workload].seed,
               "entry_point": "tg_gemm_relu_f16" if case.ws_bytes == 0 else "tg_gemm_relu_f16_ws",
               "path": tg.path_name(case.chosen), "workspace_bytes": case.ws_bytes, "l2": case.l2_note,
               "steps": steps, "warmup": args.warmup, "ms_per_step": ms,
               "value": inputs.flops(M, N, K) / (ms * 1e-3) / 1e12, "unit": UNIT,
               "roofline": roofline_for(M, N, K, ms, peaks, peak_src),
               "gpu_launches": steps * case.launches_per_step, "clocks": clocks}
        # A profile is keyed by path, and by "_ws" when a workspace changes what the path runs.
        key = tg.path_name(case.chosen) + ("_ws" if case.ws_bytes > 0 and case.chosen == tg.Path.RC else "")
        rec["roofline"]["traffic"] = committed_traffic(key, spec)
        if not args.no_cpu_baseline:
            rec["cpu_baseline"] = cpu_baseline(A, B, args.config_cpu_seconds)
        case.release()
        del A, B
        records.append(rec)
    return records


def run_ours(args):
    if args.workload in inputs.MX_WORKLOADS or args.workload in inputs.NVF4_WORKLOADS:
        return run_ours_mx(args)
    if args.workload in inputs.W4_WORKLOADS:
        return run_ours_w4(args)
    import torch
    import tiled_dense_gemm_fp16_b200 as tg

    world, rank, dev, dist = _init_ranks(args)
    path = {"auto": tg.Path.AUTO, "tc": tg.Path.TC, "tc_edge": tg.Path.TC_EDGE, "skinny": tg.Path.SKINNY,
            "tc_pair": tg.Path.TC_PAIR, "tc_pair512": tg.Path.TC_PAIR512, "rc": tg.Path.RC}[args.path]
    rows_mode = world > 1 and args.parallel == "rows"
    cols_mode = world > 1 and args.parallel == "cols"
    split = rows_mode or cols_mode
    # Row partition: every rank draws the workload itself (same seed) and keeps its rows of A; B is
    # replicated.  Column partition: it keeps its column block of B; A is replicated.  Replicas:
    # every rank runs its own independent problem.
    name, M, N_full, K, A, B = workload_problem(args.workload, 0 if split else rank)
    linear = name == "linear8192"
    bias = None
    if linear:
        B, bias = B
        if cols_mode:
            raise SystemExit("--parallel cols: the linear workload stores its weight N x K; split rows instead")
    r0, r1 = row_range(M, world, rank) if rows_mode else (0, M)
    c0, c1 = col_range(N_full, world, rank) if cols_mode else (0, N_full)
    Mr, N = r1 - r0, c1 - c0
    A_r = np.ascontiguousarray(A[r0:r1])
    if cols_mode:
        B = np.ascontiguousarray(B[:, c0:c1])
    stream = torch.cuda.Stream(dev)
    mode = "linear" if linear else ("none" if args.workspace == "none" else "auto")
    case = Fp16Case(tg, torch, dev, stream, Mr, N, K, A_r, B, mode=mode,
                    path=None if path == tg.Path.AUTO else path, bias=bias)
    case.warm(args.warmup)
    kern_ms, clocks = case.time(args.steps, dist)
    step_ms = max_over_ranks(dist, kern_ms, dev) if dist is not None else kern_ms
    flops_rank = inputs.flops(Mr, N, K)
    flops_total = inputs.flops(M, N_full, K) if split else world * flops_rank
    value = flops_total / (step_ms * 1e-3) / 1e12

    gather = None
    if split:
        # Stitch C once (outside the timed region) so every rank holds the full result; with
        # --gather-c the all-gather is also timed on its own over the same steps.
        c_block = case.sets[0][2]
        stitch = ((lambda: gather_rows(dist, c_block, M, world, rank)) if rows_mode else
                  (lambda: gather_cols(dist, c_block, N_full, world, rank)))
        full = stitch()
        assert full.shape == (M, N_full)
        gather = {"stitched": True}
        if args.gather_c:
            with torch.cuda.stream(stream):
                stitch()
            g_ms, _ = timed_region(torch, dev, stream, stitch, args.steps, None, dist)
            gather["all_gather_ms"] = max_over_ranks(dist, g_ms, dev)
            gather["step_ms_with_gather"] = step_ms + gather["all_gather_ms"]
        del full

    # End to end through the C ABI from pinned host buffers: every step copies A and B in and C out,
    # pipelined over two buffer sets (pipelined_e2e).
    Ad0, Bd0 = case.sets[0][0], case.sets[0][1]
    hosts = [torch.from_numpy(A_r).pin_memory(), torch.from_numpy(B).pin_memory()]
    e2e_ms = pipelined_e2e(dev, stream, hosts, lambda: [torch.empty_like(Ad0), torch.empty_like(Bd0)], (Mr, N),
                           torch.float16, case.call, args.e2e_steps)
    if dist is not None:
        e2e_ms = max_over_ranks(dist, e2e_ms, dev)
    h2d, d2h = 2 * (Mr * K + K * N), 2 * Mr * N
    link = host_link(dev, h2d, d2h)
    floor_ms = max(h2d / (link["h2d_gbs"] * 1e9) * 1e3, d2h / (link["d2h_gbs"] * 1e9) * 1e3, link["both_ms"])

    peaks, peak_src = load_peaks()
    roof = roofline_for(Mr, N, K, kern_ms, peaks, peak_src)
    roof["traffic"] = committed_traffic(tg.path_name(case.chosen), name) if rank == 0 else None
    if rows_mode:
        parallelism = (f"rows{world}: rank r computes rows [floor(rM/{world}), floor((r+1)M/{world})) of one "
                       f"{M}x{N}x{K} problem with B replicated; C stitched by an NCCL all-gather")
    elif cols_mode:
        parallelism = (f"cols{world}: rank r computes the columns [8 floor(floor(rN/{world})/8), ...) of one "
                       f"{M}x{N_full}x{K} problem, holding only its column block of B, with A replicated; "
                       f"C stitched by an NCCL all-gather")
    elif world > 1:
        parallelism = f"dp{world} independent problems"
    else:
        parallelism = "1 GPU"
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "strong" if split else "weak",
        "vs_baseline": None, "dtype": "f16 (fp32 accumulate)", "data": "synthetic",
        "config": {**describe(name, M, N_full, K), "path": tg.path_name(case.chosen),
                   "workspace_bytes": case.ws_bytes, "l2": case.l2_note, "parallelism": parallelism,
                   **({"rows_per_rank": [row_range(M, world, r)[1] - row_range(M, world, r)[0]
                                         for r in range(world)]} if rows_mode else {}),
                   **({"cols_per_rank": [col_range(N_full, world, r)[1] - col_range(N_full, world, r)[0]
                                         for r in range(world)]} if cols_mode else {})},
        "roofline": roof,
        "e2e": {"value": flops_total / (e2e_ms * 1e-3) / 1e12, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "mode": E2E_MODE,
                "host_link": {**link, "copy_floor_ms": floor_ms, "e2e_over_floor": e2e_ms / floor_ms,
                              "note": "floor = the longest of the upload alone, the download alone and both "
                                      "at once on two streams (separate copy engines sharing the link), "
                                      "measured with pinned host buffers of the step's sizes"}},
        "gpu_launches": args.steps * case.launches_per_step,
        "clocks": clocks,
    }
    if gather is not None:
        line["gather"] = gather
    if rank == 0 and world == 1 and args.sustained_seconds > 0:
        sus = sustained_record(case, args.sustained_seconds, peaks, peak_src)
        line["sustained"] = sus
        if sus.get("ms_x_sm_mhz"):
            # The kernel is clock-bound (tensor pipe), so time x clock is about constant: the
            # sustained run's product over the headline's time estimates the clock the headline
            # steps actually ran at, which NVML's sampled clock need not show for a short burst.
            line["clocks"]["effective_sm_mhz_estimate"] = sus["ms_x_sm_mhz"] / step_ms
    if args.cublas and not linear:
        # Context only (a library GEMM, not this path): the same operand sets, events around the region.
        def cublas_step():
            a_, b_, _ = case.sets[case.cur % len(case.sets)]
            case.cur += 1
            torch.relu(torch.matmul(a_, b_))
        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                cublas_step()
        cms, _ = timed_region(torch, dev, stream, cublas_step, args.steps, case.flush)
        line["context_cublas"] = {"op": "torch.relu(torch.matmul(A, B))", "ms_per_step": cms,
                                  "tflops": flops_rank / (cms * 1e-3) / 1e12}
    case.release()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(A, B, args.cpu_seconds)
    if rank == 0 and world == 1 and args.configs != "none" and not linear:
        del A, B, A_r, hosts
        line["configs"] = measure_configs(tg, torch, dev, stream, args, peaks, peak_src)
        line["gpu_launches"] += sum(r["gpu_launches"] for r in line["configs"])
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def _init_ranks(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    return world, rank, dev, dist


def mx_flops(m_sizes, N, K) -> int:
    return 2 * int(sum(m_sizes)) * N * K


def cpu_baseline_mx(kind, ops, m_sizes, N, K, target_s: float):
    """The oracle on the first rows of group 0, grown until one run takes about target_s."""
    import oracle
    A, SFA, B, SFB = ops
    fn = oracle.gemm_mxf8_grouped if kind == "mxf8" else oracle.gemm_nvf4_grouped
    cores = os.cpu_count() or 1
    rows = 1
    while True:
        t0 = time.perf_counter()
        fn(A[:rows], SFA[:rows], B[:1], SFB[:1], [rows], [0], N, K, nthreads=cores)
        dt = time.perf_counter() - t0
        if dt >= target_s or rows >= m_sizes[0]:
            break
        rows = min(int(m_sizes[0]), max(rows * 2, int(rows * target_s / max(dt, 1e-3) * 0.9)))
    value = mx_flops([rows], N, K) / dt / 1e12
    return {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"rows 0..{rows - 1} of group 0 ({rows} x {N} x {K}), {dt:.1f} s on {cores} threads",
            "seconds": dt}


def run_ours_mx(args):
    """A block-scaled grouped GEMM (MXFP8 or NVF4) on one of its workloads, operands resident in HBM."""
    import torch
    import tiled_dense_gemm_fp16_b200 as tg
    world, rank, dev, dist = _init_ranks(args)
    kind = "mxf8" if args.workload in inputs.MX_WORKLOADS else "nvf4"
    m_sizes, N, K, seed = (inputs.MX_WORKLOADS if kind == "mxf8" else inputs.NVF4_WORKLOADS)[args.workload]
    m_sizes = list(m_sizes)
    wseed = seed if rank == 0 else rank_seed(seed, rank)
    if kind == "mxf8":
        ops = inputs.mx_operands(m_sizes, N, K, wseed, "normal")
    else:
        ops = inputs.nvf4_operands(m_sizes, N, K, wseed, "codes")
    A, SFA, B, SFB = ops
    sfa_b, sfb_b = inputs.mx_scales_blocked(SFA), inputs.mx_scales_blocked(SFB)
    rows = A.shape[0]
    Ad, Bd = torch.from_numpy(A).to(dev), torch.from_numpy(B).to(dev)
    SFAd, SFBd = torch.from_numpy(sfa_b).to(dev), torch.from_numpy(sfb_b).to(dev)
    Cd = torch.empty((rows, N), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.Stream(dev)
    sh = stream.cuda_stream
    flops = mx_flops(m_sizes, N, K)
    in_bytes = A.nbytes + B.nbytes + sfa_b.nbytes + sfb_b.nbytes
    work_bytes = in_bytes + 2 * rows * N

    def call():
        if kind == "mxf8":
            st = tg.gemm_mxf8_grouped_raw(Ad.data_ptr(), SFAd.data_ptr(), Bd.data_ptr(), SFBd.data_ptr(),
                                          Cd.data_ptr(), m_sizes, N, K, 0, 0, False, sh)
        else:
            st = tg.gemm_nvf4_grouped_raw(Ad.data_ptr(), SFAd.data_ptr(), Bd.data_ptr(), SFBd.data_ptr(),
                                          Cd.data_ptr(), m_sizes, N, K, 1.0, False, sh)
        if st != tg.Status.OK:
            raise tg.TGError(st, f"tg_gemm_{kind}_grouped")

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            call()
    torch.cuda.synchronize(dev)
    st, word = tg.device_status()
    if st != tg.Status.OK:
        raise SystemExit(f"device error after warm-up: {tg.status_string(st)} 0x{word:x}")
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    with torch.cuda.stream(stream):
        r0.record(stream)
        for _ in range(args.steps):
            call()
        r1.record(stream)
    torch.cuda.synchronize(dev)
    sampler.stop()
    if dist is not None:
        dist.barrier()
    step_ms = r0.elapsed_time(r1) / args.steps
    kern_ms = step_ms
    if dist is not None:
        step_ms = max_over_ranks(dist, step_ms, dev)
    st, word = tg.device_status()
    if st != tg.Status.OK:
        raise SystemExit(f"device error in timed region: {tg.status_string(st)} 0x{word:x}")
    value = aggregate_throughput(world, flops, step_ms)

    hosts = [torch.from_numpy(x).pin_memory() for x in (A, B, sfa_b, sfb_b)]

    def call_sets(a, b, sa, sb, c):
        fn = tg.gemm_mxf8_grouped_raw if kind == "mxf8" else tg.gemm_nvf4_grouped_raw
        extra = (0, 0, False) if kind == "mxf8" else (1.0, False)
        st = fn(a.data_ptr(), sa.data_ptr(), b.data_ptr(), sb.data_ptr(), c.data_ptr(), m_sizes, N, K, *extra, sh)
        if st != tg.Status.OK:
            raise tg.TGError(st, f"tg_gemm_{kind}_grouped")

    e2e_ms = pipelined_e2e(dev, stream, hosts, lambda: [torch.empty_like(x) for x in (Ad, Bd, SFAd, SFBd)],
                           (rows, N), torch.bfloat16, call_sets, args.e2e_steps)
    if dist is not None:
        e2e_ms = max_over_ranks(dist, e2e_ms, dev)

    peaks, peak_src = load_peaks()
    ratio = 2.0 if kind == "mxf8" else 4.0
    peak = ratio * float(peaks["bf16_tflops"])
    achieved = flops / (kern_ms * 1e-3) / 1e12
    if kind == "mxf8":
        dtype = "e4m3 x e4m3, ue8m0 scales per 32 (fp32 accumulate, bf16 out)"
        values = "N(0,1) rounded to e4m3, scales 2^-3..2^3"
    else:
        dtype = "e2m1 x e2m1, ue4m3 scales per 16, alpha 1 (fp32 accumulate, bf16 out)"
        values = "uniform E2M1 codes, UE4M3 scale codes 0x28..0x48 (2^-2..2^2)"
    line = {
        "metric": MX_METRIC if kind == "mxf8" else NVF4_METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": dtype, "data": "synthetic",
        "config": {"workload": args.workload, "groups": len(m_sizes), "m_sizes": m_sizes, "N": N, "K": K,
                   "layout": "A stacked rows x K (groups on 128-row boundaries), B groups x N x K, blocked scales",
                   "values": values, "seed": seed, "path": f"{kind}_grouped",
                   "l2": "inputs larger than L2" if work_bytes > 2 * L2_BYTES else "operands partly L2-resident",
                   "parallelism": f"dp{world} independent problems" if world > 1 else "1 GPU"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": committed_traffic(kind, args.workload) if rank == 0 else None,
                     "peak_source": f"{peak_src} cuBLAS bf16 burst peak x {ratio:g} (nominal dense ratio to bf16)",
                     "kernel_ms": kern_ms},
        "e2e": {"value": aggregate_throughput(world, flops, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": in_bytes,
                "d2h_bytes_per_step": 2 * rows * N, "ms_per_step": e2e_ms, "mode": E2E_MODE},
        "gpu_launches": args.steps,
        "clocks": sampler.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_mx(kind, ops, m_sizes, N, K, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def w4_min_bytes(M, N, K, group) -> int:
    """Compulsory HBM bytes of one W4A16 GEMM: packed codes, scales, A and C once each."""
    return N * K // 2 + 2 * N * (K // group) + 2 * M * K + 2 * M * N


def run_ours_w4(args):
    """The 4-bit weight-only GEMM on one of inputs.W4_WORKLOADS (operands resident in HBM)."""
    import torch
    import tiled_dense_gemm_fp16_b200 as tg
    world, rank, dev, dist = _init_ranks(args)
    M, N, K, group, seed = inputs.W4_WORKLOADS[args.workload]
    A, Wq, S = inputs.w4_operands(M, N, K, group, seed if rank == 0 else rank_seed(seed, rank), "uniform")
    stream = torch.cuda.Stream(dev)
    sh = stream.cuda_stream
    need = tg.w4a16_workspace_size(M, N, K, group)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    flops = inputs.flops(M, N, K)
    nbytes = w4_min_bytes(M, N, K, group)
    # Rotate operand copies when one set fits in L2 (the decode case), so each step reads cold data.
    sets = []
    reps = max(1, -(-3 * L2_BYTES // nbytes)) if nbytes <= 2 * L2_BYTES else 1
    for _ in range(min(reps, 16)):
        sets.append((torch.from_numpy(A).to(dev), torch.from_numpy(Wq).to(dev), torch.from_numpy(S).to(dev),
                     torch.empty((M, N), dtype=torch.float16, device=dev)))
    cur = [0]

    def call(a, w, s_, c):
        st = tg.gemm_relu_w4a16_raw(a.data_ptr(), w.data_ptr(), s_.data_ptr(), c.data_ptr(), M, N, K, group, sh,
                                    ws.data_ptr(), need)
        if st != tg.Status.OK:
            raise tg.TGError(st, "tg_gemm_relu_w4a16")

    def step():
        call(*sets[cur[0] % len(sets)])
        cur[0] += 1

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize(dev)
    st, word = tg.device_status()
    if st != tg.Status.OK:
        raise SystemExit(f"device error after warm-up: {tg.status_string(st)} 0x{word:x}")
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    with torch.cuda.stream(stream):
        r0.record(stream)
        for _ in range(args.steps):
            step()
        r1.record(stream)
    torch.cuda.synchronize(dev)
    sampler.stop()
    if dist is not None:
        dist.barrier()
    step_ms = r0.elapsed_time(r1) / args.steps
    kern_ms = step_ms
    if dist is not None:
        step_ms = max_over_ranks(dist, step_ms, dev)
    st, word = tg.device_status()
    if st != tg.Status.OK:
        raise SystemExit(f"device error in timed region: {tg.status_string(st)} 0x{word:x}")
    value = aggregate_throughput(world, flops, step_ms)

    hosts = [torch.from_numpy(x).pin_memory() for x in (A, Wq, S)]
    e2e_ms = pipelined_e2e(dev, stream, hosts, lambda: [torch.empty_like(x) for x in sets[0][:3]], (M, N),
                           torch.float16, call, args.e2e_steps)
    if dist is not None:
        e2e_ms = max_over_ranks(dist, e2e_ms, dev)

    peaks, peak_src = load_peaks()
    fused = need == 0
    kind = tg.w4a16_kernel(M, N, K, group)
    path_name = {tg.W4Kernel.DECODE: "w4a16 decode (register dequantization, mma.sync, cluster split-K)",
                 tg.W4Kernel.FUSED: "w4a16 fused (tcgen05)"}.get(kind, "dequantize + tc (fp16 GEMM)")
    if fused:
        roof = {"bound": "hbm", "achieved": nbytes / (kern_ms * 1e-3) / 1e9, "peak": float(peaks["hbm_gbs"]),
                "unit": "GB/s", "peak_source": f"{peak_src} STREAM-copy HBM bandwidth"}
    else:
        roof = {"bound": "tensor", "achieved": flops / (kern_ms * 1e-3) / 1e12, "peak": float(peaks["bf16_tflops"]),
                "unit": "TFLOP/s", "peak_source": f"{peak_src} cuBLAS bf16 burst peak (fp16 runs at the bf16 rate)"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = committed_traffic("w4a16", args.workload) if rank == 0 else None
    roof["kernel_ms"] = kern_ms
    line = {
        "metric": W4_METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16 activations x 4-bit weights (fp16 scales per group), fp32 accumulate",
        "data": "synthetic",
        "config": {"workload": args.workload, "M": M, "N": N, "K": K, "group": group, "seed": seed,
                   "path": path_name,
                   "workspace_bytes": need, "min_bytes": nbytes,
                   "l2": (f"rotating {len(sets)} operand copies" if len(sets) > 1 else "inputs larger than L2"),
                   "parallelism": f"dp{world} independent problems" if world > 1 else "1 GPU"},
        "roofline": roof,
        "e2e": {"value": aggregate_throughput(world, flops, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": A.nbytes + Wq.nbytes + S.nbytes, "d2h_bytes_per_step": 2 * M * N,
                "ms_per_step": e2e_ms, "mode": E2E_MODE},
        "gpu_launches": args.steps * (1 if fused else 2),
        "clocks": sampler.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        cores = os.cpu_count() or 1
        rows = 1
        while True:
            t0 = time.perf_counter()
            oracle.gemm_relu_w4a16(A[:rows], Wq, S, group, nthreads=cores)
            dt = time.perf_counter() - t0
            if dt >= args.cpu_seconds or rows >= M:
                break
            rows = min(M, max(rows * 2, int(rows * args.cpu_seconds / max(dt, 1e-3) * 0.9)))
        line["cpu_baseline"] = {"value": inputs.flops(rows, N, K) / dt / 1e12, "unit": UNIT, "cores": cores,
                                "kind": "oracle", "seconds": dt,
                                "sample": f"rows 0..{rows - 1} ({rows} x {N} x {K}), {dt:.1f} s on {cores} threads"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
