#!/usr/bin/env python
"""Benchmark of the B200 LLM.int8() decomposed matmul.

One step = one forward of the whole path (outlier detection, row
quantisation, fused int8 GEMM with dequantisation and the fp16 outlier
product) over one batch of synthetic activations, through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 175b|opt13b]
                    [--impl ours|reference] [--sections ...] [--profile-forwards F]

Under torchrun (N > 1) every rank runs an independent replica of the problem
on its own GPU (weak scaling: the path has no exchange step); the reported
time is the maximum over ranks.  Rank 0 prints one JSON line.

Metric: effective TOPS = 2*M*N*K / time per step (the int8 contraction over
the full K), inputs resident in HBM.  Every timed step is preceded by an L2
flush outside the timed events: a 256 MB write, then a 256 MB read.
The headline workload is the 175B-scale FFN expansion prefill (M=2048,
K=12288, N=49152); the same JSON line carries further sections: the OPT-13B
prefill, the OPT-13B FFN contraction, the memory-saving weight, decode (few
tokens, HBM-bound) and the K=N=8192 sweep over M and the outlier count.

--profile-forwards F runs F plain forwards of the chosen workload (after the
warm-up) and exits without timing or printing: the command the committed ncu
summaries under profiles/ were taken with.
"""
from __future__ import annotations

import argparse
import datetime
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

import workloads  # noqa: E402

METRIC = "int8-decomp matmul effective TOPS & % INT8 tensor peak; decode-shape HBM GB/s"
# Dense tensor-core throughput ratio int8 : bf16 on B200 (4.5 POPS : 2.25 PFLOP/s).
INT8_PER_BF16 = 2.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_SCRUB_BYTES = 256 << 20
L2_BYTES = 126 << 20  # B200
# The prefill GEMM's device code (its launcher declarations in kernels.cuh
# also describe the other kernels, so they are left out of the hash).
GEMM_SOURCES = ["int8_quantized_matmul_outlier_b200/csrc/gemm_i8.cu",
                "int8_quantized_matmul_outlier_b200/csrc/ptx.cuh"]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="175b",
                    help="175b or opt13b (the headline workload); with --profile-forwards also "
                         "ffn2 (OPT-13B FFN contraction), decode:M (M tokens against the 175B-scale "
                         "weight) or sweep:M:O (K=N=8192, O planted outlier columns)")
    ap.add_argument("--sections", default="all",
                    help="comma-separated extra sections: opt13b,ffn_contraction,static_weight,decode,"
                         "sweep (or all, or none)")
    ap.add_argument("--sweep-steps", type=int, default=30, help="timed steps per sweep point")
    ap.add_argument("--profile-forwards", type=int, default=0,
                    help="run this many forwards after the warm-up and exit (for ncu)")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-rows", type=int, default=0,
                    help="rows of the oracle CPU sample (0: sized to about 10 s)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--decode-steps", type=int, default=200,
                    help="timed steps per decode shape (0 skips the decode measurement)")
    a = ap.parse_args()
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    headline = a.config in ("175b", "opt13b")
    if not headline and (a.profile_forwards <= 0 or a.impl != "ours"):
        ap.error("--config other than 175b/opt13b only with --profile-forwards")
    try:
        make_problem(a.config, 0, check_only=True)
    except ValueError as e:
        ap.error(str(e))
    known = {"opt13b", "ffn_contraction", "static_weight", "decode", "sweep"}
    if a.sections == "all":
        a.sections = set(known)
    elif a.sections == "none":
        a.sections = set()
    else:
        a.sections = {x.strip() for x in a.sections.split(",") if x.strip()}
        if not a.sections <= known:
            ap.error(f"unknown sections {sorted(a.sections - known)}")
    return a


def make_problem(config: str, rank: int, check_only: bool = False):
    """The workload named by --config (see parse_args)."""
    parts = config.split(":")
    try:
        if parts == ["opt13b"]:
            return None if check_only else workloads.opt13b_prefill(repeat=rank)
        if parts == ["175b"]:
            return None if check_only else workloads.gpt175b_prefill(repeat=rank)
        if parts == ["ffn2"]:
            return None if check_only else workloads.opt13b_contraction(repeat=rank)
        if parts[0] == "decode" and len(parts) == 2 and int(parts[1]) in DECODE_MS:
            if check_only:
                return None
            p = workloads.decode(int(parts[1]), repeat=rank, with_weight=False)
            p.W = workloads.weight(DECODE_K, DECODE_N, 3 * 1000 + 500_000 + rank)
            return p
        if parts[0] == "sweep" and len(parts) == 3 and int(parts[1]) in SWEEP_MS and int(parts[2]) in SWEEP_OUTLIERS:
            if check_only:
                return None
            p = workloads.sweep(int(parts[1]), int(parts[2]), repeat=rank, with_weight=False)
            p.W = workloads.weight(SWEEP_K, SWEEP_N, 4 * 1000 + 500_000 + rank)
            return p
    except ValueError:
        pass
    raise ValueError(f"unknown --config {config!r}")


def workload_config(p: workloads.Problem) -> dict:
    M, K, N = p.shape
    return {"workload": p.name, "M": M, "K": K, "N": N, "alpha": p.alpha,
            "planted_outlier_columns": int(p.planted.size),
            "inputs": "seeded synthetic fp16 (FFN-input statistics of the pages' OPT-13B example)",
            "l2": L2Flush.describe(forward_bytes(M, K, N))}


def forward_bytes(M: int, K: int, N: int) -> int:
    """Bytes a forward streams: X in, the int8 weight, Y out."""
    return 2 * M * K + N * K + 2 * M * N


class L2Flush:
    """Keeps every timed step cold in L2: before each step, a 256 MB write
    replaces the L2's lines and a 256 MB read then pushes the written (dirty)
    lines back to HBM, so the timed step neither finds its data in L2 nor
    pays for the write-back of the flush's own lines."""

    def __init__(self, torch, dev):
        self.w = torch.empty(L2_SCRUB_BYTES // 4, dtype=torch.float32, device=dev)
        self.r = torch.ones(L2_SCRUB_BYTES // 4, dtype=torch.float32, device=dev)

    @staticmethod
    def describe(nbytes: int) -> str:
        return ("flushed between steps (256 MB write, then 256 MB read), outside the timed events; "
                f"the step streams {nbytes / 1e6:.0f} MB (L2 126 MB)")

    def for_bytes(self, nbytes: int):
        """The flush to run between steps of a workload of nbytes."""
        def flush():
            self.w.zero_()
            self.r.sum()
        return flush


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return dict(FALLBACK_PEAKS, source="fallback")


def gemm_source_hash() -> str:
    h = hashlib.sha256()
    for rel in GEMM_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def recorded_traffic(workload: str):
    """DRAM bytes (read + write) per GEMM launch for `workload`, as recorded
    from an ncu capture in profiles/traffic.json, if it was taken on the
    current GEMM source (else None)."""
    try:
        with open(TRAFFIC_FILE, encoding="utf-8") as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    g = d.get("gemm_i8_decomp_kernel", {})
    if g.get("gemm_source_sha256_16") != gemm_source_hash():
        return None
    v = g.get("bytes_per_launch", {}).get(workload)
    return float(v) if v is not None else None


class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML while running."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device, period_s: float = 0.01):
        self.samples = []
        self.max_mhz = None
        self.ok = False
        self._stop = threading.Event()
        self._period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = self._handle(pynvml, device)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report no clocks
            self.err = str(e)
        self._t = threading.Thread(target=self._run, daemon=True)

    @staticmethod
    def _handle(nv, device):
        """NVML handle of the torch device, matched by PCI bus id (CUDA and
        NVML number devices differently under CUDA_VISIBLE_DEVICES)."""
        import torch
        pr = torch.cuda.get_device_properties(device)
        try:
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            return nv.nvmlDeviceGetHandleByPciBusId_v2(bus)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(device.index)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                try:
                    reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                except Exception:
                    reasons = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                self.samples.append((mhz, reasons))
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self.ok:
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self) -> dict:
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [s[0] for s in self.samples]
        active = set()
        for _, r in self.samples:
            for name, bit in self.REASONS.items():
                if r & bit:
                    active.add(name)
        return {"sm_mhz": float(statistics.median(mhz)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(active), "samples": len(mhz), "source": "nvml"}


# --------------------------------------------------------------------------
# CPU oracle timing (the reported baseline and the reference arm)

def oracle_rows_sample(p: workloads.Problem, rows: int, wq=None):
    """Time the oracle's forward on a batch made of the first `rows` rows of
    X (a bounded sample of the workload: same K, N, alpha and value
    distributions): outlier detection, row quantisation, the int8
    contraction, dequantisation and the fp16 outlier product.  The weight
    codes, prepared once per weight, are made outside the timed region."""
    import oracle
    if wq is None:
        wq = oracle.quantize_cols(p.W)
    qw, c_w = wq
    Xr = np.ascontiguousarray(p.X[:rows])
    t0 = time.perf_counter()
    _, idx = oracle.outlier_columns(Xr, p.alpha)
    qx, c_x = oracle.quantize_rows(Xr, idx)
    acc = oracle.int8_matmul(qx, qw)
    oracle.dequant_add_outliers(acc, c_x, c_w, Xr, p.W, idx)
    return time.perf_counter() - t0, wq


def cpu_rows_for(p, target_s: float, wq):
    t, _ = oracle_rows_sample(p, 16, wq)
    M = p.shape[0]
    return int(max(1, min(M, 16 * target_s / max(t, 1e-4))))


def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo), or "unknown"."""
    try:
        with open("/proc/cpuinfo", encoding="utf-8", errors="replace") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(p: workloads.Problem, rows: int, acc_rows=None, exact=None) -> dict:
    """The oracle timed on the host cores on a bounded sample of the
    workload.  With acc_rows / exact (the fp64 products of those rows, from
    the accuracy report), the oracle's own output on those rows is compared
    with them too, so the accuracy block carries the error of both paths."""
    import oracle
    wq = oracle.quantize_cols(p.W)
    if rows <= 0:
        rows = cpu_rows_for(p, 10.0, wq)
    t, _ = oracle_rows_sample(p, rows, wq)
    M, K, N = p.shape
    cores = oracle.num_threads()
    # the Tiny configuration on one thread, for scale
    tiny = workloads.tiny()
    oracle.set_num_threads(1)
    try:
        t1, _ = oracle_rows_sample(tiny, tiny.shape[0])
    finally:
        oracle.set_num_threads(cores)
    out = {"value": 2.0 * rows * N * K / t / 1e12, "unit": "TOPS", "cores": cores,
           "kind": "oracle",
           "sample": f"batch of the first {rows} of {M} rows, whole forward on it; "
                     f"weight codes prepared outside the timed region",
           "seconds": t,
           "single_thread_tiny_forward_s": t1,
           "cpu_model": cpu_model(), "host_threads": os.cpu_count()}
    if acc_rows is not None and exact is not None:
        r = oracle.decomp_matmul(p.X, p.W, p.alpha, rows=acc_rows, wq=wq)
        out["oracle_accuracy"] = error_vs(r["Y"].astype(np.float64), exact)
    return out


def error_vs(v: np.ndarray, exact: np.ndarray) -> dict:
    d = v - exact
    return {"max_abs": float(np.abs(d).max()), "rel_fro": float(np.linalg.norm(d) / np.linalg.norm(exact))}


# --------------------------------------------------------------------------

def max_over_ranks(x: float, device=None) -> float:
    """Maximum of x over all ranks of the default process group (x itself
    when no group is initialised).  NCCL needs a CUDA device tensor; gloo
    (CPU tests) a CPU one."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(ops_per_step: float, steps: int, world: int, max_total_ms: float) -> float:
    """Whole-job TOPS: the operations of all ranks over the slowest rank's time."""
    return ops_per_step * steps * world / (max_total_ms * 1e-3) / 1e12


DECODE_K, DECODE_N, DECODE_MS = 12288, 49152, (1, 8, 32)


def decode_algorithmic_bytes(M: int, K: int, N: int, n_out: int) -> int:
    """Bytes a decode forward must move: the int8 weight, its fp32 scales, the
    fp16 outlier rows of W, X in and Y out (intermediates excluded)."""
    return N * K + 4 * N + 2 * n_out * N + 2 * M * K + 2 * M * N


def run_decode(m, torch, dev, stream, l2, steps: int, peaks: dict, max_over, rank: int, w=None):
    """Decode steps (few tokens against the 175B-scale weight, K=12288 x
    N=49152): each step one forward, timed with events around it only, so the
    GEMM stays a programmatic dependent launch of the activation pass.  `w`
    may be a prepared weight of that shape (the headline's); else one is
    made here."""
    own = w is None
    if own:
        Wnp = workloads.weight(DECODE_K, DECODE_N, 3 * 1000 + 500_000 + rank)
        W = torch.from_numpy(Wnp).to(dev)
        del Wnp
        w = m.int8mm_prepare_weight(W)
    out = []
    for M in DECODE_MS:
        p = workloads.decode(M, repeat=rank, with_weight=False)
        X = torch.from_numpy(p.X).to(dev)
        Y = torch.empty((M, DECODE_N), dtype=torch.float16, device=dev)
        ms = max_over(time_forwards(m, torch, w, X, p.alpha, Y, stream,
                                    l2.for_bytes(forward_bytes(M, DECODE_K, DECODE_N)), steps))
        nbytes = decode_algorithmic_bytes(M, DECODE_K, DECODE_N, int(p.planted.size))
        gbps = nbytes / (ms * 1e-3) / 1e9
        out.append({"M": M, "K": DECODE_K, "N": DECODE_N, "ms_per_step": ms, "GBps": gbps,
                    "l2": L2Flush.describe(forward_bytes(M, DECODE_K, DECODE_N)),
                    "frac_hbm": gbps / peaks["hbm_gbs"], "algorithmic_bytes": nbytes,
                    "gpu_launches_per_step": m.int8mm_launches_per_forward(w, M)})
    if own:
        m.int8mm_free(w)
    return out


def accuracy_report(torch, dev, X, W, Y, rows: int = 32, seed: int = 0):
    """Error of the GPU's Y against the exact matmul of the fp16 inputs (fp64,
    on seeded sampled rows), next to tensor-wise absmax int8 (one scale for X,
    one for W, no decomposition) on the same rows.  Plain torch reference
    arithmetic, outside the timed regions.  Returns the report, the sampled
    rows and their exact products (numpy fp64)."""
    M = X.shape[0]
    g = np.random.default_rng(seed)
    r = np.unique(np.concatenate([[0, M - 1], g.choice(M, size=min(M, rows) - 2, replace=False)]))
    ri = torch.from_numpy(r).to(dev)
    Xr = X.index_select(0, ri).double()
    Wd = W.double()
    exact = Xr @ Wd
    y = Y.index_select(0, ri).double()
    cx = 127.0 / X.abs().max().double()
    cw = 127.0 / W.abs().max().double()
    qx = torch.round(Xr * cx).clamp(-127, 127)   # round half to even
    qw = torch.round(Wd * cw).clamp(-127, 127)
    tw = (qx @ qw) / (cx * cw)
    del Wd, qw
    exact_np = exact.cpu().numpy()
    e_gpu, e_tw = error_vs(y.cpu().numpy(), exact_np), error_vs(tw.cpu().numpy(), exact_np)
    rep = {"rows_sampled": int(r.size), "reference": "fp64 matmul of the fp16 inputs",
           "decomposed_gpu": e_gpu, "tensorwise_absmax_int8": e_tw,
           "rel_fro_ratio_tensorwise_over_decomposed": e_tw["rel_fro"] / max(e_gpu["rel_fro"], 1e-30)}
    return rep, r, exact_np


def time_forwards(m, torch, w, X, alpha, Y, stream, flush, steps: int, warm: int = 5) -> float:
    """Mean device time (ms) of whole forwards, CUDA events around each one
    only (the GEMM stays a programmatic dependent of the activation pass),
    `flush` run between steps outside the events."""
    for _ in range(warm):
        m.int8mm_forward(w, X, alpha, Y, stream=stream)
        flush()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    for e0, e1 in ev:
        e0.record(stream)
        m.int8mm_forward(w, X, alpha, Y, stream=stream)
        e1.record(stream)
        flush()
    torch.cuda.synchronize()
    if m.int8mm_get_status(w) != m.INT8MM_OK:
        raise RuntimeError("device wait timed out")
    return float(np.mean([e0.elapsed_time(e1) for e0, e1 in ev]))


def time_kernels(m, torch, w, X, alpha, Y, stream, flush, steps: int):
    """Mean device times (ms) of the activation pass and of the GEMM, from
    an event between them (the GEMM then an ordinary launch)."""
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    torch.cuda.synchronize()
    for e in kev:
        m.int8mm_forward_events(w, X, alpha, Y, e, stream=stream)
        flush()
    torch.cuda.synchronize()
    seg = np.array([[e[i].elapsed_time(e[i + 1]) for i in range(2)] for e in kev])
    return float(seg[:, 0].mean()), float(seg[:, 1].mean())


def run_prefill_section(m, torch, dev, stream, l2, p, steps: int, peak_tops: float, max_over) -> dict:
    """Another prefill workload: whole forwards, plus the GEMM alone."""
    M, K, N = p.shape
    X = torch.from_numpy(p.X).to(dev)
    W = torch.from_numpy(p.W).to(dev)
    w = m.int8mm_prepare_weight(W)
    Y = torch.empty((M, N), dtype=torch.float16, device=dev)
    flush = l2.for_bytes(forward_bytes(M, K, N))
    ms = max_over(time_forwards(m, torch, w, X, p.alpha, Y, stream, flush, steps))
    act_ms, gemm_ms = time_kernels(m, torch, w, X, p.alpha, Y, stream, flush, steps)
    act_ms, gemm_ms = max_over(act_ms), max_over(gemm_ms)
    flops = 2.0 * M * N * K
    tops = flops / (ms * 1e-3) / 1e12
    out = {"workload": p.name, "M": M, "K": K, "N": N, "ms_per_step": ms, "TOPS": tops,
           "frac_int8_peak": tops / peak_tops, "gpu_launches_per_step": m.int8mm_launches_per_forward(w, M),
           "l2": L2Flush.describe(forward_bytes(M, K, N)),
           "kernels_ms": {"activation pass": act_ms, "gemm_i8_decomp": gemm_ms},
           "gemm_TOPS": flops / (gemm_ms * 1e-3) / 1e12,
           "gemm_frac_int8_peak": flops / (gemm_ms * 1e-3) / 1e12 / peak_tops,
           "traffic_bytes_per_gemm_launch": recorded_traffic(p.name)}
    m.int8mm_free(w)
    return out


SWEEP_K = SWEEP_N = 8192
SWEEP_MS = (16, 128, 1024, 8192)
SWEEP_OUTLIERS = (0, 1, 7, 32, 128)


def run_sweep(m, torch, dev, stream, l2, steps: int, peaks: dict, peak_tops: float, max_over, rank: int) -> dict:
    """K = N = 8192 sweep: M in (16, 128, 1024, 8192) x outlier count in
    (0, 1, 7, 32, 128) at alpha = 6, plus alpha = inf (pure vector-wise int8)
    on the 7-outlier activations; the 0-outlier points stand for a small model
    with no outliers (detection runs and finds none).  Whole forwards, L2
    flushed between steps (the 64 MB weight would otherwise stay in L2).
    M <= 128 is weight-bandwidth bound (GB/s vs measured HBM), M >= 1024 tensor
    bound (TOPS vs the int8 peak); both figures are given for every point."""
    W = torch.from_numpy(workloads.weight(SWEEP_K, SWEEP_N, 4 * 1000 + 500_000 + rank)).to(dev)
    w = m.int8mm_prepare_weight(W)
    m.int8mm_reserve(w, max(SWEEP_MS))
    points = []
    for M in SWEEP_MS:
        Y = torch.empty((M, SWEEP_N), dtype=torch.float16, device=dev)
        runs = [(n, 6.0) for n in SWEEP_OUTLIERS] + [(7, math.inf)]
        for n_out, alpha in runs:
            p = workloads.sweep(M, n_out, repeat=rank, alpha=alpha, with_weight=False)
            X = torch.from_numpy(p.X).to(dev)
            ms = max_over(time_forwards(m, torch, w, X, alpha, Y, stream,
                                        l2.for_bytes(forward_bytes(M, SWEEP_K, SWEEP_N)), steps))
            flops = 2.0 * M * SWEEP_N * SWEEP_K
            n_used = 0 if math.isinf(alpha) else n_out
            nbytes = decode_algorithmic_bytes(M, SWEEP_K, SWEEP_N, n_used)
            tops = flops / (ms * 1e-3) / 1e12
            gbps = nbytes / (ms * 1e-3) / 1e9
            bound = "hbm" if M <= 128 else "tensor"
            points.append({"M": M, "outliers": n_out, "alpha": "inf" if math.isinf(alpha) else alpha,
                           "ms_per_step": ms, "TOPS": tops, "frac_int8_peak": tops / peak_tops,
                           "GBps": gbps, "frac_hbm": gbps / peaks["hbm_gbs"], "bound": bound,
                           "frac": gbps / peaks["hbm_gbs"] if bound == "hbm" else tops / peak_tops,
                           "algorithmic_bytes": nbytes})
            del X
    m.int8mm_free(w)
    return {"workload": "sweep: K=N=8192, M in (16,128,1024,8192) x |O| in (0,1,7,32,128), alpha=6; "
                        "plus alpha=inf on the |O|=7 activations",
            "timing": "CUDA events around each whole forward; L2 flushed between steps (256 MB write, then "
                      "256 MB read), outside the events",
            "steps_per_point": steps, "points": points}


def run_static_weight(m, torch, dev, stream, l2, p, X, W, Y_ref, steps: int, peak_tops: float,
                      max_over) -> dict:
    """The headline workload with the memory-saving weight: fp16 rows kept
    only for the planted outlier dimensions (standing in for a calibrated
    set), whole forwards timed as for the other sections."""
    M, K, N = p.shape
    w = m.int8mm_prepare_weight_static(W, p.planted.tolist(), max_outliers=64)
    Y = torch.empty((M, N), dtype=torch.float16, device=dev)
    ms = max_over(time_forwards(m, torch, w, X, p.alpha, Y, stream, l2.for_bytes(forward_bytes(M, K, N)), steps))
    tops = 2.0 * M * N * K / (ms * 1e-3) / 1e12
    out = {"workload": p.name, "stored_rows": int(p.planted.size), "max_outliers": 64,
           "ms_per_step": ms, "TOPS": tops, "frac_int8_peak": tops / peak_tops,
           "gpu_launches_per_step": m.int8mm_launches_per_forward(w, M),
           "handle_bytes": m.int8mm_weight_bytes(w), "fp16_weight_bytes_not_kept": K * N * 2,
           "y_equals_borrowed_weight": bool(torch.equal(Y, Y_ref)),
           "status_ok": m.int8mm_get_status(w) == m.INT8MM_OK}
    m.int8mm_free(w)
    return out


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    p = make_problem(args.config, 0)
    M, K, N = p.shape
    wq = oracle.quantize_cols(p.W)
    # each step is a bounded sample sized so that the whole run stays within minutes
    budget_s = 120.0 / max(1, args.steps + args.warmup)
    rows = min(M, max(1, cpu_rows_for(p, min(budget_s, 5.0), wq)))
    for _ in range(args.warmup):
        oracle_rows_sample(p, rows, wq)
    ts = [oracle_rows_sample(p, rows, wq)[0] for _ in range(args.steps)]
    t = sum(ts)
    value = 2.0 * rows * N * K * args.steps / t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * t / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic", "config": workload_config(p),
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": oracle.num_threads(), "kind": "oracle",
                         "cpu_model": cpu_model(),
                         "sample": f"each step: whole forward on a batch of the first {rows} of {M} rows; "
                                   f"weight codes prepared once, untimed"},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch

    import int8_quantized_matmul_outlier_b200 as m

    world, rank, local = dist_env()
    distributed = world > 1
    if distributed:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())

    def barrier():
        if distributed:
            dist.barrier()

    def max_over(x):
        return max_over_ranks(x, dev)

    p = make_problem(args.config, rank)
    M, K, N = p.shape
    X = torch.from_numpy(p.X).to(dev)
    W = torch.from_numpy(p.W).to(dev)
    w = m.int8mm_prepare_weight(W)
    m.int8mm_reserve(w, M)
    Y = torch.empty((M, N), dtype=torch.float16, device=dev)
    l2 = L2Flush(torch, dev)
    flush = l2.for_bytes(forward_bytes(M, K, N))
    stream = torch.cuda.current_stream()

    # warm-up (untimed)
    for _ in range(args.warmup):
        m.int8mm_forward(w, X, p.alpha, Y)
        flush()
    torch.cuda.synchronize()
    if m.int8mm_get_status(w) != m.INT8MM_OK:
        raise RuntimeError("device wait timed out during warm-up")
    if args.profile_forwards > 0:
        # plain forwards for an ncu capture: no timing, no output
        for _ in range(args.profile_forwards):
            m.int8mm_forward(w, X, p.alpha, Y)
            flush()
        torch.cuda.synchronize()
        ok = m.int8mm_get_status(w) == m.INT8MM_OK
        m.int8mm_free(w)
        if distributed:
            dist.destroy_process_group()
        return 0 if ok else 1

    steps = args.steps
    launches = m.int8mm_launches_per_forward(w, M)
    # Each step: events around the whole forward only, so that the GEMM stays
    # a programmatic dependent launch of the activation pass, as in use.
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev, period_s=0.002) as clocks:
        t0 = time.perf_counter()
        for e0, e1 in ev:
            e0.record(stream)
            m.int8mm_forward(w, X, p.alpha, Y, stream=stream)
            e1.record(stream)
            flush()
        torch.cuda.synchronize()
        wall = time.perf_counter() - t0
    barrier()
    if m.int8mm_get_status(w) != m.INT8MM_OK:
        raise RuntimeError("device wait timed out in the timed region")
    step_ms = np.array([e0.elapsed_time(e1) for e0, e1 in ev])
    total_ms = max_over(float(step_ms.sum()))
    ms_per_step = total_ms / steps
    flops = 2.0 * M * N * K
    value = job_throughput(flops, steps, world, total_ms)

    # Per-kernel times (the GEMM's launch duration for the roofline): an event
    # between the activation pass and the GEMM makes the GEMM an ordinary
    # launch, so these steps are timed apart from the headline ones.
    ksteps = max(1, min(steps, 200))
    barrier()
    xprep_ms, gemm_ms = time_kernels(m, torch, w, X, p.alpha, Y, stream, flush, ksteps)
    xprep_ms, gemm_ms = max_over(xprep_ms), max_over(gemm_ms)

    # end to end through the host-buffer entry point: pinned X in, pinned Y out
    Xh = torch.from_numpy(p.X).pin_memory()
    Yh = torch.empty((M, N), dtype=torch.float16).pin_memory()
    e2e_steps = max(1, min(args.e2e_steps, steps))
    for _ in range(3):
        m.int8mm_forward_host(w, Xh, p.alpha, Yh)
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        m.int8mm_forward_host(w, Xh, p.alpha, Yh)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over(e0.elapsed_time(e1) / e2e_steps)
    e2e_value = job_throughput(flops, 1, world, e2e_ms)
    e2e_equal = bool(torch.equal(Yh, Y.cpu()))
    del Xh, Yh

    peaks = measured_peaks()
    peak_tops = peaks["bf16_tflops"] * INT8_PER_BF16
    achieved = flops / (gemm_ms * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": workload_config(p),
        "roofline": {
            "bound": "tensor", "achieved": achieved, "peak": peak_tops, "unit": "TFLOP/s",
            "frac": achieved / peak_tops, "traffic": recorded_traffic(p.name),
            "kernel": "gemm_i8_decomp_kernel",
            "peak_note": (f"dense int8 = {INT8_PER_BF16:g} x {peaks['source']} bf16 burst "
                          f"{peaks['bf16_tflops']:g} TFLOP/s; int8 ops counted as 2*M*N*K"),
        },
        "kernels_ms": {"activation pass": xprep_ms, "gemm_i8_decomp": gemm_ms,
                       "note": f"mean over {ksteps} separately timed forwards, GEMM launched without PDL"},
        "pct_int8_peak_whole_step": 100.0 * value / world / peak_tops,
        "e2e": {"value": e2e_value, "unit": "TOPS", "h2d_bytes_per_step": M * K * 2,
                "d2h_bytes_per_step": M * N * 2, "ms_per_step": e2e_ms,
                "entry_point": "int8mm_forward_host (pinned host buffers)",
                "y_equals_device_forward": e2e_equal},
        "gpu_launches": launches * steps,
        "clocks": clocks.summary(),
        "wall_s_timed_region": wall,
    }
    acc, acc_rows, acc_exact = accuracy_report(torch, dev, X, W, Y)
    line["accuracy"] = acc
    sec = args.sections
    sec_steps = max(1, min(args.decode_steps, 100))
    if "opt13b" in sec and args.config != "opt13b":
        line["opt13b_prefill"] = run_prefill_section(m, torch, dev, stream, l2, workloads.opt13b_prefill(repeat=rank),
                                                     sec_steps, peak_tops, max_over)
    if "ffn_contraction" in sec:
        line["ffn_contraction"] = run_prefill_section(m, torch, dev, stream, l2,
                                                      workloads.opt13b_contraction(repeat=rank), sec_steps, peak_tops,
                                                      max_over)
    if "static_weight" in sec:
        line["static_weight"] = run_static_weight(m, torch, dev, stream, l2, p, X, W, Y, sec_steps, peak_tops,
                                                  max_over)
    if "decode" in sec and args.decode_steps > 0:
        same = (K, N) == (DECODE_K, DECODE_N)
        line["decode"] = {
            "workload": "decode: M in (1, 8, 32) tokens x K=12288 x N=49152, 7 outlier columns in every row",
            "timing": "CUDA events around each whole forward (no event between its kernels); GB/s = "
                      "algorithmic bytes / step time, vs measured HBM copy bandwidth",
            "weight": "the headline's prepared 175B-scale weight" if same else "a seeded K=12288 x N=49152 weight",
            "hbm_peak_gbs": peaks["hbm_gbs"],
            "shapes": run_decode(m, torch, dev, stream, l2, args.decode_steps, peaks, max_over, rank,
                                 w=w if same else None)}
    if "sweep" in sec and args.sweep_steps > 0:
        line["sweep"] = run_sweep(m, torch, dev, stream, l2, args.sweep_steps, peaks, peak_tops, max_over, rank)
    m.int8mm_free(w)
    del W
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(p, args.cpu_rows, acc_rows, acc_exact)
        oa = cb.pop("oracle_accuracy", None)
        if oa is not None:
            line["accuracy"]["decomposed_oracle"] = oa
            line["accuracy"]["oracle_note"] = "the CPU oracle's Y on the same rows (from the cpu_baseline leg)"
        line["cpu_baseline"] = cb
    if rank == 0:
        print(json.dumps(line), flush=True)
    if distributed:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
