#!/usr/bin/env python3
"""Benchmark of the fused Kronecker transform + INT4 path on B200.

Workload: the hidden-size-8192 configuration -- T = 8192 tokens of
n = 8192 (= 64 x 128) bf16, per-channel cinv, alpha = 0.85.  One step is one
kq_transform_quant call over the T tokens (the whole path: scale, both
contractions, absmax, quantise, pack).  Inputs rotate over buffer sets whose
total exceeds 2x the L2 size, so each step reads x from HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

With N > 1 it runs under torch.distributed (one process per GPU, NCCL); every
rank processes its own shard of T tokens (weak scaling, no data-path
collective); the timed region is bracketed by barriers and the reported time
is the max over ranks.  ``--impl reference`` times the fp64 CPU oracle on the
host cores instead (rank 0 only).  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from kronecker_factored_transforms_b200.workloads import (make_workload, workload_bytes,  # noqa: E402
                                                          workload_flops)

WORKLOAD = "hidden8192"
E2E_CHUNKS = 8  # chunks of a step in the end-to-end leg
METRIC = "tokens/s and % roofline (HBM/tensor) for fused Kronecker transform+INT4 at n=8192"
UNIT = "tokens/s"
PROFILES = os.path.join(ROOT, "profiles")
KERNEL_SOURCES = ["kronecker_factored_transforms_b200/csrc/kq_fused.cu",
                  "kronecker_factored_transforms_b200/csrc/kq_tc05.cu",
                  "kronecker_factored_transforms_b200/csrc/kq_tc05_ptx.cuh",
                  "kronecker_factored_transforms_b200/csrc/kq_warp_mma.cu",
                  "kronecker_factored_transforms_b200/csrc/kq_common.cuh",
                  "kronecker_factored_transforms_b200/csrc/kq_tile.cuh",
                  "kronecker_factored_transforms_b200/csrc/kq_wait.cuh"]


def parse():
    global WORKLOAD
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["transform", "gemm", "two_stage", "headwise"], default="transform",
                    help="transform: the fused transform + INT4 path (default); gemm: the W4A4 product "
                         "of packed codes that consumes it (M = N = K = 8192); two_stage: the path for "
                         "factors above 128 (--two-stage-config); headwise: the per-head key/value "
                         "transform + INT4 (8192 tokens x 32 heads x 128)")
    ap.add_argument("--config", choices=["hidden8192", "llama7b_hidden", "mlp14336", "mlp14336_cinv", "hidden5120",
                                         "sweep4096"],
                    default=WORKLOAD,
                    help="configuration of the transform workload (both arms); the default is the headline one")
    ap.add_argument("--two-stage-config", choices=["square65536", "ffn28672"], default="square65536")
    ap.add_argument("--gemm-out", choices=["fp32", "bf16"], default="fp32",
                    help="output dtype of the gemm workload (kq_w4a4_gemm or kq_w4a4_gemm_bf16)")
    ap.add_argument("--headwise-format", choices=["int4", "nvfp4"], default="int4",
                    help="rows of the headwise workload: INT4 with one scale, or NVFP4 (E2M1, an E4M3 scale per 16)")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-seconds", type=float, default=120.0,
                    help="CPU time the reference arm's warm-up + timed steps aim at")
    ap.add_argument("--sustained-ms", type=float, default=250.0,
                    help="length of the sustained leg (back-to-back launches with their own clock record); 0 skips it")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer leg (profiling runs)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="token count of the transform workload instead of its own (profiling runs on a "
                         "smaller case; the JSON line's config names the count used)")
    args = ap.parse_args()
    WORKLOAD = args.config
    return args


def metric_for(w):
    """The headline metric; other transform configurations name their own n."""
    return METRIC if w.n == 8192 else METRIC.replace("at n=8192", "at n=%d" % w.n)


def config_dict(w, extra=None):
    d = {"workload": "%s: T=%d tokens/GPU, n=%d (n1=%d, n2=%d), %s, alpha=%g"
         % (WORKLOAD, w.T, w.n, w.n1, w.n2, "cinv per channel" if w.cinv is not None else "no cinv", w.alpha),
         "T": w.T, "n": w.n, "n1": w.n1, "n2": w.n2, "alpha": w.alpha, "cinv": w.cinv is not None}
    if extra:
        d.update(extra)
    return d


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        p = os.path.join(ROOT, rel)
        if os.path.exists(p):
            h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_name):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources; else None."""
    p = os.path.join(PROFILES, "traffic_%s.json" % WORKLOAD)
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("kernel") != kernel_name or d.get("source_hash") != kernel_source_hash():
        return None
    return d.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# Multi-rank host logic: every rank owns one T-token shard; the step time is
# the maximum over ranks and the value counts the tokens of all ranks.

def max_over_ranks(x, device, world):
    """Max of a per-rank float over the process group (identity when world == 1)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(world, tokens_per_rank, steps, ms):
    """Tokens processed by all ranks over ``steps`` steps, divided by the
    slowest rank's elapsed time ``ms``."""
    return world * tokens_per_rank * steps / (ms / 1e3)


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline leg and the reference arm).

def cpu_model():
    """The host CPU's model name from /proc/cpuinfo (None where unavailable)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def cpu_fields():
    """Host facts for a cpu_baseline record: the CPU model and the logical CPUs
    the process may use (the oracle's thread count is reported as `cores`)."""
    try:
        avail = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        avail = os.cpu_count()
    return {"cpu_model": cpu_model(), "hardware_concurrency": os.cpu_count(), "cpus_available": avail}


def time_oracle(w, seconds, max_tokens=None):
    """The oracle on the host cores for about `seconds`: passes over the
    workload's rows, in pieces of about a second, until the time is reached
    (or `max_tokens`).  Returns (tokens/s, threads, tokens, seconds)."""
    import oracle
    oracle.build()
    nth = oracle.default_threads()
    probe = min(w.T, max(nth, 16))
    t0 = time.perf_counter()
    oracle.transform_quant(w.x[:probe], w.P1, w.P2, w.cinv, w.alpha, w.n1, w.n2, nthreads=nth,
                           want_codes=False)
    per_tok = (time.perf_counter() - t0) / probe
    piece = int(max(probe, min(w.T, 1.0 / max(per_tok, 1e-9))))
    done, row = 0, 0
    t0 = time.perf_counter()
    while True:
        take = min(piece, w.T - row)
        if max_tokens:
            take = min(take, max_tokens - done)
        oracle.transform_quant(w.x[row:row + take], w.P1, w.P2, w.cinv, w.alpha, w.n1, w.n2, nthreads=nth,
                               want_codes=False)
        done += take
        row = (row + take) % w.T
        el = time.perf_counter() - t0
        if el >= seconds or (max_tokens and done >= max_tokens):
            return done / el, nth, done, el


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = make_workload(WORKLOAD)
    import oracle
    oracle.build()
    nth = oracle.default_threads()
    # size each step so that warm-up + timed steps stay within ~2 minutes
    probe = min(w.T, max(nth, 16))
    t0 = time.perf_counter()
    oracle.transform_quant(w.x[:probe], w.P1, w.P2, w.cinv, w.alpha, w.n1, w.n2, nthreads=nth,
                           want_codes=False)
    per_tok = (time.perf_counter() - t0) / probe
    budget = args.ref_seconds / max(1, args.steps + args.warmup)
    sample = int(max(1, min(w.T, budget / max(per_tok, 1e-9))))
    for _ in range(args.warmup):
        oracle.transform_quant(w.x[:sample], w.P1, w.P2, w.cinv, w.alpha, w.n1, w.n2, nthreads=nth,
                               want_codes=False)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.transform_quant(w.x[:sample], w.P1, w.P2, w.cinv, w.alpha, w.n1, w.n2, nthreads=nth,
                               want_codes=False)
    el = time.perf_counter() - t0
    value = sample * args.steps / el
    line = {"impl": "reference", "metric": metric_for(w), "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(w, {"sample_tokens_per_step": sample}),
            "cpu_baseline": dict({"value": value, "unit": UNIT, "cores": nth, "kind": "oracle",
                                  "sample": "first %d of %d tokens per step, fp64 C oracle, %d threads"
                                            % (sample, w.T, nth)}, **cpu_fields()),
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# Clock sampling during the timed region (NVML, read-only).

class ClockSampler:
    REASONS = {"gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
               "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
               "display_clock_setting": 0x100}

    def __init__(self, device_index):
        self.samples, self.reasons, self.ok = [], 0, False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def sample(self):
        if not self.ok:
            return
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
        except Exception:
            pass

    def _loop(self):
        while not self._stop.wait(0.005):
            self.sample()

    def __enter__(self):
        self.sample()
        self._t = threading.Thread(target=self._loop, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        self._t.join()
        self.sample()

    def report(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"]}
        names = [k for k, v in self.REASONS.items() if self.reasons & v and k != "gpu_idle"]
        other = self.reasons & ~sum(self.REASONS.values())
        if other:
            names.append("0x%x" % other)  # a reason bit this table does not name
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------------------

def run_gemm(args):
    """The W4A4 product y = sx sw (qx qw^T) of a hidden-8192 layer: M tokens x
    N output channels x K = n, packed INT4 codes in, fp32 (or bf16) out.  One
    step is one kq_w4a4_gemm (kq_w4a4_gemm_bf16) call; ops = 2 M N K.  Single
    GPU only."""
    import torch
    from kronecker_factored_transforms_b200 import _lib
    M = N = K = 8192
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(8192)
    qx = torch.randint(0, 256, (M, K // 2), dtype=torch.uint8, device=dev, generator=g)
    qw = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=dev, generator=g)
    sx = torch.rand(M, device=dev, generator=g)
    sw = torch.rand(N, device=dev, generator=g)
    bf16 = args.gemm_out == "bf16"
    y = torch.empty((M, N), dtype=torch.bfloat16 if bf16 else torch.float32, device=dev)
    gemm = _lib.kq_w4a4_gemm_bf16 if bf16 else _lib.kq_w4a4_gemm
    stream = torch.cuda.current_stream(dev)
    for _ in range(max(3, args.warmup)):
        gemm(qx, sx, qw, sw, y, M, N, K, stream=stream.cuda_stream)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(0)
    with sampler:
        e0.record(stream)
        for _ in range(args.steps):
            gemm(qx, sx, qw, sw, y, M, N, K, stream=stream.cuda_stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / args.steps
    tops = 2.0 * M * N * K / (ms * 1e-3) / 1e12
    hbm_peak, tf_peak, kind = measured_peaks()
    int8_peak = 2.0 * tf_peak  # dense int8 runs at twice the bf16 rate
    line = {"metric": "TOPS of the W4A4 product of packed INT4 codes (M = N = K = 8192)", "value": tops,
            "unit": "TOPS", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int4 (int8 MMA)",
            "data": "synthetic", "config": {"workload": "w4a4 gemm M=N=K=8192, random codes and scales, %s out"
                                                         % args.gemm_out, "M": M, "N": N, "K": K,
                                             "out": args.gemm_out},
            "roofline": {"bound": "tensor", "achieved": tops, "peak": int8_peak, "unit": "TOP/s",
                         "frac": tops / int8_peak, "traffic": None,
                         "peak_source": "2 x %s bf16 TF/s (int8 dense rate)" % kind},
            "gpu_launches": args.steps, "clocks": sampler.report()}
    print(json.dumps(line), flush=True)
    return 0


def run_two_stage(args):
    """The two-stage path for factors above 128 on one large-factor workload.
    One step is one kq_transform_quant_two_stage call (stage 1 and stage 2
    kernels); x and the outputs rotate over two buffer sets, and the 4 T n
    byte workspace is rewritten every step.  Roofline: the slower of the
    algorithmic bytes (2.5 n + 4 per token) at the measured HBM peak and the
    factored flops 2 n (n1 + n2) per token at the measured bf16 peak.
    Single GPU only."""
    import torch
    from kronecker_factored_transforms_b200 import _lib
    name = args.two_stage_config
    w = make_workload(name)
    T, n1, n2, n = w.T, w.n1, w.n2, w.n
    dev = torch.device("cuda", 0)
    R = 2
    xs = [torch.from_numpy(w.x.view(np.int16)).to(dev) for _ in range(R)]
    qs = [torch.empty((T, n // 2), dtype=torch.uint8, device=dev) for _ in range(R)]
    ss = [torch.empty((T,), dtype=torch.float32, device=dev) for _ in range(R)]
    need = _lib.kq_two_stage_workspace_bytes(T, n1, n2)
    ws = torch.empty((need,), dtype=torch.uint8, device=dev)
    P1 = torch.from_numpy(w.P1.view(np.int16)).to(dev)
    P2 = torch.from_numpy(w.P2.view(np.int16)).to(dev)
    cinv = torch.from_numpy(w.cinv).to(dev) if w.cinv is not None else None
    stream = torch.cuda.current_stream(dev)

    def step(i):
        _lib.kq_transform_quant_two_stage(xs[i % R], P1, P2, cinv, w.alpha, qs[i % R], ss[i % R], ws, need,
                                          T, n1, n2, stream=stream.cuda_stream)

    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(0)
    with sampler:
        e0.record(stream)
        for i in range(args.steps):
            step(i)
        e1.record(stream)
        torch.cuda.synchronize(dev)
    if _lib.kq_device_error(stream) != 0:
        raise RuntimeError("a bounded wait timed out inside the kernel")
    ms = e0.elapsed_time(e1) / args.steps
    hbm_peak, tf_peak, kind = measured_peaks()
    bytes_launch, flops_launch = workload_bytes(T, n), workload_flops(T, n1, n2)
    t_hbm, t_tc = bytes_launch / (hbm_peak * 1e9), flops_launch / (tf_peak * 1e12)
    sec = ms / 1e3
    if t_hbm >= t_tc:
        roof = {"bound": "hbm", "achieved": bytes_launch / sec / 1e9, "peak": hbm_peak, "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": flops_launch / sec / 1e12, "peak": tf_peak, "unit": "TFLOP/s"}
    roof.update({"frac": roof["achieved"] / roof["peak"], "traffic": None,
                 "peak_source": "%s (MEASURED_PEAKS.json)" % kind, "bytes_per_launch": bytes_launch,
                 "flops_per_launch": flops_launch, "roofline_time_us": 1e6 * max(t_hbm, t_tc),
                 "measured_time_us": 1e3 * ms, "workspace_bytes": need})
    line = {"metric": "tokens/s and % roofline of the two-stage Kronecker transform+INT4 (factors above 128)",
            "value": T / sec, "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": "%s: T=%d, n=%d (n1=%d, n2=%d), alpha=%g, cinv %s" % (
                name, T, n, n1, n2, w.alpha, "per channel" if w.cinv is not None else "none"),
                       "T": T, "n1": n1, "n2": n2, "l2": "x and outputs rotate over 2 sets; the workspace "
                                                          "(%d MB) is rewritten every step" % (need >> 20)},
            "roofline": roof, "gpu_launches": 2 * args.steps, "clocks": sampler.report()}
    print(json.dumps(line), flush=True)
    return 0


def run_headwise(args):
    """The per-head transform of the key/value cache: 8192 tokens x 32 heads of
    head_dim 128 (262144 rows), one bf16 factor, INT4 per row.  One step is one
    kq_headwise_transform_quant call; inputs rotate over enough buffer sets to
    exceed 2x L2.  Roofline: algorithmic bytes 2.5 D + 4 per row at the measured
    HBM peak (2 D^2 flops per row are far below the tensor peak).  Single GPU."""
    import torch
    from kronecker_factored_transforms_b200 import _lib
    T, heads, D = 8192, 32, 128
    R = T * heads
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(4096)
    set_bytes = R * (2 * D + D // 2 + 4)
    props = torch.cuda.get_device_properties(dev)
    l2 = int(getattr(props, "L2_cache_size", 126 * 2 ** 20))
    nset = max(2, math.ceil(2 * l2 / set_bytes) + 1)
    xs = [torch.randn((T, heads * D), device=dev, generator=g).to(torch.bfloat16) for _ in range(nset)]
    Q, _ = torch.linalg.qr(torch.randn((D, D), device=dev, generator=g, dtype=torch.float64))
    Ph = Q.to(torch.bfloat16).contiguous()
    qs = [torch.empty((T, heads * D // 2), dtype=torch.uint8, device=dev) for _ in range(nset)]
    ss = [torch.empty((T, heads), dtype=torch.float32, device=dev) for _ in range(nset)]
    fp4 = args.headwise_format == "nvfp4"
    bs = [torch.empty((T, heads * D // 16), dtype=torch.uint8, device=dev) for _ in range(nset)] if fp4 else None
    stream = torch.cuda.current_stream(dev)

    def step(i):
        if fp4:
            _lib.kq_headwise_transform_quant_nvfp4(xs[i % nset], Ph, qs[i % nset], bs[i % nset], ss[i % nset], T,
                                                   heads, D, stream=stream.cuda_stream)
        else:
            _lib.kq_headwise_transform_quant(xs[i % nset], Ph, 0.9, qs[i % nset], ss[i % nset], T, heads, D,
                                             stream=stream.cuda_stream)

    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(0)
    with sampler:
        e0.record(stream)
        for i in range(args.steps):
            step(i)
        e1.record(stream)
        torch.cuda.synchronize(dev)
    if _lib.kq_device_error(stream) != 0:
        raise RuntimeError("a bounded wait timed out inside the kernel")
    ms = e0.elapsed_time(e1) / args.steps
    hbm_peak, _, kind = measured_peaks()
    bytes_launch = R * (2 * D + D // 2 + 4 + (D // 16 if fp4 else 0))
    achieved = bytes_launch / (ms / 1e3) / 1e9
    fmt = "NVFP4" if fp4 else "INT4"
    line = {"metric": "rows/s and %% HBM roofline of the per-head key/value transform + %s" % fmt, "value": R / (ms / 1e3),
            "unit": "rows/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "headwise: %d tokens x %d heads x head_dim %d, N(0,1) rows, orthogonal bf16 "
                                   "factor, %s" % (T, heads, D, "NVFP4" if fp4 else "INT4, alpha 0.9"), "rows": R,
                       "head_dim": D, "format": fmt,
                       "l2": "inputs rotate over %d buffer sets (%.0f MB > 2x L2)" % (nset, nset * set_bytes / 1e6)},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                         "frac": achieved / hbm_peak, "traffic": None, "peak_source": "%s (MEASURED_PEAKS.json)" % kind,
                         "bytes_per_launch": bytes_launch},
            "gpu_launches": args.steps, "clocks": sampler.report()}
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "gemm":
        return run_gemm(args)
    if args.workload == "two_stage":
        return run_two_stage(args)
    if args.workload == "headwise":
        return run_headwise(args)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world > 1:
        raise SystemExit("--gpus %d but WORLD_SIZE=%d" % (args.gpus, world))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    from kronecker_factored_transforms_b200 import _lib

    w = make_workload(WORKLOAD, T=args.tokens, shard=rank)
    T, n1, n2, n = w.T, w.n1, w.n2, w.n
    kernel = _lib.kq_kernel_for(T, n1, n2, w.cinv is not None, w.alpha)

    # Rotating device buffer sets: total > 2x L2 so x comes from HBM every step.
    props = torch.cuda.get_device_properties(dev)
    l2 = int(getattr(props, "L2_cache_size", 126 * 2 ** 20))
    set_bytes = T * n * 2 + T * n // 2 + T * 4
    R = max(2, math.ceil(2 * l2 / set_bytes) + 1)
    x0 = torch.from_numpy(w.x.view(np.int16)).to(dev)
    xs = [x0] + [x0.clone() for _ in range(R - 1)]
    qs = [torch.empty((T, n // 2), dtype=torch.uint8, device=dev) for _ in range(R)]
    ss = [torch.empty((T,), dtype=torch.float32, device=dev) for _ in range(R)]
    P1 = torch.from_numpy(w.P1.view(np.int16)).to(dev)
    P2 = torch.from_numpy(w.P2.view(np.int16)).to(dev)
    cinv = torch.from_numpy(w.cinv).to(dev) if w.cinv is not None else None

    stream = torch.cuda.current_stream(dev)
    sptr = stream.cuda_stream
    fn = _lib.lib.kq_transform_quant
    ptrs = [(xs[i].data_ptr(), qs[i].data_ptr(), ss[i].data_ptr()) for i in range(R)]
    p1, p2, ci = P1.data_ptr(), P2.data_ptr(), cinv.data_ptr() if cinv is not None else None
    alpha = w.alpha

    def step(i):
        xp, qp, sp = ptrs[i % R]
        st = fn(xp, p1, p2, ci, alpha, qp, sp, T, n1, n2, sptr)
        if st != 0:
            raise RuntimeError("kq_transform_quant: %s" % _lib.kq_status_string(st))

    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize(dev)

    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with sampler:
        ev0.record(stream)
        for i in range(args.steps):
            step(i)
        ev1.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1), dev, world)

    # Sustained leg: the same launches back to back for about --sustained-ms, with
    # a clock record of their own (a short timed region may see only boost
    # clocks); reported beside `value`, which stays on the requested step count.
    sustained = None
    if args.sustained_ms > 0:
        n_sus = max(args.steps, int(math.ceil(args.sustained_ms / max(ms / args.steps, 1e-3))))
        sampler_sus = ClockSampler(dev.index if dev.index is not None else 0)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        with sampler_sus:
            ev0.record(stream)
            for i in range(n_sus):
                step(i)
            ev1.record(stream)
            torch.cuda.synchronize(dev)
        ms_sus = max_over_ranks(ev0.elapsed_time(ev1), dev, world)
        sustained = {"launches": n_sus, "ms": ms_sus, "us_per_launch": 1e3 * ms_sus / n_sus,
                     "clocks": sampler_sus.report()}
    if _lib.kq_device_error(stream) != 0:
        raise RuntimeError("a bounded wait timed out inside the kernel")

    # End to end through the C ABI from pinned host buffers: H2D inputs,
    # kernel, D2H codes + scales, every step.  The step's tokens go in
    # E2E_CHUNKS chunks on three streams, so the copy in of chunk k + 1, the
    # kernel on chunk k and the copy out of chunk k - 1 overlap.
    hx = torch.from_numpy(w.x.view(np.int16)).pin_memory()
    hp1 = torch.from_numpy(w.P1.view(np.int16)).pin_memory()
    hp2 = torch.from_numpy(w.P2.view(np.int16)).pin_memory()
    hci = torch.from_numpy(w.cinv).pin_memory() if w.cinv is not None else None
    hq = torch.empty((T, n // 2), dtype=torch.uint8).pin_memory()
    hs = torch.empty((T,), dtype=torch.float32).pin_memory()
    dx, dq, dsc = xs[0], qs[0], ss[0]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    cs = (T + E2E_CHUNKS - 1) // E2E_CHUNKS
    chunks = [(lo, min(T, lo + cs)) for lo in range(0, T, cs)]
    ev_in = [torch.cuda.Event() for _ in chunks]
    ev_k = [torch.cuda.Event() for _ in chunks]
    ev_done = torch.cuda.Event()

    def e2e_step():
        s_in.wait_stream(stream)  # the previous step's kernels have read their inputs
        with torch.cuda.stream(s_in):
            P1.copy_(hp1, non_blocking=True)
            P2.copy_(hp2, non_blocking=True)
            if hci is not None:
                cinv.copy_(hci, non_blocking=True)
        for k, (lo, hi) in enumerate(chunks):
            with torch.cuda.stream(s_in):
                dx[lo:hi].copy_(hx[lo:hi], non_blocking=True)
                ev_in[k].record(s_in)
            stream.wait_event(ev_in[k])
            _lib.kq_transform_quant(dx[lo:hi], P1, P2, cinv, alpha, dq[lo:hi], dsc[lo:hi], hi - lo, n1, n2,
                                    stream=sptr)
            ev_k[k].record(stream)
            s_out.wait_event(ev_k[k])
            with torch.cuda.stream(s_out):
                hq[lo:hi].copy_(dq[lo:hi], non_blocking=True)
                hs[lo:hi].copy_(dsc[lo:hi], non_blocking=True)
        ev_done.record(s_out)
        stream.wait_event(ev_done)  # the step ends when its last result is on the host

    h2d = hx.numel() * 2 + hp1.numel() * 2 + hp2.numel() * 2 + (hci.numel() * 4 if hci is not None else 0)
    d2h = hq.numel() + hs.numel() * 4
    e2e_ms = float("nan")
    if not args.no_e2e:
        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_ms, dev, world)

    clocks = sampler.report()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    ms_step = ms / args.steps
    value = whole_job_tokens_per_s(world, T, args.steps, ms)
    hbm_peak, tf_peak, peak_kind = measured_peaks()
    bytes_launch = workload_bytes(T, n)
    flops_launch = workload_flops(T, n1, n2)
    achieved = bytes_launch / (ms_step / 1e3) / 1e9
    t_hbm = bytes_launch / (hbm_peak * 1e9)
    t_tc = flops_launch / (tf_peak * 1e12)
    roof = {"bound": "hbm" if t_hbm >= t_tc else "tensor", "achieved": achieved, "peak": hbm_peak,
            "unit": "GB/s", "frac": achieved / hbm_peak, "traffic": recorded_traffic(kernel) if args.tokens is None else None,
            "peak_source": "%s (MEASURED_PEAKS.json hbm_gbs)" % peak_kind if peak_kind == "measured"
            else "fallback 6650 GB/s",
            "kernel": kernel, "bytes_per_launch": bytes_launch, "flops_per_launch": flops_launch,
            "tensor_frac_algorithmic": (flops_launch / (ms_step / 1e3) / 1e12) / tf_peak,
            "roofline_time_us": 1e6 * max(t_hbm, t_tc), "measured_time_us": 1e3 * ms_step}
    line = {"metric": metric_for(w), "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_dict(w, {"parallelism": "token-row shards, %d rank(s)" % world,
                                      "l2": "inputs rotate over %d buffer sets (%.0f MB > 2x L2)"
                                            % (R, R * set_bytes / 1e6),
                                      "kernel": kernel}),
            "roofline": roof,
            "e2e": None if args.no_e2e else
                   {"value": whole_job_tokens_per_s(world, T, args.e2e_steps, e2e_ms), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": args.steps, "clocks": clocks}
    if sustained is not None:
        us = sustained["us_per_launch"]
        sustained.update({"tokens_per_s": whole_job_tokens_per_s(world, T, sustained["launches"], sustained["ms"]),
                          "achieved_gbs": bytes_launch / (us / 1e6) / 1e9,
                          "frac": bytes_launch / (us / 1e6) / 1e9 / hbm_peak})
        line["sustained"] = sustained
    if world == 1 and not args.no_cpu_baseline:
        v, cores, sample, el = time_oracle(w, args.cpu_seconds)
        line["cpu_baseline"] = dict({"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                                     "sample": "%d tokens (the workload's rows, repeated if needed) of %d per step, "
                                               "fp64 C oracle, %.1f s" % (sample, T, el)}, **cpu_fields())
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
