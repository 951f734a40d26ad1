#!/usr/bin/env python
"""Throughput of the block-scaled FP4 hot path on B200 (one JSON line on stdout).

Default workload (N=1): the decode-shaped NVFP4 GEMM -- M=16 tokens, N=28672, K=8192;
weights N(0, 0.02) pre-quantized to NVFP4 once (untimed); BF16 activations N(0,1) with
0.1% outliers x50 quantized on the fly every step; BF16 output.  One step = tensor
amax + NVFP4 quantize of the activations + the FP4 GEMM.  Memory-bound, so the metric
is GB/s of algorithmic bytes (each operand's stored bytes read once, output written
once; the activations are read twice, once for the amax and once for the encode).

The same JSON line carries a sub-record for each other configuration (prefill 8192^3 with
BF16 activations quantized every step; the training step at S = 16384; the MXFP4 grouped
MoE GEMM; the quantize kernels alone), each with its roofline, its own clock sample, an
end-to-end figure with host buffers and the oracle's rate on a bounded sample.
--workload prefill | moe | train | quantize prints one of them alone.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--workload ...]

Multi-GPU (torchrun, one rank per GPU): every rank runs its own copy of the workload
(independent problems; no data-path collective), timed between a barrier and
synchronize on both sides; the slowest rank's time gives the whole-job value.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "NVFP4 GEMM TFLOPS & % dense-FP4 peak; quantize/decode GB/s & % HBM BW"
L2_BYTES = 126 * 1024 * 1024


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p.get("hbm_gbs", 6650.0), p.get("bf16_tflops", 1590.0), p.get("bf16_tflops_sustained", 1400.0), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------- distributed plumbing
class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None

    def init(self, backend="nccl"):
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self):
        if self.pg:
            if self.pg.get_backend() == "nccl":
                self.pg.barrier(device_ids=[torch.cuda.current_device()])
            else:
                self.pg.barrier()

    def max(self, v: float, device=None) -> float:
        if not self.pg:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


def whole_job_value(units_per_rank: float, world: int, max_ms: float) -> float:
    """Units all ranks processed per second, on the slowest rank's clock."""
    return units_per_rank * world / (max_ms * 1e-3)


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""

    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.proc = subprocess.Popen(["nvidia-smi", "-i", ident, f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append((time.time(), ln.strip()))

    def mark(self):
        return time.time()

    def stop(self, t0, t1):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.12)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = [ln for (t, ln) in self.lines if t0 - 0.06 <= t <= t1 + 0.06] or [ln for _, ln in self.lines[-3:]]
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in rows:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                smax.append(float(f[1]))
            except ValueError:
                continue
            for name, val in zip(names, f[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- decode workload
def decode_bytes(m: int, n: int, k: int):
    """Algorithmic bytes: (activation quantize, GEMM, whole step)."""
    quant = 2 * (m * k * 2) + m * k // 2 + m * k // 16          # amax read + encode read + codes + scales
    gemm = n * k // 2 + n * k // 16 + m * k // 2 + m * k // 16 + m * n * 2
    return quant, gemm, quant + gemm


def traffic_for(kernel_key: str):
    """Per-launch DRAM bytes from the committed ncu summary, if the kernel's sources (the
    entry's "sources", else the whole library) have not changed since it was taken
    (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    try:
        with open(path) as f:
            t = json.load(f)
        from block_scaled_fp4_04_b200 import build as fp4_build
        entry = t.get(kernel_key)
        if not entry:
            return None
        srcs = entry.get("sources")
        fp = fp4_build.sources_fingerprint(srcs) if srcs else fp4_build._fingerprint()
        if entry.get("fingerprint") != fp:
            return None
        return entry.get("dram_bytes_per_launch")
    except Exception:
        return None


def run_decode(args, dist: Dist, dev):
    import block_scaled_fp4_04_b200 as fp4
    m, n, k = 16, 28672, 8192
    x, w = workloads.decode_inputs(device="cpu")
    x = x.to(dev)
    # weight copies so that the rotating working set is larger than L2 (untimed setup)
    w_dev = w.to(dev)
    per_copy = n * k // 2 + fp4.fp4_scales_bytes(n, k, fp4.NVFP4)
    copies = max(2, int(np.ceil(3 * L2_BYTES / per_copy)))
    wq = [fp4.quantize(w_dev, fp4.NVFP4, 16) for _ in range(copies)]
    del w_dev
    xq_codes = torch.empty(m, k // 2, dtype=torch.uint8, device=dev)
    xq_scales = torch.empty(fp4.fp4_scales_bytes(m, k, fp4.NVFP4), dtype=torch.uint8, device=dev)
    xq_g = torch.empty(1, dtype=torch.float32, device=dev)
    ws_n = fp4.fp4_gemm_bf16a_workspace_size(m, n, k)
    ws = torch.zeros(ws_n, dtype=torch.uint8, device=dev)
    d = torch.empty(m, n, dtype=torch.bfloat16, device=dev)
    L = fp4.lib()
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    P = lambda t: t.data_ptr()
    xp, xcp, xsp, xgp, wsp, dp = P(x), P(xq_codes), P(xq_scales), P(xq_g), P(ws), P(d)
    wp = [(P(q.codes), P(q.scales), P(q.g)) for q in wq]

    def step(i, src=xp):
        # one launch: every CTA of the decode kernel derives the activations' global scale,
        # quantizes its K segment of them to NVFP4 and streams its share of the
        # pre-quantized weights through the tensor cores
        c, s, g = wp[i % copies]
        rc = L.fp4_gemm_bf16a(src, c, s, g, m, n, k, dp, fp4.BF16, xcp, xsp, xgp, wsp, ws_n,
                              fp4.GEMM_WEIGHTS_READY, sp)
        if rc:
            raise RuntimeError(fp4.fp4_last_error())

    gws_n = fp4.fp4_gemm_workspace_size(m, n, k, fp4.NVFP4)
    gws = torch.zeros(gws_n, dtype=torch.uint8, device=dev)
    gwsp = P(gws)

    def gemm_only(i):
        # the same GEMM on the activations the last step quantized (no quantize work)
        c, s, g = wp[i % copies]
        rc = L.fp4_gemm_ex(fp4.NVFP4, xcp, xsp, xgp, c, s, g, m, n, k, dp, fp4.BF16, gwsp, gws_n,
                           fp4.GEMM_WEIGHTS_READY, sp)
        if rc:
            raise RuntimeError(fp4.fp4_last_error())

    qb, gb, step_bytes = decode_bytes(m, n, k)
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if fp4.fp4_get_status() != fp4.OK:
        raise RuntimeError("device status latched an error during warm-up")

    # Timed region: exactly K steps between a barrier and a synchronize on both sides,
    # repeated back to back until at least half a second of timed work, so that the clock
    # samples cover what is measured; the reported time is the median batch (each batch's
    # time the maximum over ranks).  Every rank runs the same number of batches.
    K = args.steps
    clocks = ClockSampler(dev.index or 0)
    time.sleep(0.15)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    batch_ms, total_ms = [], 0.0
    min_ms = 500.0 if MIN_S_OVERRIDE is None else MIN_S_OVERRIDE * 1e3
    c0 = clocks.mark()
    while True:
        dist.barrier()
        torch.cuda.synchronize()
        t_start.record()
        for i in range(K):
            step(i)
        t_end.record()
        torch.cuda.synchronize()
        dist.barrier()
        b = dist.max(t_start.elapsed_time(t_end), dev)
        batch_ms.append(b)
        total_ms += b
        if total_ms >= min_ms and len(batch_ms) >= 3:
            break
    c1 = clocks.mark()
    clk = clocks.stop(c0, c1)
    if fp4.fp4_get_status() != fp4.OK:
        raise RuntimeError("device status latched an error during the timed steps")
    max_ms = statistics.median(batch_ms)

    # The step is one launch of one kernel, so the events around the timed batch give its
    # average launch duration.  For reference, the same GEMM on pre-quantized activations
    # is timed in a batch of its own.
    for i in range(args.warmup):
        gemm_only(i)
    torch.cuda.synchronize()
    g0 = torch.cuda.Event(enable_timing=True)
    g1 = torch.cuda.Event(enable_timing=True)
    g0.record()
    for i in range(K):
        gemm_only(i)
    g1.record()
    torch.cuda.synchronize()
    if fp4.fp4_get_status() != fp4.OK:
        raise RuntimeError("device status latched an error in the GEMM batch")
    prequant_ms = dist.max(g0.elapsed_time(g1), dev) / K
    step_avg_ms = max_ms / K

    # end to end through the C ABI with host buffers: H2D of the step's activations
    # (pinned), quantize + GEMM, D2H of the result, every step.
    x_host = x.cpu().pin_memory()
    d_host = torch.empty(m, n, dtype=torch.bfloat16).pin_memory()
    x_stage = torch.empty_like(x)
    xs = P(x_stage)
    for i in range(min(args.warmup, 20)):
        x_stage.copy_(x_host, non_blocking=True)
        step(i, xs)
        d_host.copy_(d, non_blocking=True)
    torch.cuda.synchronize()
    dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(K):
        x_stage.copy_(x_host, non_blocking=True)
        step(i, xs)
        d_host.copy_(d, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    dist.barrier()
    e2e_ms = dist.max(e0.elapsed_time(e1), dev)

    hbm, bf16, bf16_s, src = load_peaks()
    achieved = step_bytes / (step_avg_ms * 1e-3) / 1e9
    res = {
        "metric": METRIC,
        "value": whole_job_value(step_bytes * K, dist.world, max_ms) / 1e9,
        "unit": "GB/s",
        "n_gpus": dist.world,
        "steps": K,
        "warmup": args.warmup,
        "batches": len(batch_ms),
        "timing": f"median of {len(batch_ms)} back-to-back batches of exactly {K} steps, each between a barrier "
                  "and a synchronize, max over ranks",
        "ms_per_step": max_ms / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 codes, e4m3 block scales, fp32 accumulate), bf16 in/out",
        "data": "synthetic (seeded: W ~ N(0,0.02) fp32, X ~ N(0,1) bf16 with 0.1% x50 outliers)",
        "config": {"workload": "decode-shaped NVFP4 GEMM M=16 N=28672 K=8192, bf16 activations quantized "
                               "every step, bf16 out",
                   "M": m, "N": n, "K": k,
                   "step": "fp4_gemm_bf16a: amax + quantize(X) + FP4 GEMM in one launch",
                   "bytes_per_step": step_bytes,
                   "l2": f"weights rotate over {copies} pre-quantized copies "
                         f"({copies * per_copy / 2**20:.0f} MiB > 126 MiB L2)",
                   "parallelism": f"replicas x{dist.world} (independent problems)"},
        "tflops": 2.0 * m * n * k * dist.world / (max_ms / K * 1e-3) / 1e12,
        "roofline": {"bound": "hbm", "kernel": "fp4_decode_kernel<16, bf16 activations> (the whole step)",
                     "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "peak_source": f"{src} hbm_gbs (MEASURED_PEAKS.json)" if src == "measured" else src,
                     "algorithmic_bytes_per_launch": step_bytes, "launch_ms": step_avg_ms,
                     "launch_timing": f"{K} launches back to back, CUDA events around the batch",
                     "traffic": traffic_for("decode_step")},
        "prequantized_gemm": {"kernel": "fp4_decode_kernel<16, pre-quantized activations>",
                              "ms": prequant_ms, "GB/s": gb / (prequant_ms * 1e-3) / 1e9,
                              "frac": gb / (prequant_ms * 1e-3) / 1e9 / hbm},
        "e2e": {"value": whole_job_value(step_bytes * K, dist.world, e2e_ms) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": m * k * 2, "d2h_bytes_per_step": m * n * 2,
                "ms_per_step": e2e_ms / K},
        # one kernel launch per timed step
        "gpu_launches": K,
        "clocks": clk,
    }
    return res


# ---------------------------------------------------------------- the other configurations
FP4_PER_BF16 = 4.0  # nominal dense FP4 / BF16 tensor throughput ratio (9 / 2.25 PFLOP/s)
FP8_PER_BF16 = 2.0  # nominal dense FP8 / BF16 ratio (4.5 / 2.25 PFLOP/s): the mixed FP4 x FP8 MMA's rate
MIN_TIMED_S = 0.4   # each sub-workload is timed over at least this long (clock samples cover it)
MIN_S_OVERRIDE = None  # --min-seconds: one minimum for every timed loop (short runs under a profiler)


def _check(fp4):
    if fp4.fp4_get_status() != fp4.OK:
        raise RuntimeError("device status latched an error")


def _copies(per_copy_bytes: int) -> int:
    """Rotating copies so that one pass over them exceeds the L2 three times."""
    return max(1, int(np.ceil(3 * L2_BYTES / max(per_copy_bytes, 1))))


def timed_batches(fn, steps: int, warmup: int, dev_index: int, min_s: float = MIN_TIMED_S):
    """Warm-up, then back-to-back batches of `steps` calls of fn(i), each batch bracketed by
    CUDA events on the current stream, until at least min_s of timed work; returns the
    median ms per call over the batches, the batches, and the clocks sampled meanwhile."""
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    clocks = ClockSampler(dev_index)
    time.sleep(0.15)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if MIN_S_OVERRIDE is not None:
        min_s = MIN_S_OVERRIDE
    batches, total, i = [], 0.0, 0
    c0 = clocks.mark()
    while total < min_s * 1e3 or len(batches) < 3:
        e0.record()
        for _ in range(steps):
            fn(i)
            i += 1
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        batches.append(ms / steps)
        total += ms
    c1 = clocks.mark()
    clk = clocks.stop(c0, c1)
    return statistics.median(batches), batches, clk


def mma_peak(dev) -> dict:
    """The block-scaled MMA loop's throughput on every SM (library probe fp4_mma_peak)."""
    import block_scaled_fp4_04_b200 as fp4
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    cyc = torch.zeros(sms, dtype=torch.int64, device=dev)
    iters = 20000
    fp4.fp4_mma_peak(iters, sms, cyc)  # warm
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    fp4.fp4_mma_peak(iters, sms, cyc)
    e1.record()
    torch.cuda.synchronize()
    _check(fp4)
    ms = e0.elapsed_time(e1)
    flop = 2.0 * 128 * 256 * 64 * 4 * iters
    c = float(cyc.double().mean().item())
    return {"TFLOP/s": flop * sms / (ms * 1e-3) / 1e12, "flop_per_clk_per_sm": flop / c,
            "sm_ghz": c / (ms * 1e-3) / 1e9, "probe": "fp4_mma_peak: 4 x tcgen05.mma.kind::mxf4nvf4 "
            "M=128 N=256 K=64 per K step from shared memory, no loads, one CTA per SM"}


def _tensor_roofline(kernel: str, flop: float, ms: float, peaks: dict, traffic_key: str, extra=None) -> dict:
    achieved = flop / (ms * 1e-3) / 1e12
    r = {"bound": "tensor", "kernel": kernel, "achieved": achieved, "peak": peaks["fp4"], "unit": "TFLOP/s",
         "frac": achieved / peaks["fp4"], "peak_source": peaks["fp4_source"], "launch_ms": ms,
         "frac_of_mma_loop": achieved / peaks["mma_loop"] if peaks.get("mma_loop") else None,
         "frac_of_nominal_9pf": achieved / 9000.0, "traffic": traffic_for(traffic_key)}
    if extra:
        r.update(extra)
    return r


def _e2e(step_on, host_in: list, dev_in: list, host_out: list, dev_out: list, steps: int, warmup: int) -> float:
    """ms per step through the library with host buffers: every step copies the inputs from
    pinned host memory, runs the step, and reads the outputs back."""
    def one(i):
        for h, d in zip(host_in, dev_in):
            d.copy_(h, non_blocking=True)
        step_on(i)
        for h, d in zip(host_out, dev_out):
            h.copy_(d, non_blocking=True)
    ms, _, _ = timed_batches(one, max(1, min(steps, 20)), min(warmup, 3), torch.cuda.current_device(), min_s=0.2)
    return ms


def _oracle_rows_gemm_rate(x_rows: np.ndarray, fmt: int, blk: int, w_hat: np.ndarray, g=None, budget_s=4.0):
    """The oracle, as it stands, on a sample: quantize the given activation rows and take
    their FP64 product with the (already dequantized) weights; returns TFLOP/s of the
    sampled rows, the threads used, and the repetitions."""
    import oracle
    t0 = time.perf_counter()
    reps = 0
    while True:
        q = oracle.quantize(x_rows, fmt, blk, g_in=g)
        a_hat = oracle.dequantize(q["codes"], q["scales"], q["g"], fmt)
        oracle.gemm_reference(a_hat, w_hat)
        reps += 1
        if time.perf_counter() - t0 > budget_s or reps >= 50:
            break
    dt = time.perf_counter() - t0
    flop = 2.0 * x_rows.shape[0] * w_hat.shape[0] * w_hat.shape[1] * reps
    return flop / dt / 1e12, oracle.num_threads(), reps


def measure_prefill(args, dev, peaks, cpu: bool) -> dict:
    """Prefill-shaped NVFP4 GEMM 8192^3: BF16 activations (0.1% outliers x50) quantized every
    step (tensor amax, then 16-blocks), weights pre-quantized; BF16 out; tensor-bound."""
    import block_scaled_fp4_04_b200 as fp4
    m = n = k = 8192
    x, w = workloads.prefill_inputs(device="cpu")
    xd = x.to(dev)
    per_copy = n * k // 2 + fp4.fp4_scales_bytes(n, k, fp4.NVFP4)
    copies = _copies(per_copy)
    w_dev = w.to(dev)
    wq = [fp4.quantize(w_dev, fp4.NVFP4, 16) for _ in range(copies)]
    del w_dev
    L = fp4.lib()
    P = lambda t: t.data_ptr()
    xc = torch.empty(m, k // 2, dtype=torch.uint8, device=dev)
    xs = torch.empty(fp4.fp4_scales_bytes(m, k, fp4.NVFP4), dtype=torch.uint8, device=dev)
    xg = torch.empty(1, dtype=torch.float32, device=dev)
    wn = fp4.fp4_gemm_bf16a_workspace_size(m, n, k)
    ws = torch.zeros(wn, dtype=torch.uint8, device=dev)
    d = torch.empty(m, n, dtype=torch.bfloat16, device=dev)
    sp = torch.cuda.current_stream().cuda_stream

    def step(i, src=None):
        q = wq[i % copies]
        if L.fp4_gemm_bf16a(P(src if src is not None else xd), P(q.codes), P(q.scales), P(q.g), m, n, k, P(d),
                            fp4.BF16, P(xc), P(xs), P(xg), P(ws), wn, fp4.GEMM_WEIGHTS_READY, sp):
            raise RuntimeError(fp4.fp4_last_error())

    def gemm(i):
        q = wq[i % copies]
        if L.fp4_gemm_ex(fp4.NVFP4, P(xc), P(xs), P(xg), P(q.codes), P(q.scales), P(q.g), m, n, k, P(d), fp4.BF16,
                         P(ws), wn, 0, sp):
            raise RuntimeError(fp4.fp4_last_error())

    # the GEMM with the epilogue of the next row: + bias, ReLU, and an NVFP4 copy of the result
    bias = torch.randn(n, device=dev)
    q_codes = torch.empty(m, n // 2, dtype=torch.uint8, device=dev)
    q_scales = torch.empty(fp4.fp4_scales_bytes(m, n, fp4.NVFP4), dtype=torch.uint8, device=dev)
    q_g = torch.tensor([0.05], dtype=torch.float32, device=dev)
    d_amax = torch.empty(1, dtype=torch.float32, device=dev)
    # one quantize pass: the activations' global scale supplied by the kernel that produced
    # them (fp4_gemm_epilogue's amax_out), here computed once before timing
    gx_in = torch.empty(1, dtype=torch.float32, device=dev)
    fp4.fp4_amax(xd, m * k, fp4.BF16, d_amax, ws, wn)
    fp4.fp4_global_scale(d_amax, gx_in)

    def step_one_pass(i):
        q = wq[i % copies]
        if L.fp4_quantize(P(xd), m, k, fp4.BF16, fp4.NVFP4, 16, P(xc), P(xs), P(xg), None, None, P(gx_in), P(ws),
                          wn, sp):
            raise RuntimeError(fp4.fp4_last_error())
        if L.fp4_gemm_ex(fp4.NVFP4, P(xc), P(xs), P(xg), P(q.codes), P(q.scales), P(q.g), m, n, k, P(d), fp4.BF16,
                         P(ws), wn, fp4.GEMM_WEIGHTS_READY, sp):
            raise RuntimeError(fp4.fp4_last_error())

    def gemm_epi(i):
        q = wq[i % copies]
        if L.fp4_gemm_epilogue(fp4.NVFP4, P(xc), P(xs), P(xg), P(q.codes), P(q.scales), P(q.g), m, n, k, P(bias),
                               fp4.ACT_RELU, P(d), fp4.BF16, P(q_codes), P(q_scales), P(q_g), P(d_amax), P(ws), wn, sp):
            raise RuntimeError(fp4.fp4_last_error())

    di = dev.index or 0
    step_ms, batches, clk = timed_batches(step, args.steps, args.warmup, di)
    gemm_ms, _, gclk = timed_batches(gemm, args.steps, args.warmup, di)
    epi_ms, _, eclk = timed_batches(gemm_epi, args.steps, args.warmup, di)
    one_ms, _, oclk = timed_batches(step_one_pass, args.steps, args.warmup, di)
    _check(fp4)
    flop = 2.0 * m * n * k
    x_host = x.pin_memory()
    d_host = torch.empty(m, n, dtype=torch.bfloat16).pin_memory()
    x_stage = torch.empty_like(xd)
    e2e_ms = _e2e(lambda i: step(i, x_stage), [x_host], [x_stage], [d_host], [d], args.steps, args.warmup)
    _check(fp4)
    rec = {"value": flop / (step_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": step_ms,
           "steps_per_batch": args.steps, "batches": len(batches), "timing": "median over batches",
           "config": {"workload": "prefill-shaped NVFP4 GEMM M=N=K=8192, bf16 activations (0.1% outliers x50) "
                                  "quantized every step, weights N(0,0.02) pre-quantized, bf16 out",
                      "step": "fp4_gemm_bf16a: tensor amax + NVFP4 quantize of X + FP4 GEMM (3 launches)",
                      "l2": f"weights rotate over {copies} pre-quantized copies "
                            f"({copies * per_copy / 2**20:.0f} MiB); X (128 MiB) exceeds the L2"},
           "roofline": _tensor_roofline("fp4_gemm_kernel<256, nvfp4, 1 acc, CTA pair>", flop, gemm_ms, peaks,
                                        "prefill_gemm", {"gemm_clocks": gclk}),
           "e2e": {"value": flop / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                   "h2d_bytes_per_step": m * k * 2, "d2h_bytes_per_step": m * n * 2},
           "step_one_pass": {"what": "quantize X in one pass with its global scale supplied by the kernel that "
                                     "produced X (fp4_gemm_epilogue's amax_out), then the GEMM (2 launches)",
                             "ms": one_ms, "TFLOP/s": flop / (one_ms * 1e-3) / 1e12, "clocks": oclk},
           "epilogue_gemm": {"what": "fp4_gemm_epilogue: + bias, ReLU, BF16 out, an NVFP4 copy of the result and "
                                     "its amax",
                             "ms": epi_ms, "TFLOP/s": flop / (epi_ms * 1e-3) / 1e12,
                             "frac": flop / (epi_ms * 1e-3) / 1e12 / peaks["fp4"], "clocks": eclk,
                             "traffic": traffic_for("prefill_gemm_epilogue")},
           "gpu_launches_per_step": 3, "clocks": clk}
    if cpu:
        import oracle
        rows = 8
        xb = workloads.bf16_bits(x)
        g = oracle.global_scale(oracle.amax(xb))
        ow = oracle.quantize(w.numpy(), oracle.NVFP4, 16)
        w_hat = oracle.dequantize(ow["codes"], ow["scales"], ow["g"])
        v, cores, reps = _oracle_rows_gemm_rate(np.ascontiguousarray(xb[:rows]), oracle.NVFP4, 16, w_hat, g)
        rec["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                               "sample": f"{reps} x (quantize {rows} rows of X with the tensor's g, FP64 product "
                                         f"with the 8192 x 8192 dequantized weights)"}
    del wq, xd, xc, xs, ws, d, x_stage, q_codes, q_scales, bias, d_amax, gx_in
    torch.cuda.empty_cache()
    return rec


def measure_train(args, dev, peaks, cpu: bool, s: int = 16384) -> dict:
    """Training-recipe step at S: W quantized once with 16x16 blocks (W and W^T); per step X
    and dY quantized (16-blocks), forward D = X W^T and backward dX = dY W, bf16 out."""
    import block_scaled_fp4_04_b200 as fp4
    x, w, dy = workloads.train_inputs(s, device="cpu")
    xd, dyd = x.to(dev), dy.to(dev)
    qw = fp4.quantize(w.to(dev), fp4.NVFP4, 256)
    wt = fp4.transposed(qw)
    ws = fp4.Workspace(dev)
    dout = torch.empty(s, s, dtype=torch.bfloat16, device=dev)
    dxout = torch.empty(s, s, dtype=torch.bfloat16, device=dev)
    state = {}

    def step(i, xs=None, dys=None):
        qx = fp4.quantize(xs if xs is not None else xd, fp4.NVFP4, 16, workspace=ws)
        qd = fp4.quantize(dys if dys is not None else dyd, fp4.NVFP4, 16, workspace=ws)
        fp4.gemm(qx, qw, out=dout, workspace=ws)
        fp4.gemm(qd, wt, out=dxout, workspace=ws)
        state["qx"], state["qd"] = qx, qd

    di = dev.index or 0
    steps = max(3, args.steps // 4)
    step_ms, batches, clk = timed_batches(step, steps, args.warmup, di)
    qx, qd = state["qx"], state["qd"]
    fwd_ms, _, fclk = timed_batches(lambda i: fp4.gemm(qx, qw, out=dout, workspace=ws), args.steps, args.warmup, di)
    bwd_ms, _, _ = timed_batches(lambda i: fp4.gemm(qd, wt, out=dxout, workspace=ws), args.steps, args.warmup, di)
    _check(fp4)
    flop = 2.0 * s ** 3
    x_host, dy_host = x.pin_memory(), dy.pin_memory()
    d_host = torch.empty(s, s, dtype=torch.bfloat16).pin_memory()
    dx_host = torch.empty(s, s, dtype=torch.bfloat16).pin_memory()
    xs_, dys_ = torch.empty_like(xd), torch.empty_like(dyd)
    e2e_ms = _e2e(lambda i: step(i, xs_, dys_), [x_host, dy_host], [xs_, dys_], [d_host, dx_host], [dout, dxout],
                  steps, args.warmup)
    _check(fp4)
    rec = {"value": 2 * flop / (step_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": step_ms,
           "steps_per_batch": steps, "batches": len(batches), "timing": "median over batches",
           "config": {"workload": f"training-recipe step M=N=K={s}: 16x16-block NVFP4 W (and W^T) quantized once, "
                                  "X and dY (bf16 N(0,1)) quantized every step, forward X W^T and backward dY W, "
                                  "bf16 out", "S": s,
                      "step": "amax + quantize X, amax + quantize dY, forward GEMM, backward GEMM (6 launches)",
                      "l2": "X, dY (512 MiB each) and the quantized W (144 MiB) exceed the L2"},
           "roofline": _tensor_roofline("fp4_gemm_kernel<256, nvfp4, 1 acc, CTA pair> (forward)", flop, fwd_ms, peaks,
                                        f"train_gemm_{s}", {"gemm_clocks": fclk,
                                                            "backward_TFLOP/s": flop / (bwd_ms * 1e-3) / 1e12,
                                                            "backward_ms": bwd_ms}),
           "e2e": {"value": 2 * flop / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                   "h2d_bytes_per_step": 2 * s * s * 2, "d2h_bytes_per_step": 2 * s * s * 2},
           "gpu_launches_per_step": 6, "clocks": clk}
    if cpu:
        import oracle
        rows = 2
        xb = workloads.bf16_bits(x)
        g = oracle.global_scale(oracle.amax(xb))
        ow = oracle.quantize(w.numpy(), oracle.NVFP4, 256)
        w_hat = oracle.dequantize(ow["codes"], ow["scales"], ow["g"])
        del ow
        v, cores, reps = _oracle_rows_gemm_rate(np.ascontiguousarray(xb[:rows]), oracle.NVFP4, 16, w_hat, g)
        rec["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                               "sample": f"{reps} x (quantize {rows} rows of X with the tensor's g, FP64 product "
                                         f"with the {s} x {s} dequantized 2-D-quantized weights)"}
        del w_hat
    del qw, wt, ws, dout, dxout, xd, dyd, state, xs_, dys_
    torch.cuda.empty_cache()
    return rec


def measure_moe(args, dev, peaks, cpu: bool) -> dict:
    """MXFP4 grouped MoE GEMM: 32 experts, 4096 tokens top-4 (16384 rows), K=2880, N=5760;
    the activations are quantized (grouped layout) every step; BF16 out."""
    import block_scaled_fp4_04_b200 as fp4
    a, w, offsets, _ = workloads.moe_inputs(device="cpu")
    E, N, K = w.shape
    rows = a.shape[0]
    ad = a.to(dev)
    wq = [fp4.quantize(w[e].to(dev), fp4.MXFP4, 32) for e in range(E)]
    B = torch.stack([q.codes for q in wq])
    sB = torch.cat([q.scales for q in wq])
    del wq
    off = offsets.to(dev)
    cap = fp4.fp4_scales_bytes_grouped(rows, E, K, fp4.MXFP4)
    codes = torch.empty(rows, K // 2, dtype=torch.uint8, device=dev)
    scales = torch.empty(cap, dtype=torch.uint8, device=dev)
    D = torch.empty(rows, N, dtype=torch.bfloat16, device=dev)
    L = fp4.lib()
    P = lambda t: t.data_ptr()
    sp = torch.cuda.current_stream().cuda_stream

    def quant(i, src=None):
        if L.fp4_quantize_grouped(P(src if src is not None else ad), rows, K, fp4.BF16, fp4.MXFP4, E, P(off), P(codes),
                                  P(scales), None, None, None, 0, sp):
            raise RuntimeError(fp4.fp4_last_error())

    def gemm(i):
        if L.fp4_gemm_grouped(fp4.MXFP4, E, P(off), P(codes), P(scales), None, P(B), P(sB), None, rows, N, K, P(D),
                              fp4.BF16, None, 0, sp):
            raise RuntimeError(fp4.fp4_last_error())

    di = dev.index or 0
    step_ms, batches, clk = timed_batches(lambda i: (quant(i), gemm(i)), args.steps, args.warmup, di)
    gemm_ms, _, gclk = timed_batches(gemm, args.steps, args.warmup, di)
    quant_ms, _, _ = timed_batches(quant, args.steps, args.warmup, di)
    _check(fp4)
    flop = 2.0 * rows * N * K
    gemm_bytes = E * N * K // 2 + sB.numel() + rows * K // 2 + rows * (K // 32) + rows * N * 2
    quant_bytes = rows * K * 2 + rows * K // 2 + rows * K // 32
    t_roof_ms = max(flop / (peaks["fp4"] * 1e12), gemm_bytes / (peaks["hbm"] * 1e9)) * 1e3
    a_host = a.pin_memory()
    d_host = torch.empty(rows, N, dtype=torch.bfloat16).pin_memory()
    a_stage = torch.empty_like(ad)
    e2e_ms = _e2e(lambda i: (quant(i, a_stage), gemm(i)), [a_host], [a_stage], [d_host], [D], args.steps, args.warmup)
    _check(fp4)
    achieved = flop / (gemm_ms * 1e-3) / 1e12
    rec = {"value": flop / (step_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": step_ms,
           "steps_per_batch": args.steps, "batches": len(batches), "timing": "median over batches",
           "config": {"workload": "MXFP4 grouped MoE GEMM: 32 experts, 4096 tokens routed top-4 by uniform gates "
                                  "(16384 rows), K=2880, N=5760 per expert, bf16 activations quantized every step, "
                                  "bf16 out",
                      "step": "grouped MXFP4 quantize of the activations + grouped GEMM (2 launches)",
                      "l2": "expert weights (265 MiB) exceed the L2"},
           "roofline": {"bound": "tensor" if flop / peaks["fp4"] * 1e-9 > gemm_bytes / peaks["hbm"] else "hbm",
                        "kernel": "fp4_gemm_kernel<256, mxfp4, 1 acc> (grouped, 128-row tiles)",
                        "achieved": achieved, "peak": peaks["fp4"], "unit": "TFLOP/s",
                        "frac": t_roof_ms / gemm_ms,
                        "frac_definition": "roofline time (slower of tensor and HBM) / measured kernel time",
                        "t_roof_ms": t_roof_ms, "launch_ms": gemm_ms, "algorithmic_bytes": gemm_bytes,
                        "hbm_GB/s": gemm_bytes / (gemm_ms * 1e-3) / 1e9, "peak_source": peaks["fp4_source"] +
                        "; hbm " + peaks["hbm_source"], "traffic": traffic_for("moe_gemm"), "gemm_clocks": gclk},
           "quantize": {"ms": quant_ms, "GB/s": quant_bytes / (quant_ms * 1e-3) / 1e9,
                        "frac": quant_bytes / (quant_ms * 1e-3) / 1e9 / peaks["hbm"],
                        "traffic": traffic_for("moe_quantize")},
           "e2e": {"value": flop / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                   "h2d_bytes_per_step": rows * K * 2, "d2h_bytes_per_step": rows * N * 2},
           "gpu_launches_per_step": 2, "clocks": clk}
    if cpu:
        import oracle
        ab = workloads.bf16_bits(a)
        e = 0
        lo = int(offsets[e])
        ow = oracle.quantize(w[e].numpy(), oracle.MXFP4, 32)
        w_hat = oracle.dequantize(ow["codes"], ow["scales"], ow["g"], oracle.MXFP4)
        v, cores, reps = _oracle_rows_gemm_rate(np.ascontiguousarray(ab[lo:lo + 32]), oracle.MXFP4, 32, w_hat)
        rec["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                               "sample": f"{reps} x (MXFP4-quantize 32 rows of expert 0's activations, FP64 product "
                                         "with its 5760 x 2880 dequantized weights)"}
    del B, sB, codes, scales, D, ad, a_stage
    torch.cuda.empty_cache()
    return rec


def measure_quantize(args, dev, peaks, cpu: bool) -> dict:
    """The quantize kernels alone (GB/s of algorithmic bytes; NVFP4 reads x twice: the tensor
    amax, then the encode)."""
    import block_scaled_fp4_04_b200 as fp4
    moe = {}

    def moe_activations():
        a, _, offsets, _ = workloads.moe_inputs(device="cpu", n=32)
        moe["offsets"] = offsets
        return a

    cases = [
        ("moe_quantize", "MoE activations bf16 [16384, 2880] -> MXFP4, grouped by expert (32 experts, one pass)",
         moe_activations, fp4.MXFP4, 32),
        ("quantize_train_x", "train X bf16 [16384, 16384] -> NVFP4 (amax + encode)",
         lambda: workloads.train_inputs(16384, device="cpu")[0], fp4.NVFP4, 16),
        ("quantize_decode_w", "decode W fp32 [28672, 8192] -> NVFP4 (amax + encode)",
         lambda: workloads.decode_inputs(device="cpu")[1], fp4.NVFP4, 16),
        ("quantize_2d_w", "2-D W fp32 [16384, 16384] -> NVFP4 W and W^T (amax + encode)",
         lambda: workloads.train_inputs(16384, device="cpu")[1], fp4.NVFP4, 256),
    ]
    out = []
    di = dev.index or 0
    train = {}

    def train_tensor(j):
        if not train:
            x, w, _ = workloads.train_inputs(16384, device="cpu")
            train.update(x=x, w=w)
        return train["x" if j == 0 else "w"]

    cases[1] = cases[1][:2] + (lambda: train_tensor(0),) + cases[1][3:]
    cases[3] = cases[3][:2] + (lambda: train_tensor(1),) + cases[3][3:]
    for key, name, make, fmt, blk in cases:
        if args.case and key != args.case:
            continue
        xh = make()
        x = xh.to(dev)
        rows, cols = x.shape
        esz = x.element_size()
        ws = fp4.Workspace(dev)
        codes = rows * cols // 2
        sc = fp4.fp4_scales_bytes(rows, cols, fmt)
        if blk == 256:
            nbytes = 2 * rows * cols * esz + 2 * (codes + sc)
        elif fmt == fp4.NVFP4:
            nbytes = 2 * rows * cols * esz + codes + sc
        else:
            nbytes = rows * cols * esz + codes + sc
        run = lambda i: fp4.quantize(x, fmt, blk, workspace=ws)
        if key == "moe_quantize":
            # the grouped layout an MoE layer's GEMM reads: one scale byte per block written
            off = moe["offsets"].to(dev)
            E = off.numel() - 1
            gcodes = torch.empty(rows, cols // 2, dtype=torch.uint8, device=dev)
            gsc = torch.empty(fp4.fp4_scales_bytes_grouped(rows, E, cols, fmt), dtype=torch.uint8, device=dev)
            L = fp4.lib()
            sp = torch.cuda.current_stream().cuda_stream
            nbytes = rows * cols * esz + codes + rows * (cols // blk)

            def run(i):
                if L.fp4_quantize_grouped(x.data_ptr(), rows, cols, fp4.BF16, fmt, E, off.data_ptr(),
                                          gcodes.data_ptr(), gsc.data_ptr(), None, None, None, 0, sp):
                    raise RuntimeError(fp4.fp4_last_error())
        ms, batches, clk = timed_batches(run, max(3, args.steps // 4), args.warmup, di, min_s=0.25)
        _check(fp4)
        gbs = nbytes / (ms * 1e-3) / 1e9
        rec = {"case": name, "ms": ms, "GB/s": gbs, "bytes": nbytes,
               "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm"], "unit": "GB/s",
                            "frac": gbs / peaks["hbm"], "peak_source": peaks["hbm_source"],
                            "traffic": traffic_for(key)}, "clocks": clk}
        if cpu and key in ("moe_quantize", "quantize_train_x"):
            import oracle
            xb = workloads.bf16_bits(xh) if xh.dtype == torch.bfloat16 else xh.numpy()
            sample = np.ascontiguousarray(xb[:256])
            t0 = time.perf_counter()
            reps = 0
            while time.perf_counter() - t0 < 2.0 and reps < 50:
                oracle.quantize(sample, fmt, blk)
                reps += 1
            dt = time.perf_counter() - t0
            per = sample.shape[0] * cols * esz * (2 if fmt == fp4.NVFP4 else 1) + sample.shape[0] * cols // 2
            rec["cpu_baseline"] = {"value": per * reps / dt / 1e9, "unit": "GB/s", "cores": oracle.num_threads(),
                                   "kind": "oracle", "sample": f"{reps} x 256 rows of the same tensor"}
        out.append(rec)
        del x, ws, xh
        torch.cuda.empty_cache()
    if not args.case or args.case in ("quantize_sr", "quantize_rht", "quantize_mx_floor"):
        out.extend(measure_quantize_variants(args, dev, peaks, train_tensor))
    return {"cases": out}


def measure_quantize_variants(args, dev, peaks, train_tensor) -> list:
    """The quantizer variants of the next rows, on the training tensors: stochastic rounding
    (one 4-byte random word per element read as well), the 16-point Hadamard transform
    before quantizing (the amax pass transforms too), and MXFP4 with the rounded-down
    scale."""
    import block_scaled_fp4_04_b200 as fp4
    di = dev.index or 0
    s = 16384
    x = train_tensor(0).to(dev)
    ws = torch.zeros(fp4.fp4_quantize_workspace_size(), dtype=torch.uint8, device=dev)
    codes = torch.empty(s, s // 2, dtype=torch.uint8, device=dev)
    sc16 = torch.empty(fp4.fp4_scales_bytes(s, s, fp4.NVFP4), dtype=torch.uint8, device=dev)
    sc32 = torch.empty(fp4.fp4_scales_bytes(s, s, fp4.MXFP4), dtype=torch.uint8, device=dev)
    g = torch.empty(1, dtype=torch.float32, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(11)
    rbits = torch.randint(-2 ** 31, 2 ** 31 - 1, (s, s), dtype=torch.int32, device=dev, generator=gen)
    L = fp4.lib()
    P = lambda t: t.data_ptr()
    sp = torch.cuda.current_stream().cuda_stream
    n = s * s

    def sr(i):
        if L.fp4_quantize_sr(P(x), s, s, fp4.BF16, P(rbits), P(codes), P(sc16), P(g), None, P(ws), ws.numel(), sp):
            raise RuntimeError(fp4.fp4_last_error())

    def rht(i):
        if L.fp4_quantize_rht(P(x), s, s, fp4.BF16, fp4.NVFP4, 0xA5C3, P(codes), P(sc16), P(g), None, P(ws),
                              ws.numel(), sp):
            raise RuntimeError(fp4.fp4_last_error())

    def floor(i):
        if L.fp4_quantize_ex(P(x), s, s, fp4.BF16, fp4.MXFP4, 32, fp4.QUANT_E8M0_FLOOR, P(codes), P(sc32), P(g), None,
                             None, None, P(ws), ws.numel(), sp):
            raise RuntimeError(fp4.fp4_last_error())

    cases = [("quantize_sr", "train X bf16 [16384, 16384] -> NVFP4 with stochastic rounding (amax + encode; "
              "one 4-byte random word per element)", sr, 2 * n * 2 + n * 4 + n // 2 + sc16.numel()),
             ("quantize_rht", "train X bf16 [16384, 16384] -> NVFP4 after the 16-point Hadamard transform "
              "(transforming amax + encode)", rht, 2 * n * 2 + n // 2 + sc16.numel()),
             ("quantize_mx_floor", "train X bf16 [16384, 16384] -> MXFP4 with the E8M0 scale rounded down (one pass)",
              floor, n * 2 + n // 2 + sc32.numel())]
    out = []
    for key, name, fn, nbytes in cases:
        if args.case and key != args.case:
            continue
        ms, _, clk = timed_batches(fn, max(3, args.steps // 4), args.warmup, di, min_s=0.25)
        _check(fp4)
        gbs = nbytes / (ms * 1e-3) / 1e9
        out.append({"case": name, "ms": ms, "GB/s": gbs, "bytes": nbytes,
                    "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm"], "unit": "GB/s",
                                 "frac": gbs / peaks["hbm"], "peak_source": peaks["hbm_source"],
                                 "traffic": traffic_for(key)}, "clocks": clk})
    del x, rbits, codes, sc16, sc32, ws
    torch.cuda.empty_cache()
    return out


def load_peak_table(dev) -> dict:
    hbm, bf16, bf16_s, src = load_peaks()
    pk = {"hbm": hbm, "hbm_source": f"{src} hbm_gbs (MEASURED_PEAKS.json)" if src == "measured" else src,
          "fp4": bf16 * FP4_PER_BF16,
          "fp4_source": f"{src} bf16_tflops {bf16:g} x {FP4_PER_BF16:g} (nominal FP4/BF16 dense ratio)"}
    try:
        pk["mma_loop_record"] = mma_peak(dev)
        pk["mma_loop"] = pk["mma_loop_record"]["TFLOP/s"]
    except Exception as e:  # the probe is context; its failure does not stop the bench
        pk["mma_loop_record"] = {"error": str(e)[:200]}
    return pk


def measure_mixed(args, dev, peaks, cpu: bool) -> dict:
    """The FP4 x FP8 GEMM (next row f4) on the prefill shape 8192^3: BF16 activations
    quantized to MXFP8 every step (one pass: E8M0 scales need no tensor amax), weights
    pre-quantized to MXFP4 and rotating past L2, BF16 out.  The MMA runs at the FP8 rate,
    so the tensor roofline is the measured BF16 peak x 2."""
    import block_scaled_fp4_04_b200 as fp4
    m = n = k = 8192
    x, w = workloads.prefill_inputs(device="cpu")
    xd = x.to(dev)
    per_copy = n * k // 2 + fp4.fp4_scales_bytes(n, k, fp4.MXFP4)
    copies = _copies(per_copy)
    w_dev = w.to(dev)
    wq = [fp4.quantize(w_dev, fp4.MXFP4, 32) for _ in range(copies)]
    del w_dev
    L = fp4.lib()
    P = lambda t: t.data_ptr()
    xc = torch.empty(m, k, dtype=torch.uint8, device=dev)
    xs = torch.empty(fp4.fp4_scales_bytes(m, k, fp4.MXFP8), dtype=torch.uint8, device=dev)
    d = torch.empty(m, n, dtype=torch.bfloat16, device=dev)
    sp = torch.cuda.current_stream().cuda_stream

    def quant(src=None):
        if L.fp4_quantize(P(src if src is not None else xd), m, k, fp4.BF16, fp4.MXFP8, 32, P(xc), P(xs), None, None,
                          None, None, None, 0, sp):
            raise RuntimeError(fp4.fp4_last_error())

    def gemm(i):
        q = wq[i % copies]
        if L.fp4_gemm_mixed(fp4.MXFP8, P(xc), P(xs), fp4.MXFP4, P(q.codes), P(q.scales), m, n, k, P(d), fp4.BF16, sp):
            raise RuntimeError(fp4.fp4_last_error())

    def step(i, src=None):
        quant(src)
        gemm(i)

    di = dev.index or 0
    step_ms, batches, clk = timed_batches(step, args.steps, args.warmup, di)
    gemm_ms, _, gclk = timed_batches(gemm, args.steps, args.warmup, di)
    _check(fp4)
    flop = 2.0 * m * n * k
    fp8_peak = peaks["fp4"] / FP4_PER_BF16 * FP8_PER_BF16
    achieved = flop / (gemm_ms * 1e-3) / 1e12
    x_host = x.pin_memory()
    d_host = torch.empty(m, n, dtype=torch.bfloat16).pin_memory()
    x_stage = torch.empty_like(xd)
    e2e_ms = _e2e(lambda i: step(i, x_stage), [x_host], [x_stage], [d_host], [d], args.steps, args.warmup)
    _check(fp4)
    rec = {"value": flop / (step_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": step_ms,
           "steps_per_batch": args.steps, "batches": len(batches), "timing": "median over batches",
           "config": {"workload": "mixed FP4 x FP8 GEMM M=N=K=8192: bf16 activations quantized to MXFP8 every "
                                  "step, weights MXFP4 pre-quantized, bf16 out",
                      "step": "fp4_quantize (MXFP8, one pass) + fp4_gemm_mixed (2 launches)",
                      "l2": f"weights rotate over {copies} pre-quantized copies ({copies * per_copy / 2**20:.0f} MiB)"},
           "roofline": {"bound": "tensor", "kernel": "fp4_gemm_kernel<256, mx, 1 acc, kind::mxf8f6f4>",
                        "achieved": achieved, "peak": fp8_peak, "unit": "TFLOP/s", "frac": achieved / fp8_peak,
                        "peak_source": peaks["fp4_source"].replace(f"x {FP4_PER_BF16:g} (nominal FP4/BF16",
                                                                   f"x {FP8_PER_BF16:g} (nominal FP8/BF16"),
                        "launch_ms": gemm_ms, "traffic": traffic_for("mixed_gemm"), "gemm_clocks": gclk},
           "e2e": {"value": flop / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                   "h2d_bytes_per_step": m * k * 2, "d2h_bytes_per_step": m * n * 2},
           "gpu_launches_per_step": 2, "clocks": clk}
    if cpu:
        import oracle
        rows = 8
        xb = workloads.bf16_bits(x)
        ow = oracle.quantize(w.numpy(), oracle.MXFP4, 32)
        w_hat = oracle.dequantize(ow["codes"], ow["scales"], ow["g"], oracle.MXFP4)
        v, cores, reps = _oracle_rows_gemm_rate(np.ascontiguousarray(xb[:rows]), oracle.MXFP8, 32, w_hat)
        rec["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                               "sample": f"{reps} x (MXFP8-quantize {rows} rows of X, FP64 product with the "
                                         "8192 x 8192 dequantized MXFP4 weights)"}
    del wq, xd, xc, xs, d, x_stage
    torch.cuda.empty_cache()
    return rec


MEASURES = {"prefill": measure_prefill, "train": measure_train, "moe": measure_moe, "quantize": measure_quantize,
            "mixed": measure_mixed}


def cpu_baseline_decode(budget_s: float = 12.0):
    """The oracle, as it stands, on a bounded sample of one decode step: quantize the 16
    activation rows, dequantize a sample of pre-quantized weight rows and take the
    FP64 product.  Returns (GB/s of the sample's algorithmic bytes, cores, sample)."""
    import oracle
    m, n, k = 16, 28672, 8192
    x, w = workloads.decode_inputs(device="cpu")
    rows = 1024
    g_w = oracle.global_scale(oracle.amax(w.numpy()))
    wq = oracle.quantize(w[:rows].numpy(), oracle.NVFP4, 16, g_in=g_w)
    xb = workloads.bf16_bits(x)
    t0 = time.perf_counter()
    reps = 0
    while True:
        xq = oracle.quantize(xb, oracle.NVFP4, 16)
        xh = oracle.dequantize(xq["codes"], xq["scales"], xq["g"])
        wh = oracle.dequantize(wq["codes"], wq["scales"], wq["g"])
        oracle.gemm_reference(xh, wh)
        reps += 1
        if time.perf_counter() - t0 > budget_s or reps >= 64:
            break
    dt = time.perf_counter() - t0
    _, _, per_step = decode_bytes(m, rows, k)
    gbs = per_step * reps / dt / 1e9
    return gbs, oracle.num_threads(), f"{reps} x (quantize X 16x8192 + {rows} weight rows of 28672) in {dt:.1f} s"


def run_reference(args, dist: Dist):
    """The oracle on the host cores, on the same workload, metric and unit; each step a
    bounded sample of the decode step sized so that the whole run takes about a minute."""
    import oracle
    m, n, k = 16, 28672, 8192
    x, w = workloads.decode_inputs(device="cpu")
    steps = args.warmup + args.steps
    # measured oracle costs on this kind of host: ~0.5 ms per activation row quantized,
    # ~0.2 ms per weight row dequantized and multiplied; keep the run near a minute
    per_step = 60.0 / max(steps, 1)
    xrows = 16 if per_step > 0.05 else 1
    rows = int(max(1, min(n, (per_step - xrows * 0.5e-3) / 0.2e-3)))
    g_w = oracle.global_scale(oracle.amax(w.numpy()))
    wq = oracle.quantize(w[:rows].numpy(), oracle.NVFP4, 16, g_in=g_w)
    xb = workloads.bf16_bits(x)

    def step():
        xq = oracle.quantize(xb[:xrows], oracle.NVFP4, 16)
        xh = oracle.dequantize(xq["codes"], xq["scales"], xq["g"])
        wh = oracle.dequantize(wq["codes"], wq["scales"], wq["g"])
        oracle.gemm_reference(xh, wh)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    _, _, per_step = decode_bytes(xrows, rows, k)
    v = per_step * args.steps / dt / 1e9
    sample = f"per step: quantize {xrows} activation row(s) of 8192 + {rows} of 28672 weight rows"
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64 oracle (fp32 quantize arithmetic)",
        "data": "synthetic (seeded, same recipe as the GPU arm)",
        "config": {"workload": "decode-shaped NVFP4 GEMM M=16 N=28672 K=8192 (bounded sample per step)",
                   "sample": sample},
        "cpu_baseline": {"value": v, "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode", choices=["decode", "prefill", "moe", "train", "quantize", "mixed"],
                    help="decode: the headline line, with the other configurations as sub-records; any other "
                         "value prints that configuration's record alone")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the other configurations' sub-records")
    ap.add_argument("--min-seconds", type=float, default=None,
                    help="minimum timed duration of every timed loop (default 0.5 s for the step, 0.2-0.4 s for "
                         "the sub-records); small values keep runs under a profiler short")
    ap.add_argument("--case", default=None,
                    help="with --workload quantize: only this case (moe_quantize, quantize_train_x, "
                         "quantize_decode_w, quantize_2d_w, quantize_sr, quantize_rht, quantize_mx_floor)")
    args = ap.parse_args()
    global MIN_S_OVERRIDE
    MIN_S_OVERRIDE = args.min_seconds
    if args.warmup < 3:
        raise SystemExit("at least 3 warm-up steps")
    dist = Dist()
    if args.gpus != dist.world:
        raise SystemExit(f"--gpus {args.gpus} needs {args.gpus} ranks (WORLD_SIZE is {dist.world}): launch with "
                         f"python -m torch.distributed.run --nproc-per-node {args.gpus} bench.py --gpus {args.gpus}")
    if args.impl == "reference":
        if dist.rank == 0:
            print(json.dumps(run_reference(args, dist)))
        return
    torch.cuda.set_device(dist.local)
    dev = torch.device("cuda", dist.local)
    dist.init("nccl")
    cpu = not args.no_cpu_baseline
    try:
        if args.workload != "decode":
            if dist.world > 1:
                raise SystemExit("the other configurations run on one GPU")
            peaks = load_peak_table(dev)
            rec = MEASURES[args.workload](args, dev, peaks, cpu)
            rec.update({"metric": METRIC, "n_gpus": 1, "peaks": {k: v for k, v in peaks.items() if k != "mma_loop"}})
            print(json.dumps(rec), flush=True)
            return
        res = run_decode(args, dist, dev)
        if dist.rank == 0:
            if dist.world == 1 and cpu:
                v, cores, sample = cpu_baseline_decode()
                res["cpu_baseline"] = {"value": v, "unit": "GB/s", "cores": cores, "kind": "oracle",
                                       "sample": sample}
            if dist.world == 1 and not args.no_extra:
                peaks = load_peak_table(dev)
                res["peaks"] = {k: v for k, v in peaks.items() if k != "mma_loop"}
                res["workloads"] = {}
                for name, fn in MEASURES.items():
                    res["workloads"][name] = fn(args, dev, peaks, cpu)
            print(json.dumps(res))
    finally:
        dist.close()


if __name__ == "__main__":
    main()
