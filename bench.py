#!/usr/bin/env python
"""Throughput of the block-scaled FP4 hot path on B200 (one JSON line on stdout).

Default workload (N=1): the decode-shaped NVFP4 GEMM -- M=16 tokens, N=28672, K=8192;
weights N(0, 0.02) pre-quantized to NVFP4 once (untimed); BF16 activations N(0,1) with
0.1% outliers x50 quantized on the fly every step; BF16 output.  One step = tensor
amax + NVFP4 quantize of the activations + the FP4 GEMM.  Memory-bound, so the metric
is GB/s of algorithmic bytes (each operand's stored bytes read once, output written
once; the activations are read twice, once for the amax and once for the encode).

Other workloads (--workload prefill | moe | train | quantize) measure the remaining
configurations the same way.

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

    K = args.steps
    clocks = ClockSampler(dev.index or 0)
    time.sleep(0.15)
    dist.barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    c0 = clocks.mark()
    t_start.record()
    for i in range(K):
        step(i)
    t_end.record()
    torch.cuda.synchronize()
    dist.barrier()
    c1 = clocks.mark()
    ms = t_start.elapsed_time(t_end)
    clk = clocks.stop(c0, c1)
    if fp4.fp4_get_status() != fp4.OK:
        raise RuntimeError("device status latched an error during the timed steps")
    max_ms = dist.max(ms, dev)

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


# ---------------------------------------------------------------- other workloads
FP4_PER_BF16 = 4.0  # nominal dense FP4 / BF16 tensor throughput ratio (9 / 2.25 PFLOP/s)


def _events_ms(fn, iters: int, warmup: int) -> float:
    """Average device ms per call of fn(i), events around a batch on the current stream."""
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(iters):
        fn(i)
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / iters


def _check(fp4):
    if fp4.fp4_get_status() != fp4.OK:
        raise RuntimeError("device status latched an error")


def _copies(per_copy_bytes: int) -> int:
    """Rotating copies so that one pass over them exceeds the L2 three times."""
    return max(1, int(np.ceil(3 * L2_BYTES / max(per_copy_bytes, 1))))


def _line(workload: str, value, unit: str, ms: float, args, extra: dict) -> dict:
    res = {"metric": METRIC, "value": value, "unit": unit, "n_gpus": 1, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "data": "synthetic (seeded, same recipes as the tests)", "config": {"workload": workload}}
    res.update(extra)
    return res


def run_prefill(args, dev):
    """Prefill-shaped NVFP4 GEMM 8192^3: BF16 activations quantized every step (tensor amax,
    then 16-blocks), weights pre-quantized; tensor-bound."""
    import block_scaled_fp4_04_b200 as fp4
    m = n = k = 8192
    x, w = workloads.prefill_inputs(device="cpu")
    x = x.to(dev)
    qw = fp4.quantize(w.to(dev), fp4.NVFP4, 16)
    L = fp4.lib()
    P = lambda t: t.data_ptr()
    xc = torch.empty(m, k // 2, dtype=torch.uint8, device=dev)
    xs = torch.empty(fp4.fp4_scales_bytes(m, k, fp4.NVFP4), dtype=torch.uint8, device=dev)
    xg = torch.empty(1, dtype=torch.float32, device=dev)
    wn = fp4.fp4_gemm_bf16a_workspace_size(m, n, k)
    ws = torch.zeros(wn, dtype=torch.uint8, device=dev)
    d = torch.empty(m, n, dtype=torch.bfloat16, device=dev)
    sp = torch.cuda.current_stream().cuda_stream

    def step(i):
        if L.fp4_gemm_bf16a(P(x), P(qw.codes), P(qw.scales), P(qw.g), m, n, k, P(d), fp4.BF16, P(xc), P(xs),
                            P(xg), P(ws), wn, fp4.GEMM_WEIGHTS_READY, sp):
            raise RuntimeError(fp4.fp4_last_error())

    def gemm(i):
        if L.fp4_gemm_ex(fp4.NVFP4, P(xc), P(xs), P(xg), P(qw.codes), P(qw.scales), P(qw.g), m, n, k, P(d),
                         fp4.BF16, P(ws), wn, 0, sp):
            raise RuntimeError(fp4.fp4_last_error())

    step_ms = _events_ms(step, args.steps, args.warmup)
    gemm_ms = _events_ms(gemm, args.steps, args.warmup)
    _check(fp4)
    flop = 2.0 * m * n * k
    hbm, bf16, bf16_s, src = load_peaks()
    peak = bf16 * FP4_PER_BF16
    gemm_tf = flop / (gemm_ms * 1e-3) / 1e12
    step_tf = flop / (step_ms * 1e-3) / 1e12
    return _line("prefill-shaped NVFP4 GEMM M=N=K=8192, bf16 activations quantized every step, bf16 out",
                 step_tf, "TFLOP/s", step_ms, args, {
                     "dtype": "nvfp4 x nvfp4 -> fp32 accumulate, bf16 out",
                     "roofline": {"bound": "tensor", "kernel": "fp4_gemm_kernel<256, nvfp4, 1, CTA pair>",
                                  "achieved": gemm_tf, "peak": peak, "unit": "TFLOP/s", "frac": gemm_tf / peak,
                                  "peak_source": f"{src} bf16_tflops x {FP4_PER_BF16:g} (nominal FP4/BF16 ratio)",
                                  "frac_of_nominal_9pf": gemm_tf / 9000.0, "launch_ms": gemm_ms,
                                  "traffic": None},
                     "step": {"ms": step_ms, "TFLOP/s": step_tf, "contents": "amax + quantize(X) + GEMM"},
                     "gpu_launches": 3 * args.steps})


def run_moe(args, dev):
    """MXFP4 grouped MoE GEMM: 4096 tokens x top-4 of 32 experts, K=2880, N=5760; the
    activations are quantized (grouped layout) every step."""
    import block_scaled_fp4_04_b200 as fp4
    a, w, offsets, _ = workloads.moe_inputs(device="cpu")
    E, N, K = w.shape
    rows = a.shape[0]
    a = a.to(dev)
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

    def quant(i):
        if L.fp4_quantize_grouped(P(a), rows, K, fp4.BF16, fp4.MXFP4, E, P(off), P(codes), P(scales), None, None,
                                  None, 0, sp):
            raise RuntimeError(fp4.fp4_last_error())

    def gemm(i):
        if L.fp4_gemm_grouped(fp4.MXFP4, E, P(off), P(codes), P(scales), None, P(B), P(sB), None, rows, N, K, P(D),
                              fp4.BF16, None, 0, sp):
            raise RuntimeError(fp4.fp4_last_error())

    step_ms = _events_ms(lambda i: (quant(i), gemm(i)), args.steps, args.warmup)
    gemm_ms = _events_ms(gemm, args.steps, args.warmup)
    quant_ms = _events_ms(quant, args.steps, args.warmup)
    _check(fp4)
    flop = 2.0 * rows * N * K
    gemm_bytes = E * N * K // 2 + sB.numel() + rows * K // 2 + scales.numel() + rows * N * 2
    quant_bytes = rows * K * 2 + rows * K // 2 + rows * K // 32
    hbm, bf16, bf16_s, src = load_peaks()
    peak = bf16 * FP4_PER_BF16
    t_roof = max(flop / (peak * 1e12), gemm_bytes / (hbm * 1e9)) * 1e3
    gemm_tf = flop / (gemm_ms * 1e-3) / 1e12
    return _line("MXFP4 grouped MoE GEMM: 32 experts, 4096 tokens top-4 (16384 rows), K=2880, N=5760, bf16 out",
                 flop / (step_ms * 1e-3) / 1e12, "TFLOP/s", step_ms, args, {
                     "dtype": "mxfp4 x mxfp4 -> fp32 accumulate, bf16 out",
                     "roofline": {"bound": "tensor" if flop / peak > gemm_bytes / hbm * 1e-3 else "hbm",
                                  "kernel": "fp4_gemm_kernel<256, mxfp4, 1, CTA pair> (grouped)",
                                  "achieved": gemm_tf, "peak": peak, "unit": "TFLOP/s",
                                  "frac": t_roof / gemm_ms,
                                  "frac_definition": "roofline time (slower of tensor and HBM) / measured time",
                                  "hbm_GB/s": gemm_bytes / (gemm_ms * 1e-3) / 1e9, "algorithmic_bytes": gemm_bytes,
                                  "peak_source": f"{src} bf16_tflops x {FP4_PER_BF16:g}; {src} hbm_gbs",
                                  "launch_ms": gemm_ms, "traffic": None},
                     "quantize": {"ms": quant_ms, "GB/s": quant_bytes / (quant_ms * 1e-3) / 1e9,
                                  "frac": quant_bytes / (quant_ms * 1e-3) / 1e9 / hbm},
                     "gpu_launches": 2 * args.steps})


def run_train(args, dev):
    """Training-recipe sweep: W quantized once with 16x16 blocks (W and W^T); per step X and
    dY quantized (16-blocks), forward D = X W^T and backward dX = dY W."""
    import block_scaled_fp4_04_b200 as fp4
    hbm, bf16, bf16_s, src = load_peaks()
    peak = bf16 * FP4_PER_BF16
    out = []
    for s in (1024, 2048, 4096, 8192, 16384):
        x, w, dy = workloads.train_inputs(s, device="cpu")
        per_copy = 2 * s * s * 2
        ncopy = _copies(per_copy) if s <= 2048 else 1
        xs = [x.to(dev) for _ in range(ncopy)]
        dys = [dy.to(dev) for _ in range(ncopy)]
        qw = fp4.quantize(w.to(dev), fp4.NVFP4, 256)
        wt = fp4.transposed(qw)
        ws = fp4.Workspace(dev)
        dout = torch.empty(s, s, dtype=torch.bfloat16, device=dev)
        dxout = torch.empty(s, s, dtype=torch.bfloat16, device=dev)
        state = {}

        def step(i):
            qx = fp4.quantize(xs[i % ncopy], fp4.NVFP4, 16, workspace=ws)
            qd = fp4.quantize(dys[i % ncopy], fp4.NVFP4, 16, workspace=ws)
            fp4.gemm(qx, qw, out=dout, workspace=ws)
            fp4.gemm(qd, wt, out=dxout, workspace=ws)
            state["qx"], state["qd"] = qx, qd

        step_ms = _events_ms(step, max(3, args.steps // 4), args.warmup)
        qx, qd = state["qx"], state["qd"]
        fwd_ms = _events_ms(lambda i: fp4.gemm(qx, qw, out=dout, workspace=ws), args.steps, args.warmup)
        bwd_ms = _events_ms(lambda i: fp4.gemm(qd, wt, out=dxout, workspace=ws), args.steps, args.warmup)
        _check(fp4)
        flop = 2.0 * s * s * s
        out.append({"S": s, "step_ms": step_ms, "fwd_ms": fwd_ms, "bwd_ms": bwd_ms,
                    "fwd_TFLOP/s": flop / (fwd_ms * 1e-3) / 1e12, "bwd_TFLOP/s": flop / (bwd_ms * 1e-3) / 1e12,
                    "fwd_frac": flop / (fwd_ms * 1e-3) / 1e12 / peak,
                    "step_TFLOP/s": 2 * flop / (step_ms * 1e-3) / 1e12,
                    "l2": f"{ncopy} rotating copies of X, dY" if ncopy > 1 else "inputs larger than L2"})
        del xs, dys, qw, wt, ws, dout, dxout, state
        torch.cuda.empty_cache()
    big = out[-1]
    return _line("training-recipe sweep M=N=K in {1024..16384}: 2-D NVFP4 W (and W^T) once, X and dY quantized "
                 "per step, forward X W^T and backward dY W, bf16 out", big["step_TFLOP/s"], "TFLOP/s",
                 big["step_ms"], args, {
                     "dtype": "nvfp4 x nvfp4 -> fp32 accumulate, bf16 out",
                     "roofline": {"bound": "tensor", "kernel": "fp4_gemm_kernel<256, nvfp4, 1, CTA pair> at S=16384",
                                  "achieved": big["fwd_TFLOP/s"], "peak": peak, "unit": "TFLOP/s",
                                  "frac": big["fwd_frac"], "traffic": None,
                                  "peak_source": f"{src} bf16_tflops x {FP4_PER_BF16:g}"},
                     "sweep": out, "gpu_launches": None})


def run_quantize(args, dev):
    """Quantize kernels alone: GB/s of algorithmic bytes (NVFP4 reads x twice: amax, encode)."""
    import block_scaled_fp4_04_b200 as fp4
    hbm, bf16, bf16_s, src = load_peaks()
    rows_out = []
    cases = [
        ("moe activations bf16 [16384, 2880] -> MXFP4", lambda: workloads.moe_inputs(device="cpu")[0], fp4.MXFP4, 32),
        ("train X bf16 [16384, 16384] -> NVFP4", lambda: workloads.train_inputs(16384, device="cpu")[0], fp4.NVFP4, 16),
        ("decode W fp32 [28672, 8192] -> NVFP4", lambda: workloads.decode_inputs(device="cpu")[1], fp4.NVFP4, 16),
        ("2-D W fp32 [16384, 16384] -> NVFP4 W and W^T", lambda: workloads.train_inputs(16384, device="cpu")[1],
         fp4.NVFP4, 256),
    ]
    for name, make, fmt, blk in cases:
        x = make().to(dev)
        rows, cols = x.shape
        esz = x.element_size()
        ws = fp4.Workspace(dev)
        codes = rows * cols // 2
        sc = fp4.fp4_scales_bytes(rows, cols, fmt)
        if blk == 256:
            nbytes = 2 * rows * cols * esz + 2 * (codes + sc)   # amax read + encode read; W and W^T
        elif fmt == fp4.NVFP4:
            nbytes = 2 * rows * cols * esz + codes + sc
        else:
            nbytes = rows * cols * esz + codes + sc
        ms = _events_ms(lambda i: fp4.quantize(x, fmt, blk, workspace=ws), max(3, args.steps // 4), args.warmup)
        _check(fp4)
        gbs = nbytes / (ms * 1e-3) / 1e9
        rows_out.append({"case": name, "ms": ms, "GB/s": gbs, "frac": gbs / hbm, "bytes": nbytes})
        del x, ws
        torch.cuda.empty_cache()
    best = rows_out[0]
    return _line("quantize kernels alone (MoE activations, train X, decode W, 2-D W)", best["GB/s"], "GB/s",
                 best["ms"], args, {
                     "dtype": "bf16/fp32 in -> nvfp4/mxfp4 codes + scales",
                     "roofline": {"bound": "hbm", "kernel": "quantize (first case)", "achieved": best["GB/s"],
                                  "peak": hbm, "unit": "GB/s", "frac": best["frac"], "traffic": None,
                                  "peak_source": f"{src} hbm_gbs"},
                     "cases": rows_out, "gpu_launches": None})


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
    done = 0
    reps = 0
    while True:
        xq = oracle.quantize(xb, oracle.NVFP4, 16)
        xh = oracle.dequantize(xq["codes"], xq["scales"], xq["g"])
        wh = oracle.dequantize(wq["codes"], wq["scales"], wq["g"])
        oracle.gemm_reference(xh, wh)
        done += rows
        reps += 1
        if time.perf_counter() - t0 > budget_s or reps >= 64:
            break
    dt = time.perf_counter() - t0
    _, _, per_step = decode_bytes(m, rows, k)
    gbs = per_step * reps / dt / 1e9
    return gbs, _cores(), f"{reps} x (quantize X 16x8192 + {rows} weight rows of 28672) in {dt:.1f} s"


def _cores() -> int:
    try:
        from threadpoolctl import threadpool_info
        th = [i.get("num_threads", 1) for i in threadpool_info()]
        return max([1] + th)
    except Exception:
        return 1


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
        "cpu_baseline": {"value": v, "unit": "GB/s", "cores": _cores(), "kind": "oracle", "sample": sample},
        "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode", choices=["decode", "prefill", "moe", "train", "quantize", "all"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("at least 3 warm-up steps")
    dist = Dist()
    if args.impl == "reference":
        if dist.rank == 0:
            print(json.dumps(run_reference(args, dist)))
        return
    torch.cuda.set_device(dist.local)
    dev = torch.device("cuda", dist.local)
    dist.init("nccl")
    try:
        if args.workload != "decode":
            if dist.world > 1:
                raise SystemExit("the additional workloads run on one GPU")
            names = ["prefill", "moe", "train", "quantize"] if args.workload == "all" else [args.workload]
            for name in names:
                print(json.dumps({"prefill": run_prefill, "moe": run_moe, "train": run_train,
                                  "quantize": run_quantize}[name](args, dev)), flush=True)
            return
        res = run_decode(args, dist, dev)
        if dist.rank == 0:
            if dist.world == 1 and not args.no_cpu_baseline:
                v, cores, sample = cpu_baseline_decode()
                res["cpu_baseline"] = {"value": v, "unit": "GB/s", "cores": cores, "kind": "oracle",
                                       "sample": sample}
            print(json.dumps(res))
    finally:
        dist.close()


if __name__ == "__main__":
    main()
