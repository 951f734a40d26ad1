"""Helpers shared by the GPU parity tests: run one input through the CUDA path (via the
C ABI binding) and through the CPU oracle, in the layouts both sides define."""
from __future__ import annotations

import numpy as np
import torch

import block_scaled_fp4_04_b200 as fp4
import oracle
import workloads

FMT = {"nvfp4": fp4.NVFP4, "mxfp4": fp4.MXFP4}


def host_input(x: torch.Tensor) -> np.ndarray:
    """The oracle's view of a tensor: float32 values or bf16 bit patterns."""
    x = x.detach().cpu().contiguous()
    if x.dtype == torch.bfloat16:
        return workloads.bf16_bits(x)
    return x.float().numpy()


def oracle_quantize(x: torch.Tensor, fmt: int, block: int, g_in=None):
    """Oracle codes, row-major scales and the swizzled scale buffer(s)."""
    q = oracle.quantize(host_input(x), fmt, block, g_in=g_in)
    q["scales_sw"] = oracle.swizzle_scales(q["scales"])
    if block == 256:
        q["scalesT_sw"] = oracle.swizzle_scales(q["scalesT"])
    return q


def gpu_quantize(x: torch.Tensor, fmt: int, block: int, g_in=None) -> fp4.Quantized:
    gin = None
    if g_in is not None:
        gin = torch.tensor([g_in], dtype=torch.float32, device=x.device)
    q = fp4.quantize(x, fmt, block, global_in=gin)
    torch.cuda.synchronize()
    return q


def assert_quant_equal(gq: fp4.Quantized, oq: dict, label=""):
    codes = gq.codes.cpu().numpy()
    assert codes.shape == oq["codes"].shape, label
    bad = np.argwhere(codes != oq["codes"])
    assert bad.size == 0, f"{label}: {len(bad)} code bytes differ, first at {bad[:3].tolist()}"
    sc = gq.scales.cpu().numpy()
    assert sc.shape == oq["scales_sw"].shape, label
    bad = np.flatnonzero(sc != oq["scales_sw"])
    assert bad.size == 0, f"{label}: {bad.size} scale bytes differ, first at {bad[:3].tolist()}"
    g = np.float32(gq.g.cpu().numpy()[0])
    assert g.tobytes() == np.float32(oq["g"]).tobytes(), f"{label}: g {g} vs {oq['g']}"
    if "codesT" in oq:
        assert np.array_equal(gq.codesT.cpu().numpy(), oq["codesT"]), label
        assert np.array_equal(gq.scalesT.cpu().numpy(), oq["scalesT_sw"]), label


def dequant_oracle(oq: dict, fmt: int) -> np.ndarray:
    return oracle.dequantize(oq["codes"], oq["scales"], oq["g"], fmt)


def check_gemm(d_gpu: torch.Tensor, a_hat: np.ndarray, b_hat: np.ndarray, rows=None, label=""):
    """GEMM output vs the FP64 oracle within |D - D_ref| <= 1e-6 sum|a b| (+ half a BF16
    ulp for BF16 output).  Returns the worst ratio error / tolerance."""
    bf16 = d_gpu.dtype == torch.bfloat16
    d_ref, s = oracle.gemm_reference(a_hat, b_hat, rows)
    d = d_gpu.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        d = d[np.asarray(rows)]
    tol = oracle.gemm_tolerance(d_ref, s, bf16)
    err = np.abs(d - d_ref)
    bad = np.argwhere(~(err <= tol))
    assert bad.size == 0, (f"{label}: {len(bad)} outputs outside tolerance; first {bad[:3].tolist()} "
                           f"gpu={d[tuple(bad[0])]} ref={d_ref[tuple(bad[0])]} tol={tol[tuple(bad[0])]}")
    return float(np.max(err / np.maximum(tol, 1e-300)))


def random_input(rows, cols, seed, dtype=torch.float32, std=1.0, outliers=True):
    x = workloads.normal((rows, cols), std, seed)
    if outliers:
        workloads.with_outliers(x, seed)
    return x.to(dtype)
