"""Python binding of libfp4 (block-scaled FP4 quantization and GEMM for B200).

Argument marshalling only: every step of the quantize / GEMM path runs in the CUDA
kernels of ``libfp4.so`` (built from ``csrc/`` by ``build.py``).  PyTorch provides
device memory and streams.  There is no CPU fallback: if the shared library is
missing or the device is not an sm_100 GPU, the calls raise.

The functions named ``fp4_*`` mirror the C entry points of ``include/fp4.h`` one to
one (tensors stand in for device pointers).  ``quantize`` and ``gemm`` below are
conveniences that allocate the outputs with torch and call them.
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp4.so")

NVFP4, MXFP4, MXFP8 = 0, 1, 2  # MXFP8: E4M3 elements, one byte each (the mixed GEMM's FP8 operand)
F32, BF16 = 0, 1
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_NONFINITE = range(6)
GEMM_WEIGHTS_READY = 1
QUANT_E8M0_FLOOR = 1
ACT_NONE, ACT_RELU = 0, 1
_STATUS_NAMES = {0: "FP4_OK", 1: "FP4_ERR_INVALID_ARG", 2: "FP4_ERR_UNSUPPORTED", 3: "FP4_ERR_CUDA",
                 4: "FP4_ERR_TIMEOUT", 5: "FP4_ERR_NONFINITE"}

_lib = None
_lock = threading.Lock()


class Fp4Error(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


def lib() -> ctypes.CDLL:
    """Load libfp4.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m block_scaled_fp4_04_b200.build` (no CPU fallback exists)")
            L = ctypes.CDLL(LIB_PATH)
            P, I64, I32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
            sigs = {
                "fp4_version": (ctypes.c_char_p, []),
                "fp4_last_error": (ctypes.c_char_p, []),
                "fp4_scales_bytes": (SZ, [I64, I64, I32]),
                "fp4_scales_bytes_grouped": (SZ, [I64, I32, I64, I32]),
                "fp4_quantize_workspace_size": (SZ, []),
                "fp4_amax": (I32, [P, I64, I32, P, P, SZ, P]),
                "fp4_quantize": (I32, [P, I64, I64, I32, I32, I32, P, P, P, P, P, P, P, SZ, P]),
                "fp4_quantize_grouped": (I32, [P, I64, I64, I32, I32, I32, P, P, P, P, P, P, SZ, P]),
                "fp4_quantize_ex": (I32, [P, I64, I64, I32, I32, I32, ctypes.c_uint, P, P, P, P, P, P, P, SZ, P]),
                "fp4_quantize_sr": (I32, [P, I64, I64, I32, P, P, P, P, P, P, SZ, P]),
                "fp4_quantize_rht": (I32, [P, I64, I64, I32, I32, ctypes.c_uint32, P, P, P, P, P, SZ, P]),
                "fp4_global_scale": (I32, [P, P, P]),
                "fp4_dequantize": (I32, [P, P, P, I64, I64, I32, P, P]),
                "fp4_gemm_workspace_size": (SZ, [I64, I64, I64, I32]),
                "fp4_gemm": (I32, [I32, P, P, P, P, P, P, I64, I64, I64, P, I32, P, SZ, P]),
                "fp4_gemm_ex": (I32, [I32, P, P, P, P, P, P, I64, I64, I64, P, I32, P, SZ, ctypes.c_uint, P]),
                "fp4_gemm_noalloc": (I32, [I32, P, P, P, P, P, P, I64, I64, I64, P, I32, P]),
                "fp4_gemm_mixed": (I32, [I32, P, P, I32, P, P, I64, I64, I64, P, I32, P]),
                "fp4_gemm_epilogue_workspace_size": (SZ, [I64, I64, I64, I32, I32]),
                "fp4_gemm_epilogue": (I32, [I32, P, P, P, P, P, P, I64, I64, I64, P, I32, P, I32, P, P, P, P, P,
                                            SZ, P]),
                "fp4_gemm_bf16a_workspace_size": (SZ, [I64, I64, I64]),
                "fp4_gemm_bf16a": (I32, [P, P, P, P, I64, I64, I64, P, I32, P, P, P, P, SZ, ctypes.c_uint, P]),
                "fp4_gemm_grouped": (I32, [I32, I32, P, P, P, P, P, P, P, I64, I64, I64, P, I32, P, SZ, P]),
                "fp4_get_status": (I32, [P]),
                "fp4_debug_encode": (I32, [P, I64, I32, P, P]),
                "fp4_debug_stall_next_decode": (I32, [I32]),
                "fp4_mma_peak": (I32, [I32, I32, P, P]),
            }
            for name, (res, args) in sigs.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def _p(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _s(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int):
    if rc != OK:
        raise Fp4Error(rc, lib().fp4_last_error().decode())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"input must be float32 or bfloat16, got {t.dtype}")


# ---------------------------------------------------------------- C entry points
def fp4_version() -> str:
    return lib().fp4_version().decode()


def fp4_last_error() -> str:
    return lib().fp4_last_error().decode()


def fp4_scales_bytes(rows: int, cols: int, fmt: int) -> int:
    return int(lib().fp4_scales_bytes(rows, cols, fmt))


def fp4_scales_bytes_grouped(total_rows: int, num_groups: int, cols: int, fmt: int) -> int:
    return int(lib().fp4_scales_bytes_grouped(total_rows, num_groups, cols, fmt))


def fp4_quantize_workspace_size() -> int:
    return int(lib().fp4_quantize_workspace_size())


def fp4_gemm_workspace_size(M: int, N: int, K: int, fmt: int) -> int:
    return int(lib().fp4_gemm_workspace_size(M, N, K, fmt))


def fp4_amax(x, n, in_dtype, amax_out, workspace, workspace_bytes, stream=None):
    _check(lib().fp4_amax(_p(x), n, in_dtype, _p(amax_out), _p(workspace), workspace_bytes, _s(stream)))


def fp4_quantize(x, rows, cols, in_dtype, fmt, block, codes_out, scales_out, global_out,
                 codesT_out=None, scalesT_out=None, global_in=None, workspace=None, workspace_bytes=0,
                 stream=None):
    _check(lib().fp4_quantize(_p(x), rows, cols, in_dtype, fmt, block, _p(codes_out), _p(scales_out),
                              _p(global_out), _p(codesT_out), _p(scalesT_out), _p(global_in), _p(workspace),
                              workspace_bytes, _s(stream)))


def fp4_quantize_grouped(x, rows, cols, in_dtype, fmt, num_groups, offsets, codes_out, scales_out, global_out,
                         global_in=None, workspace=None, workspace_bytes=0, stream=None):
    _check(lib().fp4_quantize_grouped(_p(x), rows, cols, in_dtype, fmt, num_groups, _p(offsets), _p(codes_out),
                                      _p(scales_out), _p(global_out), _p(global_in), _p(workspace),
                                      workspace_bytes, _s(stream)))


def fp4_quantize_ex(x, rows, cols, in_dtype, fmt, block, flags, codes_out, scales_out, global_out,
                    codesT_out=None, scalesT_out=None, global_in=None, workspace=None, workspace_bytes=0,
                    stream=None):
    _check(lib().fp4_quantize_ex(_p(x), rows, cols, in_dtype, fmt, block, flags, _p(codes_out), _p(scales_out),
                                 _p(global_out), _p(codesT_out), _p(scalesT_out), _p(global_in), _p(workspace),
                                 workspace_bytes, _s(stream)))


def fp4_quantize_sr(x, rows, cols, in_dtype, rbits, codes_out, scales_out, global_out, global_in=None,
                    workspace=None, workspace_bytes=0, stream=None):
    _check(lib().fp4_quantize_sr(_p(x), rows, cols, in_dtype, _p(rbits), _p(codes_out), _p(scales_out),
                                 _p(global_out), _p(global_in), _p(workspace), workspace_bytes, _s(stream)))


def fp4_quantize_rht(x, rows, cols, in_dtype, fmt, signs, codes_out, scales_out, global_out, global_in=None,
                     workspace=None, workspace_bytes=0, stream=None):
    _check(lib().fp4_quantize_rht(_p(x), rows, cols, in_dtype, fmt, signs, _p(codes_out), _p(scales_out),
                                  _p(global_out), _p(global_in), _p(workspace), workspace_bytes, _s(stream)))


def fp4_global_scale(amax, global_out, stream=None):
    _check(lib().fp4_global_scale(_p(amax), _p(global_out), _s(stream)))


def fp4_dequantize(codes, scales, global_, rows, cols, fmt, out, stream=None):
    _check(lib().fp4_dequantize(_p(codes), _p(scales), _p(global_), rows, cols, fmt, _p(out), _s(stream)))


def fp4_gemm(fmt, A, sA, gA, B, sB, gB, M, N, K, D, out_dtype, workspace=None, workspace_bytes=0, stream=None):
    _check(lib().fp4_gemm(fmt, _p(A), _p(sA), _p(gA), _p(B), _p(sB), _p(gB), M, N, K, _p(D), out_dtype,
                          _p(workspace), workspace_bytes, _s(stream)))


def fp4_gemm_ex(fmt, A, sA, gA, B, sB, gB, M, N, K, D, out_dtype, workspace=None, workspace_bytes=0, flags=0,
                stream=None):
    _check(lib().fp4_gemm_ex(fmt, _p(A), _p(sA), _p(gA), _p(B), _p(sB), _p(gB), M, N, K, _p(D), out_dtype,
                             _p(workspace), workspace_bytes, flags, _s(stream)))


def fp4_gemm_epilogue_workspace_size(M: int, N: int, K: int, fmt: int, rows_in_place: bool) -> int:
    return int(lib().fp4_gemm_epilogue_workspace_size(M, N, K, fmt, 1 if rows_in_place else 0))


def fp4_gemm_epilogue(fmt, A, sA, gA, B, sB, gB, M, N, K, bias, act, D, out_dtype, Dcodes=None, Dscales=None,
                      gD=None, amax_out=None, workspace=None, workspace_bytes=0, stream=None):
    _check(lib().fp4_gemm_epilogue(fmt, _p(A), _p(sA), _p(gA), _p(B), _p(sB), _p(gB), M, N, K, _p(bias), act, _p(D),
                                   out_dtype, _p(Dcodes), _p(Dscales), _p(gD), _p(amax_out), _p(workspace),
                                   workspace_bytes, _s(stream)))


def fp4_gemm_bf16a_workspace_size(M: int, N: int, K: int) -> int:
    return int(lib().fp4_gemm_bf16a_workspace_size(M, N, K))


def fp4_gemm_bf16a(X, B, sB, gB, M, N, K, D, out_dtype, Xcodes, Xscales, gX, workspace, workspace_bytes, flags=0,
                   stream=None):
    _check(lib().fp4_gemm_bf16a(_p(X), _p(B), _p(sB), _p(gB), M, N, K, _p(D), out_dtype, _p(Xcodes), _p(Xscales),
                                _p(gX), _p(workspace), workspace_bytes, flags, _s(stream)))


def fp4_gemm_noalloc(fmt, A, sA, gA, B, sB, gB, M, N, K, D, out_dtype, stream=None):
    """fp4_gemm without a caller workspace: the split-K scratch is a fixed 4 MiB array
    inside the library, shared by all calls on a device (calls that overlap race)."""
    _check(lib().fp4_gemm_noalloc(fmt, _p(A), _p(sA), _p(gA), _p(B), _p(sB), _p(gB), M, N, K, _p(D), out_dtype,
                                  _s(stream)))


def fp4_gemm_mixed(a_fmt, A, sA, b_fmt, B, sB, M, N, K, D, out_dtype, stream=None):
    """D = A B^T with A and B each MXFP4 or MXFP8 (the FP4 x FP8 GEMM)."""
    _check(lib().fp4_gemm_mixed(a_fmt, _p(A), _p(sA), b_fmt, _p(B), _p(sB), M, N, K, _p(D), out_dtype, _s(stream)))


def fp4_gemm_grouped(fmt, num_groups, offsets, A, sA, gA, B, sB, gB, total_rows, N, K, D, out_dtype,
                     workspace=None, workspace_bytes=0, stream=None):
    _check(lib().fp4_gemm_grouped(fmt, num_groups, _p(offsets), _p(A), _p(sA), _p(gA), _p(B), _p(sB), _p(gB),
                                  total_rows, N, K, _p(D), out_dtype, _p(workspace), workspace_bytes,
                                  _s(stream)))


def fp4_get_status(stream=None) -> int:
    """Synchronizes the stream and returns (and clears) the latched device status."""
    return int(lib().fp4_get_status(_s(stream)))


def fp4_mma_peak(iters: int, grid: int, cycles, stream=None):
    _check(lib().fp4_mma_peak(iters, grid, _p(cycles), _s(stream)))


def fp4_debug_stall_next_decode(cta: int):
    _check(lib().fp4_debug_stall_next_decode(cta))


def fp4_debug_encode(inp, n, which, out, stream=None):
    _check(lib().fp4_debug_encode(_p(inp), n, which, _p(out), _s(stream)))


# ---------------------------------------------------------------- conveniences
@dataclass
class Quantized:
    """A quantized [rows, cols] tensor in libfp4's layouts (see include/fp4.h)."""
    codes: torch.Tensor                 # uint8 [rows, cols/2]
    scales: torch.Tensor                # uint8, swizzled atoms
    g: torch.Tensor                     # float32 [1] on the device
    rows: int
    cols: int
    fmt: int
    codesT: Optional[torch.Tensor] = None
    scalesT: Optional[torch.Tensor] = None


class Workspace:
    """Zero-filled device scratch owned by the caller, reused across calls."""

    def __init__(self, device=None):
        self.device = torch.device(device or "cuda")
        self.buf = torch.zeros(0, dtype=torch.uint8, device=self.device)

    def get(self, nbytes: int) -> torch.Tensor:
        if nbytes > self.buf.numel():
            self.buf = torch.zeros(max(nbytes, 4096), dtype=torch.uint8, device=self.device)
        return self.buf


def quantize(x: torch.Tensor, fmt: int = NVFP4, block: Optional[int] = None, global_in=None,
             workspace: Optional[Workspace] = None, stream=None) -> Quantized:
    """Allocate outputs and run fp4_quantize on a contiguous [rows, cols] CUDA tensor."""
    if block is None:
        block = 16 if fmt == NVFP4 else 32
    x = x.contiguous()
    rows, cols = (1, x.numel()) if x.dim() == 1 else tuple(x.shape)
    dev = x.device
    codes = torch.empty(rows, cols if fmt == MXFP8 else cols // 2, dtype=torch.uint8, device=dev)
    scales = torch.empty(fp4_scales_bytes(rows, cols, fmt), dtype=torch.uint8, device=dev)
    g = torch.empty(1, dtype=torch.float32, device=dev)
    codesT = scalesT = None
    if block == 256:
        codesT = torch.empty(cols, rows // 2, dtype=torch.uint8, device=dev)
        scalesT = torch.empty(fp4_scales_bytes(cols, rows, NVFP4), dtype=torch.uint8, device=dev)
    ws = (workspace or Workspace(dev)).get(fp4_quantize_workspace_size())
    fp4_quantize(x, rows, cols, _dtype_code(x), fmt, block, codes, scales, g, codesT, scalesT, global_in, ws,
                 ws.numel(), stream)
    return Quantized(codes, scales, g, rows, cols, fmt, codesT, scalesT)


def gemm(a: Quantized, b: Quantized, out_dtype=torch.bfloat16, workspace: Optional[Workspace] = None,
         stream=None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """D[M, N] = A . B^T for quantized A [M, K] and B [N, K]."""
    assert a.fmt == b.fmt and a.cols == b.cols
    M, N, K = a.rows, b.rows, a.cols
    if out is None:
        out = torch.empty(M, N, dtype=out_dtype, device=a.codes.device)
    oc = BF16 if out.dtype == torch.bfloat16 else F32
    nbytes = fp4_gemm_workspace_size(M, N, K, a.fmt)
    ws = (workspace or Workspace(a.codes.device)).get(nbytes) if nbytes else None
    fp4_gemm(a.fmt, a.codes, a.scales, a.g, b.codes, b.scales, b.g, M, N, K, out, oc, ws,
             ws.numel() if ws is not None else 0, stream)
    return out


def gemm_mixed(a: Quantized, b: Quantized, out_dtype=torch.bfloat16, stream=None,
               out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """D[M, N] = A . B^T for A and B each quantized as MXFP4 or MXFP8 (K % 128 == 0)."""
    assert a.cols == b.cols
    M, N, K = a.rows, b.rows, a.cols
    if out is None:
        out = torch.empty(M, N, dtype=out_dtype, device=a.codes.device)
    oc = BF16 if out.dtype == torch.bfloat16 else F32
    fp4_gemm_mixed(a.fmt, a.codes, a.scales, b.fmt, b.codes, b.scales, M, N, K, out, oc, stream)
    return out


def transposed(w: Quantized) -> Quantized:
    """The W^T operand a 16x16 (block 256) quantization produced alongside W."""
    assert w.codesT is not None
    return Quantized(w.codesT, w.scalesT, w.g, w.cols, w.rows, w.fmt)
