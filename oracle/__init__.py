"""CPU oracle for block-scaled FP4 (NVFP4 / MXFP4) quantization and the FP4 GEMM.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this package.
It shares no code with the CUDA library (``block_scaled_fp4_04_b200``) and neither
imports the other; the product path never falls back to it.

The element-level definitions (code tables, encoders, quantizers, scale layout,
dequantization) live in ``fp4_oracle.c`` and are loaded through ctypes.  The GEMM
reference is the plain definition written out: the FP64 product of the dequantized
operands, ``D_ref = A_hat @ B_hat^T``, with NumPy's matmul as the one library step.

Sources: "Rubin FP4 GEMM overview" (yfxerp.com) 3.1 and 3.2 -- FP4 inputs, block
scale factors re-applied to the FP32 accumulators; "FP4" glossary entry
(ultralytics.com) "How FP4 works" -- E2M1 grid, block scale amax/6, MXFP4 and NVFP4;
"MXFP4 / NVFP4 video transcript" (prism.simon-ai.net) -- NVFP4's FP32 tensor scale,
16x16 weight blocks.

The next steps after the hot path have their definitions here too, ahead of any
kernel: the epilogue's bias and activation ("Rubin FP4 GEMM overview" 3.2 and 4.2),
the random Hadamard transform and stochastic rounding of the NVFP4 training recipe
("MXFP4 / NVFP4 video transcript", training-recipe passage; "FP4" glossary entry,
section "Inference and training in FP4").

Parity pins: every function here is pinned by a ``-m "not gpu"`` test in
``tests/test_oracle_*.py`` (code enumeration, library conversions, the glossary's
printed block-size experiment, hand-worked blocks, invariants, exact-rational brute
force for the GEMM).  Parity unpinned: none of the functions below; the hardware's
internal accumulation order is outside the oracle (covered by the GEMM tolerance).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None
_lock = threading.Lock()

NVFP4 = 0
MXFP4 = 1
MXFP8 = 2  # E4M3 elements, E8M0 scale per 32 (the FP8 operand of the mixed GEMM)
F32 = 0
BF16 = 1
ERR_NONFINITE = 5

# IEEE single-precision arithmetic as written: no FMA contraction, no fast-math.
CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11", "-Wall", "-fopenmp", "-shared", "-fPIC"]


def build(force: bool = False) -> str:
    """Compile fp4_oracle.c into oracle/liboracle.so with gcc (no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def configure(lib: ctypes.CDLL) -> ctypes.CDLL:
    """Declares the C functions' signatures on a loaded copy of the oracle library."""
    P, I64, I32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    sig = {
        "orc_e2m1_decode": (ctypes.c_double, [ctypes.c_uint8]),
        "orc_e2m1_encode": (ctypes.c_uint8, [ctypes.c_float]),
        "orc_e4m3_decode": (ctypes.c_double, [ctypes.c_uint8]),
        "orc_e4m3_encode": (ctypes.c_uint8, [ctypes.c_float]),
        "orc_e8m0_decode": (ctypes.c_double, [ctypes.c_uint8]),
        "orc_e8m0_encode": (ctypes.c_uint8, [ctypes.c_float]),
        "orc_e2m1_encode_array": (None, [P, I64, P]),
        "orc_e4m3_encode_array": (None, [P, I64, P]),
        "orc_e8m0_encode_array": (None, [P, I64, P]),
        "orc_amax": (I32, [P, I64, I32, P]),
        "orc_global_scale": (ctypes.c_float, [ctypes.c_float]),
        "orc_quantize_nvfp4_1d": (I32, [P, I64, I64, I32, P, P, P, P]),
        "orc_quantize_nvfp4_1d_r": (I32, [P, I64, I64, I32, P, P, P, P, P]),
        "orc_e2m1_encode_sr": (ctypes.c_uint8, [ctypes.c_float, ctypes.c_uint32]),
        "orc_rht16": (I32, [P, I64, I64, I32, ctypes.c_uint32, P]),
        "orc_quantize_mxfp4_1d": (I32, [P, I64, I64, I32, P, P]),
        "orc_quantize_mxfp4_1d_r": (I32, [P, I64, I64, I32, I32, P, P]),
        "orc_e8m0_encode_floor": (ctypes.c_uint8, [ctypes.c_float]),
        "orc_quantize_nvfp4_2d": (I32, [P, I64, I64, I32, P, P, P, P, P, P]),
        "orc_scales_bytes": (I64, [I64, I64]),
        "orc_swizzle_offset": (I64, [I64, I64, I64]),
        "orc_swizzle_scales": (None, [P, I64, I64, P]),
        "orc_unswizzle_scales": (None, [P, I64, I64, P]),
        "orc_scales_bytes_grouped": (I64, [P, I32, I64]),
        "orc_swizzle_scales_grouped": (None, [P, P, I32, I64, P]),
        "orc_dequantize": (None, [P, P, ctypes.c_float, I64, I64, I32, P]),
        "orc_quantize_mxfp8_1d": (I32, [P, I64, I64, I32, P, P]),
        "orc_dequantize_mxfp8": (None, [P, P, I64, I64, P]),
        "orc_fake_quant_fp32_scale": (None, [P, I64, I64, P]),
        "orc_e2m1_count_mismatch": (I64, [ctypes.c_uint64, I64, P]),
        "orc_num_threads": (I32, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def _L():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = configure(ctypes.CDLL(_LIB_PATH))
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


class NonFiniteInput(ValueError):
    """The tensor holds inf or NaN; no FP4 encoding is defined for it."""


# ---------------------------------------------------------------- scalar codes
def e2m1_decode(code: int) -> float:
    return _L().orc_e2m1_decode(code)


def e4m3_decode(code: int) -> float:
    return _L().orc_e4m3_decode(code)


def e8m0_decode(code: int) -> float:
    return _L().orc_e8m0_decode(code)


def e2m1_encode(v) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.uint8)
    _L().orc_e2m1_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def e4m3_encode(v) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.uint8)
    _L().orc_e4m3_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def e8m0_encode(v) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.uint8)
    _L().orc_e8m0_encode_array(_ptr(v), v.size, _ptr(out))
    return out


# ---------------------------------------------------------------- tensors
def _as_input(x: np.ndarray):
    """float32 arrays pass as fp32; uint16 arrays are bf16 bit patterns."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.uint16:
        return x, BF16
    raise TypeError(f"oracle input must be float32 or uint16 (bf16 bits), got {x.dtype}")


def amax(x: np.ndarray) -> float:
    x, dt = _as_input(x)
    out = np.zeros(1, np.float32)
    if _L().orc_amax(_ptr(x), x.size, dt, _ptr(out)) != 0:
        raise NonFiniteInput("non-finite element")
    return float(out[0])


def global_scale(amax_t: float) -> np.float32:
    return np.float32(_L().orc_global_scale(amax_t))


def e8m0_encode_floor(amax_b: float) -> int:
    """E8M0 scale code rounded down: 2^(floor(log2 amax_b) - 2), by brute force."""
    return int(_L().orc_e8m0_encode_floor(ctypes.c_float(amax_b)))


def quantize(x: np.ndarray, fmt: int = NVFP4, block: int = 16, g_in=None, e8m0_floor: bool = False):
    """Quantize a row-major [rows, cols] tensor.

    Returns a dict with ``codes`` [rows, cols/2] uint8 (even element in the low
    nibble), ``scales`` row-major [rows, cols/16 or /32] uint8, ``g`` (float32; 1.0
    for MXFP4) and, for the 16x16 mode (block=256), ``codesT`` [cols, rows/2] and
    ``scalesT`` [cols, rows/16].  ``e8m0_floor`` (MXFP4 only) picks the rounded-down
    power-of-two scale instead of the nearest one.
    """
    x, dt = _as_input(x)
    if x.ndim == 1:
        x = x.reshape(1, -1)
    rows, cols = x.shape
    L = _L()
    gbuf = np.zeros(1, np.float32)
    gin = None
    if g_in is not None:
        gin = np.array([g_in], np.float32)
    out = {}
    if fmt == NVFP4 and block == 16:
        codes = np.zeros((rows, cols // 2), np.uint8)
        sc = np.zeros((rows, cols // 16), np.uint8)
        rc = L.orc_quantize_nvfp4_1d(_ptr(x), rows, cols, dt, _ptr(gin) if gin is not None else None,
                                     _ptr(codes), _ptr(sc), _ptr(gbuf))
        out.update(codes=codes, scales=sc, g=np.float32(gbuf[0]))
    elif fmt == MXFP4 and block == 32:
        codes = np.zeros((rows, cols // 2), np.uint8)
        sc = np.zeros((rows, cols // 32), np.uint8)
        rc = L.orc_quantize_mxfp4_1d_r(_ptr(x), rows, cols, dt, 1 if e8m0_floor else 0, _ptr(codes), _ptr(sc))
        out.update(codes=codes, scales=sc, g=np.float32(1.0))
    elif fmt == MXFP8 and block == 32:
        codes = np.zeros((rows, cols), np.uint8)
        sc = np.zeros((rows, cols // 32), np.uint8)
        rc = L.orc_quantize_mxfp8_1d(_ptr(x), rows, cols, dt, _ptr(codes), _ptr(sc))
        out.update(codes=codes, scales=sc, g=np.float32(1.0))
    elif fmt == NVFP4 and block == 256:
        codes = np.zeros((rows, cols // 2), np.uint8)
        sc = np.zeros((rows, cols // 16), np.uint8)
        codesT = np.zeros((cols, rows // 2), np.uint8)
        scT = np.zeros((cols, rows // 16), np.uint8)
        rc = L.orc_quantize_nvfp4_2d(_ptr(x), rows, cols, dt, _ptr(gin) if gin is not None else None,
                                     _ptr(codes), _ptr(sc), _ptr(codesT), _ptr(scT), _ptr(gbuf))
        out.update(codes=codes, scales=sc, codesT=codesT, scalesT=scT, g=np.float32(gbuf[0]))
    else:
        raise ValueError(f"unsupported fmt/block {fmt}/{block}")
    if e8m0_floor and fmt != MXFP4:
        raise ValueError("e8m0_floor applies to MXFP4 only")
    if rc != 0:
        raise NonFiniteInput("non-finite element")
    return out


def scales_bytes(rows: int, scols: int) -> int:
    return int(_L().orc_scales_bytes(rows, scols))


def swizzle_offset(r: int, c: int, scols: int) -> int:
    return int(_L().orc_swizzle_offset(r, c, scols))


def swizzle_scales(rm: np.ndarray) -> np.ndarray:
    rm = np.ascontiguousarray(rm, dtype=np.uint8)
    rows, scols = rm.shape
    out = np.zeros(scales_bytes(rows, scols), np.uint8)
    _L().orc_swizzle_scales(_ptr(rm), rows, scols, _ptr(out))
    return out


def unswizzle_scales(sw: np.ndarray, rows: int, scols: int) -> np.ndarray:
    sw = np.ascontiguousarray(sw, dtype=np.uint8)
    out = np.zeros((rows, scols), np.uint8)
    _L().orc_unswizzle_scales(_ptr(sw), rows, scols, _ptr(out))
    return out


def scales_bytes_grouped(offsets: np.ndarray, scols: int) -> int:
    off = np.ascontiguousarray(offsets, dtype=np.int32)
    return int(_L().orc_scales_bytes_grouped(_ptr(off), len(off) - 1, scols))


def swizzle_scales_grouped(rm: np.ndarray, offsets: np.ndarray) -> np.ndarray:
    rm = np.ascontiguousarray(rm, dtype=np.uint8)
    off = np.ascontiguousarray(offsets, dtype=np.int32)
    scols = rm.shape[1]
    out = np.zeros(scales_bytes_grouped(off, scols), np.uint8)
    _L().orc_swizzle_scales_grouped(_ptr(rm), _ptr(off), len(off) - 1, scols, _ptr(out))
    return out


def dequantize(codes: np.ndarray, scales_rm: np.ndarray, g: float, fmt: int = NVFP4) -> np.ndarray:
    """x_hat = E2M1(code) * dec(scale) (* g for NVFP4), or E4M3(code) * dec(scale) for
    MXFP8 (one code per byte), in float64, shape [rows, cols]."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales_rm = np.ascontiguousarray(scales_rm, dtype=np.uint8)
    if fmt == MXFP8:
        rows, cols = codes.shape
        out = np.zeros((rows, cols), np.float64)
        _L().orc_dequantize_mxfp8(_ptr(codes), _ptr(scales_rm), rows, cols, _ptr(out))
        return out
    rows, half = codes.shape
    cols = half * 2
    out = np.zeros((rows, cols), np.float64)
    _L().orc_dequantize(_ptr(codes), _ptr(scales_rm), float(g), rows, cols, fmt, _ptr(out))
    return out


def e2m1_count_mismatch(start_bits: int, codes: np.ndarray) -> int:
    """Mismatches between codes[i] and the oracle's E2M1 code of float32 bit pattern
    start_bits + i (NaN patterns skipped)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    return int(_L().orc_e2m1_count_mismatch(start_bits, codes.size, _ptr(codes)))


def num_threads() -> int:
    return int(_L().orc_num_threads())


def fake_quant_fp32_scale(x: np.ndarray, block: int) -> np.ndarray:
    """The glossary experiment's procedure: unrounded FP32 block scale amax/6,
    nearest E2M1 grid point; returns the dequantized float32 values."""
    x = np.ascontiguousarray(x, dtype=np.float32).reshape(-1)
    out = np.zeros_like(x)
    _L().orc_fake_quant_fp32_scale(_ptr(x), x.size, block, _ptr(out))
    return out


# ---------------------------------------------------------------- GEMM
def gemm_reference(a_hat: np.ndarray, b_hat: np.ndarray, rows=None):
    """FP64 definition of the block-scaled GEMM on dequantized operands.

    ``D_ref[m, n] = sum_k a_hat[m, k] * b_hat[n, k]`` (A row-major [M, K], B
    row-major [N, K], both already multiplied by their block and global scales),
    and the tolerance base ``S[m, n] = sum_k |a_hat[m, k] * b_hat[n, k]|``.
    ``rows`` restricts both to the listed output rows.
    """
    a = a_hat if rows is None else a_hat[np.asarray(rows)]
    d = a @ b_hat.T
    s = np.abs(a) @ np.abs(b_hat).T
    return d, s


def gemm_tolerance(d_ref: np.ndarray, abs_sum: np.ndarray, bf16_out: bool) -> np.ndarray:
    """|D - D_ref| <= 1e-6 * sum_k |a_k b_k|, plus half a BF16 ulp of D_ref when the
    output is BF16 (the larger ulp at a binade edge)."""
    tol = 1e-6 * abs_sum
    if bf16_out:
        tol = tol + 0.5 * bf16_ulp(np.abs(d_ref) + tol)
    return tol


def epilogue_tolerance(t_ref: np.ndarray, d_ref: np.ndarray, abs_sum: np.ndarray, bias, bf16_out: bool) -> np.ndarray:
    """Tolerance of t = act(D + bias) computed in FP32 after the product ("Rubin FP4 GEMM
    overview" 3.2 order: scale, bias, activation).  The product keeps its bound
    1e-6 * sum_k |a_k b_k|; adding the bias in FP32 rounds once more, by at most 2^-24 of
    |D + bias| <= |D_ref| + bound + |bias|; ReLU moves no value further from its reference
    (it is 1-Lipschitz); a BF16 output adds half a BF16 ulp of the result.  ``t_ref`` is
    ``epilogue(d_ref, bias, act)``."""
    tol = 1e-6 * abs_sum
    b = 0.0 if bias is None else np.abs(np.asarray(bias, dtype=np.float64))[None, :]
    tol = tol + 2.0 ** -24 * (np.abs(d_ref) + tol + b)
    if bf16_out:
        tol = tol + 0.5 * bf16_ulp(np.abs(t_ref) + tol)
    return tol


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """Spacing of BF16 values around |v| (8 significant bits); at an exact power of
    two the larger spacing (above it) is used."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126.0)
    return np.ldexp(1.0, (e - 7).astype(np.int64))


# ---------------------------------------------------------------- next steps
def epilogue(d: np.ndarray, bias=None, act: str = "none") -> np.ndarray:
    """The epilogue after the scale factors ("Rubin FP4 GEMM overview" 3.2: the FP32
    result is multiplied by the scale factors, the bias is added, the activation is
    applied, then it is converted to the output format; 4.2: C = (A.B)(sA.sB) + bias).
    ``d`` is the scaled product (``gemm_reference`` of the dequantized operands);
    ``bias`` [N] is added to every row; ``act`` is "none" or "relu" (the cited sources
    name no activation; ReLU is the plainest).  FP64."""
    out = np.asarray(d, dtype=np.float64)
    if bias is not None:
        out = out + np.asarray(bias, dtype=np.float64)[None, :]
    if act == "relu":
        out = np.maximum(out, 0.0)
    elif act != "none":
        raise ValueError(f"unknown activation {act}")
    return out


def hadamard16() -> np.ndarray:
    """The 16x16 Sylvester Hadamard matrix by its definition, H[i, j] =
    (-1)^popcount(i & j)."""
    i = np.arange(16)[:, None]
    j = np.arange(16)[None, :]
    return np.where(np.vectorize(lambda v: bin(v).count("1") % 2)(i & j) == 1, -1.0, 1.0)


def rht16_reference(x: np.ndarray, signs: int) -> np.ndarray:
    """Random Hadamard transform, FP64 definition: each 16-element block b of a row
    becomes Q b with Q = (1/4) H16 diag(s), s_i = -1 where bit i of ``signs`` is set
    ("MXFP4 / NVFP4 video transcript", training-recipe passage: the values are mixed,
    the vector's magnitude is kept, a dot product of two transformed operands is
    unchanged)."""
    x = np.asarray(x, dtype=np.float64)
    rows, cols = x.shape
    s = np.array([-1.0 if (signs >> i) & 1 else 1.0 for i in range(16)])
    q = hadamard16() * s[None, :] / 4.0
    return (x.reshape(rows, cols // 16, 16) @ q.T).reshape(rows, cols)


def rht16(x: np.ndarray, signs: int) -> np.ndarray:
    """The same transform in FP32, in the fast Walsh-Hadamard order (the signs, the
    butterfly stages of half-width 1, 2, 4, 8, then the factor 1/4): the order a kernel
    uses, so that both sides quantize the same FP32 values."""
    xa, dt = _as_input(x)
    if xa.ndim == 1:
        xa = xa.reshape(1, -1)
    rows, cols = xa.shape
    out = np.zeros((rows, cols), np.float32)
    if _L().orc_rht16(_ptr(xa), rows, cols, dt, ctypes.c_uint32(signs & 0xFFFF), _ptr(out)) != 0:
        raise NonFiniteInput("non-finite element")
    return out


def e2m1_encode_sr(v: float, bits: int) -> int:
    """Stochastic E2M1 rounding of one FP32 value with one 32-bit random word."""
    return int(_L().orc_e2m1_encode_sr(ctypes.c_float(v), ctypes.c_uint32(bits)))


def quantize_sr(x: np.ndarray, rbits: np.ndarray, g_in=None):
    """NVFP4 1-D quantize with stochastic rounding of the elements (the block scales
    are the round-to-nearest quantizer's; "MXFP4 / NVFP4 video transcript",
    training-recipe passage, fourth part).  ``rbits``: one uint32 per element, the
    random numbers the method draws, passed in.  Returns codes / scales / g as
    ``quantize``."""
    xa, dt = _as_input(x)
    if xa.ndim == 1:
        xa = xa.reshape(1, -1)
    rows, cols = xa.shape
    rb = np.ascontiguousarray(rbits, dtype=np.uint32).reshape(rows, cols)
    codes = np.zeros((rows, cols // 2), np.uint8)
    sc = np.zeros((rows, cols // 16), np.uint8)
    gbuf = np.zeros(1, np.float32)
    gin = None if g_in is None else np.array([g_in], np.float32)
    rc = _L().orc_quantize_nvfp4_1d_r(_ptr(xa), rows, cols, dt, _ptr(gin) if gin is not None else None, _ptr(rb),
                                      _ptr(codes), _ptr(sc), _ptr(gbuf))
    if rc != 0:
        raise NonFiniteInput("non-finite element")
    return {"codes": codes, "scales": sc, "g": np.float32(gbuf[0])}

