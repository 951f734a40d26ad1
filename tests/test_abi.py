"""C-ABI checks that need no GPU: the library loads, exports every function that
include/fp4.h declares, sizes buffers as documented, and rejects bad arguments on the
host before touching the device."""
import ctypes
import os
import re

import pytest

import block_scaled_fp4_04_b200 as fp4
from block_scaled_fp4_04_b200 import build as fp4_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    fp4_build.build()


def _declared():
    with open(os.path.join(ROOT, "include", "fp4.h")) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fp4_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert len(names) >= 14
    lib = ctypes.CDLL(fp4.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_binding_covers_every_declared_symbol():
    for n in _declared():
        assert hasattr(fp4, n), n


def test_version():
    assert "sm_100a" in fp4.fp4_version()


def test_scale_buffer_sizes():
    assert fp4.fp4_scales_bytes(1, 32, fp4.NVFP4) == 128 * 4
    assert fp4.fp4_scales_bytes(130, 96, fp4.NVFP4) == 256 * 8      # 6 scale cols pad to 8
    assert fp4.fp4_scales_bytes(16384, 2880, fp4.MXFP4) == 16384 * 92  # 90 pad to 92
    assert fp4.fp4_scales_bytes(28672, 8192, fp4.NVFP4) == 28672 * 512
    assert fp4.fp4_scales_bytes_grouped(16384, 32, 2880, fp4.MXFP4) == (128 + 32) * 128 * 92
    assert fp4.fp4_quantize_workspace_size() >= 1024


def test_gemm_workspace_sizes():
    # decode runs split over K and needs [N, M] floats plus tile counters
    ws = fp4.fp4_gemm_workspace_size(16, 28672, 8192, fp4.NVFP4)
    assert ws >= 16 * 28672 * 4
    assert fp4.fp4_gemm_workspace_size(8192, 8192, 8192, fp4.NVFP4) == 0


def _rc_quantize(**kw):
    L = fp4.lib()
    a = dict(x=16, rows=4, cols=64, dt=fp4.F32, fmt=fp4.NVFP4, block=16, codes=16, scales=16, gout=16,
             codesT=None, scalesT=None, gin=None, ws=16, wsb=1 << 20)
    a.update(kw)
    return L.fp4_quantize(a["x"], a["rows"], a["cols"], a["dt"], a["fmt"], a["block"], a["codes"], a["scales"],
                          a["gout"], a["codesT"], a["scalesT"], a["gin"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw", [
    dict(x=None), dict(cols=48), dict(rows=0), dict(fmt=7), dict(block=32), dict(fmt=fp4.MXFP4, block=16),
    dict(block=256), dict(codesT=16), dict(x=8), dict(wsb=16), dict(gout=None), dict(dt=9),
    dict(block=256, codesT=16, scalesT=16, rows=48),
])
def test_quantize_rejects_bad_arguments(kw):
    assert _rc_quantize(**kw) == fp4.ERR_INVALID_ARG


def test_gemm_rejects_bad_arguments():
    L = fp4.lib()
    good = [fp4.NVFP4, 16, 16, 16, 16, 16, 16, 128, 128, 256, 16, fp4.BF16, None, 0, None]

    def call(i, v):
        a = list(good)
        a[i] = v
        return L.fp4_gemm(*a)

    assert call(1, None) == fp4.ERR_INVALID_ARG          # null A
    assert call(9, 48) == fp4.ERR_INVALID_ARG            # K % 32
    assert call(7, 0) == fp4.ERR_INVALID_ARG             # M
    assert call(10, 8) == fp4.ERR_INVALID_ARG            # misaligned D
    assert call(0, 5) == fp4.ERR_INVALID_ARG             # fmt
    assert L.fp4_gemm_grouped(fp4.MXFP4, 0, 16, 16, 16, None, 16, 16, None, 64, 128, 64, 16, fp4.BF16,
                              None, 0, None) == fp4.ERR_INVALID_ARG
    assert L.fp4_gemm_grouped(fp4.MXFP4, 4, 16, 16, 16, None, 16, 16, None, 64, 100, 64, 16, fp4.BF16,
                              None, 0, None) == fp4.ERR_INVALID_ARG   # N % 128
    assert L.fp4_gemm_grouped(fp4.MXFP4, 1025, 16, 16, 16, None, 16, 16, None, 64, 128, 64, 16, fp4.BF16,
                              None, 0, None) == fp4.ERR_INVALID_ARG   # more than 1024 groups
    assert L.fp4_gemm_grouped(fp4.MXFP4, 4, None, 16, 16, None, 16, 16, None, 64, 128, 64, 16, fp4.BF16,
                              None, 0, None) == fp4.ERR_INVALID_ARG   # no offsets


def test_mixed_gemm_rejects_bad_arguments():
    L = fp4.lib()
    good = [fp4.MXFP4, 32, 16, fp4.MXFP8, 64, 16, 128, 128, 256, 16, fp4.BF16, None]

    def call(i, v):
        a = list(good)
        a[i] = v
        return L.fp4_gemm_mixed(*a)

    assert call(0, fp4.NVFP4) == fp4.ERR_INVALID_ARG     # NVFP4 operands use fp4_gemm
    assert call(3, 7) == fp4.ERR_INVALID_ARG             # b_fmt
    assert call(8, 192) == fp4.ERR_INVALID_ARG           # K % 128
    assert call(1, 16) == fp4.ERR_INVALID_ARG            # A only 16-byte aligned
    assert call(4, 48) == fp4.ERR_INVALID_ARG            # B only 16-byte aligned
    assert call(9, None) == fp4.ERR_INVALID_ARG          # null D
    assert call(10, 3) == fp4.ERR_INVALID_ARG            # out dtype
    assert call(6, 0) == fp4.ERR_INVALID_ARG             # M


def test_mxfp8_quantize_arguments():
    assert fp4.fp4_scales_bytes(300, 1024, fp4.MXFP8) == fp4.fp4_scales_bytes(300, 1024, fp4.MXFP4)
    assert _rc_quantize(fmt=fp4.MXFP8, block=16) == fp4.ERR_INVALID_ARG
    assert _rc_quantize(fmt=fp4.MXFP8, block=256) == fp4.ERR_INVALID_ARG
    L = fp4.lib()
    assert L.fp4_quantize_grouped(16, 64, 64, fp4.F32, fp4.MXFP8, 2, 16, 16, 16, None, None, 16, 1 << 20, None) \
        == fp4.ERR_UNSUPPORTED
    assert L.fp4_quantize_ex(16, 4, 64, fp4.F32, fp4.MXFP8, 32, fp4.QUANT_E8M0_FLOOR, 16, 16, 16, None, None,
                             None, 16, 1 << 20, None) == fp4.ERR_UNSUPPORTED


def test_gemm_ex_rejects_unknown_flags():
    L = fp4.lib()
    assert L.fp4_gemm_ex(fp4.NVFP4, 16, 16, 16, 16, 16, 16, 128, 128, 256, 16, fp4.BF16, None, 0, 6, None) \
        == fp4.ERR_INVALID_ARG


def test_last_error_message():
    _rc_quantize(cols=48)
    assert b"multiple of 32" in fp4.lib().fp4_last_error()


def test_no_oracle_import_in_product():
    """The product package never imports or loads the oracle."""
    pkg = os.path.join(ROOT, "block_scaled_fp4_04_b200")
    for dp, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                with open(os.path.join(dp, f)) as fh:
                    assert "oracle" not in fh.read().lower(), f
