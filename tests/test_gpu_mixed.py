"""The FP4 x FP8 path ("Rubin FP4 GEMM overview" 3.4: an FP4 operand opposite an FP8 one)
against the oracle: the MXFP8 quantizer bit-exact (codes, swizzled scales with their pads,
g = 1), and the mixed GEMM within the GEMM tolerance for every pairing of MXFP4 and MXFP8
operands, on both tile widths, ragged M and N, FP32 and BF16 output."""
import numpy as np
import pytest
import torch

import block_scaled_fp4_04_b200 as fp4
import oracle
from fp4_testutil import (assert_quant_equal, check_gemm, dequant_oracle, gpu_quantize, host_input, oracle_quantize,
                          random_input)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,cols,dtype", [(1, 32, torch.float32), (130, 96, torch.bfloat16),
                                             (300, 1024, torch.float32), (257, 2880, torch.bfloat16)])
def test_mxfp8_quantize_bit_exact(rows, cols, dtype):
    x = random_input(rows, cols, rows + 5 * cols, dtype)
    gq = gpu_quantize(x.cuda(), fp4.MXFP8, 32)
    assert fp4.fp4_get_status() == fp4.OK
    assert_quant_equal(gq, oracle_quantize(x, fp4.MXFP8, 32), f"mxfp8 {rows}x{cols}")


def test_mxfp8_quantize_every_e4m3_code_and_midpoint():
    """Rows of [448, v, -v, 0...]: scale 2^0, so v encodes directly; v runs over every E4M3
    magnitude and every midpoint between neighbours (ties to the even code)."""
    mags = [oracle.e4m3_decode(c) for c in range(0x7F)]
    vals = mags + [(mags[i] + mags[i + 1]) / 2 for i in range(len(mags) - 1)]
    x = torch.zeros(len(vals), 64, dtype=torch.float32)
    x[:, 0] = 448.0
    x[:, 1] = torch.tensor(vals)
    x[:, 2] = -torch.tensor(vals)
    x[:, 40] = torch.tensor(vals) * 2.0 ** -20     # second block: a small scale, subnormal elements
    gq = gpu_quantize(x.cuda(), fp4.MXFP8, 32)
    assert_quant_equal(gq, oracle_quantize(x, fp4.MXFP8, 32), "e4m3 codes and midpoints")


PAIRS = [(fp4.MXFP4, fp4.MXFP8), (fp4.MXFP8, fp4.MXFP4), (fp4.MXFP8, fp4.MXFP8), (fp4.MXFP4, fp4.MXFP4)]


@pytest.mark.parametrize("a_fmt,b_fmt", PAIRS)
@pytest.mark.parametrize("m,n,k,out", [(128, 256, 128, "f32"), (300, 200, 1024, "bf16"), (1000, 640, 2048, "f32")])
def test_mixed_gemm_matches_oracle(a_fmt, b_fmt, m, n, k, out):
    xa = random_input(m, k, m + k, torch.bfloat16)
    xb = random_input(n, k, n + 3 * k, torch.float32, std=0.02, outliers=False)
    qa, qb = gpu_quantize(xa.cuda(), a_fmt, 32), gpu_quantize(xb.cuda(), b_fmt, 32)
    d = fp4.gemm_mixed(qa, qb, torch.float32 if out == "f32" else torch.bfloat16)
    torch.cuda.synchronize()
    assert fp4.fp4_get_status() == fp4.OK
    oa, ob = oracle_quantize(xa, a_fmt, 32), oracle_quantize(xb, b_fmt, 32)
    assert np.array_equal(qa.codes.cpu().numpy(), oa["codes"]) and np.array_equal(qb.codes.cpu().numpy(), ob["codes"])
    check_gemm(d, dequant_oracle(oa, a_fmt), dequant_oracle(ob, b_fmt), label=f"{a_fmt}x{b_fmt} {m}x{n}x{k}")


@pytest.mark.parametrize("a_fmt,b_fmt", [(fp4.MXFP8, fp4.MXFP4), (fp4.MXFP4, fp4.MXFP8)])
def test_mixed_gemm_256_wide_tiles(a_fmt, b_fmt):
    """Enough 256-wide tiles to fill the SMs: the 256-column tile configuration (two B
    scale row-blocks per stage); every column checked on sampled rows."""
    m, n, k = 4096, 2560, 512
    xa = random_input(m, k, 17, torch.bfloat16)
    xb = random_input(n, k, 18, torch.float32, std=0.02, outliers=False)
    qa, qb = gpu_quantize(xa.cuda(), a_fmt, 32), gpu_quantize(xb.cuda(), b_fmt, 32)
    d = fp4.gemm_mixed(qa, qb, torch.bfloat16)
    torch.cuda.synchronize()
    assert fp4.fp4_get_status() == fp4.OK
    rows = np.unique(np.concatenate([[0, m - 1], np.random.default_rng(19).integers(0, m, 64)]))
    oa = oracle.quantize(np.ascontiguousarray(host_input(xa)[rows]), a_fmt, 32)   # 1-D blocks: rows independent
    ob = oracle_quantize(xb, b_fmt, 32)
    d_rows = d[torch.from_numpy(rows).cuda()]
    check_gemm(d_rows, dequant_oracle(oa, a_fmt), dequant_oracle(ob, b_fmt), label="256-wide")
