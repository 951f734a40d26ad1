"""Pins of the oracle's MXFP8 quantizer (E4M3 elements, an E8M0 scale per 32), the FP8
operand of the mixed FP4 x FP8 GEMM ("Rubin FP4 GEMM overview" 3.4; MXFP8 beside MXFP4
in 3.1).  Reading: the scale is the nearest power of two of amax_b / 448, as MXFP4's is
of amax_b / 6.  The pins: hand-worked blocks, every E4M3 code, every midpoint, the scale
rule at and between powers of two, sign and power-of-two symmetry, the error bound."""
import os

import numpy as np
import pytest

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mxfp8_blocks.txt")


def _golden():
    out = []
    for ln in open(GOLDEN):
        if ln.startswith("mxfp8"):
            kv = dict(p.split("=") for p in ln.split()[1:])
            out.append((np.array([float(v) for v in kv["values"].split(",")], np.float32), int(kv["scale"], 16),
                        bytes.fromhex(kv["codes"])))
    return out


@pytest.mark.parametrize("idx", range(3))
def test_mxfp8_worked_blocks(idx):
    vals, scale, codes = _golden()[idx]
    q = oracle.quantize(vals.reshape(1, -1), oracle.MXFP8, 32)
    assert q["scales"].ravel().tolist() == [scale]
    assert q["codes"].tobytes() == codes


def _e4m3_codes():
    return [c for c in range(256) if (c & 0x7F) != 0x7F]   # 0x7F / 0xFF are NaN


def test_mxfp8_every_e4m3_code_round_trips():
    """A block holding 448 has scale 2^0, so each other element must come back as its own
    code: row r carries the decoded value of code r in its second place."""
    codes = _e4m3_codes()
    x = np.zeros((len(codes), 32), np.float32)
    x[:, 0] = 448.0
    x[:, 1] = [oracle.e4m3_decode(c) for c in codes]
    q = oracle.quantize(x, oracle.MXFP8, 32)
    assert np.all(q["scales"] == 127)
    assert q["codes"][:, 1].tolist() == codes
    assert np.array_equal(oracle.dequantize(q["codes"], q["scales"], 1.0, oracle.MXFP8)[:, 1], x[:, 1].astype(np.float64))


def test_mxfp8_midpoints_go_to_the_even_code():
    mags = [c for c in range(0x7F)]
    x = np.zeros((len(mags) - 1, 32), np.float32)
    x[:, 0] = 448.0
    want = []
    for i, c in enumerate(mags[:-1]):
        lo, hi = oracle.e4m3_decode(c), oracle.e4m3_decode(c + 1)
        x[i, 1] = np.float32((lo + hi) / 2)
        assert float(x[i, 1]) == (lo + hi) / 2   # exact in FP32
        want.append(c if c % 2 == 0 else c + 1)
    q = oracle.quantize(x, oracle.MXFP8, 32)
    assert q["codes"][:, 1].tolist() == want


@pytest.mark.parametrize("amax,code", [(448.0, 127), (896.0, 128), (224.0, 126), (448.0 * 1.5, 128),
                                       (448.0 * 1.49, 127), (448.0 * 0.75, 127), (448.0 * 0.74, 126),
                                       (1.0, 127 - 9), (0.0, 0)])
def test_mxfp8_scale_is_the_nearest_power_of_two_of_amax_over_448(amax, code):
    x = np.zeros((1, 32), np.float32)
    x[0, 3] = amax
    assert int(oracle.quantize(x, oracle.MXFP8, 32)["scales"][0, 0]) == code


def _rand(rows, cols, seed):
    x = workloads.normal((rows, cols), 1.0, seed)
    workloads.with_outliers(x, seed)
    return x.numpy()


def test_mxfp8_sign_symmetry():
    x = _rand(16, 256, 1)
    a, b = oracle.quantize(x, oracle.MXFP8, 32), oracle.quantize(-x, oracle.MXFP8, 32)
    assert np.array_equal(a["codes"] ^ 0x80, b["codes"])
    assert np.array_equal(a["scales"], b["scales"])


@pytest.mark.parametrize("k", [-3, 5])
def test_mxfp8_power_of_two_invariance(k):
    x = _rand(16, 256, 2)
    a = oracle.quantize(x, oracle.MXFP8, 32)
    b = oracle.quantize((x * np.float32(2.0 ** k)).astype(np.float32), oracle.MXFP8, 32)
    assert np.array_equal(a["codes"], b["codes"])
    assert np.array_equal(a["scales"].astype(int) + k, b["scales"].astype(int))


def test_mxfp8_error_bound():
    """Within half an E4M3 step: 2^-4 |x| for normals, 2^-10 scale in the subnormal range;
    elements past 448 scale (the scale rounds amax / 448 down by up to 1.5x) saturate."""
    x = _rand(64, 512, 3)
    q = oracle.quantize(x, oracle.MXFP8, 32)
    xh = oracle.dequantize(q["codes"], q["scales"], 1.0, oracle.MXFP8)
    scale = np.repeat(np.ldexp(1.0, q["scales"].astype(int) - 127), 32, axis=1)
    ratio = np.abs(x.astype(np.float64)) / scale
    sat = ratio > 448
    assert np.all(np.abs(xh[sat]) == 448 * scale[sat])
    err = np.abs(xh - x)[~sat]
    bound = np.maximum(2.0 ** -4 * np.abs(x.astype(np.float64)), 2.0 ** -10 * scale)[~sat]
    assert np.all(err <= bound)


def test_mixed_fp4_fp8_reference_is_exact_on_representable_operands():
    """The mixed GEMM's reference is the FP64 product of the two dequantized operands: on
    operands that both formats hold exactly (scale 2^0) it is the plain matrix product."""
    rng = np.random.default_rng(4)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float32)
    a = grid[rng.integers(0, 8, (8, 64))] * np.where(rng.random((8, 64)) < 0.5, -1, 1).astype(np.float32)
    a[:, 0] = 6.0                              # scale 2^0 in every MXFP4 block (6 / 6 = 1)
    a[:, 32] = 6.0
    b = np.array([oracle.e4m3_decode(c) for c in rng.integers(0, 0x7E, 6 * 64)], np.float32).reshape(6, 64)
    b[:, 0] = 448.0                            # scale 2^0 in every MXFP8 block
    b[:, 32] = 448.0
    qa, qb = oracle.quantize(a, oracle.MXFP4, 32), oracle.quantize(b, oracle.MXFP8, 32)
    a_hat = oracle.dequantize(qa["codes"], qa["scales"], 1.0, oracle.MXFP4)
    b_hat = oracle.dequantize(qb["codes"], qb["scales"], 1.0, oracle.MXFP8)
    assert np.array_equal(a_hat, a.astype(np.float64)) and np.array_equal(b_hat, b.astype(np.float64))
    d, _ = oracle.gemm_reference(a_hat, b_hat)
    assert np.array_equal(d, a.astype(np.float64) @ b.astype(np.float64).T)
