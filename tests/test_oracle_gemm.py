"""Pins for the oracle's GEMM reference (CPU only).

The FP64 reference is checked against exact rational arithmetic on small,
non-square shapes (so a transposed operand or a swapped index fails), against
closed forms (identity and rank-1 operands) and against the tolerance rule.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads


def _quantized(rows, cols, seed, fmt=oracle.NVFP4):
    x = workloads.with_outliers(workloads.normal((rows, cols), 1.0, seed), seed).numpy()
    blk = 16 if fmt == oracle.NVFP4 else 32
    q = oracle.quantize(x, fmt, blk)
    return oracle.dequantize(q["codes"], q["scales"], q["g"], fmt)


@pytest.mark.parametrize("m,n,k,fmt", [(3, 5, 64, oracle.NVFP4), (4, 2, 96, oracle.MXFP4), (1, 7, 32, oracle.NVFP4)])
def test_gemm_reference_vs_exact_rationals(m, n, k, fmt):
    a = _quantized(m, k, 11, fmt)
    b = _quantized(n, k, 12, fmt)
    d, s = oracle.gemm_reference(a, b)
    assert d.shape == (m, n)
    for i in range(m):
        for j in range(n):
            exact = sum(Fraction(float(a[i, t])) * Fraction(float(b[j, t])) for t in range(k))
            mag = sum(abs(Fraction(float(a[i, t])) * Fraction(float(b[j, t]))) for t in range(k))
            assert abs(Fraction(float(d[i, j])) - exact) <= Fraction(1, 10 ** 12) * (mag + 1)
            assert abs(Fraction(float(s[i, j])) - mag) <= Fraction(1, 10 ** 12) * (mag + 1)


def test_gemm_identity_operand():
    """A = identity (code 1.0 on the diagonal) gives D = B_hat^T exactly."""
    k = 64
    b = _quantized(24, k, 13)
    eye = np.eye(k)[:40]
    d, _ = oracle.gemm_reference(eye, b)
    assert np.array_equal(d, b[:, :40].T)


def test_gemm_rank_one_integer_sums():
    a = np.ones((3, 128))
    b = np.arange(5 * 128, dtype=np.float64).reshape(5, 128) % 7 - 3
    d, s = oracle.gemm_reference(a, b)
    assert np.array_equal(d, np.tile(b.sum(1), (3, 1)))
    assert np.array_equal(s, np.tile(np.abs(b).sum(1), (3, 1)))


def test_sampled_rows_equal_full():
    a = _quantized(20, 64, 14)
    b = _quantized(9, 64, 15)
    d, s = oracle.gemm_reference(a, b)
    rows = [0, 7, 19]
    d2, s2 = oracle.gemm_reference(a, b, rows)
    # BLAS may sum in another order for another shape: equal to rounding
    assert np.allclose(d[rows], d2, rtol=1e-12, atol=1e-12) and np.allclose(s[rows], s2, rtol=1e-12)


def test_tolerance_rule():
    d = np.array([1.0, 1.0, 3.0, 0.0])
    s = np.array([1e3, 1e3, 1e3, 1e3])
    tol32 = oracle.gemm_tolerance(d, s, bf16_out=False)
    assert np.allclose(tol32, 1e-3)
    tol16 = oracle.gemm_tolerance(d, s, bf16_out=True)
    # bf16 keeps 8 significant bits: ulp(1) = 2^-7, ulp(3) = 2^-6
    assert np.isclose(tol16[0], 1e-3 + 2.0 ** -8)
    assert np.isclose(tol16[2], 1e-3 + 2.0 ** -7)
    assert oracle.bf16_ulp(np.array([1.0]))[0] == 2.0 ** -7
    assert oracle.bf16_ulp(np.array([1.99]))[0] == 2.0 ** -7
    assert oracle.bf16_ulp(np.array([2.0]))[0] == 2.0 ** -6
