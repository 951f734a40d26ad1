"""Pins for the oracle's definitions of the steps after the hot path: the epilogue's bias
and activation, the random Hadamard transform and stochastic rounding.  Each pin rests
on something other than the function's own formula: a library routine (SciPy's
Hadamard matrix), closed forms, invariants the pages state (a transformed vector keeps
its magnitude and two transformed operands keep their dot products; a stochastically
rounded value keeps its expectation), exact counts over uniform grids of random numbers,
or hand-built operands whose products are exact."""
import numpy as np
import pytest
import scipy.linalg

import oracle

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


# ---------------------------------------------------------------- Hadamard transform
def test_hadamard16_matches_scipy():
    assert np.array_equal(oracle.hadamard16(), scipy.linalg.hadamard(16).astype(np.float64))


@pytest.mark.parametrize("signs", [0x0000, 0xFFFF, 0x8421, 0x1234])
def test_rht_is_orthonormal(signs):
    # the transform of the identity's rows gives Q^T; entries are +-1/4, so Q^T Q is exact
    qt = oracle.rht16_reference(np.eye(16), signs)
    assert np.array_equal(qt.T @ qt, np.eye(16))


@pytest.mark.parametrize("signs", [0x0000, 0x00FF, 0xA5A5])
@pytest.mark.parametrize("j", [0, 5, 15])
def test_rht_spreads_a_spike_evenly(signs, j):
    """An outlier alone in its block becomes 16 values of a quarter of its size: the
    block amax falls 4x (closed form: column j of H, times s_j, times c / 4)."""
    c = 48.0
    x = np.zeros((1, 32), np.float32)
    x[0, 16 + j] = c
    s_j = -1.0 if (signs >> j) & 1 else 1.0
    want = np.zeros(32)
    want[16:] = scipy.linalg.hadamard(16)[:, j] * s_j * c / 4.0
    assert np.array_equal(oracle.rht16_reference(x, signs)[0], want)
    assert np.array_equal(oracle.rht16(x, signs)[0].astype(np.float64), want)  # exact in FP32 too


def test_rht_keeps_block_norms():
    x = np.random.default_rng(1).normal(size=(8, 64))
    y = oracle.rht16_reference(x, 0x3C5A)
    nx = np.linalg.norm(x.reshape(8, 4, 16), axis=2)
    ny = np.linalg.norm(y.reshape(8, 4, 16), axis=2)
    assert np.allclose(nx, ny, rtol=1e-14, atol=0)


def test_rht_keeps_dot_products():
    """Transforming both operands along K alike leaves A.B^T unchanged."""
    rng = np.random.default_rng(2)
    a, b = rng.normal(size=(5, 128)), rng.normal(size=(7, 128))
    d = oracle.rht16_reference(a, 0xBEEF) @ oracle.rht16_reference(b, 0xBEEF).T
    assert np.allclose(d, a @ b.T, rtol=1e-12, atol=1e-12)


def test_rht_without_signs_is_its_own_inverse():
    x = np.random.default_rng(3).normal(size=(4, 32))
    assert np.allclose(oracle.rht16_reference(oracle.rht16_reference(x, 0), 0), x, rtol=0, atol=1e-14)


def test_rht_fp32_within_the_butterfly_bound():
    """Four butterfly stages each round once: |fp32 - exact| <= 2^-24 * sum|x| of the
    block (the factor 1/4 is exact)."""
    rng = np.random.default_rng(4)
    x = (rng.normal(size=(64, 256)) * np.exp(rng.normal(size=(64, 256)))).astype(np.float32)
    for signs in (0, 0xFFFF, 0x6E29):
        y32 = oracle.rht16(x, signs).astype(np.float64)
        ref = oracle.rht16_reference(x.astype(np.float64), signs)
        bound = 2.0 ** -24 * np.repeat(np.abs(x.astype(np.float64)).reshape(64, 16, 16).sum(2), 16, axis=1)
        assert np.all(np.abs(y32 - ref) <= bound)


def test_rht_bf16_input_equals_widened_fp32():
    rng = np.random.default_rng(5)
    bits = (rng.normal(size=(3, 48)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    wide = (bits.astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(oracle.rht16(bits, 0x0F0F), oracle.rht16(wide, 0x0F0F))


def test_rht_lowers_the_block_scale_of_blocks_with_an_outlier():
    """What the pages claim: mixing lowers the scale factor a block needs (its amax),
    here about 4x for blocks whose one large value dominates.  (It does not promise a
    lower quantization error: a lone spike spreads into 16 values near +-amax/4 that
    fall on E2M1's coarse top steps.)"""
    rng = np.random.default_rng(6)
    x = rng.normal(size=(64, 256)).astype(np.float32)
    x.reshape(64, 16, 16)[:, :, 3] = 50.0 * np.sign(x.reshape(64, 16, 16)[:, :, 3])  # one outlier per block
    y = oracle.rht16(x, 0x5AC3)
    before = np.abs(x).reshape(64, 16, 16).max(2)
    after = np.abs(y).reshape(64, 16, 16).max(2)
    ratio = after / before
    assert np.all(ratio < 0.4) and 0.25 < ratio.mean() < 0.35


# ---------------------------------------------------------------- stochastic rounding
def _bits_for(u_index: int, levels_log2: int) -> int:
    return (u_index << (32 - levels_log2)) & 0xFFFFFFFF


@pytest.mark.parametrize("sign", [1.0, -1.0])
def test_sr_keeps_grid_values(sign):
    for k, m in enumerate(GRID):
        for bits in (0, 0x80000000, 0xFFFFFFFF):
            code = oracle.e2m1_encode_sr(float(sign * m), bits)
            assert oracle.e2m1_decode(code) == sign * m
            assert code == int(oracle.e2m1_encode(np.float32(sign * m))[0])


def test_sr_returns_one_of_the_two_neighbours():
    rng = np.random.default_rng(7)
    v = rng.uniform(-5.99, 5.99, 4000).astype(np.float32)
    bits = rng.integers(0, 2 ** 32, 4000, dtype=np.uint64)
    for vi, bi in zip(v, bits):
        a = abs(float(vi))
        lo = GRID[GRID <= a].max()
        hi = GRID[GRID >= a].min()
        got = oracle.e2m1_decode(oracle.e2m1_encode_sr(float(vi), int(bi)))
        assert abs(got) in (lo, hi) and (got == 0 or np.sign(got) == np.sign(vi))


@pytest.mark.parametrize("v", [0.3, 0.75, 1.25, 1.9, 2.2, 3.7, 5.5, 0.125, 4.0 + 2.0 / 4096])
def test_sr_expectation_over_a_uniform_grid_of_u(v):
    """u = k / 4096 for k = 0..4095 rounds up exactly ceil(frac * 4096) times (up iff
    u < frac), so the mean is v to within gap / 4096 (the pages' 0.3 example: up with
    probability 0.3)."""
    n = 12
    lo = GRID[GRID <= v].max()
    hi = GRID[GRID > v].min()
    frac = (v - lo) / (hi - lo)
    got = np.array([oracle.e2m1_decode(oracle.e2m1_encode_sr(v, _bits_for(k, n))) for k in range(1 << n)])
    ups = int(np.sum(got == hi))
    assert set(np.unique(got)) <= {lo, hi}
    assert ups == int(np.ceil(np.float32(frac) * (1 << n)))
    assert abs(got.mean() - v) <= (hi - lo) / (1 << n)


def test_sr_saturates_beyond_six():
    for v in (6.0, 6.5, 100.0, 3.0e38):
        for bits in (0, 0x7FFFFFFF, 0xFFFFFFFF):
            assert oracle.e2m1_decode(oracle.e2m1_encode_sr(v, bits)) == 6.0
            assert oracle.e2m1_decode(oracle.e2m1_encode_sr(-v, bits)) == -6.0


def test_sr_sign_symmetry():
    rng = np.random.default_rng(8)
    for v, b in zip(rng.uniform(0.01, 5.9, 500), rng.integers(0, 2 ** 32, 500, dtype=np.uint64)):
        assert oracle.e2m1_encode_sr(-float(v), int(b)) == oracle.e2m1_encode_sr(float(v), int(b)) | 8


def test_quantize_sr_keeps_the_block_scales_and_is_unbiased():
    """The block scales are the round-to-nearest ones; over a uniform grid of 64 values
    of u (the same u for every element in one pass) the mean dequantized tensor is the
    input to within 1/64 of each element's gap.  Elements whose ratio to the block scale
    exceeds 6 (the E4M3 scale rounded down) saturate to 6 on every pass instead."""
    rng = np.random.default_rng(9)
    x = (rng.normal(size=(8, 64)) * np.exp(rng.normal(size=(8, 64)))).astype(np.float32)
    rtn = oracle.quantize(x, oracle.NVFP4, 16)
    acc = np.zeros(x.shape)
    n = 6
    for k in range(1 << n):
        q = oracle.quantize_sr(x, np.full(x.size, _bits_for(k, n), np.uint32))
        assert np.array_equal(q["scales"], rtn["scales"]) and q["g"] == rtn["g"]
        acc += oracle.dequantize(q["codes"], q["scales"], q["g"])
    mean = acc / (1 << n)
    scale = np.repeat(np.vectorize(oracle.e4m3_decode)(rtn["scales"]), 16, axis=1) * float(rtn["g"])
    ratio = np.abs(x) / scale
    sat = ratio >= 6.0
    assert sat.any() and (~sat).sum() > 400
    assert np.allclose(mean[sat], np.sign(x[sat]) * 6.0 * scale[sat], rtol=1e-12, atol=0)
    gap = np.where(ratio < 2, 0.5, np.where(ratio < 4, 1.0, 2.0)) * scale
    assert np.all(np.abs(mean - x)[~sat] <= (gap / (1 << n) + 1e-6 * np.abs(x))[~sat])


def test_quantize_sr_with_zero_bits_rounds_every_magnitude_up():
    x = np.array([[0.1, 0.26, 0.51, 1.1, 2.1, 3.1, 4.1, 5.0] * 2], np.float32)
    q = oracle.quantize_sr(x, np.zeros(16, np.uint32), g_in=np.float32(1.0 / 448))
    d = oracle.dequantize(q["codes"], q["scales"], q["g"])
    # the block amax 5.0 maps near 6, so every other magnitude sits between grid points
    assert np.all(np.abs(d) >= np.abs(x) - 1e-7)


# ---------------------------------------------------------------- epilogue
def test_epilogue_order_scale_bias_activation():
    """Hand-built operands with exact products.  A = 2 * identity (rows 0..3), B's rows
    hold grid values; gA * gB = 2.  Scaling first, then the bias, then ReLU gives
    max(0, 2 * 2 * B[n, m] + bias[n]); adding the bias before the scale, or ReLU before
    the bias, gives other values for these inputs."""
    k = 16
    a_hat = np.zeros((4, k))
    for i in range(4):
        a_hat[i, i] = 2.0 * 2.0  # code 2.0, global scale 2
    b = np.array([[1.0, -0.5, 3.0, 0.0] + [0.0] * 12,
                  [-2.0, 1.5, -6.0, 0.5] + [0.0] * 12,
                  [0.5, 0.5, -1.0, -3.0] + [0.0] * 12])
    b_hat = b * 1.0
    d, _ = oracle.gemm_reference(a_hat, b_hat)
    bias = np.array([1.0, 3.0, -1.5])
    got = oracle.epilogue(d, bias, "relu")
    want = np.array([[max(0.0, 4.0 * b[n, m] + bias[n]) for n in range(3)] for m in range(4)])
    assert np.array_equal(got, want)
    assert np.array_equal(oracle.epilogue(d), d)
    assert np.array_equal(oracle.epilogue(d, bias), d + bias[None, :])


# ---------------------------------------------------------------- E8M0 rounded down
# The MXFP4 scale may also be rounded down to a power of two ("MXFP4 / NVFP4 video
# transcript", MXFP4 passage: 70 must become 64 or 128).  Reading: the largest power of two
# not above the block amax, divided by 4 (the largest power of two on the E2M1 grid), so
# that the block's largest element lands in [4, 8) after scaling.
@pytest.mark.parametrize("amax,code", [
    (6.0, 127), (4.0, 127), (3.99, 126), (8.0, 128), (7.99, 127), (0.75, 124), (1.0, 125),
    (420.0, 133),            # scale 420 / 6 = 70 becomes 64 = 2^6, code 127 + 6
    (0.0, 0), (2.0 ** -126, 0), (2.0 ** -124, 1), (2.0 ** 127, 252)])
def test_e8m0_floor_hand_cases(amax, code):
    assert oracle.e8m0_encode_floor(amax) == code


def test_e8m0_floor_puts_the_block_amax_in_four_to_eight():
    rng = np.random.default_rng(11)
    for a in np.float32(2.0) ** rng.uniform(-100, 100, 2000).astype(np.float32):
        x = oracle.e8m0_decode(oracle.e8m0_encode_floor(float(a)))
        assert 4.0 * x <= float(a) < 8.0 * x, (a, x)


def test_e8m0_floor_never_above_nearest():
    """The rounded-down scale is within one binade of the nearest power of two of amax / 6
    (both are powers of two within a factor of two of amax / 6 or of amax / 4, and
    amax / 4 is 1.5 times amax / 6)."""
    rng = np.random.default_rng(12)
    for a in np.float32(2.0) ** rng.uniform(-60, 60, 2000).astype(np.float32):
        f = oracle.e8m0_encode_floor(float(a))
        n = int(oracle.e8m0_encode(np.array([np.float32(a) / np.float32(6.0)], np.float32))[0])
        assert n - 1 <= f <= n + 1, (a, f, n)


def test_quantize_mxfp4_floor_block_maximum_codes():
    """With the rounded-down scale every non-zero block's largest element encodes as 4 or 6
    (its scaled magnitude is in [4, 8): 4..5 rounds to 4, 5..8 to 6), and the codes equal
    a plain E2M1 encode of x / scale."""
    rng = np.random.default_rng(13)
    x = (rng.standard_normal((8, 256)) * np.float32(2.0) ** rng.integers(-20, 20, (8, 1))).astype(np.float32)
    q = oracle.quantize(x, oracle.MXFP4, 32, e8m0_floor=True)
    codes = np.zeros((8, 256), np.uint8)
    codes[:, 0::2] = q["codes"] & 15
    codes[:, 1::2] = q["codes"] >> 4
    for r in range(8):
        for b in range(8):
            blk = x[r, b * 32:(b + 1) * 32]
            sc = q["scales"][r, b]
            assert sc == oracle.e8m0_encode_floor(float(np.abs(blk).max()))
            scale = np.float32(oracle.e8m0_decode(sc))
            want = oracle.e2m1_encode(blk / scale)      # exact: scale is a power of two
            assert np.array_equal(codes[r, b * 32:(b + 1) * 32], want)
            top = int(codes[r, b * 32 + int(np.abs(blk).argmax())] & 7)
            assert GRID[top] in (4.0, 6.0)


def test_quantize_mxfp4_floor_off_is_the_nearest_quantizer():
    x = np.random.default_rng(14).standard_normal((4, 128)).astype(np.float32)
    a = oracle.quantize(x, oracle.MXFP4, 32)
    b = oracle.quantize(x, oracle.MXFP4, 32, e8m0_floor=False)
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["scales"], b["scales"])


# ---------------------------------------------------------------- epilogue tolerance
def test_epilogue_tolerance_covers_an_fp32_epilogue():
    """An FP32 epilogue of an FP32-accurate product (the product rounded once, the bias
    added in FP32, ReLU) stays inside the bound; the same bound without its bias term
    does not cover large biases."""
    rng = np.random.default_rng(21)
    d = rng.standard_normal((64, 96)) * 3.0
    s = np.abs(d) + 1.0
    bias = (rng.standard_normal(96) * 1000.0).astype(np.float32).astype(np.float64)  # the bias is FP32 data
    t_ref = oracle.epilogue(d, bias, "relu")
    t32 = np.maximum(d.astype(np.float32) + bias.astype(np.float32), np.float32(0)).astype(np.float64)
    tol = oracle.epilogue_tolerance(t_ref, d, s, bias, False)
    assert np.all(np.abs(t32 - t_ref) <= tol)
    no_bias_term = 1e-6 * s + 2.0 ** -24 * np.abs(d)
    assert np.any(np.abs(t32 - t_ref) > no_bias_term)


def test_epilogue_tolerance_reduces_to_the_gemm_tolerance_without_bias():
    rng = np.random.default_rng(22)
    d = rng.standard_normal((8, 16))
    s = np.abs(d) + 0.5
    tol = oracle.epilogue_tolerance(d, d, s, None, True)
    base = oracle.gemm_tolerance(d, s, True)
    # the extra FP32 rounding term is the only difference
    assert np.all(tol >= base) and np.all(tol - base <= 2.0 ** -24 * (np.abs(d) + 1e-6 * s) * (1 + 1e-9) + 1e-300 + 0.5 * oracle.bf16_ulp(np.abs(d) + tol))
