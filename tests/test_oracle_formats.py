"""Pins for the oracle's code tables and scalar encoders (CPU only).

Each test checks the oracle against something other than itself: the value grid
printed on the "FP4" glossary page (ultralytics.com), torch's own FP8 conversions
(a library routine), the tie rule spelled out per midpoint, or a second, threshold
formulation of the E2M1 rounding.
"""
import os

import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _golden_rows(name):
    with open(os.path.join(GOLD, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


# ------------------------------------------------------------------ E2M1
def test_e2m1_grid_matches_glossary():
    grid = [float(v) for v in _golden_rows("e2m1_grid.txt")[0]]
    assert [oracle.e2m1_decode(c) for c in range(8)] == grid
    for c in range(8):
        neg = oracle.e2m1_decode(c | 8)
        assert neg == -grid[c] and np.signbit(neg)
    distinct = {oracle.e2m1_decode(c) for c in range(16)}
    assert len(distinct) == 15  # +0 and -0 compare equal: 15 distinct values, no inf/NaN


def test_e2m1_round_trip_all_codes():
    vals = np.array([oracle.e2m1_decode(c) for c in range(16)], np.float32)
    assert oracle.e2m1_encode(vals).tolist() == list(range(16))


# Ties between neighbouring grid points go to the even mantissa bit (RNE).
TIES = [(0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6)]


@pytest.mark.parametrize("v,code", TIES)
def test_e2m1_ties_to_even(v, code):
    assert oracle.e2m1_encode(np.float32(v)).item() == code
    assert oracle.e2m1_encode(np.float32(-v)).item() == code | 8


def _e2m1_by_thresholds(v: np.ndarray) -> np.ndarray:
    """A second formulation: count the decision thresholds |v| passes.  Ties listed
    above fall on the lower side for the first threshold of each pair ('>') or the
    upper side ('>=') exactly as the table says."""
    a = np.abs(v.astype(np.float64))
    c = ((a > 0.25).astype(np.int32) + (a >= 0.75) + (a > 1.25) + (a >= 1.75)
         + (a > 2.5) + (a >= 3.5) + (a > 5.0))
    return (c | np.where(np.signbit(v), 8, 0)).astype(np.uint8)


def test_e2m1_matches_threshold_formulation():
    rng = np.random.default_rng(123)
    parts = [rng.standard_normal(200_000).astype(np.float32) * s for s in (0.3, 1, 3, 10)]
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 0.0], np.float32)
    for m in mids:  # every midpoint and its fp32 neighbours, both signs
        nb = [m]
        lo = hi = np.float32(m)
        for _ in range(4):
            lo = np.nextafter(lo, np.float32(-np.inf))
            hi = np.nextafter(hi, np.float32(np.inf))
            nb += [lo, hi]
        parts.append(np.array(nb, np.float32))
        parts.append(-np.array(nb, np.float32))
    parts.append(np.array([np.inf, -np.inf, 1e30, -1e30, 6.0, 7.0, 1e-40, -1e-40], np.float32))
    v = np.concatenate(parts)
    assert np.array_equal(oracle.e2m1_encode(v), _e2m1_by_thresholds(v))


def test_e2m1_monotone():
    v = np.linspace(-8, 8, 100_001, dtype=np.float32)
    mags = np.array([oracle.e2m1_decode(c) for c in oracle.e2m1_encode(v)])
    assert np.all(np.diff(mags) >= 0)


# ------------------------------------------------------------------ E4M3
def test_e4m3_decode_matches_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    ours = np.array([oracle.e4m3_decode(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert oracle.e4m3_decode(0x7E) == 448.0
    assert nan[0x7F] and nan[0xFF]


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(7)
    codes = np.arange(0, 0x7F)
    vals = np.array([oracle.e4m3_decode(c) for c in codes])
    mids = (vals[:-1] + vals[1:]) / 2                     # exact in fp32
    parts = [vals, mids, np.nextafter(mids.astype(np.float32), 0), np.nextafter(mids.astype(np.float32), 1e9),
             rng.uniform(0, 464, 200_000), np.exp2(rng.uniform(-14, 8.8, 200_000))]
    v = np.concatenate([p.astype(np.float32) for p in parts])
    v = v[(v >= 0) & (v <= 464)]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(v), ref)


def test_e4m3_saturates():
    v = np.array([464.0001, 500, 1e9, 1e30, 3.4e38, np.inf], np.float32)
    assert oracle.e4m3_encode(v).tolist() == [0x7E] * 6
    # below half the smallest subnormal (2^-10) -> 0; the midpoint itself ties to 0
    assert oracle.e4m3_encode(np.array([2.0 ** -10, 2.0 ** -11, 0.0], np.float32)).tolist() == [0, 0, 0]
    assert oracle.e4m3_encode(np.float32(2.0 ** -10 * 1.01)).item() == 1


def test_e4m3_round_trip_all_finite():
    vals = np.array([oracle.e4m3_decode(c) for c in range(0x7F)], np.float32)
    assert oracle.e4m3_encode(vals).tolist() == list(range(0x7F))


# ------------------------------------------------------------------ E8M0
def test_e8m0_decode_matches_torch():
    codes = torch.arange(255, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e8m0fnu).float().numpy().astype(np.float64)
    ours = np.array([oracle.e8m0_decode(c) for c in range(255)])
    # torch widens to fp32, where 2^-127 is a subnormal: still exact
    assert np.array_equal(ours, ref)
    assert np.isnan(oracle.e8m0_decode(255))


def test_e8m0_encode_matches_torch():
    rng = np.random.default_rng(11)
    e = rng.integers(-126, 127, 100_000)
    f = rng.uniform(1.0, 2.0, 100_000)
    v = np.ldexp(f, e).astype(np.float32)
    ties = np.ldexp(1.5, np.arange(-126, 126)).astype(np.float32)
    v = np.concatenate([v, ties, np.ldexp(1.0, np.arange(-126, 127)).astype(np.float32)])
    ref = torch.from_numpy(v).to(torch.float8_e8m0fnu).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e8m0_encode(v), ref)


def test_e8m0_midpoint_goes_up():
    # a scale that should be 96 = 1.5 * 64 becomes 128; 70 becomes 64
    assert oracle.e8m0_encode(np.float32(96.0)).item() == 127 + 7
    assert oracle.e8m0_encode(np.float32(70.0)).item() == 127 + 6
    assert oracle.e8m0_encode(np.float32(0.0)).item() == 0
