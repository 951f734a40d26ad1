"""Pins for the oracle's quantizers, scale layout and dequantization (CPU only)."""
import os

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLD, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


# ------------------------------------------------------------ printed experiment
def test_glossary_block_size_experiment_exact():
    """The glossary page prints 0.7238 / 0.0901 / 0.0747 for blocks 4096 / 32 / 16."""
    x = workloads.glossary_experiment_input().numpy()
    for block, mae in _rows("glossary_block_size_mae.txt"):
        deq = oracle.fake_quant_fp32_scale(x, int(block))
        assert f"{np.abs(deq - x).mean():.4f}" == mae


def test_format_true_scales_near_printed_shape():
    """With scales stored in their formats the error keeps the page's shape:
    one tensor-wide scale ~0.72, 32-blocks ~0.09, 16-blocks ~0.075."""
    x = workloads.glossary_experiment_input().numpy()
    q16 = oracle.quantize(x, oracle.NVFP4, 16)
    e16 = np.abs(oracle.dequantize(q16["codes"], q16["scales"], q16["g"]).ravel() - x).mean()
    q32 = oracle.quantize(x, oracle.MXFP4, 32)
    e32 = np.abs(oracle.dequantize(q32["codes"], q32["scales"], 1.0, oracle.MXFP4).ravel() - x).mean()
    assert abs(e16 - 0.0747) < 0.01 and abs(e32 - 0.0901) < 0.025 and e16 < e32 < 0.7238


# ------------------------------------------------------------ hand-worked blocks
def _parse_block(parts):
    fmt = parts[0]
    kv = dict(p.split("=") for p in parts[1:])
    vals = np.array([float(v) for v in kv["values"].split(",")], np.float32)
    return fmt, float(kv["g"]), vals, int(kv["scale"], 16), bytes.fromhex(kv["codes"])


@pytest.mark.parametrize("idx", range(4))
def test_worked_blocks(idx):
    fmt, g, vals, scale, codes = _parse_block(_rows("worked_blocks.txt")[idx])
    if fmt == "nvfp4":
        q = oracle.quantize(vals.reshape(1, -1), oracle.NVFP4, 16, g_in=g)
    else:
        q = oracle.quantize(vals.reshape(1, -1), oracle.MXFP4, 32)
    assert q["scales"].ravel().tolist() == [scale]
    assert q["codes"].tobytes() == codes


# ------------------------------------------------------------ invariants
def _rand(rows, cols, seed, outliers=True):
    x = workloads.normal((rows, cols), 1.0, seed)
    if outliers:
        workloads.with_outliers(x, seed)
    return x.numpy()


@pytest.mark.parametrize("fmt,block", [(oracle.NVFP4, 16), (oracle.MXFP4, 32), (oracle.NVFP4, 256)])
def test_sign_symmetry(fmt, block):
    x = _rand(32, 64, 1)
    a, b = oracle.quantize(x, fmt, block), oracle.quantize(-x, fmt, block)
    assert np.array_equal(a["codes"] ^ 0x88, b["codes"])
    assert np.array_equal(a["scales"], b["scales"])


@pytest.mark.parametrize("k", [-20, -3, 1, 7, 30])
def test_power_of_two_invariance(k):
    x = _rand(16, 128, 2)
    a = oracle.quantize(x, oracle.NVFP4, 16)
    b = oracle.quantize((x * np.float32(2.0 ** k)).astype(np.float32), oracle.NVFP4, 16)
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["scales"], b["scales"])
    assert b["g"] == np.float32(a["g"] * np.float32(2.0 ** k))
    m1 = oracle.quantize(x, oracle.MXFP4, 32)
    m2 = oracle.quantize((x * np.float32(2.0 ** k)).astype(np.float32), oracle.MXFP4, 32)
    assert np.array_equal(m1["codes"], m2["codes"])
    assert np.array_equal(m1["scales"].astype(int) + k, m2["scales"].astype(int))


def test_permutation_within_block_permutes_codes():
    x = _rand(4, 64, 3)
    perm = np.random.default_rng(0).permutation(16)
    xp = x.reshape(4, 4, 16)[:, :, perm].reshape(4, 64)
    a, b = oracle.quantize(x, oracle.NVFP4, 16), oracle.quantize(xp, oracle.NVFP4, 16)

    def unpack(c):
        return np.stack([c & 15, c >> 4], -1).reshape(c.shape[0], -1)

    assert np.array_equal(unpack(a["codes"]).reshape(4, 4, 16)[:, :, perm].reshape(4, 64), unpack(b["codes"]))
    assert np.array_equal(a["scales"], b["scales"])


def test_error_bound_unsaturated():
    """|x - x_hat| <= half the grid gap at x's magnitude, times the block scale."""
    x = _rand(64, 256, 4)
    q = oracle.quantize(x, oracle.NVFP4, 16)
    xh = oracle.dequantize(q["codes"], q["scales"], q["g"])
    s = np.repeat(np.array([[oracle.e4m3_decode(c) for c in row] for row in q["scales"]]), 16, 1) * float(q["g"])
    r = np.abs(x) / np.where(s > 0, s, 1)
    gap = np.select([r < 2, r < 4], [0.5, 1.0], 2.0)
    ok = (r <= 6) & (s > 0)
    # the FP32 ratio is the product by a rounded reciprocal: allow a few ulps of slack
    assert np.all(np.abs(x - xh)[ok] <= (0.5 * gap * s * (1 + 1e-6))[ok])


def test_no_element_beyond_the_block_range():
    """The block scale covers the block's largest magnitude: with a normal E4M3 scale
    below the 448 clamp, sb = E4M3(amax_b / (6 g)) is within half an E4M3 ulp (2^-4
    relative) of its argument, so every |x| / (dec(sb) g) <= 6 (1 + 2^-4).  For MXFP4
    the power of two rounds amax_b / 6 by at most a factor 1.5: |x| / dec(sb) < 9."""
    x = _rand(64, 512, 12)
    q = oracle.quantize(x, oracle.NVFP4, 16)
    s = np.repeat(np.array([[oracle.e4m3_decode(c) for c in row] for row in q["scales"]]), 16, 1)
    normal = np.repeat((q["scales"] >= 8) & (q["scales"] < 0x7E), 16, 1)
    r = np.abs(x) / (s * float(q["g"]))
    assert normal.mean() > 0.9 and np.all(r[normal] <= 6 * (1 + 2.0 ** -4))
    m = oracle.quantize(x, oracle.MXFP4, 32)
    sm = np.repeat(np.array([[oracle.e8m0_decode(c) for c in row] for row in m["scales"]]), 32, 1)
    assert np.all(np.abs(x) / sm < 9.0)


def test_global_scale():
    assert oracle.global_scale(2688.0) == 1.0
    assert oracle.global_scale(0.0) == 1.0
    x = _rand(8, 32, 5)
    q = oracle.quantize(x, oracle.NVFP4, 16)
    assert q["g"] == np.float32(np.float32(np.abs(x).max()) / np.float32(2688.0))
    # the largest scale byte is within rounding of 448 (the E4M3 maximum)
    assert 416 <= max(oracle.e4m3_decode(c) for c in q["scales"].ravel()) <= 448


def test_all_zero_and_tiny_blocks():
    x = np.zeros((2, 32), np.float32)
    x[1, 16:] = -0.0
    q = oracle.quantize(x, oracle.NVFP4, 16)
    assert q["g"] == 1.0 and not q["scales"].any()
    assert q["codes"][0].tolist() == [0] * 16 and q["codes"][1, 8:].tolist() == [0x88] * 8
    # one block far below the tensor amax: its scale rounds to 0 -> zero codes
    y = np.full((1, 32), 1e-3, np.float32)
    y[0, 0] = 1e4
    q = oracle.quantize(y, oracle.NVFP4, 16)
    assert q["scales"][0, 1] == 0 and not q["codes"][0, 8:].any()


def test_nonfinite_rejected():
    for bad in (np.nan, np.inf, -np.inf):
        x = np.ones((1, 32), np.float32)
        x[0, 5] = bad
        for fmt, block in ((oracle.NVFP4, 16), (oracle.MXFP4, 32), (oracle.NVFP4, 256)):
            if block == 256:
                x2 = np.ones((16, 32), np.float32)
                x2[3, 3] = bad
                with pytest.raises(oracle.NonFiniteInput):
                    oracle.quantize(x2, fmt, block)
                continue
            with pytest.raises(oracle.NonFiniteInput):
                oracle.quantize(x, fmt, block)
        with pytest.raises(oracle.NonFiniteInput):
            oracle.quantize(x, oracle.NVFP4, 16, g_in=1.0)


def test_bf16_input_equals_widened_fp32():
    x = workloads.with_outliers(workloads.normal((16, 64), 1.0, 6), 6).to(torch.bfloat16)
    a = oracle.quantize(workloads.bf16_bits(x), oracle.NVFP4, 16)
    b = oracle.quantize(x.float().numpy(), oracle.NVFP4, 16)
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["scales"], b["scales"])
    assert a["g"] == b["g"]


def test_grid_valued_inputs_round_trip():
    """Values already on the grid times a representable scale dequantize exactly."""
    rng = np.random.default_rng(9)
    grid = np.array([oracle.e2m1_decode(c) for c in range(16)])
    codes = rng.integers(0, 16, (8, 32))
    codes[:, ::16] = 7  # each block holds a 6 so its amax maps to scale 1.0 exactly
    x = (grid[codes] * 4.0).astype(np.float32)  # MXFP4: scale 4 -> code 129
    q = oracle.quantize(x, oracle.MXFP4, 32)
    assert np.all(q["scales"] == 129)
    assert np.array_equal(oracle.dequantize(q["codes"], q["scales"], 1.0, oracle.MXFP4), x.astype(np.float64))


# ------------------------------------------------------------ 2-D weights
def test_2d_transpose_identity():
    w = _rand(64, 96, 7)
    q = oracle.quantize(w, oracle.NVFP4, 256)
    qt = oracle.quantize(np.ascontiguousarray(w.T), oracle.NVFP4, 256)
    assert np.array_equal(q["codesT"], qt["codes"]) and np.array_equal(q["scalesT"], qt["scales"])
    assert np.array_equal(q["codes"], qt["codesT"]) and np.array_equal(q["scales"], qt["scalesT"])
    # every 16x16 patch shares one scale
    s = q["scales"].reshape(4, 16, 6)
    assert np.all(s == s[:, :1, :])


def test_2d_equals_1d_on_constant_patch_amax():
    """If every 1x16 block of a 16x16 patch has the patch's amax, 2-D and 1-D agree."""
    w = _rand(32, 64, 8, outliers=False)
    w[:, ::16] = 5.0
    a = oracle.quantize(w, oracle.NVFP4, 256)
    b = oracle.quantize(w, oracle.NVFP4, 16)
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["scales"], b["scales"])


# ------------------------------------------------------------ scale layout
def test_swizzle_offsets_by_hand():
    # inside a 128x4 atom: (r % 32) * 16 + (r / 32) * 4 + c
    assert oracle.swizzle_offset(0, 0, 8) == 0
    assert oracle.swizzle_offset(1, 0, 8) == 16
    assert oracle.swizzle_offset(32, 0, 8) == 4
    assert oracle.swizzle_offset(0, 3, 8) == 3
    assert oracle.swizzle_offset(97, 2, 8) == 1 * 16 + 3 * 4 + 2
    assert oracle.swizzle_offset(0, 4, 8) == 512          # next atom along columns
    assert oracle.swizzle_offset(128, 0, 8) == 2 * 512    # next row-block: after 2 atoms
    assert oracle.swizzle_offset(128, 0, 6) == 2 * 512    # 6 scale columns pad to 8
    assert oracle.scales_bytes(130, 6) == 256 * 8


@pytest.mark.parametrize("rows,scols", [(1, 1), (128, 4), (130, 6), (300, 90), (17, 512)])
def test_swizzle_is_a_bijection_with_zero_pads(rows, scols):
    rng = np.random.default_rng(rows * 1000 + scols)
    rm = rng.integers(1, 256, (rows, scols)).astype(np.uint8)
    sw = oracle.swizzle_scales(rm)
    assert sw.size == oracle.scales_bytes(rows, scols)
    assert np.count_nonzero(sw) == rows * scols          # pads are zero
    assert np.array_equal(oracle.unswizzle_scales(sw, rows, scols), rm)
    offs = {oracle.swizzle_offset(r, c, scols) for r in range(rows) for c in range(scols)}
    assert len(offs) == rows * scols


def test_grouped_swizzle():
    offsets = np.array([0, 3, 3, 200, 201], np.int32)   # an empty group and a ragged tail
    rm = np.random.default_rng(0).integers(1, 256, (201, 6)).astype(np.uint8)
    sw = oracle.swizzle_scales_grouped(rm, offsets)
    # row-blocks: ceil(3/128)=1, 0, ceil(197/128)=2, 1 -> 4 blocks of 128 x 8
    assert sw.size == 4 * 128 * 8
    for e, (lo, hi) in enumerate(zip(offsets[:-1], offsets[1:])):
        rb = sum((offsets[i + 1] - offsets[i] + 127) // 128 for i in range(e))
        base = sw[rb * 128 * 8:]
        if hi > lo:
            got = oracle.unswizzle_scales(base[:((hi - lo + 127) // 128) * 128 * 8], hi - lo, 6)
            assert np.array_equal(got, rm[lo:hi])
