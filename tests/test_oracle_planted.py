"""Planted mistakes (CPU only): each case edits one plausible error into a private copy
of the oracle -- its C source, rebuilt under a temporary directory, or one of its
Python steps -- and checks that at least one pin test fails on that copy.  A pin set
that let such a mistake through would not pin the oracle.  The committed oracle is
never modified; every case runs against its own build.
"""
import ctypes
import subprocess

import numpy as np
import pytest

import oracle
import test_oracle_formats as tf
import test_oracle_gemm as tg
import test_oracle_quantize as tq

with open(oracle._SRC) as _f:
    SRC = _f.read()

WORKED = [lambda i=i: tq.test_worked_blocks(i) for i in range(4)]

# (name, text in fp4_oracle.c, the mistaken text, pins expected to notice)
C_MUTATIONS = [
    ("e2m1 ties go to the smaller magnitude",
     "double d = fabs(a - e2m1_magnitude(c));\n        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {",
     "double d = fabs(a - e2m1_magnitude(c));\n        if (d < best_d) {",
     [lambda: tf.test_e2m1_ties_to_even(0.75, 2), tf.test_e2m1_matches_threshold_formulation]),
    ("e2m1 drops the sign of a zero code",
     "return (uint8_t)(best | sign);",
     "return (uint8_t)(best ? (best | sign) : 0);",
     [tf.test_e2m1_round_trip_all_codes, lambda: tq.test_sign_symmetry(oracle.NVFP4, 16)]),
    ("e2m1 without saturation",
     "if (a >= 6.0) return (uint8_t)(7 | sign);",
     "",
     [tf.test_e2m1_matches_threshold_formulation]),
    ("e4m3 exponent bias 8",
     "else v = (1.0 + m / 8.0) * ldexp(1.0, e - 7);",
     "else v = (1.0 + m / 8.0) * ldexp(1.0, e - 8);",
     [tf.test_e4m3_decode_matches_torch, lambda: tq.test_worked_blocks(0)]),
    ("e4m3 mantissa of 2 bits",
     "else v = (1.0 + m / 8.0) * ldexp(1.0, e - 7);",
     "else v = (1.0 + m / 4.0) * ldexp(1.0, e - 7);",
     [tf.test_e4m3_decode_matches_torch]),
    ("e8m0 midpoint goes down",
     "if (d <= best_d) {  /* ascending c",
     "if (d < best_d) {  /* ascending c",
     [tf.test_e8m0_midpoint_goes_up, tf.test_e8m0_encode_matches_torch]),
    ("global scale maps amax to 6 * 256",
     "if (amax_t > 0.0f) return amax_t / 2688.0f;",
     "if (amax_t > 0.0f) return amax_t / 1536.0f;",
     [tq.test_global_scale]),
    ("tensor amax without the absolute value",
     "float a = fabsf(v);\n        if (a > m) m = a;",
     "float a = v;\n        if (a > m) m = a;",
     [lambda: tq.test_sign_symmetry(oracle.NVFP4, 16), tq.test_global_scale]),
    ("block scale maps the block amax to 4",
     "float t = amax_b / 6.0f;",
     "float t = amax_b / 4.0f;",
     WORKED),
    ("nvfp4 scale applied twice (no reciprocal)",
     "float inv = 1.0f / denom;",
     "float inv = denom;",
     WORKED + [tq.test_error_bound_unsaturated]),
    ("mxfp4 divides by the inverse scale",
     "codes[i] = orc_e2m1_encode(xs[i] * f);",
     "codes[i] = orc_e2m1_encode(xs[i] / f);",
     [tq.test_grid_valued_inputs_round_trip] + WORKED),
    ("nibble order swapped",
     "out[j] = (uint8_t)((codes[2 * j] & 15) | ((codes[2 * j + 1] & 15) << 4));",
     "out[j] = (uint8_t)((codes[2 * j + 1] & 15) | ((codes[2 * j] & 15) << 4));",
     WORKED),
    ("1-D block amax over 15 elements",
     "xs[i] = load_elem(x, r * cols + b * 16 + i, dtype);\n                if (fabsf(xs[i]) > amax_b)",
     "xs[i] = load_elem(x, r * cols + b * 16 + i, dtype);\n                if (i < 15 && fabsf(xs[i]) > amax_b)",
     WORKED + [tq.test_no_element_beyond_the_block_range]),
    ("W^T codes read with swapped strides",
     "for (int64_t r = 0; r < rows; ++r) colbuf[r] = full[r * cols + c];",
     "for (int64_t r = 0; r < rows; ++r) colbuf[r] = full[c * rows + r];",
     [tq.test_2d_transpose_identity]),
    ("scale atom with the row fields exchanged",
     "return atom * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4);",
     "return atom * 512 + (r % 32) * 4 + ((r % 128) / 32) * 16 + (c % 4);",
     [tq.test_swizzle_offsets_by_hand, lambda: tq.test_swizzle_is_a_bijection_with_zero_pads(128, 4)]),
    ("scale columns not padded to a multiple of 4",
     "int64_t cpad = (scols + 3) / 4 * 4;\n    int64_t atom",
     "int64_t cpad = scols;\n    int64_t atom",
     [tq.test_swizzle_offsets_by_hand]),
    ("dequantize forgets the global scale",
     "double s = fmt == 0 ? orc_e4m3_decode(sb) * (double)g : orc_e8m0_decode(sb);",
     "double s = fmt == 0 ? orc_e4m3_decode(sb) : orc_e8m0_decode(sb);",
     [tq.test_format_true_scales_near_printed_shape, tq.test_error_bound_unsaturated]),
    ("dequantize reads the high nibble for even elements",
     "uint8_t code = (k & 1) ? (byte >> 4) : (byte & 15);",
     "uint8_t code = (k & 1) ? (byte & 15) : (byte >> 4);",
     [tq.test_grid_valued_inputs_round_trip, tq.test_format_true_scales_near_printed_shape]),
    ("glossary experiment keeps the scale unclamped at amax/5",
     "float scale = amax_b / 6.0f;",
     "float scale = amax_b / 5.0f;",
     [tq.test_glossary_block_size_experiment_exact]),
]


def _variant(tmp_path, old: str, new: str) -> ctypes.CDLL:
    assert SRC.count(old) == 1, f"planted text not found exactly once: {old!r}"
    c = tmp_path / "variant.c"
    c.write_text(SRC.replace(old, new))
    so = tmp_path / "libvariant.so"
    subprocess.check_call(["gcc", *oracle.CFLAGS, "-o", str(so), str(c), "-lm"])
    return oracle.configure(ctypes.CDLL(str(so)))


def _caught(pins) -> int:
    n = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            n += 1
    return n


@pytest.mark.parametrize("name,old,new,pins", C_MUTATIONS, ids=[m[0] for m in C_MUTATIONS])
def test_planted_c_mistake_is_caught(tmp_path, monkeypatch, name, old, new, pins):
    monkeypatch.setattr(oracle, "_lib", _variant(tmp_path, old, new))
    assert _caught(pins) > 0, f"no pin noticed: {name}"


def test_unmodified_copy_passes_the_same_pins(tmp_path, monkeypatch):
    """Control: the copy machinery itself does not make pins fail."""
    monkeypatch.setattr(oracle, "_lib", _variant(tmp_path, "float t = amax_b / 6.0f;", "float t = amax_b / 6.0f;"))
    pins = {id(p): p for m in C_MUTATIONS for p in m[3]}
    assert _caught(pins.values()) == 0


# Python-level steps of the GEMM reference and its tolerance
def _gemm_without_abs(a_hat, b_hat, rows=None):
    a = a_hat if rows is None else a_hat[np.asarray(rows)]
    return a @ b_hat.T, a @ b_hat.T


def _gemm_with_transposed_b(a_hat, b_hat, rows=None):
    a = a_hat if rows is None else a_hat[np.asarray(rows)]
    bt = b_hat.reshape(b_hat.shape[1], b_hat.shape[0]).T  # a row-major/column-major slip
    return a @ bt.T, np.abs(a) @ np.abs(bt).T


def _ulp_one_bit_short(v):
    a = np.abs(np.asarray(v, dtype=np.float64))
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.ldexp(1.0, (np.maximum(e, -126.0) - 8).astype(np.int64))


@pytest.mark.parametrize("attr,wrong,pins", [
    ("gemm_reference", _gemm_without_abs, [lambda: tg.test_gemm_reference_vs_exact_rationals(3, 5, 64, oracle.NVFP4),
                                           tg.test_gemm_rank_one_integer_sums]),
    ("gemm_reference", _gemm_with_transposed_b,
     [lambda: tg.test_gemm_reference_vs_exact_rationals(3, 5, 64, oracle.NVFP4), tg.test_gemm_identity_operand]),
    ("bf16_ulp", _ulp_one_bit_short, [tg.test_tolerance_rule]),
])
def test_planted_python_mistake_is_caught(monkeypatch, attr, wrong, pins):
    monkeypatch.setattr(oracle, attr, wrong)
    assert _caught(pins) > 0
