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
import test_oracle_mxfp8 as tm
import test_oracle_next as tn
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
    # stochastic rounding and the Hadamard transform (the steps after the hot path)
    ("stochastic rounding goes up when u equals the fraction",
     "return (uint8_t)((u < frac ? lo + 1 : lo) | sign);",
     "return (uint8_t)((u <= frac ? lo + 1 : lo) | sign);",
     [lambda: tn.test_sr_expectation_over_a_uniform_grid_of_u(0.75),
      lambda: tn.test_sr_expectation_over_a_uniform_grid_of_u(1.25)]),
    ("stochastic rounding goes up with probability 1 - fraction",
     "return (uint8_t)((u < frac ? lo + 1 : lo) | sign);",
     "return (uint8_t)((u >= frac ? lo + 1 : lo) | sign);",
     [lambda: tn.test_sr_expectation_over_a_uniform_grid_of_u(0.3), tn.test_quantize_sr_keeps_the_block_scales_and_is_unbiased]),
    ("stochastic quantize rounds to nearest",
     "rbits != NULL ? orc_e2m1_encode_sr(xs[i] * inv, rbits[i])",
     "rbits != NULL ? orc_e2m1_encode(xs[i] * inv)",
     [tn.test_quantize_sr_keeps_the_block_scales_and_is_unbiased, tn.test_quantize_sr_with_zero_bits_rounds_every_magnitude_up]),
    ("Hadamard butterfly skips the first stage",
     "for (int h = 1; h < 16; h *= 2)",
     "for (int h = 2; h < 16; h *= 2)",
     [lambda: tn.test_rht_spreads_a_spike_evenly(0x0000, 5), tn.test_rht_fp32_within_the_butterfly_bound]),
    ("Hadamard transform without the factor 1/4",
     "out[r * cols + b * 16 + i] = v[i] * 0.25f;",
     "out[r * cols + b * 16 + i] = v[i];",
     [lambda: tn.test_rht_spreads_a_spike_evenly(0x0000, 0), tn.test_rht_fp32_within_the_butterfly_bound]),
    ("Hadamard signs read from the high bit down",
     "if ((signs >> i) & 1u) v[i] = -v[i];",
     "if ((signs >> (15 - i)) & 1u) v[i] = -v[i];",
     [lambda: tn.test_rht_spreads_a_spike_evenly(0x00FF, 0), tn.test_rht_fp32_within_the_butterfly_bound]),
    ("E8M0 rounded down from amax / 6 instead of amax / 4",
     "if (4.0 * e8m0_value(c) <= a) best = c;",
     "if (6.0 * e8m0_value(c) <= a) best = c;",
     [lambda: tn.test_e8m0_floor_hand_cases(4.0, 127), tn.test_e8m0_floor_puts_the_block_amax_in_four_to_eight]),
    ("E8M0 rounded down one binade too far",
     "if (4.0 * e8m0_value(c) <= a) best = c;",
     "if (8.0 * e8m0_value(c) <= a) best = c;",
     [lambda: tn.test_e8m0_floor_hand_cases(6.0, 127), tn.test_quantize_mxfp4_floor_block_maximum_codes]),
    ("MXFP4 quantizer ignores the rounding mode",
     "uint8_t sb = floor_mode ? orc_e8m0_encode_floor(amax_b) : orc_e8m0_encode(amax_b / 6.0f);",
     "uint8_t sb = orc_e8m0_encode(amax_b / 6.0f);",
     [tn.test_quantize_mxfp4_floor_block_maximum_codes]),
    ("MXFP8 scale maps the block amax to 6 instead of 448",
     "uint8_t sb = orc_e8m0_encode(amax_b / 448.0f);",
     "uint8_t sb = orc_e8m0_encode(amax_b / 6.0f);",
     [lambda: tm.test_mxfp8_worked_blocks(0), lambda: tm.test_mxfp8_scale_is_the_nearest_power_of_two_of_amax_over_448(448.0, 127)]),
    ("MXFP8 drops the element sign",
     "codes[i] = (uint8_t)((signbit(v) ? 0x80 : 0) | orc_e4m3_encode(fabsf(v)));",
     "codes[i] = (uint8_t)orc_e4m3_encode(fabsf(v));",
     [tm.test_mxfp8_sign_symmetry, tm.test_mxfp8_every_e4m3_code_round_trips]),
    ("MXFP8 dequantize forgets the block scale",
     "out[r * cols + k] = orc_e4m3_decode(codes[r * cols + k]) * orc_e8m0_decode(scales_rm[r * (cols / 32) + k / 32]);",
     "out[r * cols + k] = orc_e4m3_decode(codes[r * cols + k]);",
     [tm.test_mxfp8_error_bound]),
    ("Hadamard butterfly difference reversed",
     "v[j + h] = p - q;",
     "v[j + h] = q - p;",
     [lambda: tn.test_rht_spreads_a_spike_evenly(0x0000, 5), tn.test_rht_fp32_within_the_butterfly_bound]),
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


# Python-level steps of the Hadamard transform's definition and of the epilogue
_H = oracle.hadamard16()


def _hadamard_sequency_order():
    """The rows sorted by their number of sign changes (Walsh order), a common slip."""
    changes = (np.diff(_H, axis=1) != 0).sum(1)
    return _H[np.argsort(changes, kind="stable")]


def _rht_norm_sixteenth(x, signs):
    return oracle_rht_reference(x, signs) / 4.0


def _rht_signs_on_rows(x, signs):
    x = np.asarray(x, dtype=np.float64)
    rows, cols = x.shape
    s = np.array([-1.0 if (signs >> i) & 1 else 1.0 for i in range(16)])
    q = s[:, None] * _H / 4.0
    return (x.reshape(rows, cols // 16, 16) @ q.T).reshape(rows, cols)


def _epilogue_relu_before_bias(d, bias=None, act="none"):
    out = np.asarray(d, dtype=np.float64)
    if act == "relu":
        out = np.maximum(out, 0.0)
    if bias is not None:
        out = out + np.asarray(bias, dtype=np.float64)[None, :]
    return out


oracle_rht_reference = oracle.rht16_reference


@pytest.mark.parametrize("attr,wrong,pins", [
    ("hadamard16", _hadamard_sequency_order, [tn.test_hadamard16_matches_scipy]),
    ("rht16_reference", _rht_norm_sixteenth, [tn.test_rht_keeps_block_norms, lambda: tn.test_rht_is_orthonormal(0x1234)]),
    ("rht16_reference", _rht_signs_on_rows, [lambda: tn.test_rht_spreads_a_spike_evenly(0x00FF, 0)]),
    ("epilogue", _epilogue_relu_before_bias, [tn.test_epilogue_order_scale_bias_activation]),
])
def test_planted_python_mistake_in_the_next_steps_is_caught(monkeypatch, attr, wrong, pins):
    monkeypatch.setattr(oracle, attr, wrong)
    assert _caught(pins) > 0

