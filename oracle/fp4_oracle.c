/*
 * fp4_oracle.c -- plain, slow CPU definition of block-scaled FP4 (NVFP4 / MXFP4).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the oracle that the CUDA path is checked
 * against.  Only the tests, the smoke check and the benchmark's CPU-baseline leg may
 * load it.  It shares no code, header, table or constant generator with the CUDA
 * library, and it must never be used as a fallback for it.
 *
 * Every encoder here is written as a brute-force search over the format's code
 * table ("pick the representable value nearest to v"), not as bit tricks, so that
 * a reader can check it against the definitions by eye.  Arithmetic is IEEE-754
 * single precision where the method fixes FP32 (block scales, the global scale,
 * the element ratio) and double precision for distances and dequantized values.
 * Build with -O2 -ffp-contract=off (no FMA contraction) and without -ffast-math.
 *
 * Sources (the pages this follows; each function names the one it uses):
 *  [P1] "Rubin FP4 GEMM overview" (yfxerp.com news 178243): 3.1 why FP4 needs scale
 *       factors; 3.2 the GEMM pipeline; 4.2 where the scale factors go; 5.2 nibble
 *       packing and alignment.
 *  [P2] "MXFP4 / NVFP4 video transcript" (prism.simon-ai.net article 7890): the MXFP4
 *       and NVFP4 passages (32-block power-of-two scale; 16-block E4M3 scale plus an
 *       FP32 tensor scale) and the training-recipe passage on 16x16 weight blocks.
 *  [P4] "FP4" glossary entry (ultralytics.com/ru/glossary/fp4): the E2M1 value set,
 *       section "How FP4 works" (block scale = block amax / 6; MXFP4 and NVFP4
 *       definitions) and its block-size experiment.
 *
 * Readings where the pages are silent (each is listed with its reason in the
 * design notes):
 *  - E2M1 ties go to the even mantissa (round-to-nearest-even); values at or beyond
 *    6 saturate to 6; the sign is kept, also on a zero code (0x8 = -0).
 *  - E4M3 is the OCP "FN" variant: bias 7, max 448, no inf, 0x7F = NaN (never
 *    produced), subnormals kept; encode is nearest-even, saturating at 448.
 *  - E8M0 is 2^(c-127), c = 0..254 (255 = NaN, never produced); encode picks the
 *    nearest power of two in the linear domain, an exact midpoint goes up.
 *  - NVFP4 global scale g = amax_t / (6*448), or 1 when amax_t == 0.
 *  - NVFP4 block scale sb = E4M3((amax_b / 6) / g) (two FP32 divisions in that
 *    order); element ratio x * (1 / (dec(sb) * g)) in FP32 (one reciprocal per
 *    block, one multiply per element); a zero denominator gives zero codes, and a
 *    zero element gives a zero code even if the reciprocal overflowed.
 *  - Packing: two codes per byte, the even element in the low nibble.
 *  - Scale-factor layout: 128x4 atoms of 512 bytes (see orc_swizzle_scales).
 *  - Stochastic rounding ([P2] training-recipe passage, its fourth part): only the
 *    element rounding changes; the block scale is the deterministic one.  u is a
 *    24-bit uniform in [0, 1) taken from caller-supplied random bits.
 *  - Random Hadamard transform ([P2] training-recipe passage, its third part; [P4]
 *    section "Inference and training in FP4"): 16-element blocks along the rows,
 *    y = (1/4) H16 diag(s) x with the Sylvester H16 and one caller-supplied sign
 *    vector s; in FP32 the four butterfly stages of the fast Walsh-Hadamard
 *    transform, in order.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>

#define ORC_OK 0
#define ORC_ERR_NONFINITE 5

/* input dtypes */
#define ORC_F32 0
#define ORC_BF16 1

/* ------------------------------------------------------------------------- */
/* Input loading                                                             */
/* ------------------------------------------------------------------------- */

/* bf16 is the upper half of an fp32 bit pattern; widening is exact. */
static float bf16_to_f32(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static float load_elem(const void* x, int64_t i, int dtype) {
    if (dtype == ORC_BF16) return bf16_to_f32(((const uint16_t*)x)[i]);
    return ((const float*)x)[i];
}

/* ------------------------------------------------------------------------- */
/* E2M1 -- 1 sign, 2 exponent, 1 mantissa bit, bias 1.  [P4] lists the only     */
/* values: 0, +-0.5, +-1, +-1.5, +-2, +-3, +-4, +-6; [P1] 3.1 gives the bit split.  */
/* ------------------------------------------------------------------------- */

/* Magnitude of code c (0..7) from the bit fields: e = c >> 1, m = c & 1.
 * e == 0 is subnormal: m * 0.5; otherwise (1 + m/2) * 2^(e-1). */
static double e2m1_magnitude_from_bits(int c) {
    int e = c >> 1, m = c & 1;
    if (e == 0) return 0.5 * m;
    return (1.0 + 0.5 * m) * ldexp(1.0, e - 1);
}

/* The same eight magnitudes, tabulated once (so that sweeps over many values do not
 * recompute them). */
static double e2m1_table[8];
static int e2m1_table_ready = 0;

static double e2m1_magnitude(int c) {
    if (!e2m1_table_ready) {
        for (int i = 0; i < 8; ++i) e2m1_table[i] = e2m1_magnitude_from_bits(i);
        e2m1_table_ready = 1;
    }
    return e2m1_table[c];
}

double orc_e2m1_decode(uint8_t code) {
    double mag = e2m1_magnitude(code & 7);
    return (code & 8) ? -mag : mag;
}

/* Nearest of the 8 magnitudes to |v|; an exact tie goes to the code whose mantissa
 * bit is 0 (even).  |v| beyond 6 has 6 as its nearest value (saturation).  The sign
 * bit copies v's sign, including for a zero result.  v must not be NaN. */
uint8_t orc_e2m1_encode(float v) {
    double a = fabs((double)v);
    int best = 0;
    double best_d = INFINITY;
    uint8_t sign = signbit(v) ? 8 : 0;
    if (a >= 6.0) return (uint8_t)(7 | sign);  /* saturate (also keeps huge |v| out of the
                                                   distance search, where all distances
                                                   would round to the same double) */
    for (int c = 0; c < 8; ++c) {
        double d = fabs(a - e2m1_magnitude(c));
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_d = d;
        }
    }
    return (uint8_t)(best | sign);
}

/* Stochastic rounding ([P2] training-recipe passage, fourth part: 0.3 between the
 * representable 0 and 1 becomes 1 with probability 0.3 and 0 otherwise, so that the
 * expected value is the value).  |v| between the neighbouring magnitudes lo < |v| < hi
 * goes to hi iff u < (|v| - lo) / (hi - lo), with u = (bits >> 8) * 2^-24 in [0, 1);
 * magnitudes on the grid are kept, magnitudes at or beyond 6 saturate to 6.  Both the
 * difference and the division are exact in FP32 (lo <= |v| < hi <= 2 lo or lo = 0,
 * and the gap is a power of two), so the decision does not depend on the precision.
 * The sign bit copies v's sign. */
uint8_t orc_e2m1_encode_sr(float v, uint32_t bits) {
    uint8_t sign = signbit(v) ? 8 : 0;
    float a = fabsf(v);
    if (a >= 6.0f) return (uint8_t)(7 | sign);
    int lo = 0;  /* the largest magnitude not above a */
    for (int c = 1; c < 8; ++c)
        if (e2m1_magnitude(c) <= (double)a) lo = c;
    float lov = (float)e2m1_magnitude(lo);
    if (a == lov) return (uint8_t)(lo | sign);
    float gap = (float)e2m1_magnitude(lo + 1) - lov;
    float frac = (a - lov) / gap;
    float u = (float)(bits >> 8) * 0x1p-24f;
    return (uint8_t)((u < frac ? lo + 1 : lo) | sign);
}

/* ------------------------------------------------------------------------- */
/* E4M3 scale byte -- 4 exponent bits, 3 mantissa bits ([P2] NVFP4 passage).     */
/* Unsigned use: sign bit always 0.  Bias 7, 0x7F NaN, max 0x7E = 448.          */
/* ------------------------------------------------------------------------- */

double orc_e4m3_decode(uint8_t code) {
    int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);               /* m/8 * 2^(1-7) */
    else v = (1.0 + m / 8.0) * ldexp(1.0, e - 7);
    return s ? -v : v;
}

/* Values of the 127 finite non-negative E4M3 codes, tabulated once from the decoder. */
static double e4m3_table[127];
static int e4m3_table_ready = 0;

static double e4m3_value(int c) {
    if (!e4m3_table_ready) {
        for (int i = 0; i < 127; ++i) e4m3_table[i] = orc_e4m3_decode((uint8_t)i);
        e4m3_table_ready = 1;
    }
    return e4m3_table[c];
}

/* v >= 0 (may be +inf).  Nearest finite non-negative code; tie -> even mantissa;
 * above 448 the nearest finite code is 448 (saturation). */
uint8_t orc_e4m3_encode(float v) {
    double a = (double)v;
    int best = 0;
    double best_d = INFINITY;
    if (a >= 448.0) return 0x7E;  /* saturate; see orc_e2m1_encode */
    for (int c = 0; c <= 0x7E; ++c) {
        double d = fabs(a - e4m3_value(c));
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_d = d;
        }
    }
    return (uint8_t)best;
}

/* ------------------------------------------------------------------------- */
/* E8M0 scale byte -- exponent only, a power of two ([P1] 3.1; the [P2] MXFP4  */
/* passage notes that a non-power-of-two ideal scale has to be rounded to one   */
/* of its neighbouring powers of two).  Bias 127, 0xFF NaN.                     */
/* ------------------------------------------------------------------------- */

double orc_e8m0_decode(uint8_t code) {
    if (code == 255) return NAN;
    return ldexp(1.0, (int)code - 127);
}

/* Values of the 255 finite E8M0 codes, tabulated once from the decoder. */
static double e8m0_table[255];
static int e8m0_table_ready = 0;

static double e8m0_value(int c) {
    if (!e8m0_table_ready) {
        for (int i = 0; i < 255; ++i) e8m0_table[i] = orc_e8m0_decode((uint8_t)i);
        e8m0_table_ready = 1;
    }
    return e8m0_table[c];
}

/* Builds the three code tables before rows are processed on several threads (each
 * table is filled on first use; filling it once up front keeps the threads from doing
 * it concurrently).  Rows are independent, so running them on OpenMP threads changes
 * no arithmetic. */
static void tables_ready(void) {
    (void)e2m1_magnitude(0);
    (void)e4m3_value(0);
    (void)e8m0_value(0);
}

/* v >= 0.  Nearest power of two 2^(c-127), c in 0..254, in the linear domain; an
 * exact midpoint (1.5 * 2^e) goes to the larger power. */
uint8_t orc_e8m0_encode(float v) {
    double a = (double)v;
    int best = 0;
    double best_d = INFINITY;
    for (int c = 0; c <= 254; ++c) {
        double d = isinf(a) ? (c == 254 ? 0.0 : INFINITY) : fabs(a - e8m0_value(c));
        if (d <= best_d) {  /* ascending c: an equal distance replaces with the larger power */
            best = c;
            best_d = d;
        }
    }
    return (uint8_t)best;
}

/* ------------------------------------------------------------------------- */
/* Tensor amax and the NVFP4 global scale ([P2] NVFP4 passage: an FP32 tensor   */
/* scale handles the global range; g maps the tensor amax to 6 * 448).          */
/* ------------------------------------------------------------------------- */

/* max |x_i|; returns ORC_ERR_NONFINITE if any element is inf or NaN. */
int orc_amax(const void* x, int64_t n, int dtype, float* amax_out) {
    float m = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float v = load_elem(x, i, dtype);
        if (!isfinite(v)) return ORC_ERR_NONFINITE;
        float a = fabsf(v);
        if (a > m) m = a;
    }
    *amax_out = m;
    return ORC_OK;
}

float orc_global_scale(float amax_t) {
    if (amax_t > 0.0f) return amax_t / 2688.0f; /* 2688 = 6 * 448 */
    return 1.0f;
}

/* ------------------------------------------------------------------------- */
/* One NVFP4 block: its 16 (or 256) values share one E4M3 scale under the      */
/* tensor's FP32 scale g ([P2] NVFP4 passage; [P4] "How FP4 works": the block's   */
/* largest magnitude maps to 6).                                                */
/* ------------------------------------------------------------------------- */

/* Encodes n values xs[] with block amax amax_b and global scale g; returns the
 * scale byte and writes the n 4-bit codes (rounded to nearest, or stochastically
 * with one 32-bit random word per element when rbits is not NULL). */
static uint8_t nvfp4_encode_block(const float* xs, int n, float amax_b, float g, const uint32_t* rbits,
                                  uint8_t* codes) {
    float t = amax_b / 6.0f;
    float r = t / g;
    uint8_t sb = orc_e4m3_encode(r);
    float denom = (float)orc_e4m3_decode(sb) * g;   /* exact decode, FP32 multiply */
    if (denom == 0.0f) {
        for (int i = 0; i < n; ++i) codes[i] = signbit(xs[i]) ? 8 : 0;
        return sb;
    }
    float inv = 1.0f / denom;
    /* A zero element encodes as a zero code even when 1/denom overflowed to inf
     * (a denominator below 2^-128): the ratio x / denom of a zero is zero. */
    for (int i = 0; i < n; ++i)
        codes[i] = xs[i] == 0.0f   ? (signbit(xs[i]) ? 8 : 0)
                   : rbits != NULL ? orc_e2m1_encode_sr(xs[i] * inv, rbits[i])
                                   : orc_e2m1_encode(xs[i] * inv);
    return sb;
}

/* The other way to reach a power of two ([P2] MXFP4 passage: a scale of 70 must become
 * 64 or 128, so one may also round down): take the largest power of two not above the
 * block amax and divide it by 4, the largest power of two on the E2M1 grid.  The block's
 * largest element then lands in [4, 8) after scaling (values from 6 up saturate).  Brute
 * force: the largest code c with 4 * 2^(c-127) <= amax_b; code 0 if none (and for a
 * zero block). */
uint8_t orc_e8m0_encode_floor(float amax_b) {
    double a = (double)amax_b;
    int best = 0;
    for (int c = 0; c <= 254; ++c)
        if (4.0 * e8m0_value(c) <= a) best = c;
    return (uint8_t)best;
}

/* One MXFP4 block of 32 values, E8M0 scale ([P2] MXFP4 passage; [P4]): the nearest power
 * of two of amax_b / 6, or (floor != 0) the rounded-down scale above. */
static uint8_t mxfp4_encode_block(const float* xs, int n, float amax_b, int floor_mode, uint8_t* codes) {
    uint8_t sb = floor_mode ? orc_e8m0_encode_floor(amax_b) : orc_e8m0_encode(amax_b / 6.0f);
    /* multiplying by 2^(127 - sb) is exact in FP32 (the factor is representable and
     * the scaling only moves the exponent), so it equals dividing by the scale */
    float f = (float)ldexp(1.0, 127 - (int)sb);
    if (amax_b == 0.0f) {
        for (int i = 0; i < n; ++i) codes[i] = signbit(xs[i]) ? 8 : 0;
        return sb;
    }
    for (int i = 0; i < n; ++i) codes[i] = orc_e2m1_encode(xs[i] * f);
    return sb;
}

/* Packing, [P1] 5.2: two codes per byte; here element 2j in the low nibble. */
static void pack_row(const uint8_t* codes, int64_t n, uint8_t* out) {
    for (int64_t j = 0; j < n / 2; ++j)
        out[j] = (uint8_t)((codes[2 * j] & 15) | ((codes[2 * j + 1] & 15) << 4));
}

/* ------------------------------------------------------------------------- */
/* 1-D quantize of a row-major [rows, cols] tensor, blocks along cols.          */
/* codes: [rows, cols/2] packed.  scales_rm: plain row-major [rows, cols/blk]. */
/* g_in: caller's global scale (NVFP4), or NULL to compute amax first.         */
/* ------------------------------------------------------------------------- */

/* rbits: NULL (round to nearest) or one random word per element, row-major
 * [rows, cols], for stochastic rounding. */
int orc_quantize_nvfp4_1d_r(const void* x, int64_t rows, int64_t cols, int dtype, const float* g_in,
                            const uint32_t* rbits, uint8_t* codes, uint8_t* scales_rm, float* g_out) {
    /* a non-finite element is an error whether or not the caller supplies g */
    float amax_t, g;
    if (orc_amax(x, rows * cols, dtype, &amax_t) != ORC_OK) return ORC_ERR_NONFINITE;
    g = g_in ? *g_in : orc_global_scale(amax_t);
    if (g_out) *g_out = g;
    tables_ready();
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        float xs[16];
        uint8_t cb[16];
        uint8_t* row_codes = (uint8_t*)malloc((size_t)cols);
        for (int64_t b = 0; b < cols / 16; ++b) {
            float amax_b = 0.0f;
            for (int i = 0; i < 16; ++i) {
                xs[i] = load_elem(x, r * cols + b * 16 + i, dtype);
                if (fabsf(xs[i]) > amax_b) amax_b = fabsf(xs[i]);
            }
            scales_rm[r * (cols / 16) + b] =
                nvfp4_encode_block(xs, 16, amax_b, g, rbits ? rbits + r * cols + b * 16 : NULL, cb);
            memcpy(row_codes + b * 16, cb, 16);
        }
        pack_row(row_codes, cols, codes + r * (cols / 2));
        free(row_codes);
    }
    return ORC_OK;
}

int orc_quantize_nvfp4_1d(const void* x, int64_t rows, int64_t cols, int dtype,
                          const float* g_in, uint8_t* codes, uint8_t* scales_rm, float* g_out) {
    return orc_quantize_nvfp4_1d_r(x, rows, cols, dtype, g_in, NULL, codes, scales_rm, g_out);
}

int orc_quantize_mxfp4_1d_r(const void* x, int64_t rows, int64_t cols, int dtype, int floor_mode,
                            uint8_t* codes, uint8_t* scales_rm);

int orc_quantize_mxfp4_1d(const void* x, int64_t rows, int64_t cols, int dtype,
                          uint8_t* codes, uint8_t* scales_rm) {
    return orc_quantize_mxfp4_1d_r(x, rows, cols, dtype, 0, codes, scales_rm);
}

/* floor_mode: 0 = nearest power of two of amax_b / 6; 1 = rounded down (see
 * orc_e8m0_encode_floor). */
int orc_quantize_mxfp4_1d_r(const void* x, int64_t rows, int64_t cols, int dtype, int floor_mode,
                            uint8_t* codes, uint8_t* scales_rm) {
    /* a non-finite element anywhere is an error (no encoding exists for it) */
    for (int64_t i = 0; i < rows * cols; ++i)
        if (!isfinite(load_elem(x, i, dtype))) return ORC_ERR_NONFINITE;
    tables_ready();
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        float xs[32];
        uint8_t cb[32];
        uint8_t* row_codes = (uint8_t*)malloc((size_t)cols);
        for (int64_t b = 0; b < cols / 32; ++b) {
            float amax_b = 0.0f;
            for (int i = 0; i < 32; ++i) {
                xs[i] = load_elem(x, r * cols + b * 32 + i, dtype);
                if (fabsf(xs[i]) > amax_b) amax_b = fabsf(xs[i]);
            }
            scales_rm[r * (cols / 32) + b] = mxfp4_encode_block(xs, 32, amax_b, floor_mode, cb);
            memcpy(row_codes + b * 32, cb, 32);
        }
        pack_row(row_codes, cols, codes + r * (cols / 2));
        free(row_codes);
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* MXFP8: E4M3 elements with an E8M0 scale per 32 ([P1] 3.1 names MXFP8 beside     */
/* MXFP4 in the OCP microscaling family, pure-exponent scales; [P1] 3.4 wants an     */
/* FP8 operand opposite an FP4 one).  The pages fix no scale rule for it; the       */
/* reading follows the MXFP4 one: the nearest power of two of amax_b / 448, 448     */
/* being E4M3's largest value as 6 is E2M1's.  Elements: sign in bit 7, magnitude   */
/* by the E4M3 encoder above (nearest, ties to the even mantissa, saturating).      */
/* ------------------------------------------------------------------------- */

static uint8_t mxfp8_encode_block(const float* xs, int n, float amax_b, uint8_t* codes) {
    uint8_t sb = orc_e8m0_encode(amax_b / 448.0f);
    float f = (float)ldexp(1.0, 127 - (int)sb);  /* exact scaling, as for MXFP4 */
    for (int i = 0; i < n; ++i) {
        float v = xs[i] * f;
        codes[i] = (uint8_t)((signbit(v) ? 0x80 : 0) | orc_e4m3_encode(fabsf(v)));
    }
    return sb;
}

/* [rows, cols] -> codes [rows, cols] (one byte per element), scales_rm [rows, cols / 32]. */
int orc_quantize_mxfp8_1d(const void* x, int64_t rows, int64_t cols, int dtype, uint8_t* codes,
                          uint8_t* scales_rm) {
    for (int64_t i = 0; i < rows * cols; ++i)
        if (!isfinite(load_elem(x, i, dtype))) return ORC_ERR_NONFINITE;
    tables_ready();
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        float xs[32];
        for (int64_t b = 0; b < cols / 32; ++b) {
            float amax_b = 0.0f;
            for (int i = 0; i < 32; ++i) {
                xs[i] = load_elem(x, r * cols + b * 32 + i, dtype);
                if (fabsf(xs[i]) > amax_b) amax_b = fabsf(xs[i]);
            }
            scales_rm[r * (cols / 32) + b] = mxfp8_encode_block(xs, 32, amax_b, codes + r * cols + b * 32);
        }
    }
    return ORC_OK;
}

/* x_hat = E4M3(code) * 2^(scale - 127), in FP64. */
void orc_dequantize_mxfp8(const uint8_t* codes, const uint8_t* scales_rm, int64_t rows, int64_t cols,
                          double* out) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < cols; ++k)
            out[r * cols + k] = orc_e4m3_decode(codes[r * cols + k]) * orc_e8m0_decode(scales_rm[r * (cols / 32) + k / 32]);
}

/* ------------------------------------------------------------------------- */
/* 2-D NVFP4 weight quantize ([P2] training-recipe passage: one scale per 16x16 */
/* weight patch, so the forward W and the backward W^T share one quantization). */
/* Emits W's codes and 1x16-expanded scales, and W^T's codes and scales.        */
/* rows and cols are multiples of 16; cols, rows even.                         */
/* ------------------------------------------------------------------------- */

int orc_quantize_nvfp4_2d(const void* x, int64_t rows, int64_t cols, int dtype, const float* g_in,
                          uint8_t* codes, uint8_t* scales_rm, uint8_t* codesT, uint8_t* scalesT_rm,
                          float* g_out) {
    /* a non-finite element is an error whether or not the caller supplies g */
    float amax_t, g;
    if (orc_amax(x, rows * cols, dtype, &amax_t) != ORC_OK) return ORC_ERR_NONFINITE;
    g = g_in ? *g_in : orc_global_scale(amax_t);
    if (g_out) *g_out = g;
    uint8_t* full = (uint8_t*)malloc((size_t)(rows * cols)); /* unpacked codes of W */
    tables_ready();
#pragma omp parallel for schedule(static)
    for (int64_t tr = 0; tr < rows / 16; ++tr) {
        float xs[256];
        uint8_t cb[256];
        for (int64_t tc = 0; tc < cols / 16; ++tc) {
            float amax_b = 0.0f;
            for (int i = 0; i < 16; ++i)
                for (int j = 0; j < 16; ++j) {
                    float v = load_elem(x, (tr * 16 + i) * cols + tc * 16 + j, dtype);
                    xs[i * 16 + j] = v;
                    if (fabsf(v) > amax_b) amax_b = fabsf(v);
                }
            uint8_t sb = nvfp4_encode_block(xs, 256, amax_b, g, NULL, cb);
            for (int i = 0; i < 16; ++i) {
                for (int j = 0; j < 16; ++j) full[(tr * 16 + i) * cols + tc * 16 + j] = cb[i * 16 + j];
                scales_rm[(tr * 16 + i) * (cols / 16) + tc] = sb;       /* row of W    */
            }
            for (int j = 0; j < 16; ++j)
                scalesT_rm[(tc * 16 + j) * (rows / 16) + tr] = sb;      /* row of W^T  */
        }
    }
    for (int64_t r = 0; r < rows; ++r) pack_row(full + r * cols, cols, codes + r * (cols / 2));
#pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < cols; ++c) {
        uint8_t* colbuf = (uint8_t*)malloc((size_t)rows);
        for (int64_t r = 0; r < rows; ++r) colbuf[r] = full[r * cols + c];
        pack_row(colbuf, rows, codesT + c * (rows / 2));
        free(colbuf);
    }
    free(full);
    return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* Scale-factor layout.  [P1] 4.2 and 4.4 only require that the scale layout   */
/* be tile-loadable with the matrix.  Reading: 128-row x 4-column atoms of 512   */
/* bytes, row-blocks outermost; inside an atom entry (r, c) sits at             */
/* (r % 32) * 16 + (r / 32) * 4 + c.  Rows pad to 128, columns to 4, pads 0.      */
/* ------------------------------------------------------------------------- */

int64_t orc_scales_bytes(int64_t rows, int64_t scols) {
    int64_t rp = (rows + 127) / 128 * 128, cp = (scols + 3) / 4 * 4;
    return rp * cp;
}

int64_t orc_swizzle_offset(int64_t r, int64_t c, int64_t scols) {
    int64_t cpad = (scols + 3) / 4 * 4;
    int64_t atom = (r / 128) * (cpad / 4) + c / 4;
    return atom * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4);
}

void orc_swizzle_scales(const uint8_t* rm, int64_t rows, int64_t scols, uint8_t* out) {
    memset(out, 0, (size_t)orc_scales_bytes(rows, scols));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < scols; ++c) out[orc_swizzle_offset(r, c, scols)] = rm[r * scols + c];
}

void orc_unswizzle_scales(const uint8_t* sw, int64_t rows, int64_t scols, uint8_t* rm) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < scols; ++c) rm[r * scols + c] = sw[orc_swizzle_offset(r, c, scols)];
}

/* Grouped (MoE) activations: rows [offsets[e], offsets[e+1]) belong to group e.
 * Each group's scale rows start on a fresh 128-row block, so that every 128-row
 * tile of one group reads whole atoms.  Group e's first row-block is
 * sum_{e' < e} ceil(rows_e' / 128). */
int64_t orc_scales_bytes_grouped(const int32_t* offsets, int num_groups, int64_t scols) {
    int64_t rb = 0;
    for (int e = 0; e < num_groups; ++e) rb += ((int64_t)offsets[e + 1] - offsets[e] + 127) / 128;
    return rb * 128 * ((scols + 3) / 4 * 4);
}

void orc_swizzle_scales_grouped(const uint8_t* rm, const int32_t* offsets, int num_groups, int64_t scols,
                                uint8_t* out) {
    memset(out, 0, (size_t)orc_scales_bytes_grouped(offsets, num_groups, scols));
    int64_t rb = 0, cpad = (scols + 3) / 4 * 4;
    for (int e = 0; e < num_groups; ++e) {
        int64_t n = (int64_t)offsets[e + 1] - offsets[e];
        uint8_t* base = out + rb * 128 * cpad;
        for (int64_t lr = 0; lr < n; ++lr)
            for (int64_t c = 0; c < scols; ++c)
                base[orc_swizzle_offset(lr, c, scols)] = rm[(offsets[e] + lr) * scols + c];
        rb += (n + 127) / 128;
    }
}

/* ------------------------------------------------------------------------- */
/* Dequantize ([P4] experiment: value = grid[code] * sign * scale; NVFP4 also   */
/* multiplies the tensor scale, [P2]).  Output in double.                        */
/* fmt: 0 = NVFP4 (E4M3 scales, block 16), 1 = MXFP4 (E8M0 scales, block 32).   */
/* scales_rm row-major [rows, cols/block].                                      */
/* ------------------------------------------------------------------------- */

void orc_dequantize(const uint8_t* codes, const uint8_t* scales_rm, float g, int64_t rows, int64_t cols,
                    int fmt, double* out) {
    int blk = fmt == 0 ? 16 : 32;
    tables_ready();
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < cols; ++k) {
            uint8_t byte = codes[r * (cols / 2) + k / 2];
            uint8_t code = (k & 1) ? (byte >> 4) : (byte & 15);
            uint8_t sb = scales_rm[r * (cols / blk) + k / blk];
            double s = fmt == 0 ? orc_e4m3_decode(sb) * (double)g : orc_e8m0_decode(sb);
            out[r * cols + k] = orc_e2m1_decode(code) * s;
        }
}

/* ------------------------------------------------------------------------- */
/* [P4] block-size experiment: the block scale is the unrounded FP32 amax / 6   */
/* and each value goes to the nearest E2M1 grid point of |x| / scale.           */
/* Writes the dequantized FP32 values.  n is a multiple of block.               */
/* ------------------------------------------------------------------------- */

void orc_fake_quant_fp32_scale(const float* x, int64_t n, int64_t block, float* deq) {
    for (int64_t b = 0; b < n / block; ++b) {
        float amax_b = 0.0f;
        for (int64_t i = 0; i < block; ++i)
            if (fabsf(x[b * block + i]) > amax_b) amax_b = fabsf(x[b * block + i]);
        float scale = amax_b / 6.0f;
        for (int64_t i = 0; i < block; ++i) {
            float v = x[b * block + i];
            float ratio = fabsf(v) / scale;
            float mag = (float)e2m1_magnitude(orc_e2m1_encode(ratio) & 7);
            float sgn = v > 0.0f ? 1.0f : (v < 0.0f ? -1.0f : 0.0f);
            deq[b * block + i] = mag * sgn * scale;
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Random Hadamard transform ([P2] training-recipe passage, third part: the values */
/* of a block are mixed so that an outlier no longer sets the block scale alone;   */
/* the vector's magnitude is unchanged, and so is a dot product when both operands */
/* are transformed alike).  Each 16-element block b of a row becomes               */
/* (1/4) H16 diag(s) b, s_i = -1 where bit i of `signs` is set, H16 the Sylvester  */
/* Hadamard matrix.  FP32, in the order of the fast Walsh-Hadamard transform: the  */
/* signs, then butterfly stages with half-widths 1, 2, 4, 8 (pairs j, j + h become */
/* their sum and difference), then the exact factor 1/4.  cols % 16 == 0.          */
/* ------------------------------------------------------------------------- */

int orc_rht16(const void* x, int64_t rows, int64_t cols, int dtype, uint32_t signs, float* out) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < cols / 16; ++b) {
            float v[16];
            for (int i = 0; i < 16; ++i) {
                v[i] = load_elem(x, r * cols + b * 16 + i, dtype);
                if (!isfinite(v[i])) return ORC_ERR_NONFINITE;
                if ((signs >> i) & 1u) v[i] = -v[i];
            }
            for (int h = 1; h < 16; h *= 2)
                for (int i = 0; i < 16; i += 2 * h)
                    for (int j = i; j < i + h; ++j) {
                        float p = v[j], q = v[j + h];
                        v[j] = p + q;
                        v[j + h] = p - q;
                    }
            for (int i = 0; i < 16; ++i) out[r * cols + b * 16 + i] = v[i] * 0.25f;
        }
    return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* Array forms of the scalar encoders, so that a caller can sweep many values    */
/* in one call.  Each is a plain loop over the scalar definition above.          */
/* ------------------------------------------------------------------------- */

void orc_e2m1_encode_array(const float* v, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m1_encode(v[i]);
}

void orc_e4m3_encode_array(const float* v, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(v[i]);
}

void orc_e8m0_encode_array(const float* v, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e8m0_encode(v[i]);
}

/* Exhaustive-sweep helper: for the n float32 bit patterns start, start+1, ... compares
 * codes[i] with orc_e2m1_encode of that pattern and returns the number of mismatches.
 * NaN patterns (no E2M1 encoding is defined for them) are skipped.  Runs the
 * independent elements on all OpenMP threads. */
int64_t orc_e2m1_count_mismatch(uint64_t start, int64_t n, const uint8_t* codes) {
    int64_t bad = 0;
    (void)e2m1_magnitude(0); /* build the tables before the threads start */
#pragma omp parallel for reduction(+ : bad) schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        uint32_t bits = (uint32_t)(start + (uint64_t)i);
        float v;
        memcpy(&v, &bits, 4);
        if (isnan(v)) continue;
        if (orc_e2m1_encode(v) != codes[i]) bad += 1;
    }
    return bad;
}

int orc_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
