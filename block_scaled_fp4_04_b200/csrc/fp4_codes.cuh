// fp4_codes.cuh -- device encoders and decoders of the three code formats.
//
// E2M1 (the values): 1 sign, 2 exponent bits (bias 1), 1 mantissa bit; magnitudes
//   0, 0.5, 1, 1.5, 2, 3, 4, 6 ("FP4" glossary entry, ultralytics.com; "Rubin FP4 GEMM
//   overview", yfxerp.com, 3.1).  Nearest value, ties to the even mantissa bit,
//   saturating at 6, sign kept on zero.
// E4M3 (NVFP4 block scale, "MXFP4 / NVFP4 video transcript", NVFP4 passage): bias 7,
//   max 448, nearest-even, saturating; used unsigned.
// E8M0 (MXFP4 block scale, same transcript, MXFP4 passage): 2^(c-127); the nearest
//   power of two, an exact midpoint (1.5 * 2^e) rounds up.
#pragma once

#include <cstdint>

namespace fp4 {

// E2M1 by counting the decision thresholds |v| passes.  Ties (0.25, 0.75, 1.25, 1.75,
// 2.5, 3.5, 5) fall on the side of the even code.  Used to validate the hardware
// conversion below and selectable as the production encoder.
__device__ __forceinline__ uint32_t e2m1_code_exact(float v) {
  const float a = fabsf(v);
  uint32_t c = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) + (a >= 3.5f) + (a > 5.0f);
  return c | ((__float_as_uint(v) >> 28) & 8u);
}

// Hardware round-to-nearest-even, saturating conversion of two floats to one byte
// (lo -> low nibble, hi -> high nibble).
__device__ __forceinline__ uint32_t e2m1x2_hw(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "cvt.u32.u8 %0, t;\n\t}\n"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// Pack 8 scaled values into 4 bytes (element 2j in the low nibble of byte j).
template <bool HW>
__device__ __forceinline__ uint32_t pack8(const float (&v)[8]) {
  if constexpr (HW) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}\n"
        : "=r"(out)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return out;
  } else {
    uint32_t out = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) out |= e2m1_code_exact(v[i]) << (4 * i);
    return out;
  }
}

template <bool HW>
__device__ __forceinline__ uint32_t pack4(const float (&v)[4]) {
  if constexpr (HW) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "mov.b32 %0, {b0, b1, b0, b1};\n\t}\n"
        : "=r"(out)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]));
    return out & 0xFFFFu;
  } else {
    uint32_t out = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) out |= e2m1_code_exact(v[i]) << (4 * i);
    return out;
  }
}

// E4M3 of a non-negative float: hardware nearest-even conversion that saturates at
// 448 (inf included).
__device__ __forceinline__ uint32_t e4m3_code(float r) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(0.0f), "f"(r));
  return d & 0xFFu;
}

// Four scaled values to four E4M3 bytes, the first in the low byte: hardware nearest-even
// conversion that saturates at +-448 and keeps the sign of zero.
__device__ __forceinline__ uint32_t pack4_e4m3(float a, float b, float c, float d) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// Exact value of an E4M3 code (< 0x7F): subnormal m * 2^-9, else (1 + m/8) * 2^(e-7).
__device__ __forceinline__ float e4m3_value(uint32_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  if (e == 0) return static_cast<float>(m) * 0.001953125f;
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// E8M0 of a non-negative float, from its bit fields.  Normal v = (1 + f) 2^(e-127):
// code e, plus one when f >= 1/2.  Subnormal v (< 2^-126): code 1 from 1.5 * 2^-127 up,
// else code 0.  Codes clamp at 254 (2^127; inf included).
__device__ __forceinline__ uint32_t e8m0_code(float v) {
  const uint32_t b = __float_as_uint(v);
  const uint32_t e = b >> 23, m = b & 0x7FFFFFu;
  if (e == 0) return m >= 0x600000u ? 1u : 0u;
  if (e >= 254u) return 254u;
  return e + (m >= 0x400000u ? 1u : 0u);
}

// 2^(127 - c) as a float (exact; 2^-127 is a subnormal).
__device__ __forceinline__ float e8m0_inverse(uint32_t c) {
  const int ex = 127 - static_cast<int>(c);
  if (ex >= -126) return __uint_as_float(static_cast<uint32_t>(ex + 127) << 23);
  return __uint_as_float(0x00400000u);
}

__device__ __forceinline__ float e8m0_value(uint32_t c) {
  const int ex = static_cast<int>(c) - 127;
  if (ex >= -126) return __uint_as_float(static_cast<uint32_t>(ex + 127) << 23);
  return __uint_as_float(0x00400000u);
}

__device__ __forceinline__ float e2m1_value(uint32_t code) {
  // magnitude from the bit fields: e = (c >> 1) & 3, m = c & 1
  const uint32_t c = code & 7u, e = c >> 1, m = c & 1u;
  float mag = e == 0 ? 0.5f * static_cast<float>(m) : (1.0f + 0.5f * static_cast<float>(m)) * static_cast<float>(1u << (e - 1));
  return (code & 8u) ? -mag : mag;
}

// NVFP4 block scale for a block with largest magnitude amax_b under global scale g:
// sb = E4M3((amax_b / 6) / g) (two IEEE divisions, in that order); returns the element
// multiplier 1 / (dec(sb) * g) (IEEE reciprocal), or 0 when that denominator is 0.
__device__ __forceinline__ float nvfp4_block_scale(float amax_b, float g, uint32_t& sb) {
  const float t = __fdiv_rn(amax_b, 6.0f);
  sb = e4m3_code(__fdiv_rn(t, g));
  const float denom = __fmul_rn(e4m3_value(sb), g);
  return denom == 0.0f ? 0.0f : __frcp_rn(denom);
}

}  // namespace fp4
