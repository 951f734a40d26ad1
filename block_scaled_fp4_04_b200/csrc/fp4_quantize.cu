// fp4_quantize.cu -- memory-bound kernels: tensor amax, 1-D and 16x16 block
// quantization (NVFP4 / MXFP4), dequantization and the encoder check kernel.
//
// Method ("FP4" glossary entry, ultralytics.com, "How FP4 works"; "MXFP4 / NVFP4 video
// transcript", prism.simon-ai.net, MXFP4 / NVFP4 / training-recipe passages):
//   NVFP4: g = amax_t / (6*448) (1 if amax_t == 0); per 16 values sb = E4M3((amax_b/6)/g),
//          codes = E2M1(x * (1 / (dec(sb) * g))).
//   MXFP4: per 32 values sb = E8M0(amax_b / 6), codes = E2M1(x * 2^(127 - sb)).
//   2-D:   NVFP4 with amax_b over a 16x16 patch; codes for W and W^T.
// Every FP32 step is an explicit IEEE round-to-nearest operation (__fdiv_rn, __fmul_rn,
// __frcp_rn) so that codes and scales are bit-identical to the CPU definition.
//
// Scale bytes are written straight into the 128x4-atom layout the tensor cores read:
// entry (r, c) at ((r/128)*(Cpad/4) + c/4)*512 + (r%32)*16 + ((r%128)/32)*4 + c%4.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "fp4_codes.cuh"
#include "fp4_internal.h"
#include "fp4_ptx.cuh"

namespace fp4 {

// ------------------------------------------------------------------ loads
template <typename T>
struct Elem;
template <>
struct Elem<float> {
  static constexpr int kPerChunk = 4;  // 16-byte chunk
  __device__ __forceinline__ static void unpack(const uint4& u, float* v) {
    v[0] = __uint_as_float(u.x);
    v[1] = __uint_as_float(u.y);
    v[2] = __uint_as_float(u.z);
    v[3] = __uint_as_float(u.w);
  }
};
template <>
struct Elem<__nv_bfloat16> {
  static constexpr int kPerChunk = 8;
  __device__ __forceinline__ static void unpack(const uint4& u, float* v) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
};

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint32_t abs_bits(float v) { return __float_as_uint(v) & 0x7FFFFFFFu; }

// ------------------------------------------------------------------ quantizer variants
// Variants of the 1-D quantizer (the steps around the hot path, "MXFP4 / NVFP4 video
// transcript", training-recipe and MXFP4 passages):
//   kQuantPlain    the method as stated;
//   kQuantMxFloor  MXFP4 with the block scale rounded down to a power of two;
//   kQuantSR       NVFP4 with stochastic rounding of the elements (caller's random words);
//   kQuantRHT      a 16-point random Hadamard transform of every 16-element block first.

// Hadamard transform of the 16-element blocks that lanes hold EPC elements of: this
// lane holds elements [j0, j0 + EPC) of its block (j0 = (lane % (16 / EPC)) * EPC), its
// partners hold the rest.  Signs first (bit j of `signs` negates element j), then the
// butterfly stages of half-width 1, 2, 4, 8 in that order (pair (j, j + h) becomes
// (sum, difference)), then the exact factor 1/4: the same FP32 operations, in the same
// order, as the definition.  Stages narrower than EPC stay in the thread; wider ones pair
// lanes by a shuffle.  All lanes of the warp take part.
template <int EPC>
__device__ __forceinline__ void rht16_lanes(float (&v)[EPC], uint32_t signs, int j0) {
#pragma unroll
  for (int i = 0; i < EPC; ++i)
    if ((signs >> (j0 + i)) & 1u) v[i] = -v[i];
#pragma unroll
  for (int h = 1; h < EPC; h <<= 1)
#pragma unroll
    for (int i = 0; i < EPC; ++i)
      if ((i & h) == 0) {
        const float a = v[i], b = v[i + h];
        v[i] = __fadd_rn(a, b);
        v[i + h] = __fsub_rn(a, b);
      }
#pragma unroll
  for (int h = EPC; h < 16; h <<= 1) {
    const int lane_bit = h / EPC;
    const bool upper = ((j0 / EPC) & lane_bit) != 0;  // this lane holds the j + h half
#pragma unroll
    for (int i = 0; i < EPC; ++i) {
      const float o = __shfl_xor_sync(0xFFFFFFFFu, v[i], lane_bit);
      v[i] = upper ? __fsub_rn(o, v[i]) : __fadd_rn(v[i], o);
    }
  }
#pragma unroll
  for (int i = 0; i < EPC; ++i) v[i] = __fmul_rn(v[i], 0.25f);
}

// Stochastic E2M1 rounding of a scaled value s with one 32-bit random word: |s| between
// grid neighbours lo < |s| < hi goes up iff u < (|s| - lo) / (hi - lo), u = (bits >> 8)
// * 2^-24.  The difference is exact (lo <= |s| < 2 lo, or lo = 0) and the gap a power of
// two, so the fraction is exact in FP32.  Grid values stay, |s| >= 6 saturates; the sign
// bit copies s's sign.
__device__ __forceinline__ uint32_t e2m1_code_sr(float s, uint32_t bits) {
  const uint32_t sb = __float_as_uint(s), ab = sb & 0x7FFFFFFFu;
  const uint32_t sign = (sb >> 28) & 8u;
  if (ab > 0x7F800000u) return sign;        // NaN: code 0 (the status word reports it)
  if (ab >= 0x40C00000u) return 7u | sign;  // |s| >= 6 saturates
  const uint32_t n = bits >> 8;             // u = n * 2^-24
  const bool ge1 = ab >= 0x3F800000u;
  // [1, 6): the lower neighbour's code is 2 + 2 (exponent - 127) + the top mantissa bit, and
  // the fraction toward the upper one is the 22 mantissa bits below that bit, times 2^-22;
  // [0.5, 1): the lower neighbour is 0.5 and the fraction the 23 mantissa bits, times 2^-23
  uint32_t lo = ge1 ? (ab >> 22) - 252u : 1u;
  bool up = n < (ge1 ? (ab & 0x3FFFFFu) << 2 : (ab & 0x7FFFFFu) << 1);
  if (ab < 0x3F000000u) {  // [0, 0.5): lower neighbour 0, fraction 2 |s|
    lo = 0u;
    up = __fmul_rn(__uint2float_rn(n), 5.9604644775390625e-08f) < __fmul_rn(__uint_as_float(ab), 2.0f);
  }
  return (lo + (up ? 1u : 0u)) | sign;
}

// E8M0 scale rounded down: 2^(floor(log2 amax_b) - 2), i.e. the exponent field less 2,
// clamped to [0, 254] (subnormal and zero amax give 0).
__device__ __forceinline__ uint32_t e8m0_floor_code(float amax_b) {
  const uint32_t e = __float_as_uint(amax_b) >> 23;
  if (e >= 255u) return 254u;
  return e >= 2u ? e - 2u : 0u;
}

// Programmatic dependent launch: let the next kernel on the stream start its prologue
// early / wait until the previous kernel's writes are visible (no-ops without the
// launch attribute).
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void wait_prior_grids() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ------------------------------------------------------------------ amax
// Grid-stride max of |x| (as bit patterns: for non-negative floats the integer order is
// the numeric order, and inf / NaN patterns exceed every finite one).  Each block writes
// its partial; the last block to finish (ticket from a self-resetting atomicInc) reduces
// them, latches non-finite input, and writes amax and / or g.
// RHT: the maximum of the Hadamard-transformed values (n a multiple of 16; each thread
// transforms whole 16-element blocks, in the same FP32 order as the quantize kernel).
template <typename T, bool RHT = false>
__global__ void __launch_bounds__(512) amax_kernel(const T* __restrict__ x, int64_t n, uint32_t* ws,
                                                    float* amax_out, float* g_out, unsigned* status,
                                                    uint32_t signs) {
  allow_dependents();
  wait_prior_grids();  // x may be the output of the kernel just before
  constexpr int EPC = Elem<T>::kPerChunk;
  const int64_t nchunks = RHT ? 0 : n / EPC;
  const uint4* xc = reinterpret_cast<const uint4*>(x);
  uint32_t m = 0;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if constexpr (RHT) {
    constexpr int CPB = 16 / EPC;  // 16-byte chunks per 16-element block
    for (int64_t b = i; b < n / 16; b += stride) {
      float v[16];
#pragma unroll
      for (int c = 0; c < CPB; ++c) {
        float t[EPC];
        Elem<T>::unpack(ld_stream(xc + b * CPB + c), t);
#pragma unroll
        for (int e = 0; e < EPC; ++e) v[c * EPC + e] = t[e];
      }
      rht16_lanes<16>(v, signs, 0);
#pragma unroll
      for (int e = 0; e < 16; ++e) m = max(m, abs_bits(v[e]));
    }
  }
  for (; i + 3 * stride < nchunks; i += 4 * stride) {
    uint4 u[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) u[j] = ld_stream(xc + i + j * stride);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float v[EPC];
      Elem<T>::unpack(u[j], v);
#pragma unroll
      for (int e = 0; e < EPC; ++e) m = max(m, abs_bits(v[e]));
    }
  }
  for (; i < nchunks; i += stride) {
    float v[EPC];
    Elem<T>::unpack(ld_stream(xc + i), v);
#pragma unroll
    for (int e = 0; e < EPC; ++e) m = max(m, abs_bits(v[e]));
  }
  if (!RHT && blockIdx.x == 0) {  // tail elements that do not fill a 16-byte chunk
    for (int64_t t = nchunks * EPC + threadIdx.x; t < n; t += blockDim.x) {
      float v;
      if constexpr (sizeof(T) == 4) v = reinterpret_cast<const float*>(x)[t];
      else v = __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t*>(x)[t]) << 16);
      m = max(m, abs_bits(v));
    }
  }
  m = __reduce_max_sync(0xFFFFFFFFu, m);
  __shared__ uint32_t s_m[16];
  __shared__ bool s_last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) s_m[warp] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t bm = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) bm = max(bm, s_m[w]);
    volatile uint32_t* partial = ws + 2;
    partial[blockIdx.x] = bm;
    __threadfence();
    const unsigned ticket = atomicInc(ws, gridDim.x - 1);  // wraps back to 0 on the last block
    s_last = (ticket == gridDim.x - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  uint32_t bm = 0;
  volatile uint32_t* partial = ws + 2;
  for (unsigned b = threadIdx.x; b < gridDim.x; b += blockDim.x) {
    bm = max(bm, partial[b]);
    partial[b] = 0;  // leave the workspace zero-filled
  }
  bm = __reduce_max_sync(0xFFFFFFFFu, bm);
  if (lane == 0) s_m[warp] = bm;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t am = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) am = max(am, s_m[w]);
    if (am >= 0x7F800000u) atomicOr(status, kStatusNonFinite);
    const float amax = __uint_as_float(am);
    if (amax_out) *amax_out = amax;
    if (g_out) *g_out = amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f;  // 2688 = 6 * 448
  }
}

// ------------------------------------------------------------------ group prefix
// Row-blocks of the (grouped) scale layout: group e owns blocks [rb[e], rb[e+1]) with
// rb[e+1] - rb[e] = ceil(rows_e / 128).  Computed by every block into shared memory.
__device__ void group_prefix(const int32_t* offsets, int E, int* s_rb, int* s_off) {
  // E <= kMaxGroups; simple two-level scan by one warp
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int carry = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      int cnt = 0;
      if (e < E) {
        const int lo = offsets[e], hi = offsets[e + 1];
        s_off[e] = lo;
        cnt = (hi - lo + 127) / 128;
      }
      int incl = cnt;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int t = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += t;
      }
      if (e < E) s_rb[e] = carry + incl - cnt;
      carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
    if (lane == 0) {
      s_rb[E] = carry;
      s_off[E] = offsets[E];
    }
  }
  __syncthreads();
}

// ------------------------------------------------------------------ 1-D quantize
struct Quant1DArgs {
  const void* x;
  int64_t rows, cols;
  uint8_t* codes;
  uint8_t* scales;
  const float* g;          // NVFP4 global scale (device)
  const int32_t* offsets;  // grouped rows, or null
  int num_groups;
  int64_t rb_upper;        // row-blocks covered by the launch (grouped: upper bound)
  int64_t ct_count;        // column tiles = atoms along columns
  unsigned* status;
  const uint32_t* rbits;   // kQuantSR: one random word per element, row-major [rows, cols]
  uint32_t signs;          // kQuantRHT: the 16 sign bits of the transform
};

// One tile = 128 rows x (4 * BLOCK) columns = exactly one 512-byte scale atom; one CTA of
// 256 threads per tile.  Each thread owns whole blocks (a row's BLOCK consecutive
// elements), two per tile: it loads them, takes their maximum, computes the block's scale
// once, encodes and packs the codes, and stores its scale byte straight into the
// swizzled atom.  Consecutive threads take consecutive blocks of a row, so a warp reads
// whole rows of the tile.
template <typename T>
struct BlockLoad {
  static constexpr int kChunks(int block) { return block * static_cast<int>(sizeof(T)) / 16; }
};

// max |x| over 8 BF16 values packed in a 16-byte chunk, as float bits (NaN propagates:
// its pattern exceeds every finite one, and so does inf)
__device__ __forceinline__ uint32_t chunk_absmax_bf16(const uint4& u) {
  const __nv_bfloat162 a = __hmax2_nan(__habs2(*reinterpret_cast<const __nv_bfloat162*>(&u.x)),
                                       __habs2(*reinterpret_cast<const __nv_bfloat162*>(&u.y)));
  const __nv_bfloat162 b = __hmax2_nan(__habs2(*reinterpret_cast<const __nv_bfloat162*>(&u.z)),
                                       __habs2(*reinterpret_cast<const __nv_bfloat162*>(&u.w)));
  const __nv_bfloat162 c = __hmax2_nan(a, b);
  const uint32_t w = *reinterpret_cast<const uint32_t*>(&c);
  return max(w << 16, w & 0xFFFF0000u);
}

// BF16 input in 16-blocks (plain and Hadamard) fits five CTAs per SM without spilling; the
// encode pass is issue-bound, and the extra warps took 4-5% off it (A/B, one B200 session).
template <typename T, int BLOCK, int VAR, bool GROUPED>
constexpr int q1d_min_ctas() {
  return sizeof(T) == 2 && BLOCK == 16 && VAR != kQuantSR && !GROUPED ? 5 : 0;
}

template <typename T, int BLOCK, bool MX, bool HW, int VAR = kQuantPlain, bool GROUPED = false>
__global__ void __launch_bounds__(256, q1d_min_ctas<T, BLOCK, VAR, GROUPED>()) quantize_1d_kernel(const Quant1DArgs p) {
  constexpr int EPC = Elem<T>::kPerChunk;
  constexpr int CH = BLOCK * static_cast<int>(sizeof(T)) / 16;  // 16-byte chunks per block
  constexpr int UPT = 2;                                        // blocks per thread per tile
  static_assert(VAR != kQuantMxFloor || MX, "the rounded-down scale is an E8M0 one");
  static_assert(VAR != kQuantSR || (!MX && BLOCK == 16), "stochastic rounding: NVFP4");
  static_assert(VAR != kQuantFp8 || (MX && BLOCK == 32), "MXFP8: E4M3 elements in 32-blocks");
  constexpr int RW = VAR == kQuantSR ? BLOCK / 4 : 0;  // 16-byte loads of random words per block

  // More than 32 groups: the row-block prefix in shared memory, 2 (E + 1) ints sized at
  // launch.  Up to 32 groups: every warp forms the prefix in registers (lane e holds group
  // e), with no shared memory and no barrier.  Ungrouped launches take neither (a fixed 8 KB
  // table for the largest group count, or a barrier, cost the streaming loads about 1 us of
  // a 25 us launch).
  extern __shared__ int s_grp[];
  int* const s_rb = s_grp;
  int* const s_off = s_grp + (GROUPED ? p.num_groups + 1 : 0);
  allow_dependents();
  wait_prior_grids();  // g (and x, offsets) may come from the kernels just before
  const int E = GROUPED ? p.num_groups : 1;
  const int lane = threadIdx.x & 31;
  int rb_total = static_cast<int>((p.rows + 127) / 128);
  int w_off = 0, w_end = 0, w_rb = 0, w_rbe = 0;  // lane e < E: offsets[e], offsets[e + 1], rb[e], rb[e + 1]
  if constexpr (GROUPED) {
    if (E <= 32) {
      if (lane < E) {
        w_off = p.offsets[lane];
        w_end = p.offsets[lane + 1];
      }
      const int cnt = lane < E ? (w_end - w_off + 127) / 128 : 0;
      int incl = cnt;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int t = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += t;
      }
      w_rb = incl - cnt;
      w_rbe = incl;
      rb_total = __shfl_sync(0xFFFFFFFFu, incl, 31);
    } else {
      group_prefix(p.offsets, E, s_rb, s_off);
      rb_total = s_rb[E];
    }
  }
  float g = 1.0f;
  if constexpr (!MX) g = *p.g;

  const int tid = threadIdx.x;
  const int64_t half_cols = p.cols / 2;
  const int64_t ntiles = p.rb_upper * p.ct_count;
  const int64_t nbc = p.cols / BLOCK;  // blocks per row
  unsigned bad = 0;

  for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const int64_t rb = tile / p.ct_count;
    const int64_t ct = tile % p.ct_count;
    uint8_t* atom = p.scales + (rb * p.ct_count + ct) * 512;
    if (rb >= rb_total) {  // beyond the last group's blocks: zero pad atom
      if (tid < 32) reinterpret_cast<uint4*>(atom)[tid] = make_uint4(0, 0, 0, 0);
      continue;
    }
    // group of this row-block: one ballot over the warp's prefix (<= 32 groups), else a binary
    // search of the shared table.  A tile never spans two groups: tiles of x's own 128-row
    // blocks, each scale byte sent to its group's atom, measured 20% slower (32 x ~512 rows).
    int64_t row_base = rb * 128, row_end = p.rows;
    if constexpr (GROUPED) {
      if (E <= 32) {
        // the one lane (group) whose row-blocks hold rb; none only for malformed offsets
        const unsigned own = __ballot_sync(0xFFFFFFFFu, lane < E && w_rb <= rb && rb < w_rbe);
        const int e = own ? __ffs(own) - 1 : 0;
        row_base = __shfl_sync(0xFFFFFFFFu, w_off, e) + (rb - __shfl_sync(0xFFFFFFFFu, w_rb, e)) * 128;
        row_end = own ? __shfl_sync(0xFFFFFFFFu, w_end, e) : row_base;
      } else {
        int lo = 0, hi = E - 1;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (s_rb[mid] <= rb) lo = mid;
          else hi = mid - 1;
        }
        row_base = s_off[lo] + (rb - s_rb[lo]) * 128;
        row_end = s_off[lo + 1];
      }
      if (row_end > p.rows) row_end = p.rows;  // offsets past the tensor read nothing
    }

    // this thread's blocks: unit q -> row q / 4 of the tile, block column q % 4
    uint4 u[UPT][CH];
    uint4 rw[UPT][RW > 0 ? RW : 1];
    bool ok[UPT];
#pragma unroll
    for (int i = 0; i < UPT; ++i) {
      const int q = tid + 256 * i;
      const int64_t r = row_base + (q >> 2);
      const int64_t bcol = ct * 4 + (q & 3);
      ok[i] = (!GROUPED || r >= 0) && r < row_end && bcol < nbc;
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.x) +
                                                        (r * p.cols + bcol * BLOCK) * static_cast<int64_t>(sizeof(T)));
#pragma unroll
      for (int c = 0; c < CH; ++c) u[i][c] = ok[i] ? ld_stream(src + c) : make_uint4(0, 0, 0, 0);
      if constexpr (RW > 0) {
        const uint4* rsrc = reinterpret_cast<const uint4*>(p.rbits + r * p.cols + bcol * BLOCK);
#pragma unroll
        for (int c = 0; c < RW; ++c) rw[i][c] = ok[i] ? ld_stream(rsrc + c) : make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int i = 0; i < UPT; ++i) {
      const int q = tid + 256 * i;
      const int rl = q >> 2, bc = q & 3;
      const int64_t r = row_base + rl;
      const int64_t bcol = ct * 4 + bc;
      float v[BLOCK];
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        float t[EPC];
        Elem<T>::unpack(u[i][c], t);
#pragma unroll
        for (int j = 0; j < EPC; ++j) v[c * EPC + j] = t[j];
      }
      uint32_t m = 0;
      if constexpr (VAR == kQuantRHT) {
#pragma unroll
        for (int h = 0; h < BLOCK; h += 16) {
          float (&w16)[16] = *reinterpret_cast<float(*)[16]>(v + h);
          rht16_lanes<16>(w16, p.signs, 0);
        }
#pragma unroll
        for (int j = 0; j < BLOCK; ++j) m = max(m, abs_bits(v[j]));
      } else if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int c = 0; c < CH; ++c) m = max(m, chunk_absmax_bf16(u[i][c]));
      } else {
#pragma unroll
        for (int j = 0; j < BLOCK; ++j) m = max(m, abs_bits(v[j]));
      }
      bad |= ok[i] && m >= 0x7F800000u;
      const float amax_b = __uint_as_float(m);
      uint32_t sb;
      float mul;
      if constexpr (MX) {
        // MXFP4: nearest power of two of amax_b / 6 (or rounded down); MXFP8: of amax_b / 448,
        // E4M3's largest value
        sb = VAR == kQuantMxFloor ? e8m0_floor_code(amax_b)
                                  : e8m0_code(__fdiv_rn(amax_b, VAR == kQuantFp8 ? 448.0f : 6.0f));
        mul = e8m0_inverse(sb);
      } else {
        mul = nvfp4_block_scale(amax_b, g, sb);
      }
      const bool inf_mul = !MX && isinf(mul);  // 1/denom overflowed: zeros stay zeros, not NaN
      if constexpr (VAR == kQuantFp8) {
        // one E4M3 byte per element: 32 bytes per block, two 16-byte stores
        uint32_t w8[BLOCK / 4];
#pragma unroll
        for (int o = 0; o < BLOCK / 4; ++o)
          w8[o] = pack4_e4m3(__fmul_rn(v[4 * o], mul), __fmul_rn(v[4 * o + 1], mul), __fmul_rn(v[4 * o + 2], mul),
                             __fmul_rn(v[4 * o + 3], mul));
        if (ok[i]) {
          uint4* dst = reinterpret_cast<uint4*>(p.codes + r * p.cols + bcol * BLOCK);
          dst[0] = make_uint4(w8[0], w8[1], w8[2], w8[3]);
          dst[1] = make_uint4(w8[4], w8[5], w8[6], w8[7]);
        }
      } else {
      uint32_t packed[BLOCK / 8];
#pragma unroll
      for (int o = 0; o < BLOCK / 8; ++o) {
        float sv[8];
        if (!inf_mul) {
#pragma unroll
          for (int j = 0; j < 8; ++j) sv[j] = __fmul_rn(v[o * 8 + j], mul);
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float x = v[o * 8 + j];
            sv[j] = x == 0.0f ? x : __fmul_rn(x, mul);
          }
        }
        if constexpr (VAR == kQuantSR) {
          uint32_t word = 0;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint4 w4 = rw[i][(o * 8 + j) / 4];
            const int k = (o * 8 + j) & 3;
            const uint32_t bits = k == 0 ? w4.x : k == 1 ? w4.y : k == 2 ? w4.z : w4.w;
            word |= e2m1_code_sr(sv[j], bits) << (4 * j);
          }
          packed[o] = word;
        } else {
          packed[o] = pack8<HW>(sv);
        }
      }
      if (ok[i]) {
        uint8_t* dst = p.codes + r * half_cols + bcol * (BLOCK / 2);
        if constexpr (BLOCK == 16) *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
        else *reinterpret_cast<uint4*>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      }
      }
      // the scale byte at its place in the atom (rows and blocks past the tensor: 0)
      atom[(rl & 31) * 16 + (rl >> 5) * 4 + bc] = ok[i] ? static_cast<uint8_t>(sb) : 0;
    }
  }
  if (bad) atomicOr(p.status, kStatusNonFinite);
}

// ------------------------------------------------------------------ small tensors
// A tensor of at most kSmallThreads * kSmallCtas * NB blocks (e.g. 32 x 8192 BF16
// activations of a decode step) is quantized by one thread-block cluster in a single
// launch: every thread loads its NB blocks into registers, the cluster combines the
// tensor amax through distributed shared memory, and the registers are encoded -- one
// read of x, and no second kernel waiting for the amax.
struct SmallArgs {
  const void* x;
  int64_t rows, cols;
  uint8_t* codes;
  uint8_t* scales;
  int64_t scale_bytes;  // padded size of the scale buffer (zero-filled by the kernel)
  const float* g_in;    // NVFP4: caller's global scale, or null to compute it
  float* g_out;         // may be null
  unsigned* status;
};

// Store v into the shared-memory word at local address `local` of cluster CTA `rank`.
__device__ __forceinline__ void st_cluster_u32(const void* local, uint32_t rank, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr(smem_u32(local), rank)), "r"(v) : "memory");
}

template <typename T, int BLOCK>
struct SmallCfg {
  static constexpr int kChunks = BLOCK * static_cast<int>(sizeof(T)) / 16;  // 16-byte loads per block
  static constexpr int kNB = 8 / kChunks;                                    // blocks per thread
};

template <typename T, int BLOCK, bool MX, bool HW>
__global__ void __cluster_dims__(kSmallCtas, 1, 1) __launch_bounds__(kSmallThreads)
    quantize_small_kernel(const SmallArgs p) {
  using SC = SmallCfg<T, BLOCK>;
  constexpr int CH = SC::kChunks, NB = SC::kNB, EPC = Elem<T>::kPerChunk;
  constexpr int TT = kSmallThreads * kSmallCtas;
  __shared__ uint32_t s_warp[kSmallThreads / 32];
  __shared__ uint32_t s_cta[kSmallCtas];

  allow_dependents();
  wait_prior_grids();  // x may come from the kernel just before; codes / scales may still be read by it
  const uint32_t rank = cluster_rank();
  const int gt = static_cast<int>(rank) * kSmallThreads + threadIdx.x;
  // zero-fill the padded scale buffer; the cluster barrier below orders these stores
  // before the scale bytes written after it
  for (int64_t o = static_cast<int64_t>(gt) * 16; o < p.scale_bytes; o += static_cast<int64_t>(TT) * 16)
    *reinterpret_cast<uint4*>(p.scales + o) = make_uint4(0, 0, 0, 0);

  const int64_t bpr = p.cols / BLOCK;  // blocks per row
  const int64_t nblocks = p.rows * bpr;
  uint4 u[NB][CH];
  uint32_t bm[NB];
  uint32_t tmax = 0;
#pragma unroll
  for (int i = 0; i < NB; ++i) {
    const int64_t b = gt + static_cast<int64_t>(i) * TT;
    const uint8_t* src = static_cast<const uint8_t*>(p.x) + b * BLOCK * static_cast<int64_t>(sizeof(T));
#pragma unroll
    for (int j = 0; j < CH; ++j) u[i][j] = b < nblocks ? ld_stream(src + j * 16) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int i = 0; i < NB; ++i) {
    uint32_t m = 0;
#pragma unroll
    for (int j = 0; j < CH; ++j) {
      float v[EPC];
      Elem<T>::unpack(u[i][j], v);
#pragma unroll
      for (int e = 0; e < EPC; ++e) m = max(m, abs_bits(v[e]));
    }
    bm[i] = m;
    tmax = max(tmax, m);
  }
  // tensor amax: warp -> CTA -> every CTA of the cluster
  tmax = __reduce_max_sync(0xFFFFFFFFu, tmax);
  if ((threadIdx.x & 31) == 0) s_warp[threadIdx.x >> 5] = tmax;
  __syncthreads();
  if (threadIdx.x < kSmallCtas) {
    uint32_t cm = 0;
    for (int w = 0; w < kSmallThreads / 32; ++w) cm = max(cm, s_warp[w]);
    st_cluster_u32(&s_cta[rank], threadIdx.x, cm);  // thread t delivers this CTA's max to CTA t
  }
  cluster_sync_all();
  uint32_t am = 0;
#pragma unroll
  for (int c = 0; c < kSmallCtas; ++c) am = max(am, s_cta[c]);
  float g = 1.0f;
  if constexpr (!MX) {
    const float amax = __uint_as_float(am);
    g = p.g_in ? *p.g_in : (amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f);  // 2688 = 6 * 448
  }
  if (gt == 0 && p.g_out) *p.g_out = g;
  if (gt == 0 && am >= 0x7F800000u) atomicOr(p.status, kStatusNonFinite);

  const int64_t spad = ((bpr + 3) / 4) * 4;  // scale columns padded to whole atoms
#pragma unroll
  for (int i = 0; i < NB; ++i) {
    const int64_t b = gt + static_cast<int64_t>(i) * TT;
    if (b >= nblocks) continue;
    const int64_t r = b / bpr, c = b % bpr;
    uint32_t sb;
    float mul;
    if constexpr (MX) {
      sb = e8m0_code(__fdiv_rn(__uint_as_float(bm[i]), 6.0f));
      mul = e8m0_inverse(sb);
    } else {
      mul = nvfp4_block_scale(__uint_as_float(bm[i]), g, sb);
    }
    uint32_t packed[BLOCK / 8];
#pragma unroll
    for (int j = 0; j < CH; ++j) {
      float v[EPC];
      Elem<T>::unpack(u[i][j], v);
      float s[EPC];
#pragma unroll
      for (int e = 0; e < EPC; ++e) s[e] = (!MX && v[e] == 0.0f) ? v[e] : __fmul_rn(v[e], mul);
      if constexpr (EPC == 8) {
        packed[j] = pack8<HW>(s);
      } else {
        const uint32_t h = pack4<HW>(s);
        if (j & 1) packed[j / 2] |= h << 16;
        else packed[j / 2] = h;
      }
    }
    uint8_t* dst = p.codes + b * (BLOCK / 2);
    if constexpr (BLOCK == 16) *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
    else *reinterpret_cast<uint4*>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    p.scales[((r / 128) * (spad / 4) + c / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + c % 4] =
        static_cast<uint8_t>(sb);
  }
}

// x * (1/denom) with a zero element kept zero when the reciprocal overflowed.
__device__ __forceinline__ float ratio(float x, float mul) { return x == 0.0f ? x : __fmul_rn(x, mul); }

// ------------------------------------------------------------------ 2-D quantize
struct Quant2DArgs {
  const void* x;
  int64_t rows, cols;
  uint8_t* codes;    // [rows, cols/2]
  uint8_t* scales;   // swizzled [rows, cols/16]
  uint8_t* codesT;   // [cols, rows/2]
  uint8_t* scalesT;  // swizzled [cols, rows/16]
  const float* g;
  unsigned* status;
};

// Four consecutive elements of one row, as FP32 (16-byte load for FP32, 8-byte for BF16).
template <typename T>
__device__ __forceinline__ void load4(const T* src, float (&v)[4]);
template <>
__device__ __forceinline__ void load4<float>(const float* src, float (&v)[4]) {
  const uint4 u = ld_stream(src);
  v[0] = __uint_as_float(u.x);
  v[1] = __uint_as_float(u.y);
  v[2] = __uint_as_float(u.z);
  v[3] = __uint_as_float(u.w);
}
template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16* src, float (&v)[4]) {
  uint32_t a, b;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(a), "=r"(b) : "l"(src));
  v[0] = __uint_as_float(a << 16);
  v[1] = __uint_as_float(a & 0xFFFF0000u);
  v[2] = __uint_as_float(b << 16);
  v[3] = __uint_as_float(b & 0xFFFF0000u);
}

// One CTA per 128 x 128 region of W; warp w holds the region's 16-row band w in registers,
// lane l its four columns 4l .. 4l+3, so that the four lanes of a 16 x 16 patch find the
// patch amax with two shuffles.  Each element's ratio to its patch scale is formed once and
// encoded twice: in row pairs along W's rows (W's codes) and in pairs down the columns
// (W^T's codes, eight bytes per column of the band).  The patches' scale bytes meet in
// shared memory, and both scale layouts receive two full 512-byte atoms per region.  Rows
// (a multiple of 32) and columns (a multiple of 32) beyond the tensor are zero: a band and a
// lane's four columns are either wholly inside or wholly outside.
template <typename T, bool HW>
__global__ void __launch_bounds__(256, 3) quantize_2d_kernel(const Quant2DArgs p) {
  __shared__ uint8_t s_sb[8][8];
  __shared__ __align__(16) uint8_t s_atom[2][512];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * 128;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * 128;
  const int64_t rb = r0 + warp * 16;  // this warp's first row
  const int64_t cl = c0 + lane * 4;   // this lane's first column
  const bool in = rb < p.rows && cl < p.cols;
  const float g = *p.g;

  float v[16][4];
  if (in) {
    const T* src = static_cast<const T*>(p.x) + rb * p.cols + cl;
#pragma unroll
    for (int i = 0; i < 16; ++i) load4<T>(src + i * p.cols, v[i]);
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i][0] = v[i][1] = v[i][2] = v[i][3] = 0.0f;
  }
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) m = max(m, abs_bits(v[i][j]));
  m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
  m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
  const unsigned bad = m >= 0x7F800000u;
  uint32_t sb;
  const float mul = nvfp4_block_scale(__uint_as_float(m), g, sb);
  if ((lane & 3) == 0) s_sb[warp][lane >> 2] = static_cast<uint8_t>(sb);
#pragma unroll
  for (int i = 0; i < 16; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) v[i][j] = ratio(v[i][j], mul);
  if (in) {
    // W: two rows per pack8 (four codes of each), sixteen bits per row and lane
    uint8_t* wrow = p.codes + rb * (p.cols / 2) + cl / 2;
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
      const float a[8] = {v[i][0], v[i][1], v[i][2], v[i][3], v[i + 1][0], v[i + 1][1], v[i + 1][2], v[i + 1][3]};
      const uint32_t w = pack8<HW>(a);
      *reinterpret_cast<uint16_t*>(wrow + i * (p.cols / 2)) = static_cast<uint16_t>(w);
      *reinterpret_cast<uint16_t*>(wrow + (i + 1) * (p.cols / 2)) = static_cast<uint16_t>(w >> 16);
    }
    // W^T: column j of the band is sixteen codes, eight bytes of W^T's row cl + j
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float a[8] = {v[0][j], v[1][j], v[2][j], v[3][j], v[4][j], v[5][j], v[6][j], v[7][j]};
      const float b[8] = {v[8][j], v[9][j], v[10][j], v[11][j], v[12][j], v[13][j], v[14][j], v[15][j]};
      *reinterpret_cast<uint2*>(p.codesT + (cl + j) * (p.rows / 2) + rb / 2) = make_uint2(pack8<HW>(a), pack8<HW>(b));
    }
  }
  __syncthreads();
  // scale atoms.  W: rows r0..r0+127, scale columns c0/16 .. +7 -> atoms (r0/128, c0/64 + {0,1}).
  // W^T: rows c0..c0+127, scale columns r0/16 .. +7 -> atoms (c0/128, r0/64 + {0,1}).
  for (int pass = 0; pass < 2; ++pass) {
    for (int idx = tid; idx < 2 * 128 * 4; idx += 256) {
      const int a = idx >> 9, rem = idx & 511, rl = rem >> 2, cc = rem & 3;
      const int off = (rl & 31) * 16 + (rl >> 5) * 4 + cc;
      const int b = a * 4 + cc;  // scale column inside the region (0..7)
      uint8_t byte;
      if (pass == 0) byte = ((r0 + rl) < p.rows && (c0 + b * 16) < p.cols) ? s_sb[rl >> 4][b] : 0;
      else byte = ((c0 + rl) < p.cols && (r0 + b * 16) < p.rows) ? s_sb[b][rl >> 4] : 0;
      s_atom[a][off] = byte;
    }
    __syncthreads();
    const int64_t natoms = pass == 0 ? ((p.cols / 16) + 3) / 4 : ((p.rows / 16) + 3) / 4;
    const int64_t rowblk = pass == 0 ? r0 / 128 : c0 / 128;
    const int64_t first = pass == 0 ? c0 / 64 : r0 / 64;
    uint8_t* dst = pass == 0 ? p.scales : p.scalesT;
    if (tid < 64) {
      const int a = tid >> 5;
      if (first + a < natoms)
        reinterpret_cast<uint4*>(dst + (rowblk * natoms + first + a) * 512)[lane] =
            reinterpret_cast<const uint4*>(s_atom[a])[lane];
    }
    __syncthreads();
  }
  if (bad) atomicOr(p.status, kStatusNonFinite);
}

// ------------------------------------------------------------------ dequantize
__global__ void dequantize_kernel(const uint8_t* codes, const uint8_t* scales, const float* gptr, int64_t rows,
                                  int64_t cols, int mx, float* out) {
  const int64_t n = rows * cols;
  const int blk = mx ? 32 : 16;
  const int64_t scols = cols / blk, cpad = (scols + 3) / 4 * 4;
  const float g = gptr ? *gptr : 1.0f;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / cols, k = i % cols;
    const uint8_t byte = codes[r * (cols / 2) + k / 2];
    const uint32_t code = (k & 1) ? (byte >> 4) : (byte & 15);
    const int64_t c = k / blk;
    const int64_t off = ((r / 128) * (cpad / 4) + c / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4);
    const uint32_t sb = scales[off];
    const float s = mx ? e8m0_value(sb) : __fmul_rn(e4m3_value(sb), g);
    out[i] = __fmul_rn(e2m1_value(code), s);
  }
}

__global__ void debug_encode_kernel(const float* in, int64_t n, int which, uint8_t* out) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float v = in[i];
    uint32_t r;
    switch (which) {
      case 0: {  // the production encoder of the quantize kernels
        float a[4] = {v, 0.0f, 0.0f, 0.0f};
        r = pack4<kE2M1Hardware>(a) & 15u;
        break;
      }
      case 1: r = e4m3_code(v); break;
      case 2: r = e8m0_code(v); break;
      case 3: r = e2m1_code_exact(v); break;
      default: {
        float a[4] = {v, 0.0f, 0.0f, 0.0f};
        r = pack4<true>(a) & 15u;
      }
    }
    out[i] = static_cast<uint8_t>(r);
  }
}

__global__ void set_value_kernel(float* p, float v) { *p = v; }

__global__ void global_scale_kernel(const float* amax, float* g, unsigned* status) {
  allow_dependents();
  wait_prior_grids();  // the maximum may come from the kernel (or collective) just before
  const float a = *amax;
  if (!(abs_bits(a) < 0x7F800000u)) atomicOr(status, kStatusNonFinite);
  *g = a > 0.0f ? __fdiv_rn(a, 2688.0f) : 1.0f;  // 2688 = 6 * 448
}

// ------------------------------------------------------------------ launchers
static int blocks_for(int64_t work, int per_sm) {
  const int sms = num_sms();
  int64_t b = std::min<int64_t>(work, static_cast<int64_t>(sms) * per_sm);
  return static_cast<int>(std::max<int64_t>(b, 1));
}

cudaError_t launch_amax(const void* x, int64_t n, int bf16, uint32_t* ws, float* amax_out, float* g_out,
                        unsigned* status, cudaStream_t st, int rht, uint32_t signs) {
  const int epc = bf16 ? 8 : 4;
  const int64_t chunks = (n + epc - 1) / epc;
  int blocks = static_cast<int>(std::min<int64_t>((chunks + 2047) / 2048, static_cast<int64_t>(num_sms()) * 4));
  blocks = std::max(1, std::min(blocks, kAmaxMaxBlocks));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(512);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (rht) {
    if (bf16)
      return cudaLaunchKernelEx(&cfg, amax_kernel<__nv_bfloat16, true>, static_cast<const __nv_bfloat16*>(x), n, ws,
                                amax_out, g_out, status, signs);
    return cudaLaunchKernelEx(&cfg, amax_kernel<float, true>, static_cast<const float*>(x), n, ws, amax_out, g_out,
                              status, signs);
  }
  if (bf16)
    return cudaLaunchKernelEx(&cfg, amax_kernel<__nv_bfloat16>, static_cast<const __nv_bfloat16*>(x), n, ws, amax_out,
                              g_out, status, 0u);
  return cudaLaunchKernelEx(&cfg, amax_kernel<float>, static_cast<const float*>(x), n, ws, amax_out, g_out, status,
                            0u);
}

template <typename T, int BLOCK, bool MX, int VAR = kQuantPlain>
static cudaError_t launch_q1d_t(const Quant1DArgs& a, cudaStream_t st) {
  // one CTA per tile: the hardware starts a new tile as soon as one finishes, which keeps
  // every SM's loads in flight to the end (a persistent grid would finish in waves, and
  // leave SMs idle in the last one when the tile count is a few grid sizes)
  const int blocks = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(a.rb_upper * a.ct_count, 1 << 30)));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if constexpr (VAR == kQuantPlain) {
    cfg.dynamicSmemBytes = a.offsets && a.num_groups > 32 ? 2 * (a.num_groups + 1) * sizeof(int) : 0;
    if (a.offsets) return cudaLaunchKernelEx(&cfg, quantize_1d_kernel<T, BLOCK, MX, kE2M1Hardware, VAR, true>, a);
  } else {
    if (a.offsets) return cudaErrorInvalidValue;  // the variants take no groups
  }
  return cudaLaunchKernelEx(&cfg, quantize_1d_kernel<T, BLOCK, MX, kE2M1Hardware, VAR>, a);
}

cudaError_t launch_quantize_1d(const void* x, int64_t rows, int64_t cols, int bf16, int mx, uint8_t* codes,
                               uint8_t* scales, const float* g, const int32_t* offsets, int num_groups,
                               unsigned* status, cudaStream_t st, int variant, const uint32_t* rbits,
                               uint32_t signs) {
  Quant1DArgs a;
  a.x = x;
  a.rows = rows;
  a.cols = cols;
  a.codes = codes;
  a.scales = scales;
  a.g = g;
  a.offsets = offsets;
  a.num_groups = num_groups;
  a.rb_upper = (rows + 127) / 128 + (offsets ? num_groups : 0);
  const int blk = mx ? 32 : 16;
  a.ct_count = ((cols / blk) + 3) / 4;
  a.status = status;
  a.rbits = rbits;
  a.signs = signs;
  using BF = __nv_bfloat16;
  switch (variant) {
    case kQuantMxFloor:
      if (!mx) return cudaErrorInvalidValue;
      return bf16 ? launch_q1d_t<BF, 32, true, kQuantMxFloor>(a, st) : launch_q1d_t<float, 32, true, kQuantMxFloor>(a, st);
    case kQuantSR:
      if (mx) return cudaErrorInvalidValue;
      return bf16 ? launch_q1d_t<BF, 16, false, kQuantSR>(a, st) : launch_q1d_t<float, 16, false, kQuantSR>(a, st);
    case kQuantFp8:
      if (!mx) return cudaErrorInvalidValue;
      return bf16 ? launch_q1d_t<BF, 32, true, kQuantFp8>(a, st) : launch_q1d_t<float, 32, true, kQuantFp8>(a, st);
    case kQuantRHT:
      if (bf16)
        return mx ? launch_q1d_t<BF, 32, true, kQuantRHT>(a, st) : launch_q1d_t<BF, 16, false, kQuantRHT>(a, st);
      return mx ? launch_q1d_t<float, 32, true, kQuantRHT>(a, st) : launch_q1d_t<float, 16, false, kQuantRHT>(a, st);
    default:
      break;
  }
  if (bf16) return mx ? launch_q1d_t<BF, 32, true>(a, st) : launch_q1d_t<BF, 16, false>(a, st);
  return mx ? launch_q1d_t<float, 32, true>(a, st) : launch_q1d_t<float, 16, false>(a, st);
}

template <typename T, int BLOCK>
static constexpr int64_t small_capacity_blocks() {
  return static_cast<int64_t>(kSmallThreads) * kSmallCtas * SmallCfg<T, BLOCK>::kNB;
}

bool quantize_small_fits(int64_t rows, int64_t cols, int bf16, int mx) {
  const int64_t nb = rows * (cols / (mx ? 32 : 16));
  if (bf16) return nb <= (mx ? small_capacity_blocks<__nv_bfloat16, 32>() : small_capacity_blocks<__nv_bfloat16, 16>());
  return nb <= (mx ? small_capacity_blocks<float, 32>() : small_capacity_blocks<float, 16>());
}

template <typename T, int BLOCK, bool MX>
static cudaError_t launch_small_t(const SmallArgs& a, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kSmallCtas);  // one cluster (its size is fixed by the kernel)
  cfg.blockDim = dim3(kSmallThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, quantize_small_kernel<T, BLOCK, MX, kE2M1Hardware>, a);
}

cudaError_t launch_quantize_small(const void* x, int64_t rows, int64_t cols, int bf16, int mx, uint8_t* codes,
                                  uint8_t* scales, const float* g_in, float* g_out, unsigned* status,
                                  cudaStream_t st) {
  SmallArgs a;
  a.x = x;
  a.rows = rows;
  a.cols = cols;
  a.codes = codes;
  a.scales = scales;
  const int64_t scols = cols / (mx ? 32 : 16);
  a.scale_bytes = ((rows + 127) / 128) * 128 * (((scols + 3) / 4) * 4);
  a.g_in = g_in;
  a.g_out = g_out;
  a.status = status;
  if (bf16) return mx ? launch_small_t<__nv_bfloat16, 32, true>(a, st) : launch_small_t<__nv_bfloat16, 16, false>(a, st);
  return mx ? launch_small_t<float, 32, true>(a, st) : launch_small_t<float, 16, false>(a, st);
}

cudaError_t launch_quantize_2d(const void* x, int64_t rows, int64_t cols, int bf16, uint8_t* codes,
                               uint8_t* scales, uint8_t* codesT, uint8_t* scalesT, const float* g,
                               unsigned* status, cudaStream_t st) {
  Quant2DArgs a{x, rows, cols, codes, scales, codesT, scalesT, g, status};
  dim3 grid(static_cast<unsigned>((cols + 127) / 128), static_cast<unsigned>((rows + 127) / 128));
  if (bf16)
    quantize_2d_kernel<__nv_bfloat16, kE2M1Hardware><<<grid, 256, 0, st>>>(a);
  else
    quantize_2d_kernel<float, kE2M1Hardware><<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* scales, const float* g, int64_t rows,
                              int64_t cols, int mx, float* out, cudaStream_t st) {
  dequantize_kernel<<<blocks_for((rows * cols + 255) / 256, 8), 256, 0, st>>>(codes, scales, g, rows, cols, mx, out);
  return cudaGetLastError();
}

cudaError_t launch_set_value(float* p, float v, cudaStream_t st) {
  set_value_kernel<<<1, 1, 0, st>>>(p, v);
  return cudaGetLastError();
}

cudaError_t launch_global_scale(const float* amax, float* g, unsigned* status, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, global_scale_kernel, amax, g, status);
}

cudaError_t launch_debug_encode(const float* in, int64_t n, int which, uint8_t* out, cudaStream_t st) {
  debug_encode_kernel<<<blocks_for((n + 255) / 256, 16), 256, 0, st>>>(in, n, which, out);
  return cudaGetLastError();
}

}  // namespace fp4
