// fp4_gemm.cu -- block-scaled FP4 GEMM on the sm_100a tensor cores (tcgen05).
//
// Computes D = gA * gB * (A_hat . B_hat^T) where A_hat / B_hat are E2M1 codes times
// their block scales ("Rubin FP4 GEMM overview", yfxerp.com, 3.1: the block scale
// factors are re-applied on the FP32 accumulators; 3.2: global -> shared -> tensor core
// -> FP32 accumulators -> epilogue; 4.2: the global scale product is fused into the
// epilogue so no extra pass over memory is needed).
//
// Structure (one CTA per SM, persistent).  128/256-wide tiles, one pipeline per CTA:
//   warp 0      TMA producer: per 256-wide K step, one 128 x 128-byte box of A, one
//               BN x 128-byte box of B (both 128-byte swizzled) on the stage's barrier,
//               and the matching 512-byte scale-factor atoms (issued first) on a
//               barrier of their own, into a STAGES-deep ring.
//   warp 1      TMEM owner; lane 0 issues tcgen05.mma.kind::mxf4nvf4 (NVFP4,
//               scale_vec::4X, UE4M3) or kind::mxf4 (MXFP4, scale_vec::2X, UE8M0),
//               M=128, N=BN, K=64 each, accumulating in TMEM; commits free the ring
//               slot and, at the end of a tile, hand the accumulator to the epilogue.
//   warps 2..9  epilogue: two warps per TMEM lane quarter (warp w reads lanes
//               32*(w%4)..+31), one per column half; multiply by gA*gB, BF16 (RNE) or
//               FP32 stores.  BF16 row-major tiles are packed into registers and the
//               accumulator is handed back before the stores.
//   warps 10..  scale-factor copiers (one for A's atoms, one per 128-row block of B's):
//               tcgen05.cp of a stage's atoms into a TMEM slot, replicated to the four
//               sub-partitions, while the MMA thread works on earlier stages.
// 256-wide tiles with M >= 256 run on CTA pairs (clusters of two): the pair computes a
// 256 x 256 tile with M=256 MMAs (tcgen05 .cta_group::2) issued by the leader; each CTA
// loads its own 128 rows of A and half of B's rows (so each SM moves a third fewer
// operand bytes per MMA), all TMA bytes complete on the leader's barriers, and the
// leader's commits arrive on both CTAs' barriers.
// Small-N tiles (16..64) run two independent pipelines of 6 warps per CTA, whose MMA
// thread also issues the scale-factor copies.
// Schedules: whole tiles (grouped raster for L2 reuse); stream-K over (tile, K-step)
// units when there are too few tiles to fill the SMs -- each CTA adds its FP32 partial
// tiles into a workspace with vector reductions, and the one whose part completes a
// tile's K range reads it back, scales, converts, stores and clears it; grouped MoE
// tiles enumerated on the device from the expert offsets.
// Decode-sized M (<= 64) runs with the operands swapped: the weight rows fill MMA-M and
// the few activation rows are MMA-N (16/32/64), which keeps the tensor-core work held per
// pipeline stage small and therefore many stages of weights in flight.
// Scale-factor TMEM addresses are always multiples of 4 columns (one 128-row atom per
// 4 columns); the hardware faults on other alignments.
// Launched with programmatic dependent launch: the prologue overlaps the previous
// kernel; global memory is touched only after griddepcontrol.wait.
// No TMA multicast is used anywhere.  Every wait is bounded (fp4_ptx.cuh); on a timeout
// the CTA latches the status word, drains its in-flight copies and MMAs, frees TMEM and
// returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "fp4_codes.cuh"
#include "fp4_internal.h"
#include "fp4_ptx.cuh"

namespace fp4 {

enum { kModeTile = 0, kModeStreamK = 1, kModeGrouped = 2 };

struct GemmArgs {
  const uint8_t* sfa;
  const uint8_t* sfb;
  int64_t sfa_rb_bytes;     // bytes per 128-row block of A's scales
  int64_t sfb_rb_bytes;
  int64_t sfb_group_bytes;  // grouped: bytes of one expert's B scales
  int sf_atoms_k;           // scale atoms along K per row-block
  int sfb_rbs;              // row-blocks of B (per expert)
  const float* ga;
  const float* gb;
  int Mk, Nk, K, num_kb;    // kernel orientation
  void* out;
  int64_t ldo;
  int out_bf16, transposed, vec_store;
  int indep;  // 1: kernel A, 2: kernel B may be read before the preceding kernel finishes
  float* ws;        // stream-K: FP32 partial sums [Mk, Nk], zero between calls
  int* tile_cnt;    // stream-K: K steps summed so far per tile, zero between calls
  int mode;
  int tiles_m, tiles_n, group_m;
  int64_t total_units;
  int num_groups;
  const int32_t* offsets;
  int b_rows_per_group;
  unsigned* status;
  // epilogue after the scale ("Rubin FP4 GEMM overview" 3.2 / 4.2): + bias[n], activation,
  // and optionally an NVFP4 copy of the result (16-blocks along n, caller's global scale)
  const float* bias;   // [N] (output columns), or null
  int act;             // 0: none, 1: ReLU
  uint8_t* q_codes;    // [M, N/2] NVFP4 codes of the result, or null
  uint8_t* q_scales;   // swizzled scale atoms of the [M, N/16] block scales
  const float* q_g;    // global scale of the NVFP4 result (device)
  int64_t q_atoms;     // scale atoms per 128-row block of the result: ceil(N/16, 4) / 4
  unsigned* amax_out;  // max |result| as float bits (zeroed before the launch), or null
  uint32_t f8_fmt;     // kind::mxf8f6f4: A's format | B's format << 3 (E4M3 0, E2M1 5)
};

struct Work {
  int a_row, b_row;    // TMA row coordinates of the A and B boxes
  int out_row0;        // first output row (kernel orientation)
  int rows_valid;      // rows of the tile that exist
  int n0;              // first column (kernel orientation)
  int sfa_rb;          // A scale row-block
  int64_t sfb_off;     // byte offset of B's first scale row-block
  int group;
  int kb0, kb1;
  int tile;
};

template <int BN>
struct Sched {
  const GemmArgs& p;
  const int* s_mt;   // grouped: 128-row block prefix per group (= A scale row-blocks)
  const int* s_off;  // grouped: row offsets
  const int* s_pt;   // grouped CTA pairs: 256-row tile prefix per group
  int64_t u, u_end;  // stream-K: current / end unit; tile modes: current unit
  int64_t total;

  int vgrid;         // pipelines in the grid; this one is number vb
  int mtile;         // output rows per M tile: 128, or 256 for a CTA pair
  int sub_row;       // CTA pair: this CTA's first row (and first B row) within the tile
  // vb / vg: this pipeline's index among all pipelines of the grid, and their count
  __device__ Sched(const GemmArgs& args, const int* mt, const int* off, int vb, int vg, int mtile_ = 128,
                   int sub_row_ = 0, const int* pt = nullptr)
      : p(args), s_mt(mt), s_off(off), s_pt(pt), vgrid(vg), mtile(mtile_), sub_row(sub_row_) {
    if (p.mode == kModeStreamK) {
      const int64_t T = p.total_units;
      u = T * vb / vg;
      u_end = T * (vb + 1) / vg;
      total = T;
    } else if (p.mode == kModeGrouped) {
      total = static_cast<int64_t>(tiles_prefix()[p.num_groups]) * p.tiles_n;
      u = vb;
    } else {
      total = p.total_units;
      u = vb;
    }
  }

  __device__ bool next(Work& w) {
    if (p.mode == kModeStreamK) {
      if (u >= u_end) return false;
      const int tile = static_cast<int>(u / p.num_kb);
      const int kb0 = static_cast<int>(u % p.num_kb);
      const int64_t kb1_ = static_cast<int64_t>(kb0) + (u_end - u);
      const int kb1 = static_cast<int>(kb1_ < p.num_kb ? kb1_ : p.num_kb);
      u += kb1 - kb0;
      const int mt = tile / p.tiles_n, nt = tile % p.tiles_n;
      plain(w, mt, nt);
      w.kb0 = kb0;
      w.kb1 = kb1;
      w.tile = tile;
      return true;
    }
    if (u >= total) return false;
    const int64_t cur = u;
    u += vgrid;
    if (p.mode == kModeGrouped) {
      const int E = p.num_groups;
      const int* tp = tiles_prefix();
      int lo = 0, hi = E - 1;  // last group e with tp[e] * tiles_n <= cur
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (static_cast<int64_t>(tp[mid]) * p.tiles_n <= cur) lo = mid;
        else hi = mid - 1;
      }
      const int e = lo;
      const int mte = tp[e + 1] - tp[e];
      const int64_t local = cur - static_cast<int64_t>(tp[e]) * p.tiles_n;
      const int nt = static_cast<int>(local / mte), mt = static_cast<int>(local % mte);
      // a pair's second CTA may get rows of the next group (or none): they are loaded
      // and multiplied but never stored
      w.a_row = s_off[e] + mt * mtile + sub_row;
      w.out_row0 = w.a_row;
      w.rows_valid = max(0, min(128, s_off[e + 1] - w.a_row));
      w.n0 = nt * BN;
      w.b_row = e * p.b_rows_per_group + w.n0 + sub_row;
      w.sfa_rb = s_mt[e] + mt * (mtile / 128) + sub_row / 128;
      w.sfb_off = e * p.sfb_group_bytes + static_cast<int64_t>(w.n0 / 128) * p.sfb_rb_bytes;
      w.group = e;
      w.kb0 = 0;
      w.kb1 = p.num_kb;
      w.tile = static_cast<int>(cur);
      return true;
    }
    // tile mode: rasterize in groups of group_m m-tiles so concurrently running CTAs
    // share A and B tiles in L2
    const int per_group = p.group_m * p.tiles_n;
    const int gi = static_cast<int>(cur / per_group);
    const int first_m = gi * p.group_m;
    const int gsize = min(p.tiles_m - first_m, p.group_m);
    const int r = static_cast<int>(cur % per_group);
    plain(w, first_m + r % gsize, r / gsize);
    w.kb0 = 0;
    w.kb1 = p.num_kb;
    w.tile = static_cast<int>(cur);
    return true;
  }

  // grouped: M-tile prefix per group in this schedule's tile height
  __device__ const int* tiles_prefix() const { return mtile == 256 ? s_pt : s_mt; }

  __device__ void plain(Work& w, int mt, int nt) {
    w.a_row = mt * mtile + sub_row;
    w.out_row0 = w.a_row;
    w.rows_valid = max(0, min(128, p.Mk - w.a_row));
    w.n0 = nt * BN;
    w.b_row = w.n0 + sub_row;  // a pair's CTAs each load half of the tile's B rows
    w.sfa_rb = w.a_row / 128;
    w.sfb_off = static_cast<int64_t>(w.n0 / 128) * p.sfb_rb_bytes;
    w.group = 0;
  }
};

// Small-N tiles (decode) run two independent pipelines per CTA ("sub-CTAs" of 192
// threads, each with its own producer, MMA issuer, epilogue warps, shared-memory ring
// and TMEM columns).  One thread issues all tcgen05 operations of a pipeline, and at
// N = 16..64 the issue latency of that thread -- not the tensor pipe -- bounds how fast
// weight stages are consumed, so two issuers per SM double the rate.  (Two CTAs per SM
// would do the same, but a kernel that allocates TMEM is scheduled one CTA per SM.)
#ifndef FP4_SMALL_N_PIPES
#define FP4_SMALL_N_PIPES 2
#endif
template <int BN>
constexpr int pipes_per_cta() { return BN <= 32 ? FP4_SMALL_N_PIPES : BN <= 64 ? 2 : 1; }

// F8: the kind::mxf8f6f4 MMA (E2M1 or E4M3 operands, one byte per element in shared
// memory, an E8M0 scale per 32): a stage holds 128 K elements, one scale atom per row-block.
template <int BN, bool MX, int ACC, bool PAIR = false, bool F8 = false>
struct Cfg {
  static_assert(!F8 || MX, "mixed-format MMAs: E8M0 scales");
  static_assert(!PAIR || (BN == 256 && ACC == 1), "CTA pairs run 256 x 256 tiles");
  static constexpr int kP = pipes_per_cta<BN>();
  // Single-pipeline kernels (128/256-wide tiles) add copier warps that move each stage's
  // scale factors into TMEM, so that these copies are not serialised behind the MMA
  // thread's own MMAs: one for A's atoms and one per 128-row block of B's.
  static constexpr bool kSepCp = kP == 1;
  static constexpr int kCopiers = kSepCp ? 1 + (BN >= 128 ? BN / 128 : 1) : 0;
  // One-pipeline kernels run two epilogue warps per TMEM lane quarter, one per column
  // half: twice the TMEM read and store rate, and half a row of packed BF16 per thread
  // is few enough registers to hold the tile while TMEM is already handed back.
  static constexpr int kEpiWarps = kSepCp ? 8 : 4;
  static constexpr int kEpiCols = BN * 4 / kEpiWarps;  // accumulator columns per epilogue thread
  static constexpr int kThreads = kSepCp ? 64 + 32 * kEpiWarps + 32 * kCopiers : 192 * kP;
  static constexpr int kAtomsKT = F8 ? 1 : MX ? 2 : 4;  // scale atoms per stage (256 K; 128 K for F8)
  static constexpr int kNRB = BN >= 128 ? BN / 128 : 1;  // B scale row-blocks per tile
  static constexpr int kABytes = 128 * 128;
  static constexpr int kBBytes = (PAIR ? BN / 2 : BN) * 128;  // a pair's CTA holds half of B's rows
  static constexpr int kSFABytes = kAtomsKT * 512;
  static constexpr int kSFBBytes = kNRB * kAtomsKT * 512;
  // rounded up to 1024 bytes (the 128-byte swizzle's alignment): only the mixed-format
  // stages (one scale atom per row-block) need the padding
  static constexpr int kStageBytes = (kABytes + kBBytes + kSFABytes + kSFBBytes + 1023) / 1024 * 1024;
  // grouped schedules use 128-wide tiles only, so multi-pipeline kernels skip the group tables
  static constexpr int kGroupBytes = kP == 1 ? (PAIR ? 3 : 2) * (kMaxGroups + 1) * 4 : 0;
  static constexpr int kMiscBytes = 1024 /*barriers, flags*/ + kGroupBytes;
  // the opt-in limit per block, less the alignment slack and the static shared memory
  static constexpr int kSmemLimit = 227 * 1024 - 1024 - 256;
  static constexpr int kStagesFit = (kSmemLimit / kP - kMiscBytes) / kStageBytes;
  static constexpr int kStages = kStagesFit > 12 ? 12 : kStagesFit;
  // one pipeline's share; the next pipeline's stages start 1024-byte aligned
  static constexpr int kSubBytes = (kStages * kStageBytes + kMiscBytes + 1023) / 1024 * 1024;
  static constexpr int kSmemBytes = kP == 1 ? kStages * kStageBytes + kMiscBytes + 1024 : kP * kSubBytes + 1024;
  static_assert(kSmemBytes + 256 <= 227 * 1024, "shared memory opt-in limit");
  static constexpr int kSFACols = kAtomsKT * 4;
  static constexpr int kSFBCols = kNRB * kAtomsKT * 4;
  static constexpr int kSFSlot = kSFACols + kSFBCols;
  // TMEM slots for the stages' scale factors: with a separate copier, as many as fit
  // (up to 4, and fewer than the ring's stages) so that it can run ahead of the MMAs
  static constexpr int kSlotsFit = (512 - ACC * BN) / kSFSlot;
  static constexpr int kSFSlots = !kSepCp ? 2 : (kSlotsFit < 4 ? kSlotsFit : 4) < kStages ? (kSlotsFit < 4 ? kSlotsFit : 4)
                                                                                           : kStages - 1;
  static constexpr int kColsUsed = ACC * BN + kSFSlots * kSFSlot;
  static constexpr int kTmemCols = kColsUsed <= 32 ? 32 : kColsUsed <= 64 ? 64 : kColsUsed <= 128 ? 128
                                   : kColsUsed <= 256 ? 256 : 512;  // per pipeline
  // one allocation for all pipelines: a power of two of at least 32 columns
  static constexpr int kTmemAlloc = kP * kTmemCols <= 32 ? 32 : kP * kTmemCols <= 64 ? 64
                                    : kP * kTmemCols <= 128 ? 128 : kP * kTmemCols <= 256 ? 256 : 512;
  static_assert(kP * kTmemCols <= 512, "TMEM budget");
  static_assert(kSFSlots >= 2 && kSFSlots < kStages, "scale-factor slots");
  static_assert(kStageBytes % 1024 == 0 && kSubBytes % 1024 == 0, "128-byte swizzled stages need 1024-byte alignment");
  static_assert(kStages >= 2, "shared memory budget");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
};

__device__ __forceinline__ void latch_timeout(volatile int* abort, unsigned* status) {
  *abort = 1;
  atomicOr(status, kStatusTimeout);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

// Waits until the grids this one depends on (programmatic dependent launch) have
// finished and their writes are visible; a no-op when launched without the attribute.
__device__ __forceinline__ void wait_prior_grids() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Lets the kernel launched after this one on the stream start its prologue now (it still
// waits for this grid's completion before it reads what this grid writes).
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void store_out(const GemmArgs& p, int64_t off, float v) {
  if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.out)[off] = __float2bfloat16_rn(v);
  else reinterpret_cast<float*>(p.out)[off] = v;
}

// Stores 16 consecutive kernel columns [col, col+16) of one kernel row.  With swapped
// operands (transposed) kernel row = output column and kernel column = output row.
__device__ __forceinline__ void store_row16(const GemmArgs& p, int row, int col, const float (&v)[16]) {
  if (p.transposed) {
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (col + j < p.Nk) store_out(p, static_cast<int64_t>(col + j) * p.ldo + row, v[j]);
    return;
  }
  const int64_t base = static_cast<int64_t>(row) * p.ldo + col;
  if (p.vec_store && col + 16 <= p.Nk) {
    if (p.out_bf16) {
      uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.out) + base);
      dst[0] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                          pack_bf16x2(v[6], v[7]));
      dst[1] = make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                          pack_bf16x2(v[14], v[15]));
    } else {
      float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + base);
#pragma unroll
      for (int j = 0; j < 4; ++j) dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    }
    return;
  }
#pragma unroll
  for (int j = 0; j < 16; ++j)
    if (col + j < p.Nk) store_out(p, base + j, v[j]);
}

// Bias and activation of 16 consecutive kernel columns [col, col+16) of kernel row `row`
// (values already multiplied by gA * gB).  With swapped operands the kernel row is the
// output column, which indexes the bias.
__device__ __forceinline__ void epi_bias_act(const GemmArgs& p, int row, int col, float (&v)[16]) {
  if (p.bias) {
    if (p.transposed) {
      const float b = p.bias[row];
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = __fadd_rn(v[j], b);
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (col + j < p.Nk) v[j] = __fadd_rn(v[j], __ldg(p.bias + col + j));
    }
  }
  if (p.act == 1) {
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = fmaxf(v[j], 0.0f);
  }
}

// NVFP4 copy of 16 output columns [col, col+16) of output row `row` (one block; the
// caller guarantees N % 32 == 0 and a row-major kernel orientation): block scale and
// codes exactly as the quantize kernels compute them, with the caller's global scale.
__device__ __forceinline__ void epi_quantize16(const GemmArgs& p, int row, int col, const float (&v)[16]) {
  const float g = *p.q_g;
  uint32_t m = 0;
#pragma unroll
  for (int j = 0; j < 16; ++j) m = max(m, __float_as_uint(v[j]) & 0x7FFFFFFFu);
  uint32_t sb;
  const float mul = nvfp4_block_scale(__uint_as_float(m), g, sb);
  float a[8], b[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    a[j] = v[j] == 0.0f ? v[j] : __fmul_rn(v[j], mul);  // a zero stays zero if 1/denom overflowed
    b[j] = v[8 + j] == 0.0f ? v[8 + j] : __fmul_rn(v[8 + j], mul);
  }
  *reinterpret_cast<uint2*>(p.q_codes + static_cast<int64_t>(row) * (p.Nk / 2) + col / 2) =
      make_uint2(pack8<kE2M1Hardware>(a), pack8<kE2M1Hardware>(b));
  const int c = col / 16;
  p.q_scales[((row / 128) * p.q_atoms + c / 4) * 512 + (row % 32) * 16 + ((row % 128) / 32) * 4 + c % 4] =
      static_cast<uint8_t>(sb);
}

// Finishes 16 consecutive kernel columns of one kernel row: bias, activation, the
// BF16 / FP32 store and the NVFP4 copy.
__device__ __forceinline__ void epi_row16(const GemmArgs& p, int row, int col, float (&v)[16], uint32_t& tmax) {
  epi_bias_act(p, row, col, v);
  if (p.out) store_row16(p, row, col, v);
  if (p.q_codes && col < p.Nk) epi_quantize16(p, row, col, v);
  if (p.amax_out) {  // the result's amax, for the global scale of its next quantization
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (p.transposed || col + j < p.Nk) tmax = max(tmax, __float_as_uint(v[j]) & 0x7FFFFFFFu);
  }
}

// Named barrier among the epilogue threads of one pipeline.
__device__ __forceinline__ void epi_sync(int sub, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(1 + sub), "r"(nthreads) : "memory");
}

template <int BN, bool MX, int ACC, bool PAIR, bool F8 = false>
__global__ void __launch_bounds__(Cfg<BN, MX, ACC, PAIR, F8>::kThreads, 1)
    fp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                    const GemmArgs p) {
  using C = Cfg<BN, MX, ACC, PAIR, F8>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem_base;
  const int sub = C::kP == 1 ? 0 : threadIdx.x / 192;  // pipeline of this thread
  const int lt = C::kP == 1 ? threadIdx.x : threadIdx.x % 192;
  const int warp = lt >> 5, lane = lt & 31;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023)) +
                  sub * C::kSubBytes;
  uint8_t* misc = smem + S * C::kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(misc);
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;
  uint64_t* acc_empty = acc_full + ACC;
  uint64_t* drain = acc_empty + ACC;
  uint64_t* sf_full = drain + 1;                // [kSFSlots]: stage scale factors are in TMEM slot i
  uint64_t* cp_drain = sf_full + C::kSFSlots;   // the copier warps' last copies have completed
  // [S]: a stage's scale factors have landed.  With a separate copier they complete on
  // their own barrier (and are issued first), so that the copier warps move them into TMEM
  // while the stage's operand tiles are still arriving; otherwise they complete on full.
  uint64_t* sf_landed = cp_drain + 1;
  volatile int* s_abort = reinterpret_cast<volatile int*>(sf_landed + S);
  volatile int* s_epi_fail = s_abort + 1;
  volatile int* s_last = s_abort + 2;  // stream-K: this pipeline completes the current tile
  int* s_mt = reinterpret_cast<int*>(misc + 1024);
  int* s_off = s_mt + (kMaxGroups + 1);
  int* s_pt = PAIR ? s_off + (kMaxGroups + 1) : nullptr;
  // A CTA pair (cluster of two) shares one 256 x 256 tile: rank 0, the leader, issues the
  // MMAs and scale-factor copies for both; each CTA loads its own 128 rows of A, its half
  // of B's rows, its A scales and all of the tile's B scales, and stores its 128 rows.
  const uint32_t rank = PAIR ? cluster_rank() : 0u;
  const bool leader = rank == 0;
  const int vb = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x) * C::kP + sub;
  const int vg = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x) * C::kP;
  constexpr int kMTile = PAIR ? 256 : 128;
  const int sub_row = static_cast<int>(rank) * 128;

  // prologue (overlaps the tail of the previous kernel under programmatic launch)
  if (lt == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_landed[s], 1);
    }
    for (int a = 0; a < ACC; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], (PAIR ? 2 : 1) * C::kEpiWarps);  // a pair: both CTAs' epilogue warps
    }
    mbar_init(drain, 1);
    for (int i = 0; i < C::kSFSlots; ++i) mbar_init(&sf_full[i], C::kSepCp ? C::kCopiers : 1);
    mbar_init(cp_drain, C::kSepCp ? C::kCopiers : 1);
    *s_abort = 0;
    *s_epi_fail = 0;
    *s_last = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (PAIR) {
      tma_prefetch_desc(&tmSFA);
      tma_prefetch_desc(&tmSFB);
    }
  }
  if (sub == 0 && warp == 1) {  // one allocation for all pipelines of the CTA
    if constexpr (PAIR) {       // the same columns in both CTAs of the pair
      tmem_alloc_pair(&s_tmem_base, C::kTmemAlloc);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(&s_tmem_base, C::kTmemAlloc);
      tmem_relinquish();
    }
  }
  // the next kernel on the stream may launch now; it waits for this grid to complete
  allow_dependents();
  if (p.mode == kModeGrouped && warp == 2) {
    wait_prior_grids();  // the offsets may come from the previous kernel
    // m-tile prefix per group (= scale row-block prefix of the grouped A layout)
    const int E = p.num_groups;
    // (CTA pairs: also the prefix of 256-row tiles, by which they enumerate tiles)
    int carry = 0, carry2 = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      int cnt = 0, cnt2 = 0;
      if (e < E) {
        const int lo = p.offsets[e], hi = p.offsets[e + 1];
        s_off[e] = lo;
        cnt = (hi - lo + 127) / 128;
        cnt2 = (hi - lo + 255) / 256;
      }
      int incl = cnt, incl2 = cnt2;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int t = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        const int t2 = __shfl_up_sync(0xFFFFFFFFu, incl2, d);
        if (lane >= d) {
          incl += t;
          incl2 += t2;
        }
      }
      if (e < E) {
        s_mt[e] = carry + incl - cnt;
        if (PAIR) s_pt[e] = carry2 + incl2 - cnt2;
      }
      carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
      carry2 += __shfl_sync(0xFFFFFFFFu, incl2, 31);
    }
    if (lane == 0) {
      s_mt[E] = carry;
      if (PAIR) s_pt[E] = carry2;
      s_off[E] = p.offsets[E];
    }
  }
  tc_fence_before();
  __syncthreads();
  // a pair: the peer's barriers are initialised before this CTA's loads and arrivals reach them
  if constexpr (PAIR) cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = s_tmem_base + sub * C::kTmemCols;
  const uint32_t sf_col0 = ACC * BN;
  // copies one stage's scale-factor atoms (A's, then B's row-blocks) into a TMEM slot
  auto copy_stage_sf = [&](uint32_t st, uint32_t sfa_t, int kb) {
    const uint32_t sfb_t = sfa_t + C::kSFACols;
    const int atoms = min(C::kAtomsKT, p.sf_atoms_k - kb * C::kAtomsKT);
    for (int a = 0; a < atoms; ++a) tc_cp_sf_atom(sfa_t + a * 4, smem_desc_sf(st + C::kABytes + C::kBBytes + a * 512));
#pragma unroll
    for (int rb = 0; rb < C::kNRB; ++rb)
      for (int a = 0; a < atoms; ++a)
        tc_cp_sf_atom(sfb_t + (a * C::kNRB + rb) * 4,
                      smem_desc_sf(st + C::kABytes + C::kBBytes + C::kSFABytes + (rb * C::kAtomsKT + a) * 512));
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      // swapped decode: the weights (A here) are read once -> evict first; the small
      // activations (B) are re-read by every CTA -> keep
      // otherwise both operands are re-read by other tiles -> keep (the output is stored
      // with the streaming hint, so that it does not push them out of L2)
      const uint64_t pol_a = p.transposed ? l2_policy_evict_first() : l2_policy_evict_last();
      const uint64_t pol_b = l2_policy_evict_last();
      // Loads of one stage: the A box and A scales ("a" side), the B box and B scales.
      auto load_side = [&](int st_idx, const Work& w, int kb, bool side_a) {
        uint8_t* st = smem + st_idx * C::kStageBytes;
        const int atoms = min(C::kAtomsKT, p.sf_atoms_k - kb * C::kAtomsKT);
        const uint32_t sf_bytes = static_cast<uint32_t>(atoms) * 512u;
        const int64_t koff = static_cast<int64_t>(kb) * C::kAtomsKT * 512;
        if constexpr (PAIR) {
          // every box in full (out-of-range rows read as zero), so that the leader can
          // expect a fixed byte count from both CTAs on its own barriers
          const uint32_t c_full = cluster_addr(smem_u32(&full[st_idx]), 0);
          const uint32_t c_sf = cluster_addr(smem_u32(&sf_landed[st_idx]), 0);
          if (side_a) {
            tma_load_2d_pair(st + C::kABytes + C::kBBytes, &tmSFA, c_sf, 0,
                             static_cast<int>((w.sfa_rb * p.sfa_rb_bytes + koff) / 256), pol_a);
            tma_load_2d_pair(st, &tmA, c_full, kb * 128, w.a_row, pol_a);
          } else {
#pragma unroll
            for (int rb = 0; rb < C::kNRB; ++rb)
              tma_load_2d_pair(st + C::kABytes + C::kBBytes + C::kSFABytes + rb * C::kAtomsKT * 512, &tmSFB, c_sf, 0,
                               static_cast<int>((w.sfb_off + rb * p.sfb_rb_bytes + koff) / 256), pol_b);
            tma_load_2d_pair(st + C::kABytes, &tmB, c_full, kb * 128, w.b_row, pol_b);
          }
          (void)sf_bytes;
          return;
        }
        uint64_t* sf_bar = C::kSepCp ? &sf_landed[st_idx] : &full[st_idx];
        if (side_a) {
          bulk_load(st + C::kABytes + C::kBBytes, p.sfa + w.sfa_rb * p.sfa_rb_bytes + koff, sf_bytes, sf_bar, pol_a);
          tma_load_2d(st, &tmA, &full[st_idx], kb * 128, w.a_row, pol_a);
        } else {
          const int rb0 = w.n0 / 128;
#pragma unroll
          for (int rb = 0; rb < C::kNRB; ++rb)
            if (rb0 + rb < p.sfb_rbs)
              bulk_load(st + C::kABytes + C::kBBytes + C::kSFABytes + rb * C::kAtomsKT * 512,
                        p.sfb + w.sfb_off + rb * p.sfb_rb_bytes + koff, sf_bytes, sf_bar, pol_b);
          tma_load_2d(st + C::kABytes, &tmB, &full[st_idx], kb * 128, w.b_row, pol_b);
        }
      };
      auto stage_sf_bytes = [&](const Work& w, int kb) -> uint32_t {
        const int atoms = min(C::kAtomsKT, p.sf_atoms_k - kb * C::kAtomsKT);
        const uint32_t sf_bytes = static_cast<uint32_t>(atoms) * 512u;
        const int rb0 = w.n0 / 128;
        int nrb = 0;
#pragma unroll
        for (int rb = 0; rb < C::kNRB; ++rb) nrb += (rb0 + rb < p.sfb_rbs) ? 1 : 0;
        return sf_bytes * (1 + nrb);
      };
      // With an independent operand, the first ring-full of stages loads only that side,
      // then waits for the preceding kernel, then issues the other side of those stages.
      const bool early = p.indep != 0;
      const bool early_a = p.indep == 1;
      int npend = 0;
      bool replayed = !early;
      auto replay = [&]() {
        wait_prior_grids();
        Sched<BN> rs(p, s_mt, s_off, vb, vg, kMTile, sub_row, s_pt);
        Work rw;
        int j = 0;
        while (j < npend && rs.next(rw))
          for (int kb = rw.kb0; kb < rw.kb1 && j < npend; ++kb, ++j) load_side(j, rw, kb, !early_a);
        replayed = true;
      };
      if (!early) wait_prior_grids();
      Sched<BN> sch(p, s_mt, s_off, vb, vg, kMTile, sub_row, s_pt);
      Work w;
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_par = 0;
      bool ok = true;
      // operand bytes a stage's tensor copies complete: a 4-bit operand of the mixed-format
      // MMA counts its packed bytes (half its footprint in shared memory)
      uint32_t ab_tx = C::kABytes + C::kBBytes;
      if constexpr (F8)
        ab_tx = ((p.f8_fmt & 7u) == kFmtE2M1 ? C::kABytes / 2 : C::kABytes) +
                (((p.f8_fmt >> 3) & 7u) == kFmtE2M1 ? C::kBBytes / 2 : C::kBBytes);
      while (ok && sch.next(w)) {
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, s_abort)) {
            latch_timeout(s_abort, p.status);
            ok = false;
            break;
          }
          if constexpr (PAIR) {
            if (leader) {  // the leader's barriers count the boxes of both CTAs
              mbar_arrive_expect_tx(&sf_landed[stage], 2 * (C::kSFABytes + C::kSFBBytes));
              mbar_arrive_expect_tx(&full[stage], 2 * ab_tx);
            }
          } else if constexpr (C::kSepCp) {
            mbar_arrive_expect_tx(&sf_landed[stage], stage_sf_bytes(w, kb));
            mbar_arrive_expect_tx(&full[stage], ab_tx);
          } else {
            mbar_arrive_expect_tx(&full[stage], C::kABytes + C::kBBytes + stage_sf_bytes(w, kb));
          }
          if (!replayed) {
            load_side(stage, w, kb, early_a);
            if (++npend == S) replay();
          } else {
            load_side(stage, w, kb, true);
            load_side(stage, w, kb, false);
          }
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (ok && !replayed) replay();
      // let every issued copy land before the CTA's shared memory goes away (a pair's
      // leader waits for both CTAs' boxes: they complete on its barriers)
      if (*s_abort && leader) {
        for (int s = 0; s < S; ++s)
          if (issued & (1u << s)) {
            volatile int no_abort = 0;
            mbar_wait(&full[s], (issued_par >> s) & 1u, &no_abort);
            if (C::kSepCp) mbar_wait(&sf_landed[s], (issued_par >> s) & 1u, &no_abort);
          }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------------------ MMA issuer
      Sched<BN> sch(p, s_mt, s_off, vb, vg, kMTile, sub_row, s_pt);
      const uint32_t smem_base = smem_u32(smem);
      Work w;
      int stage = 0, iter = 0, nstage = 0;
      uint32_t phase = 0, slot = 0;
      bool ok = true;
      while (ok && sch.next(w)) {
        const int acc = iter % ACC;
        if (!mbar_wait(&acc_empty[acc], ((iter / ACC) & 1) ^ 1, s_abort)) {
          latch_timeout(s_abort, p.status);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * BN;
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, s_abort)) {
            latch_timeout(s_abort, p.status);
            ok = false;
            break;
          }
          const uint32_t st = smem_base + stage * C::kStageBytes;
          const uint32_t sfa_t = tmem + sf_col0 + slot * C::kSFSlot;
          const uint32_t sfb_t = sfa_t + C::kSFACols;
          if constexpr (C::kSepCp) {
            // the copier warps have put this stage's scale factors into the slot
            if (!mbar_wait(&sf_full[slot], (nstage / C::kSFSlots) & 1, s_abort)) {
              latch_timeout(s_abort, p.status);
              ok = false;
              break;
            }
            tc_fence_after();
          } else {
            tc_fence_after();
            copy_stage_sf(st, sfa_t, kb);
          }
          ++nstage;
          const int krem = p.K - kb * (F8 ? 128 : 256);
          const int nk = F8 ? (krem >= 128 ? 4 : (krem + 31) / 32) : (krem >= 256 ? 4 : (krem + 63) / 64);
          const uint64_t adesc = smem_desc_sw128(st);
          const uint64_t bdesc = smem_desc_sw128(st + C::kABytes);
          if constexpr (F8) {
            // four K = 32 MMAs over the stage's 128-byte rows (one byte per element of
            // either format); MMA k reads byte k of each row's 32-bit scale word
            for (int k = 0; k < nk; ++k) {
              const uint32_t sfid = static_cast<uint32_t>(k);
              const uint32_t idesc = mma_idesc_f8(BN, p.f8_fmt & 7u, (p.f8_fmt >> 3) & 7u, sfid, sfid, kMTile);
              const uint32_t accum = (kb > w.kb0 || k > 0) ? 1u : 0u;
              if constexpr (PAIR)
                tc_mma_mxf8f6f4_pair(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, sfa_t | (sfid << 30),
                                     sfb_t | (sfid << 30), accum);
              else
                tc_mma_mxf8f6f4(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, sfa_t | (sfid << 30),
                                sfb_t | (sfid << 30), accum);
            }
          } else {
          for (int k = 0; k < nk; ++k) {
            const uint32_t a_idx = MX ? (k >> 1) : k;
            const uint32_t sfid = MX ? (k & 1) * 2 : 0;
            const uint32_t idesc = mma_idesc(BN, MX, sfid, sfid, kMTile);
            const uint32_t accum = (kb > w.kb0 || k > 0) ? 1u : 0u;
            const uint32_t ta = (sfa_t + a_idx * 4) | (sfid << 30);
            const uint32_t tb = (sfb_t + a_idx * C::kNRB * 4) | (sfid << 30);
            if constexpr (PAIR && MX)
              tc_mma_mxfp4_pair(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, ta, tb, accum);
            else if constexpr (PAIR)
              tc_mma_nvfp4_pair(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, ta, tb, accum);
            else if constexpr (MX)
              tc_mma_mxfp4(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, ta, tb, accum);
            else
              tc_mma_nvfp4(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, ta, tb, accum);
          }
          }
          if constexpr (PAIR)
            tc_commit_pair_mc(&empty[stage], 3);  // frees the stage in both CTAs
          else
            tc_commit(&empty[stage]);
          if (++slot == C::kSFSlots) slot = 0;
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        if constexpr (PAIR)
          tc_commit_pair_mc(&acc_full[acc], 3);  // both CTAs' epilogues
        else
          tc_commit(&acc_full[acc]);
        ++iter;
      }
      // make sure no MMA still writes TMEM when it is freed
      if constexpr (PAIR)
        tc_commit_pair(drain);
      else
        tc_commit(drain);
      volatile int no_abort = 0;
      mbar_wait(drain, 0, &no_abort);
    }
  } else if (C::kSepCp && warp >= 2 + C::kEpiWarps) {
    const int cw = warp - 2 - C::kEpiWarps;  // 0: A's atoms; 1 + rb: B's row-block rb
    if (lane == 0 && leader) {
      // ------------------------------------------------------------ scale-factor copier
      // Stage n's atoms go to TMEM slot n % kSFSlots once they have landed and the
      // MMAs of stage n - kSFSlots (the slot's previous user) have completed; each slot's
      // copies are committed to sf_full[slot] for the MMA thread.
      Sched<BN> sch(p, s_mt, s_off, vb, vg, kMTile, sub_row, s_pt);
      const uint32_t smem_base = smem_u32(smem);
      Work w;
      int stage = 0, n = 0;
      uint32_t phase = 0;
      bool ok = true;
      while (ok && sch.next(w)) {
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!mbar_wait(&sf_landed[stage], phase, s_abort)) {
            latch_timeout(s_abort, p.status);
            ok = false;
            break;
          }
          if (n >= C::kSFSlots) {
            const int prev = n - C::kSFSlots;
            if (!mbar_wait(&empty[prev % S], (prev / S) & 1, s_abort)) {
              latch_timeout(s_abort, p.status);
              ok = false;
              break;
            }
          }
          tc_fence_after();
          const uint32_t sl = n % C::kSFSlots;
          {
            const uint32_t st = smem_base + stage * C::kStageBytes;
            const uint32_t sfa_t = tmem + sf_col0 + sl * C::kSFSlot;
            const int atoms = min(C::kAtomsKT, p.sf_atoms_k - kb * C::kAtomsKT);
            auto cp = [&](uint32_t taddr, uint64_t sdesc) {
              if constexpr (PAIR)
                tc_cp_sf_atom_pair(taddr, sdesc);
              else
                tc_cp_sf_atom(taddr, sdesc);
            };
            if (cw == 0) {
              for (int a = 0; a < atoms; ++a) cp(sfa_t + a * 4, smem_desc_sf(st + C::kABytes + C::kBBytes + a * 512));
            } else {
              const int rb = cw - 1;
              for (int a = 0; a < atoms; ++a)
                cp(sfa_t + C::kSFACols + (a * C::kNRB + rb) * 4,
                   smem_desc_sf(st + C::kABytes + C::kBBytes + C::kSFABytes + (rb * C::kAtomsKT + a) * 512));
            }
          }
          if constexpr (PAIR)
            tc_commit_pair(&sf_full[sl]);
          else
            tc_commit(&sf_full[sl]);
          ++n;
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // no copy may still write TMEM when it is freed
      if constexpr (PAIR)
        tc_commit_pair(cp_drain);
      else
        tc_commit(cp_drain);
      volatile int no_abort = 0;
      mbar_wait(cp_drain, 0, &no_abort);
    }
  } else if (warp >= 2 && warp < 2 + C::kEpiWarps) {
    // ------------------------------------------------------------ epilogue
    // a warp reads the TMEM lane quarter given by its warp index in the CTA, modulo 4,
    // and (with eight epilogue warps) the column half given by its warp index over 4
    const int q = (threadIdx.x >> 5) & 3;
    const int rl = q * 32 + lane;     // accumulator row (TMEM lane) of this thread
    const int et = lt - 64;           // 0 .. 32 * kEpiWarps - 1
    constexpr int CH = C::kEpiCols;
    const int c0 = ((warp - 2) >> 2) * CH;  // first accumulator column of this thread
    // BF16 row-major tiles whose columns are all in range are converted into registers
    // and TMEM is handed back to the MMA thread before the stores, so that they overlap
    // the next tile's MMAs
    const bool early_release = C::kSepCp && p.mode != kModeStreamK && p.out && p.out_bf16 && !p.transposed &&
                               p.vec_store && !p.q_codes;
    // hands an accumulator back to the MMA thread (a pair's leader counts both CTAs' warps)
    auto release_acc = [&](int a) {
      if constexpr (PAIR)
        mbar_arrive_cluster(cluster_addr(smem_u32(&acc_empty[a]), 0));
      else
        mbar_arrive(&acc_empty[a]);
    };
    wait_prior_grids();               // the global scales come from earlier kernels
    const float ga = p.ga ? *p.ga : 1.0f;
    uint32_t tmax = 0;                // max |result| over this thread's values (amax_out)
    Sched<BN> sch(p, s_mt, s_off, vb, vg, kMTile, sub_row, s_pt);
    Work w;
    int iter = 0;
    while (sch.next(w)) {
      const int acc = iter % ACC;
      const uint32_t par = (iter / ACC) & 1;
      // the epilogue warps decide together whether to go on, so that none of them
      // is left behind at a named barrier
      if (et == 0 && !mbar_wait(&acc_full[acc], par, s_abort)) {
        latch_timeout(s_abort, p.status);
        *s_epi_fail = 1;
      }
      epi_sync(sub, 32 * C::kEpiWarps);
      if (*s_epi_fail) break;
      tc_fence_after();
      const float gb = p.gb ? p.gb[w.group] : 1.0f;
      const float scale = ga * gb;
      const bool row_ok = rl < w.rows_valid;
      const int row = w.out_row0 + rl;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + acc * BN;
      bool released = false;
      if (q * 32 < w.rows_valid && early_release && w.n0 + BN <= p.Nk) {  // warp-uniform
        uint32_t pk[CH / 2];  // this thread's columns [c0, c0 + CH) as scaled BF16 pairs
        // 32-column TMEM loads, one wait per load: the hand-back of the accumulator
        // waits for few TMEM round trips
        constexpr int kLdBatch = CH >= 32 ? 32 : CH;
        static_assert(CH % kLdBatch == 0 && kLdBatch % 16 == 0, "TMEM load batches");
#pragma unroll
        for (int cb = 0; cb < CH; cb += kLdBatch) {
          uint32_t rr[kLdBatch];
          if constexpr (kLdBatch % 32 == 0) {
#pragma unroll
            for (int h = 0; h < kLdBatch; h += 32) tmem_ld32(taddr + c0 + cb + h, rr + h);
          } else {
            tmem_ld16(taddr + c0 + cb, *reinterpret_cast<uint32_t(*)[16]>(rr));
          }
          tmem_ld_wait();
#pragma unroll
          for (int cw = 0; cw < kLdBatch; cw += 16) {
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(rr[cw + j]) * scale;
            if (p.bias || p.act) epi_bias_act(p, row, w.n0 + c0 + cb + cw, v);
            if (p.amax_out && row_ok) {
#pragma unroll
              for (int j = 0; j < 16; ++j) tmax = max(tmax, __float_as_uint(v[j]) & 0x7FFFFFFFu);
            }
#pragma unroll
            for (int j = 0; j < 16; j += 2) pk[(cb + cw + j) / 2] = pack_bf16x2(v[j], v[j + 1]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) release_acc(acc);
        released = true;
        if (row_ok) {
          __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.out) + static_cast<int64_t>(row) * p.ldo;
#pragma unroll
          for (int c = 0; c < CH; c += 8)  // streaming stores: the output is not read back here
            __stcs(reinterpret_cast<uint4*>(orow + w.n0 + c0 + c),
                   make_uint4(pk[c / 2], pk[c / 2 + 1], pk[c / 2 + 2], pk[c / 2 + 3]));
        }
      } else if (q * 32 < w.rows_valid) {  // warp-uniform: warps without a valid row skip TMEM
        // up to 64 columns per TMEM round trip (32 with eight epilogue warps), one wait
        constexpr int CW = C::kSepCp ? 32 : CH >= 64 ? 64 : CH;
#pragma unroll 1
        for (int cw = c0; cw < c0 + CH; cw += CW) {
          uint32_t rr[CW / 16][16];
#pragma unroll
          for (int h = 0; h < CW / 16; ++h) tmem_ld16(taddr + cw + h * 16, rr[h]);
          tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < CW / 16; ++h) {
          const int c = cw + h * 16;
          const uint32_t (&r)[16] = rr[h];
          const int col = w.n0 + c;
          if (!row_ok || col >= p.Nk) continue;
          if (p.mode == kModeStreamK) {
            float* dst = p.ws + static_cast<int64_t>(row) * p.Nk + col;
            if ((p.Nk & 3) == 0 && col + 16 <= p.Nk) {
#pragma unroll
              for (int j = 0; j < 16; j += 4)
                red_add_v4(dst + j, __uint_as_float(r[j]), __uint_as_float(r[j + 1]), __uint_as_float(r[j + 2]),
                           __uint_as_float(r[j + 3]));
            } else {
              for (int j = 0; j < 16 && col + j < p.Nk; ++j) atomicAdd(dst + j, __uint_as_float(r[j]));
            }
          } else {
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]) * scale;
            epi_row16(p, row, col, v, tmax);
          }
        }
        }
      }
      if (!released) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) release_acc(acc);
      }
      ++iter;
      if (p.mode == kModeStreamK) {
        // The pipeline whose partial sums complete the tile's K range writes the tile:
        // every pipeline publishes its reductions (fence), then adds the K steps it
        // covered to the tile's counter; the one that brings it to num_kb reads the
        // sums back from L2, scales, converts, stores, and clears sums and counter.
        __threadfence();
        epi_sync(sub, 32 * C::kEpiWarps);
        if (et == 0) {
          __threadfence();
          const int covered = w.kb1 - w.kb0;
          const int before = atomicAdd(p.tile_cnt + w.tile, covered);
          *s_last = before + covered == p.num_kb ? 1 : 0;
        }
        epi_sync(sub, 32 * C::kEpiWarps);
        if (*s_last) {
          __threadfence();
          if (row_ok) {
            float* src = p.ws + static_cast<int64_t>(row) * p.Nk;
            for (int c = c0; c < c0 + CH; c += 16) {
              const int col = w.n0 + c;
              if (col >= p.Nk) break;
              float v[16];
              if ((p.Nk & 3) == 0 && col + 16 <= p.Nk) {
#pragma unroll
                for (int j = 0; j < 16; j += 4) {
                  const float4 t = __ldcg(reinterpret_cast<const float4*>(src + col + j));
                  __stcg(reinterpret_cast<float4*>(src + col + j), make_float4(0.f, 0.f, 0.f, 0.f));
                  v[j] = t.x * scale;
                  v[j + 1] = t.y * scale;
                  v[j + 2] = t.z * scale;
                  v[j + 3] = t.w * scale;
                }
              } else {
                for (int j = 0; j < 16; ++j) {
                  v[j] = 0.0f;
                  if (col + j < p.Nk) {
                    v[j] = __ldcg(src + col + j) * scale;
                    __stcg(src + col + j, 0.0f);
                  }
                }
              }
              epi_row16(p, row, col, v, tmax);
            }
          }
          if (et == 0) p.tile_cnt[w.tile] = 0;
        }
      }
    }
    if (p.amax_out) {  // one atomic per warp: non-negative float bits order as integers
      tmax = __reduce_max_sync(0xFFFFFFFFu, tmax);
      if (lane == 0 && tmax) atomicMax(p.amax_out, tmax);
    }
  }

  tc_fence_before();
  __syncthreads();
  // a pair: neither CTA frees TMEM or leaves (its shared memory is the peer's operand and
  // barrier target) before both are done
  if constexpr (PAIR) cluster_sync_all();
  tc_fence_after();
  if (sub == 0 && warp == 1) {
    __syncwarp();
    if constexpr (PAIR)
      tmem_dealloc_pair(s_tmem_base, C::kTmemAlloc);
    else
      tmem_dealloc(s_tmem_base, C::kTmemAlloc);
  }
}

// ---------------------------------------------------------------------- host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// [rows, inner_bytes] uint8 matrix, boxes of box_rows x 128 bytes, 128-byte swizzle,
// out-of-bounds elements read as zero.
static bool encode_map(CUtensorMap* m, const void* base, uint64_t inner_bytes, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner_bytes, rows};
  const cuuint64_t strides[1] = {inner_bytes};
  const cuuint32_t box[2] = {128, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [rows, k] E2M1 codes, packed two per byte in global memory (row pitch k / 2 bytes),
// copied into shared memory one byte per element: each 16 codes (8 bytes) followed by an
// 8-byte gap, the operand layout of the kind::mxf8f6f4 MMA.  CUDA's documented limits for
// this data type: a 32-byte aligned base, k a multiple of 128, a row pitch that is a
// multiple of 32 bytes, and boxes 128 elements wide.
static bool encode_map_u4(CUtensorMap* m, const void* base, uint64_t k, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {k, rows};
  const cuuint64_t strides[1] = {k / 2};
  const cuuint32_t box[2] = {128, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Small host cache of encoded tensor maps keyed by (address, shape, box): decode-style
// callers pass the same buffers every step, and encoding costs host time on every call.
// A map only describes addresses, so a stale entry is just another valid encoding.
struct MapCacheEntry {
  const void* base;
  uint64_t inner, rows;
  uint32_t box;
  CUtensorMap map;
};
bool make_tensor_map_u8(CUtensorMap* m, const void* base, uint64_t inner_bytes, uint64_t rows, uint32_t box_rows) {
  constexpr int kEntries = 32;
  static MapCacheEntry cache[kEntries];
  static int used = 0, next = 0;
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i) {
      const MapCacheEntry& e = cache[i];
      if (e.base == base && e.inner == inner_bytes && e.rows == rows && e.box == box_rows) {
        *m = e.map;
        return true;
      }
    }
  }
  if (!encode_map(m, base, inner_bytes, rows, box_rows)) return false;
  std::lock_guard<std::mutex> lock(mu);
  MapCacheEntry& e = cache[next];
  e.base = base;
  e.inner = inner_bytes;
  e.rows = rows;
  e.box = box_rows;
  e.map = *m;
  next = (next + 1) % kEntries;
  if (used < kEntries) ++used;
  return true;
}

// A scale-factor buffer as a [bytes / 256, 256] uint8 matrix, boxes of box_rows x 256
// bytes, no swizzle, rows past the end read as zero: a CTA pair loads a stage's scale
// atoms with tensor copies (their completion can be counted on the leader's barrier).
static bool encode_sf_map(CUtensorMap* m, const void* base, uint64_t bytes, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {256, bytes / 256};
  const cuuint64_t strides[1] = {256};
  const cuuint32_t box[2] = {256, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static bool make_sf_map(CUtensorMap* m, const void* base, uint64_t bytes, uint32_t box_rows) {
  constexpr int kEntries = 16;
  static MapCacheEntry cache[kEntries];
  static int used = 0, next = 0;
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i) {
      const MapCacheEntry& e = cache[i];
      if (e.base == base && e.inner == 256 && e.rows == bytes / 256 && e.box == box_rows) {
        *m = e.map;
        return true;
      }
    }
  }
  if (!encode_sf_map(m, base, bytes, box_rows)) return false;
  std::lock_guard<std::mutex> lock(mu);
  MapCacheEntry& e = cache[next];
  e.base = base;
  e.inner = 256;
  e.rows = bytes / 256;
  e.box = box_rows;
  e.map = *m;
  next = (next + 1) % kEntries;
  if (used < kEntries) ++used;
  return true;
}

struct Plan {
  bool swap;
  bool pair;  // 256 x 256 tiles on CTA pairs
  int BN, ACC, mode;
  int64_t Mk, Nk;
  int tiles_m, tiles_n, num_kb;
  int64_t units;
  size_t ws_bytes;
};

// `groups` is the number of experts of a grouped problem, 0 for a plain GEMM.
static Plan make_plan(int64_t M, int64_t N, int64_t K, int groups, int mx, bool row_major_out = false) {
  Plan pl{};
  pl.num_kb = static_cast<int>((K + 255) / 256);
  (void)mx;
  if (groups) {
    // 256-wide tiles: per MMA the scale-factor copies into TMEM cost less than with
    // 128-wide ones (an expert's last N-tile may be half empty; its extra columns, read
    // from the next expert's rows, are never stored)
    pl.swap = false;
    pl.BN = N >= 256 ? 256 : 128;
    pl.ACC = pl.BN == 256 ? 1 : 2;
    // 256 x 256 tiles on CTA pairs load a third fewer bytes per MMA, but an expert's last
    // row tile is on average half empty: 128 rows of padding per expert instead of 64.
    // With experts of a few hundred rows (top-k routing of a few thousand tokens) the
    // padding costs more than the pairs save (measured on 32 experts of ~512 rows:
    // 128-row tiles 5% faster per clock); pairs from 1280 rows per expert on average.
    pl.pair = pl.BN == 256 && M >= 1280 * static_cast<int64_t>(groups);
    pl.mode = kModeGrouped;
    pl.Mk = M;
    pl.Nk = N;
    pl.tiles_n = static_cast<int>((N + pl.BN - 1) / pl.BN);
    pl.ws_bytes = 0;
    return pl;
  }
  if (M <= 64 && !row_major_out) {  // decode: weight rows fill MMA-M, the few activation rows are MMA-N
    pl.swap = true;
    pl.Mk = N;
    pl.Nk = M;
    pl.BN = M <= 16 ? 16 : M <= 32 ? 32 : 64;
    pl.ACC = 2;
  } else {
    pl.swap = false;
    pl.Mk = M;
    pl.Nk = N;
    // 256-wide tiles when there are enough of them to fill the SMs, else 128-wide
    const int64_t tiles256 = ((M + 127) / 128) * ((N + 255) / 256);
    pl.BN = (N >= 256 && tiles256 >= num_sms()) ? 256 : 128;
    pl.ACC = pl.BN == 256 ? 1 : 2;
  }
  pl.tiles_m = static_cast<int>((pl.Mk + 127) / 128);
  pl.tiles_n = static_cast<int>((pl.Nk + pl.BN - 1) / pl.BN);
  const int64_t tiles = static_cast<int64_t>(pl.tiles_m) * pl.tiles_n;
  const int sms = num_sms();
  // Too few tiles to fill the SMs: split every tile's K range across CTAs (stream-K).
  // Swapped (decode-like) shapes split whenever tiles are scarce; the others only when
  // K is long enough that the split's partial-sum traffic stays small against the MMAs.
  if (tiles < 2 * sms && pl.num_kb >= 4 && (pl.swap || (2 * tiles < sms && pl.num_kb >= 16))) {
    pl.mode = kModeStreamK;
    pl.units = tiles * pl.num_kb;
    pl.ws_bytes = (static_cast<size_t>(M * N) * 4 + 255) / 256 * 256 + (static_cast<size_t>(tiles) * 4 + 255) / 256 * 256;
  } else {
    pl.mode = kModeTile;
    pl.units = tiles;
    pl.ws_bytes = 0;
    // 256-wide tiles with at least two 128-row blocks: CTA pairs share 256 x 256 tiles,
    // so that each SM loads a third fewer operand bytes per MMA
    if (pl.BN == 256 && !pl.swap && M >= 256) {
      pl.pair = true;
      pl.tiles_m = static_cast<int>((pl.Mk + 255) / 256);
      pl.units = static_cast<int64_t>(pl.tiles_m) * pl.tiles_n;
    }
  }
  return pl;
}

size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int mx, bool fp4_out) {
  if (!mx && !fp4_out && decode_eligible(M, N, K)) return decode_workspace_bytes(M, N);
  return make_plan(M, N, K, 0, mx, fp4_out).ws_bytes;
}

// the quantize workspace (tensor amax), then the GEMM's
size_t gemm_bf16a_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  return (kQuantWorkspaceBytes + 255) / 256 * 256 + gemm_workspace_bytes(M, N, K, 0);
}

template <int BN, bool MX, int ACC, bool PAIR, bool F8 = false>
static cudaError_t run(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tsa, const CUtensorMap& tsb,
                       const GemmArgs& a, int64_t units, cudaStream_t st) {
  using C = Cfg<BN, MX, ACC, PAIR, F8>;
  auto kern = fp4_gemm_kernel<BN, MX, ACC, PAIR, F8>;
  // the shared-memory opt-in is per device; set it once per (kernel, device)
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  cudaError_t e = cudaSuccess;
  if (dev < 0 || dev >= 64 || !attr_done[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_done[dev] = true;
  }
  // programmatic dependent launch: the prologue (barriers, TMEM, descriptor prefetch,
  // and loads of an operand the caller marked as ready) overlaps the previous kernel on
  // the stream; everything else waits for it
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int grid = 0;
  if constexpr (PAIR) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
    // persistent: as many pairs as can be resident at once (asked once per device)
    static int max_pairs[64] = {0};
    int pairs = (dev >= 0 && dev < 64) ? max_pairs[dev] : 0;
    if (pairs <= 0) {
      cfg.gridDim = dim3(2 * static_cast<unsigned>(num_sms() / 2));
      e = cudaOccupancyMaxActiveClusters(&pairs, kern, &cfg);
      if (e != cudaSuccess) return e;
      if (pairs <= 0) return cudaErrorInvalidConfiguration;
      if (dev >= 0 && dev < 64) max_pairs[dev] = pairs;
    }
    // (grouped schedules count their tiles on the device: every pair)
    grid = 2 * static_cast<int>(a.mode == kModeGrouped ? pairs : std::max<int64_t>(1, std::min<int64_t>(units, pairs)));
  } else {
    grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((units + C::kP - 1) / C::kP, num_sms())));
    if (a.mode == kModeGrouped) grid = num_sms();
  }
  cfg.gridDim = dim3(grid);
  return cudaLaunchKernelEx(&cfg, kern, ta, tb, tsa, tsb, a);
}

template <bool MX>
static cudaError_t dispatch(const Plan& pl, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tsa,
                            const CUtensorMap& tsb, const GemmArgs& a, cudaStream_t st) {
  // one CTA per SM at most; a CTA holds pipes_per_cta<BN>() pipelines
  switch (pl.BN) {
    case 16: return run<16, MX, 2, false>(ta, tb, tsa, tsb, a, pl.units, st);
    case 32: return run<32, MX, 2, false>(ta, tb, tsa, tsb, a, pl.units, st);
    case 64: return run<64, MX, 2, false>(ta, tb, tsa, tsb, a, pl.units, st);
    case 128: return run<128, MX, 2, false>(ta, tb, tsa, tsb, a, pl.units, st);
    default:
      return pl.pair ? run<256, MX, 1, true>(ta, tb, tsa, tsb, a, pl.units, st)
                     : run<256, MX, 1, false>(ta, tb, tsa, tsb, a, pl.units, st);
  }
}

int launch_gemm(const GemmProblem& g, unsigned* status, cudaStream_t st, const char** why, cudaError_t* err) {
  const int grouped = g.num_groups > 0;
  if (!grouped && !g.mx && !g.q_codes && !g.amax_out && decode_eligible(g.M, g.N, g.K)) {
    // a few activation rows: the decode kernel (the weights are problem B)
    DecodeProblem q{};
    q.W = g.B;
    q.sW = g.sB;
    q.gW = g.gB;
    q.Xq = g.A;
    q.Xs = g.sA;
    q.gX = g.gA;
    q.M = g.M;
    q.N = g.N;
    q.K = g.K;
    q.D = g.D;
    q.out_bf16 = g.out_bf16;
    q.ws = g.ws;
    q.ws_bytes = g.ws_bytes;
    q.weights_ready = g.weights_ready;
    q.bias = g.bias;
    q.act = g.act;
    return launch_decode(q, status, st, why, err);
  }
  // the NVFP4 copy of the result is written by rows: keep the operands in place
  const Plan pl = make_plan(g.M, g.N, g.K, g.num_groups, g.mx, g.q_codes != nullptr || g.amax_out != nullptr);
  if (g.ws_bytes < pl.ws_bytes || (pl.ws_bytes && !g.ws)) {
    *why = "workspace too small (see fp4_gemm_workspace_size)";
    return 1;
  }
  const int64_t sf_cols = g.K / (g.mx ? 32 : 16);
  const int64_t atoms_k = (sf_cols + 3) / 4;
  const uint8_t *kA = g.A, *kB = g.B, *kSA = g.sA, *kSB = g.sB;
  const float *kgA = g.gA, *kgB = g.gB;
  int64_t rowsA = g.M, rowsB = grouped ? static_cast<int64_t>(g.num_groups) * g.N : g.N;
  if (pl.swap) {
    std::swap(kA, kB);
    std::swap(kSA, kSB);
    std::swap(kgA, kgB);
    std::swap(rowsA, rowsB);
  }
  CUtensorMap ta, tb, tsa, tsb;
  if (!make_tensor_map_u8(&ta, kA, static_cast<uint64_t>(g.K / 2), static_cast<uint64_t>(rowsA), 128) ||
      !make_tensor_map_u8(&tb, kB, static_cast<uint64_t>(g.K / 2), static_cast<uint64_t>(rowsB),
                          static_cast<uint32_t>(pl.pair ? pl.BN / 2 : pl.BN))) {
    *why = "cuTensorMapEncodeTiled failed (alignment or driver)";
    return 1;
  }
  tsa = ta;  // unused unless CTA pairs load the scale factors with tensor copies
  tsb = ta;
  if (pl.pair) {
    // one box = one stage's atoms of one 128-row block (4 atoms NVFP4, 2 MXFP4)
    const uint32_t box_rows = (g.mx ? 2u : 4u) * 512u / 256u;
    // grouped A scales: the capacity fp4_scales_bytes_grouped gives (every 128-row block
    // of every group plus one pad block per group), which the caller's buffer holds
    const int64_t sfa_blocks = (rowsA + 127) / 128 + (grouped ? g.num_groups : 0);
    if (!make_sf_map(&tsa, kSA, static_cast<uint64_t>(sfa_blocks) * atoms_k * 512, box_rows) ||
        !make_sf_map(&tsb, kSB, static_cast<uint64_t>((rowsB + 127) / 128) * atoms_k * 512, box_rows)) {
      *why = "cuTensorMapEncodeTiled failed for the scale factors (alignment or driver)";
      return 1;
    }
  }
  GemmArgs a{};
  a.sfa = kSA;
  a.sfb = kSB;
  a.sfa_rb_bytes = atoms_k * 512;
  a.sfb_rb_bytes = atoms_k * 512;
  a.sf_atoms_k = static_cast<int>(atoms_k);
  a.ga = kgA;
  a.gb = kgB;
  a.Mk = static_cast<int>(pl.Mk);
  a.Nk = static_cast<int>(pl.Nk);
  a.K = static_cast<int>(g.K);
  a.num_kb = pl.num_kb;
  a.out = g.D;
  a.out_bf16 = g.out_bf16;
  a.transposed = pl.swap ? 1 : 0;
  // the weights (problem B) are kernel A when the operands are swapped
  a.indep = g.weights_ready ? (pl.swap ? 1 : 2) : 0;
  a.ldo = g.N;
  const int esz = g.out_bf16 ? 2 : 4;
  a.vec_store = ((g.N * esz) % 16 == 0 && (reinterpret_cast<uintptr_t>(g.D) & 15) == 0) ? 1 : 0;
  a.mode = pl.mode;
  a.tiles_m = pl.tiles_m;
  a.tiles_n = pl.tiles_n;
  a.group_m = 16;
  a.total_units = pl.units;
  a.status = status;
  a.bias = g.bias;
  a.act = g.act;
  a.q_codes = g.q_codes;
  a.q_scales = g.q_scales;
  a.q_g = g.q_g;
  a.q_atoms = (g.N / 16 + 3) / 4;
  a.amax_out = reinterpret_cast<unsigned*>(g.amax_out);
  if (pl.mode == kModeStreamK) {
    a.ws = static_cast<float*>(g.ws);
    a.tile_cnt = reinterpret_cast<int*>(static_cast<uint8_t*>(g.ws) + (static_cast<size_t>(g.M * g.N) * 4 + 255) / 256 * 256);
  }
  if (grouped) {
    a.num_groups = g.num_groups;
    a.offsets = g.offsets;
    a.b_rows_per_group = static_cast<int>(g.N);
    a.sfb_rbs = static_cast<int>((g.N + 127) / 128);
    a.sfb_group_bytes = static_cast<int64_t>(a.sfb_rbs) * atoms_k * 512;
  } else {
    a.sfb_rbs = static_cast<int>((rowsB + 127) / 128);
  }
  const cudaError_t e = g.mx ? dispatch<true>(pl, ta, tb, tsa, tsb, a, st) : dispatch<false>(pl, ta, tb, tsa, tsb, a, st);
  if (e != cudaSuccess) {
    *err = e;
    return 2;
  }
  return 0;
}

// FP4 x FP8 ("Rubin FP4 GEMM overview" 3.4: an FP4 operand opposite an FP8 one): A and
// B each MXFP4 or MXFP8, D = A B^T on kind::mxf8f6f4 MMAs.  Dense, whole tiles on single
// CTAs; K a multiple of 128.
int launch_gemm_mixed(const GemmProblem& g, int a_fp8, int b_fp8, unsigned* status, cudaStream_t st,
                      const char** why, cudaError_t* err) {
  const int sms = num_sms();
  const int64_t tiles256 = ((g.M + 127) / 128) * ((g.N + 255) / 256);
  const int BN = (g.N >= 256 && tiles256 >= sms) ? 256 : 128;
  // 256-wide tiles with at least two 128-row blocks run on CTA pairs, as the FP4 GEMM's do
  const bool pair = BN == 256 && g.M >= 256;
  CUtensorMap ta, tb, tsa, tsb;
  const bool ok_a = a_fp8 ? make_tensor_map_u8(&ta, g.A, static_cast<uint64_t>(g.K), static_cast<uint64_t>(g.M), 128)
                          : encode_map_u4(&ta, g.A, static_cast<uint64_t>(g.K), static_cast<uint64_t>(g.M), 128);
  const bool ok_b = b_fp8 ? make_tensor_map_u8(&tb, g.B, static_cast<uint64_t>(g.K), static_cast<uint64_t>(g.N),
                                               static_cast<uint32_t>(pair ? BN / 2 : BN))
                          : encode_map_u4(&tb, g.B, static_cast<uint64_t>(g.K), static_cast<uint64_t>(g.N),
                                          static_cast<uint32_t>(pair ? BN / 2 : BN));
  if (!ok_a || !ok_b) {
    *why = "cuTensorMapEncodeTiled failed (alignment or driver)";
    return 1;
  }
  const int64_t atoms_k = g.K / 128;  // one E8M0 per 32 K elements, four per atom row
  tsa = ta;
  tsb = ta;
  // a pair loads a stage's scale atoms (one per 128-row block: 512 bytes, two 256-byte rows)
  // with tensor copies that complete on the leader's barrier
  if (pair && (!make_sf_map(&tsa, g.sA, static_cast<uint64_t>((g.M + 127) / 128) * atoms_k * 512, 2) ||
               !make_sf_map(&tsb, g.sB, static_cast<uint64_t>((g.N + 127) / 128) * atoms_k * 512, 2))) {
    *why = "cuTensorMapEncodeTiled failed for the scale factors (alignment or driver)";
    return 1;
  }
  GemmArgs a{};
  a.sfa = g.sA;
  a.sfb = g.sB;
  a.sfa_rb_bytes = atoms_k * 512;
  a.sfb_rb_bytes = atoms_k * 512;
  a.sf_atoms_k = static_cast<int>(atoms_k);
  a.sfb_rbs = static_cast<int>((g.N + 127) / 128);
  a.Mk = static_cast<int>(g.M);
  a.Nk = static_cast<int>(g.N);
  a.K = static_cast<int>(g.K);
  a.num_kb = static_cast<int>(g.K / 128);
  a.out = g.D;
  a.out_bf16 = g.out_bf16;
  a.ldo = g.N;
  const int esz = g.out_bf16 ? 2 : 4;
  a.vec_store = ((g.N * esz) % 16 == 0 && (reinterpret_cast<uintptr_t>(g.D) & 15) == 0) ? 1 : 0;
  a.mode = kModeTile;
  a.tiles_m = static_cast<int>((g.M + (pair ? 255 : 127)) / (pair ? 256 : 128));
  a.tiles_n = static_cast<int>((g.N + BN - 1) / BN);
  a.group_m = 16;
  a.total_units = static_cast<int64_t>(a.tiles_m) * a.tiles_n;
  a.status = status;
  a.f8_fmt = (a_fp8 ? kFmtE4M3 : kFmtE2M1) | ((b_fp8 ? kFmtE4M3 : kFmtE2M1) << 3);
  const cudaError_t e = pair        ? run<256, true, 1, true, true>(ta, tb, tsa, tsb, a, a.total_units, st)
                        : BN == 256 ? run<256, true, 1, false, true>(ta, tb, tsa, tsb, a, a.total_units, st)
                                    : run<128, true, 2, false, true>(ta, tb, tsa, tsb, a, a.total_units, st);
  if (e != cudaSuccess) {
    *err = e;
    return 2;
  }
  return 0;
}

}  // namespace fp4
