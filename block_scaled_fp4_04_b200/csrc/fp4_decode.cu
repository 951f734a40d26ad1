// fp4_decode.cu -- the decode-shaped NVFP4 GEMM: a few activation rows (M <= 32) against
// many weight rows, D [M, N] = gX * gW * (X_hat . W_hat^T).  Memory-bound: the weights
// are read once and everything else is arranged so that they stream at full bandwidth.
//
// Same arithmetic as the general GEMM ("Rubin FP4 GEMM overview", yfxerp.com, 3.1 / 3.2:
// E2M1 products scaled per block and summed in FP32; 4.2: global scales applied in the
// epilogue), with the operands swapped: the weight rows fill the MMA's M = 128, the
// activation rows are its N (16 or 32).
//
// Layout of the work:
//   K is cut into nseg segments; the grid holds nseg groups of equal size, and each CTA
//   works inside one segment.  The activations' codes for the segment stay in shared
//   memory and their scale factors in TMEM for the whole kernel, so every pipeline
//   stage carries only one 128-row weight box and its scale atoms.
//   A CTA runs two pipelines (producer thread, MMA thread, four epilogue warps each);
//   within a segment, the (weight tile, K step) units are split evenly over all its
//   pipelines (stream-K).  Each pipeline adds its FP32 partial tiles into a workspace;
//   the pipeline that completes a tile's K range (a per-tile counter) scales, converts
//   and stores it, and clears the workspace and counter behind it.
//   With BF16 activations (fused), the eight epilogue warps first compute the tensor
//   amax of all of X themselves (every CTA: no grid-wide communication), then quantize
//   the CTA's K segment straight into the shared-memory operand (128-byte swizzled, as
//   TMA would have written it) and scale atoms; the first CTA of each segment also
//   writes those codes and scales to the caller's buffers.  Meanwhile the producers are
//   already streaming weight stages into their rings.
// Every wait is bounded; a timeout latches the status word and unwinds.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "fp4_codes.cuh"
#include "fp4_internal.h"
#include "fp4_ptx.cuh"

namespace fp4 {

struct DecodeArgs {
  const uint8_t* sfw;     // weight scale atoms (swizzled layout of [N, K/16])
  int64_t sfw_rb_bytes;   // bytes per 128-row block of weight scales
  const float* gw;        // weight global scale
  const uint8_t* xs;      // pre-quantized activations: scale atoms (row-block 0)
  const float* gx;        // pre-quantized activations: global scale
  const uint16_t* x;      // fused: BF16 activations [M, K]
  uint8_t* xq_out;        // fused: activation codes [M, K/2] (written)
  uint8_t* xs_out;        // fused: activation scale atoms (written)
  float* gx_out;          // fused: activation global scale (written)
  int M, N, K, num_kb, atoms_k;
  int nseg, seg_len, ctas_per_seg, tiles;
  void* out;
  int out_bf16;
  float* ws;              // FP32 partial sums [N, M], zero between calls
  int* tile_cnt;          // K steps summed per weight tile, zero between calls
  int weights_ready;      // W was not written by the kernel just before this one
  unsigned* gbar;         // fused: [0] call counter, then one 128-byte slot per CTA
  unsigned* status;
  const float* bias;      // [N] added to every output row after the scale, or null
  int act;                // 0: none, 1: ReLU
  int stall_plus1;        // test hook for the bounded waits: CTA stall_plus1 - 1 does not
                          // publish its share of the amax (0: every CTA publishes)
};

// K steps of one segment at most (the activations' scale factors for a segment take 16
// TMEM columns per K step; longer segments measured slower: fewer partial sums, but each
// CTA quantizes twice as much of X and its rings are shallower)
constexpr int decode_max_seg(int) { return 8; }

template <int BN>
struct DecodeCfg {
  static constexpr int kP = 2;                              // pipelines per CTA
  static constexpr int kThreads = 192 * kP;
  static constexpr int kMaxSeg = decode_max_seg(BN);        // K steps of one segment (max)
  static constexpr int kBBox = BN * 128;                    // one K step of activation codes
  static constexpr int kBBytes = kMaxSeg * kBBox;
  static constexpr int kBSFBytes = kMaxSeg * 4 * 512;
  static constexpr int kABytes = 128 * 128;
  static constexpr int kSFABytes = 4 * 512;
  static constexpr int kStageBytes = kABytes + kSFABytes;  // 18 KB
  static constexpr int kMiscBytes = 1024;
  static constexpr int kSharedBytes = kBBytes + kBSFBytes + 1024;  // + shared barriers / scratch
  static constexpr int kSmemLimit = 227 * 1024 - 1024 - 256;
  static constexpr int kStagesFit = ((kSmemLimit - kSharedBytes) / kP - kMiscBytes) / kStageBytes;
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  static constexpr int kSubBytes = kStages * kStageBytes + kMiscBytes;
  static constexpr int kSmemBytes = kSharedBytes + kP * kSubBytes + 1024;
  // TMEM: the segment's activation scale factors, then per pipeline ACC accumulators and
  // two slots of weight scale factors
  static constexpr int kACC = 4;  // lets the epilogue lag behind the MMAs by up to three tiles
  static constexpr int kBSFCols = kMaxSeg * 16;
  static constexpr int kPipeCols = kACC * BN + 2 * 16;
  static constexpr int kColsUsed = kBSFCols + kP * kPipeCols;
  static constexpr int kTmemAlloc = kColsUsed <= 128 ? 128 : kColsUsed <= 256 ? 256 : 512;
  static_assert(kColsUsed <= 512, "TMEM budget");
  static_assert(kStages >= 2, "shared memory budget");
  static_assert(kSmemBytes + 256 <= 227 * 1024, "shared memory opt-in limit");
  static_assert(kBBox % 1024 == 0 && kStageBytes % 1024 == 0 && kSubBytes % 1024 == 0, "1024-byte alignment");
};

__device__ __forceinline__ void d_allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void d_wait_prior_grids() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void d_red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

__device__ __forceinline__ void named_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void d_latch_timeout(volatile int* abort, unsigned* status) {
  *abort = 1;
  atomicOr(status, kStatusTimeout);
}

// Writes v (already scaled) to D[col][row]: the kernel's rows are D's columns.
__device__ __forceinline__ void d_store(const DecodeArgs& p, int row, int col, float v) {
  const int64_t o = static_cast<int64_t>(col) * p.N + row;
  if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.out)[o] = __float2bfloat16_rn(v);
  else reinterpret_cast<float*>(p.out)[o] = v;
}

// The (weight tile, K step) units of one pipeline: units u in [u0, u1) of its segment,
// u -> tile u / seg_len, K step kb0 + u % seg_len; consecutive units of one tile form
// one accumulation.  In the fused kernel a range that starts inside a tile (and goes on
// past it) takes that partial tile last, so that the pipeline starts on the segment's
// first K step -- the one whose activations are quantized first.  (With pre-quantized
// activations every K step is ready at once and the natural order finishes tiles sooner.)
struct DecodeSched {
  int64_t u, u1;
  int64_t head0, head1;  // the deferred partial first tile: units [head0, head1), or empty
  int kb0, len;
  __device__ DecodeSched(const DecodeArgs& p, int seg, int pipe_in_seg, int pipes_in_seg, bool defer_head) {
    kb0 = seg * p.seg_len;
    len = min(p.seg_len, p.num_kb - kb0);
    const int64_t U = static_cast<int64_t>(p.tiles) * len;
    u = U * pipe_in_seg / pipes_in_seg;
    u1 = U * (pipe_in_seg + 1) / pipes_in_seg;
    head0 = head1 = 0;
    const int64_t first_end = (u / len + 1) * len;
    if (defer_head && u % len != 0 && u1 > first_end) {
      head0 = u;
      head1 = first_end;
      u = first_end;
    }
  }
  // next accumulation: tile, K steps [k0, k1)
  __device__ bool next(int& tile, int& k0, int& k1) {
    if (u >= u1 && head0 < head1) {
      u = head0;
      u1 = head1;
      head0 = head1 = 0;
    }
    if (u >= u1) return false;
    tile = static_cast<int>(u / len);
    const int j0 = static_cast<int>(u % len);
    const int64_t j1 = min(static_cast<int64_t>(len), j0 + (u1 - u));
    k0 = kb0 + j0;
    k1 = kb0 + static_cast<int>(j1);
    u += j1 - j0;
    return true;
  }
};

constexpr int kMaxBatch = 8;

// Weight stages a pipeline of the fused kernel issues before the activations are ready.
#ifndef FP4_FUSED_PREFILL
#define FP4_FUSED_PREFILL 2
#endif
constexpr int kFusedPrefill = FP4_FUSED_PREFILL;

template <int BN, bool FUSED>
__global__ void __launch_bounds__(DecodeCfg<BN>::kThreads, 1)
    fp4_decode_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                      const DecodeArgs p) {
  using C = DecodeCfg<BN>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem_base;
  __shared__ uint32_t s_red[9];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_b = base;                          // activation codes, one swizzled box per K step
  uint8_t* s_bsf = base + C::kBBytes;           // activation scale atoms, 4 per K step
  uint8_t* shared_misc = s_bsf + C::kBSFBytes;
  // The activation operand becomes ready in batches of K steps: b_ready[b] when batch b
  // is in shared memory, bsf_ready[b] when its scale factors have been copied to TMEM.
  // Pre-quantized activations arrive in one batch.
  constexpr int kKpb = FUSED ? 256 / (BN * 8) : C::kMaxSeg;  // K steps per batch
  uint64_t* b_ready = reinterpret_cast<uint64_t*>(shared_misc);  // [kMaxBatch]
  uint64_t* bsf_ready = b_ready + kMaxBatch;                     // [kMaxBatch]
  volatile int* s_xfail = reinterpret_cast<volatile int*>(bsf_ready + kMaxBatch);

  const int sub = threadIdx.x / 192, lt = threadIdx.x % 192, warp = lt >> 5, lane = lt & 31;
  uint8_t* ring = base + C::kSharedBytes + sub * C::kSubBytes;
  uint8_t* misc = ring + S * C::kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(misc);
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;
  uint64_t* acc_empty = acc_full + C::kACC;
  uint64_t* drain = acc_empty + C::kACC;
  volatile int* s_abort = reinterpret_cast<volatile int*>(drain + 1);
  volatile int* s_epi_fail = s_abort + 1;
  volatile int* s_last = s_abort + 2;

  const int seg = blockIdx.x / p.ctas_per_seg;
  const int cta_in_seg = blockIdx.x % p.ctas_per_seg;
  const int pipes_in_seg = p.ctas_per_seg * C::kP;
  const int pipe_in_seg = cta_in_seg * C::kP + sub;
  const int kb0 = seg * p.seg_len;
  const int seg_steps = min(p.seg_len, p.num_kb - kb0);
  const int nbatch = (seg_steps + kKpb - 1) / kKpb;
  const int seg_atoms = min(seg_steps * 4, p.atoms_k - kb0 * 4);  // activation scale atoms

  if (lt == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < C::kACC; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4);
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    *s_epi_fail = 0;
    *s_last = 0;
    if (sub == 0) {
      for (int b = 0; b < kMaxBatch; ++b) {
        mbar_init(&b_ready[b], 1);
        mbar_init(&bsf_ready[b], 1);
      }
      *s_xfail = 0;
    }
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmW);
    if (!FUSED) tma_prefetch_desc(&tmX);
  }
  if (sub == 0 && warp == 1) {
    tmem_alloc(&s_tmem_base, C::kTmemAlloc);
    tmem_relinquish();
  }
  d_allow_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_bsf = s_tmem_base;
  const uint32_t tmem = s_tmem_base + C::kBSFCols + sub * C::kPipeCols;  // this pipeline's columns
  const uint32_t tmem_sfa = tmem + C::kACC * BN;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      const uint64_t pol_w = l2_policy_evict_first();  // weights: read once
      // pre-quantized activations: the first pipeline loads the segment's operand once
      auto load_x = [&]() {
        if (FUSED || sub != 0) return;
        const int atoms = min(seg_steps * 4, p.atoms_k - kb0 * 4);
        mbar_arrive_expect_tx(&b_ready[0], static_cast<uint32_t>(seg_steps * C::kBBox + atoms * 512));
        const uint64_t pol_x = l2_policy_evict_last();
        for (int j = 0; j < seg_steps; ++j)
          tma_load_2d(s_b + j * C::kBBox, &tmX, &b_ready[0], (kb0 + j) * 128, 0, pol_x);
        bulk_load(s_bsf, p.xs + static_cast<int64_t>(kb0) * 4 * 512, static_cast<uint32_t>(atoms) * 512u, &b_ready[0],
                  pol_x);
      };
      if (!p.weights_ready) {
        d_wait_prior_grids();
        load_x();
      }
      DecodeSched sch(p, seg, pipe_in_seg, pipes_in_seg, FUSED);
      int tile, k0, k1, stage = 0, issued_n = 0;
      uint32_t phase = 0, issued = 0, issued_par = 0;
      bool ok = true, x_done = !p.weights_ready;
      if (FUSED && kFusedPrefill == 0 && !mbar_wait(&b_ready[0], 0, s_abort)) {
        if (!*s_xfail) d_latch_timeout(s_abort, p.status);
        ok = false;
      }
      while (ok && sch.next(tile, k0, k1)) {
        for (int kb = k0; kb < k1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, s_abort)) {
            if (!*s_xfail) d_latch_timeout(s_abort, p.status);
            ok = false;
            break;
          }
          const int atoms = min(4, p.atoms_k - kb * 4);
          mbar_arrive_expect_tx(&full[stage], static_cast<uint32_t>(C::kABytes + atoms * 512));
          uint8_t* st = ring + stage * C::kStageBytes;
          tma_load_2d(st, &tmW, &full[stage], kb * 128, tile * 128, pol_w);
          bulk_load(st + C::kABytes, p.sfw + tile * p.sfw_rb_bytes + static_cast<int64_t>(kb) * 4 * 512,
                    static_cast<uint32_t>(atoms) * 512u, &full[stage], pol_w);
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
          // weights ready: the ring is filled first, then the activations' loads wait
          // for the kernel before this one
          // fused: while the activations are being quantized, only a short prefill is in
          // flight, so that the quantizer's own loads and stores do not queue behind a
          // full ring of weight copies
          ++issued_n;
          if (FUSED && issued_n == kFusedPrefill) {
            if (!mbar_wait(&b_ready[0], 0, s_abort)) {
              if (!*s_xfail) d_latch_timeout(s_abort, p.status);
              ok = false;
              break;
            }
          }
          if (!x_done && issued_n == S) {
            d_wait_prior_grids();
            load_x();
            x_done = true;
          }
        }
      }
      if (ok && !x_done) {
        d_wait_prior_grids();
        load_x();
      }
      if (*s_abort) {  // let issued copies land before the shared memory goes away
        for (int s = 0; s < S; ++s)
          if (issued & (1u << s)) {
            volatile int no_abort = 0;
            mbar_wait(&full[s], (issued_par >> s) & 1u, &no_abort);
          }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      bool ok = true;
      // The activations' scale factors go to TMEM once for both pipelines, batch by
      // batch as the operand becomes ready: the first pipeline's MMA thread copies them
      // (in batch order, as soon as each batch is ready or needed) and commits each batch
      // to bsf_ready[b]; the second pipeline waits for the batches it needs.
      int copied = 0, known = 0;
      const uint32_t bsf_s = smem_u32(s_bsf);
      auto copy_batch = [&](int b) {
        tc_fence_after();
        const int a1 = min((b + 1) * kKpb * 4, seg_atoms);
        for (int a = b * kKpb * 4; a < a1; ++a) tc_cp_sf_atom(tmem_bsf + a * 4, smem_desc_sf(bsf_s + a * 512));
        tc_commit(&bsf_ready[b]);
      };
      // batches 0..need in TMEM (for this thread's MMAs); false on failure
      auto ensure = [&](int need) -> bool {
        if (sub == 0) {
          while (copied <= need) {
            if (!mbar_wait(&b_ready[copied], 0, s_abort) || *s_xfail) return false;
            copy_batch(copied++);
          }
          return true;  // this thread's own copies precede its MMAs
        }
        while (known <= need) {
          if (!mbar_wait(&bsf_ready[known], 0, s_abort) || *s_xfail) return false;
          ++known;
        }
        tc_fence_after();
        return true;
      };
      // later batches that are already quantized: copied after a stage's MMAs are issued,
      // so that they never delay an MMA that does not need them (a non-blocking look: a
      // batch not ready yet must not suspend the MMA thread)
      auto copy_ready = [&]() {
        if (sub != 0) return;
        while (copied < nbatch && !*s_xfail && mbar_test_wait(&b_ready[copied], 0)) copy_batch(copied++);
      };
      auto fail = [&]() {
        if (!*s_xfail) d_latch_timeout(s_abort, p.status);
        ok = false;
      };
      if (!ensure(0)) fail();
      DecodeSched sch(p, seg, pipe_in_seg, pipes_in_seg, FUSED);
      const uint32_t ring_s = smem_u32(ring), b_s = smem_u32(s_b);
      int tile, k0, k1, stage = 0, iter = 0;
      uint32_t phase = 0, slot = 0;
      while (ok && sch.next(tile, k0, k1)) {
        const int acc = iter % C::kACC;
        if (!mbar_wait(&acc_empty[acc], ((iter / C::kACC) & 1) ^ 1, s_abort)) {
          d_latch_timeout(s_abort, p.status);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * BN;
        for (int kb = k0; kb < k1; ++kb) {
          if (!mbar_wait(&full[stage], phase, s_abort)) {
            d_latch_timeout(s_abort, p.status);
            ok = false;
            break;
          }
          if (!ensure((kb - kb0) / kKpb)) {
            fail();
            break;
          }
          tc_fence_after();
          const uint32_t st = ring_s + stage * C::kStageBytes;
          const uint32_t sfa_t = tmem_sfa + slot * 16;
          const int atoms = min(4, p.atoms_k - kb * 4);
          for (int a = 0; a < atoms; ++a) tc_cp_sf_atom(sfa_t + a * 4, smem_desc_sf(st + C::kABytes + a * 512));
          const int krem = p.K - kb * 256;
          const int nk = krem >= 256 ? 4 : (krem + 63) / 64;
          const uint64_t adesc = smem_desc_sw128(st);
          const uint64_t bdesc = smem_desc_sw128(b_s + (kb - kb0) * C::kBBox);
          const uint32_t sfb_t = tmem_bsf + (kb - kb0) * 16;
          const uint32_t idesc = mma_idesc(BN, false, 0, 0);
          for (int k = 0; k < nk; ++k)
            tc_mma_nvfp4(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, sfa_t + k * 4, sfb_t + k * 4,
                         (kb > k0 || k > 0) ? 1u : 0u);
          tc_commit(&empty[stage]);
          copy_ready();
          slot ^= 1;
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc_commit(&acc_full[acc]);
        ++iter;
      }
      // the other pipeline may still need batches this one did not: copy them all (or, on
      // failure, release its waits)
      if (sub == 0) {
        if (ok && !ensure(nbatch - 1)) fail();
        for (int b = copied; b < kMaxBatch; ++b) tc_commit(&bsf_ready[b]);
      }
      tc_commit(drain);  // no MMA may still write TMEM when it is freed
      volatile int no_abort = 0;
      mbar_wait(drain, 0, &no_abort);
    }
  } else {
    const int et = lt - 64;                 // 0..127 within the pipeline
    const int xt = sub * 128 + et;          // 0..255 over both pipelines' epilogue warps
    if constexpr (FUSED) {
      // ---------------------------------------------------------- activations
      d_wait_prior_grids();  // X may come from the kernel just before
      // zero the scale atoms: rows M..127 of every atom are padding
      for (int o = xt * 16; o < C::kBSFBytes; o += 256 * 16)
        *reinterpret_cast<uint4*>(s_bsf + o) = make_uint4(0, 0, 0, 0);
      // tensor amax (bit patterns of |x|: for non-negative floats integer order is numeric
      // order): every CTA reduces its 1/grid share of X, the shares meet in the workspace
      // behind a grid-wide barrier (the launch is cooperative: all CTAs are resident)
      const int64_t nchunk = static_cast<int64_t>(p.M) * p.K / 8;
      const uint4* xv = reinterpret_cast<const uint4*>(p.x);
      const int64_t c_lo = nchunk * blockIdx.x / gridDim.x, c_hi = nchunk * (blockIdx.x + 1) / gridDim.x;
      uint32_t m = 0;
      for (int64_t c0 = c_lo + xt; c0 < c_hi; c0 += 256 * 4) {
        uint4 u[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int64_t c = c0 + i * 256;
          u[i] = c < c_hi ? __ldg(xv + c) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t w4[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
#pragma unroll
          for (int j = 0; j < 4; ++j) m = max(m, max((w4[j] << 16) & 0x7FFFFFFFu, w4[j] & 0x7FFF0000u));
        }
      }
      // The segment is quantized in batches of 256 chunks of 32 elements (one chunk per
      // thread): chunk c is row (c / 8) % BN, K step c / (8 BN), 32-element piece c % 8,
      // so that 8 consecutive threads read 512 contiguous bytes of a row and batch b
      // completes K steps [b kKpb, (b + 1) kKpb).  The first two batches are loaded now:
      // they arrive while the amax exchange below waits for the other CTAs.
      const int chunks = BN * seg_steps * 8;
      auto load_batch = [&](int b, uint4 (&u)[4]) {
        const int c = b * 256 + xt;
        const int j = c / (BN * 8), r = (c >> 3) % BN, q = c & 7;
        const int k = (kb0 + j) * 256 + q * 32;
        const bool ok = c < chunks && r < p.M && k < p.K;
        const uint4* src = reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(r) * p.K + k);
#pragma unroll
        for (int e = 0; e < 4; ++e) u[e] = ok ? __ldg(src + e) : make_uint4(0, 0, 0, 0);
      };
      uint4 ua[4], ub[4];
      load_batch(0, ua);
      load_batch(1, ub);
      m = __reduce_max_sync(0xFFFFFFFFu, m);
      if (lane == 0) s_red[xt >> 5] = m;
      named_sync(3, 256);
      // Each CTA publishes its maximum in a slot of its own (one 128-byte line each, so
      // that the polls of all CTAs spread over many L2 lines) as one 64-bit word: the
      // call's generation number in the high half, the maximum in the low half.  Every
      // CTA polls all slots until each carries this call's generation.  The generation
      // is the workspace's call counter plus one; CTA 0 stores it back once it has seen
      // every slot (by then every CTA has read the counter), so nothing needs clearing.
      uint64_t* slots = reinterpret_cast<uint64_t*>(p.gbar + 32);  // 16 words per slot
      if (xt == 0) {
        uint32_t cm = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) cm = max(cm, s_red[w]);
        const uint32_t gen = *reinterpret_cast<volatile unsigned*>(p.gbar) + 1u;
        s_red[8] = gen;
        const uint64_t word = (static_cast<uint64_t>(gen) << 32) | cm;
        if (static_cast<int>(blockIdx.x) + 1 != p.stall_plus1)
          asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(slots + blockIdx.x * 16), "l"(word) : "memory");
      }
      named_sync(3, 256);
      const uint32_t gen = s_red[8];
      uint32_t seen = 0;
      bool got = true;
      for (int b = xt; b < static_cast<int>(gridDim.x); b += 256) {
        uint64_t v = 0;
        const uint64_t t0 = globaltimer_ns();
        for (uint32_t it = 1; it < kWaitMaxIters; ++it) {
          asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(slots + b * 16) : "memory");
          if (static_cast<uint32_t>(v >> 32) == gen) break;
          if ((it & 63u) == 0 && globaltimer_ns() - t0 > kWaitTimeoutNs) break;
          __nanosleep(32);
        }
        if (static_cast<uint32_t>(v >> 32) == gen) seen = max(seen, static_cast<uint32_t>(v));
        else got = false;
      }
      seen = __reduce_max_sync(0xFFFFFFFFu, seen);
      got = __all_sync(0xFFFFFFFFu, got);
      named_sync(3, 256);  // every thread has read s_red
      if (lane == 0) s_red[xt >> 5] = got ? seen : 0xFFFFFFFFu;
      named_sync(3, 256);
      if (xt == 0) {
        uint32_t am = 0;
        bool ok = true;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          if (s_red[w] == 0xFFFFFFFFu) ok = false;
          else am = max(am, s_red[w]);
        }
        s_red[0] = ok ? am : 0x7F800000u;
        if (!ok) {
          *s_xfail = 1;
          atomicOr(p.status, kStatusTimeout);
        }
        if (ok && blockIdx.x == 0) *reinterpret_cast<volatile unsigned*>(p.gbar) = gen;
      }
      named_sync(3, 256);
      const uint32_t am = s_red[0];
      if (am >= 0x7F800000u || *s_xfail) {
        // no encoding exists (or the barrier gave up): latch the status, stop this CTA
        if (xt == 0) {
          if (!*s_xfail && blockIdx.x == 0) atomicOr(p.status, kStatusNonFinite);
          *s_xfail = 1;
        }
        if (et == 0) *s_abort = 1;
        named_sync(3, 256);
        if (xt == 0)
          for (int b = 0; b < kMaxBatch; ++b) mbar_arrive(&b_ready[b]);
      } else {
      const float amax = __uint_as_float(am);
      const float g = amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f;  // 2688 = 6 * 448
      if (blockIdx.x == 0 && xt == 0 && p.gx_out) *p.gx_out = g;
      const bool writer = cta_in_seg == 0;  // writes the segment to the caller's buffers
      // quantize this thread's chunk of batch b: two 16-element blocks of one row
      auto quantize_batch = [&](int b, const uint4 (&u)[4]) {
        const int c = b * 256 + xt;
        if (c >= chunks) return;
        const int j = c / (BN * 8), r = (c >> 3) % BN, q = c & 7;
        const int k = (kb0 + j) * 256 + q * 32;
        uint32_t packed[4];
        uint32_t sbs[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float v[16];
          uint32_t bm = 0;
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const uint4 w = u[2 * h + t];
            const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              v[t * 8 + 2 * e] = __uint_as_float(w4[e] << 16);
              v[t * 8 + 2 * e + 1] = __uint_as_float(w4[e] & 0xFFFF0000u);
              bm = max(bm, max((w4[e] << 16) & 0x7FFFFFFFu, w4[e] & 0x7FFF0000u));
            }
          }
          uint32_t sb;
          const float mul = nvfp4_block_scale(__uint_as_float(bm), g, sb);
          sbs[h] = sb;
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            float sv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float xe = v[t * 8 + e];
              sv[e] = xe == 0.0f ? xe : __fmul_rn(xe, mul);  // a zero stays zero if 1/denom overflowed
            }
            packed[2 * h + t] = pack8<kE2M1Hardware>(sv);
          }
        }
        // the operand box of K step j, 128-byte swizzled: 16-byte chunk q of row r
        *reinterpret_cast<uint4*>(s_b + j * C::kBBox + r * 128 + ((q ^ (r & 7)) << 4)) =
            make_uint4(packed[0], packed[1], packed[2], packed[3]);
        // scale bytes: blocks 2q and 2q+1 of the K step -> atom (j, q / 2), column 2 (q % 2) + h
#pragma unroll
        for (int h = 0; h < 2; ++h)
          s_bsf[(j * 4 + (q >> 1)) * 512 + (r & 31) * 16 + (r >> 5) * 4 + ((q & 1) * 2 + h)] =
              static_cast<uint8_t>(sbs[h]);
        if (writer && r < p.M && k < p.K)
          *reinterpret_cast<uint4*>(p.xq_out + static_cast<int64_t>(r) * (p.K / 2) + k / 2) =
              make_uint4(packed[0], packed[1], packed[2], packed[3]);
      };
      // batch b is in shared memory: make it visible to the tensor cores and announce it
      auto publish = [&](int b) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic writes -> tensor-core reads
        named_sync(3, 256);
        if (xt == 0) mbar_arrive(&b_ready[b]);
      };
      for (int b = 0; b < nbatch; b += 2) {
        quantize_batch(b, ua);
        publish(b);
        if (b + 2 < nbatch) load_batch(b + 2, ua);
        if (b + 1 < nbatch) {
          quantize_batch(b + 1, ub);
          publish(b + 1);
          if (b + 3 < nbatch) load_batch(b + 3, ub);
        }
      }
      if (writer) {  // the segment's scale atoms (pads included) to the caller's buffer
        for (int o = xt; o < seg_atoms * 32; o += 256)
          reinterpret_cast<uint4*>(p.xs_out + static_cast<int64_t>(kb0) * 4 * 512)[o] =
              reinterpret_cast<const uint4*>(s_bsf)[o];
      }
      }
    }
    // ------------------------------------------------------------ epilogue
    if (!FUSED) d_wait_prior_grids();  // the activations' global scale
    const float gw = p.gw ? *p.gw : 1.0f;
    float scale;
    if constexpr (FUSED) {
      const float amax = __uint_as_float(s_red[0]);
      scale = (amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f) * gw;
    } else {
      scale = (p.gx ? *p.gx : 1.0f) * gw;
    }
    const int q4 = (threadIdx.x >> 5) & 3;  // the TMEM lane quarter this warp may read
    const int rl = q4 * 32 + lane;
    // Tiles whose partial sums this pipeline added but has not yet counted.  Counting
    // needs a fence after the reductions; it is done for a batch of tiles at a time (at
    // the end, or when the list is full) instead of once per tile, so that the
    // epilogue does not sit in a fence while the weight stream is at full load.
    constexpr int kMaxPend = 8;
    int* s_pend = const_cast<int*>(s_abort) + 4;  // [kMaxPend] tiles, [kMaxPend] K steps covered
    int npend = 0;
    // publish the pending partial sums, count them, and write out the tiles they complete
    auto flush = [&]() {
      __threadfence();
      named_sync(1 + sub, 128);
      // one thread per pending tile, so that the counts are in flight together
      if (et < npend) {
        __threadfence();
        atomicAdd(p.tile_cnt + s_pend[et], s_pend[kMaxPend + et]);
      }
      named_sync(1 + sub, 128);  // the list is reused
      npend = 0;
    };
    // Write-out.  Tile t belongs to pipeline t mod (pipelines in the grid).  Its owner
    // waits (bounded) until the tile's counter shows every K step summed, then scales,
    // converts and stores the tile and clears the sums and the counter behind it.  (The
    // launch is cooperative, so an owner never waits for a CTA that cannot run.)
    const int gp = blockIdx.x * C::kP + sub, np = gridDim.x * C::kP;
    int next_owned = gp;
    auto write_owned = [&]() {
      while (next_owned < p.tiles && !*s_epi_fail && !*s_xfail) {
        const int t = next_owned;
        if (et == 0) {
          const uint64_t t0 = globaltimer_ns();
          int ready = 0;
          for (uint32_t it = 1; it < kWaitMaxIters; ++it) {
            int c;
            asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(c) : "l"(p.tile_cnt + t) : "memory");
            if (c >= p.num_kb) {
              ready = 1;
              break;
            }
            if ((it & 63u) == 0 && globaltimer_ns() - t0 > kWaitTimeoutNs) {
              d_latch_timeout(s_abort, p.status);
              *s_epi_fail = 1;
              break;
            }
            __nanosleep(64);
          }
          if (ready) __threadfence();
          *s_last = ready;
        }
        named_sync(1 + sub, 128);
        const int ready = *s_last;
        named_sync(1 + sub, 128);  // s_last is rewritten on the next turn
        if (*s_epi_fail || !ready) return;
        const int row = t * 128 + rl;
        if (row < p.N) {
          float* wsrow = p.ws + static_cast<int64_t>(row) * p.M;
          float v[BN];
          if ((p.M & 3) == 0) {
#pragma unroll
            for (int j = 0; j < BN; j += 4)
              if (j < p.M) {
                const float4 f = __ldcg(reinterpret_cast<const float4*>(wsrow + j));
                v[j] = f.x;
                v[j + 1] = f.y;
                v[j + 2] = f.z;
                v[j + 3] = f.w;
              }
#pragma unroll
            for (int j = 0; j < BN; j += 4)
              if (j < p.M) __stcg(reinterpret_cast<float4*>(wsrow + j), make_float4(0.f, 0.f, 0.f, 0.f));
          } else {
#pragma unroll
            for (int j = 0; j < BN; ++j)
              if (j < p.M) v[j] = __ldcg(wsrow + j);
#pragma unroll
            for (int j = 0; j < BN; ++j)
              if (j < p.M) __stcg(wsrow + j, 0.0f);
          }
          // the epilogue after the scale: bias of this output column, then the activation
          const float bias = p.bias ? __ldg(p.bias + row) : 0.0f;
#pragma unroll
          for (int j = 0; j < BN; ++j)
            if (j < p.M) {
              float o = v[j] * scale;
              if (p.bias) o = __fadd_rn(o, bias);
              if (p.act == 1) o = fmaxf(o, 0.0f);
              d_store(p, row, j, o);
            }
        }
        if (et == 0) p.tile_cnt[t] = 0;
        next_owned += np;
      }
    };
    DecodeSched sch(p, seg, pipe_in_seg, pipes_in_seg, FUSED);
    int tile, k0, k1, iter = 0;
    while (!*s_xfail && sch.next(tile, k0, k1)) {
      const int acc = iter % C::kACC;
      const uint32_t par = (iter / C::kACC) & 1;
      if (et == 0 && !mbar_wait(&acc_full[acc], par, s_abort)) {
        d_latch_timeout(s_abort, p.status);
        *s_epi_fail = 1;
      }
      named_sync(1 + sub, 128);
      if (*s_epi_fail) break;
      tc_fence_after();
      const int row = tile * 128 + rl;  // weight row = output column
      const bool row_ok = row < p.N;
      float* wsrow = p.ws + static_cast<int64_t>(row) * p.M;
#pragma unroll
      for (int c = 0; c < BN; c += 16) {
        uint32_t r[16];
        tmem_ld16(tmem + (static_cast<uint32_t>(q4 * 32) << 16) + acc * BN + c, r);
        tmem_ld_wait();
        if (row_ok) {
          if ((p.M & 3) == 0) {
#pragma unroll
            for (int j = 0; j < 16; j += 4)
              if (c + j < p.M)
                d_red_add_v4(wsrow + c + j, __uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                             __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
          } else {
            for (int j = 0; j < 16 && c + j < p.M; ++j) atomicAdd(wsrow + c + j, __uint_as_float(r[j]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      ++iter;
      if (et == 0) {
        s_pend[npend] = tile;
        s_pend[kMaxPend + npend] = k1 - k0;
      }
      if (++npend == kMaxPend) flush();
    }
    if (npend && !*s_epi_fail && !*s_xfail) flush();
    write_owned();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (sub == 0 && warp == 1) {
    __syncwarp();
    tmem_dealloc(s_tmem_base, C::kTmemAlloc);
  }
}

// ---------------------------------------------------------------------- host side
constexpr int kDecodeMaxCtas = 512;  // amax slots in the workspace
bool decode_eligible(int64_t M, int64_t N, int64_t K) { return M >= 1 && M <= 32 && N >= 1 && K >= 32; }

struct DecodePlan {
  int nseg, seg_len, ctas_per_seg, tiles, num_kb;
};

static DecodePlan decode_plan(int64_t N, int64_t K, int bn) {
  DecodePlan d{};
  d.num_kb = static_cast<int>((K + 255) / 256);
  d.tiles = static_cast<int>((N + 127) / 128);
  const int sms = num_sms();
  // segments of at most decode_max_seg(bn) K steps
  const int max_seg = decode_max_seg(bn);
  int nseg = (d.num_kb + max_seg - 1) / max_seg;
  const int min_seg = 4;
  if (nseg < min_seg) nseg = d.num_kb < min_seg ? d.num_kb : min_seg;
  if (nseg > sms) nseg = sms;
  const int max_ctas = sms < kDecodeMaxCtas ? sms : kDecodeMaxCtas;
  d.seg_len = (d.num_kb + nseg - 1) / nseg;
  d.nseg = (d.num_kb + d.seg_len - 1) / d.seg_len;
  d.ctas_per_seg = max_ctas / d.nseg;
  // no more pipelines than units in a segment
  const int64_t units = static_cast<int64_t>(d.tiles) * d.seg_len;
  const int64_t useful = (units + 1) / 2;
  if (d.ctas_per_seg > useful) d.ctas_per_seg = static_cast<int>(useful);
  if (d.ctas_per_seg < 1) d.ctas_per_seg = 1;
  return d;
}

// [FP32 partial sums M*N][tile counters][3 barrier words], each part 256-byte aligned
static size_t ws_partials(int64_t M, int64_t N) { return (static_cast<size_t>(M * N) * 4 + 255) / 256 * 256; }
static size_t ws_counters(int64_t N) { return (static_cast<size_t>((N + 127) / 128) * 4 + 255) / 256 * 256; }

size_t decode_workspace_bytes(int64_t M, int64_t N) {
  return ws_partials(M, N) + ws_counters(N) + 128 + static_cast<size_t>(kDecodeMaxCtas) * 128;
}

template <int BN, bool FUSED>
static cudaError_t run_decode(const CUtensorMap& tw, const CUtensorMap& tx, const DecodeArgs& a, int grid,
                              cudaStream_t st) {
  using C = DecodeCfg<BN>;
  auto kern = fp4_decode_kernel<BN, FUSED>;
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_done[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_done[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  // CTAs wait for one another (the fused kernel's amax exchange; the owners of tiles
  // wait for the other pipelines' partial sums): all must be resident at once
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, tw, tx, a);
}

int launch_decode(const DecodeProblem& q, unsigned* status, cudaStream_t st, const char** why, cudaError_t* err) {
  if (!decode_eligible(q.M, q.N, q.K)) {
    *why = "decode kernel: 1 <= M <= 32";
    return 1;
  }
  if (q.ws_bytes < decode_workspace_bytes(q.M, q.N) || !q.ws) {
    *why = "workspace too small (see fp4_gemm_workspace_size)";
    return 1;
  }
  const int BN = q.M <= 16 ? 16 : 32;
  const DecodePlan pl = decode_plan(q.N, q.K, BN);
  CUtensorMap tw, tx;
  if (!make_tensor_map_u8(&tw, q.W, static_cast<uint64_t>(q.K / 2), static_cast<uint64_t>(q.N), 128)) {
    *why = "cuTensorMapEncodeTiled failed (alignment or driver)";
    return 1;
  }
  if (q.X) {
    tx = tw;  // unused by the fused kernel
  } else if (!make_tensor_map_u8(&tx, q.Xq, static_cast<uint64_t>(q.K / 2), static_cast<uint64_t>(q.M),
                                 static_cast<uint32_t>(BN))) {
    *why = "cuTensorMapEncodeTiled failed (alignment or driver)";
    return 1;
  }
  DecodeArgs a{};
  const int64_t atoms_k = (q.K / 16 + 3) / 4;
  a.sfw = q.sW;
  a.sfw_rb_bytes = atoms_k * 512;
  a.gw = q.gW;
  a.xs = q.Xs;
  a.gx = q.gX;
  a.x = static_cast<const uint16_t*>(q.X);
  a.xq_out = q.Xq_out;
  a.xs_out = q.Xs_out;
  a.gx_out = q.gX_out;
  a.M = static_cast<int>(q.M);
  a.N = static_cast<int>(q.N);
  a.K = static_cast<int>(q.K);
  a.num_kb = pl.num_kb;
  a.atoms_k = static_cast<int>(atoms_k);
  a.nseg = pl.nseg;
  a.seg_len = pl.seg_len;
  a.ctas_per_seg = pl.ctas_per_seg;
  a.tiles = pl.tiles;
  a.out = q.D;
  a.out_bf16 = q.out_bf16;
  a.ws = static_cast<float*>(q.ws);
  a.tile_cnt = reinterpret_cast<int*>(static_cast<uint8_t*>(q.ws) + ws_partials(q.M, q.N));
  a.gbar = reinterpret_cast<unsigned*>(static_cast<uint8_t*>(q.ws) + ws_partials(q.M, q.N) + ws_counters(q.N));
  a.weights_ready = q.weights_ready;
  a.status = status;
  a.bias = q.bias;
  a.act = q.act;
  a.stall_plus1 = q.stall_plus1;
  const int grid = pl.nseg * pl.ctas_per_seg;
  cudaError_t e;
  if (q.X) e = BN == 16 ? run_decode<16, true>(tw, tx, a, grid, st) : run_decode<32, true>(tw, tx, a, grid, st);
  else e = BN == 16 ? run_decode<16, false>(tw, tx, a, grid, st) : run_decode<32, false>(tw, tx, a, grid, st);
  if (e != cudaSuccess) {
    *err = e;
    return 2;
  }
  return 0;
}

}  // namespace fp4
