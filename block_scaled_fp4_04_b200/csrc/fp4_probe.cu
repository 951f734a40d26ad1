// fp4_probe.cu -- the peak the block-scaled tensor-core MMA sustains on this GPU, measured
// rather than quoted ("NVIDIA FP4" article, hardware table: 9 PFLOP/s dense FP4 for B200 is
// a vendor figure; the roofline of the tensor-bound GEMMs is reported against a measured
// number).
//
// One CTA per SM fills an A tile (128 rows x 256 E2M1 values) and a B tile (N rows) in
// shared memory with pseudo-random codes and every scale byte with 1.0, copies the scale
// atoms into TMEM, and one thread issues `iters` K steps of four back-to-back
// tcgen05.mma.kind::mxf4nvf4 (M = 128, N = 256, K = 64) into one TMEM accumulator: no
// loads, no epilogue, only the tensor pipe.  clock64 around the loop gives cycles per SM.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "fp4_internal.h"
#include "fp4_ptx.cuh"

namespace fp4 {

constexpr int kProbeN = 256;

__global__ void __launch_bounds__(128, 1) mma_peak_kernel(int iters, unsigned long long* cycles, unsigned* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bar;
  __shared__ uint32_t s_tmem;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kA = 128 * 128, kB = kProbeN * 128, kNRB = kProbeN / 128;
  uint8_t* sfa = smem + kA + kB;   // 4 atoms
  uint8_t* sfb = sfa + 4 * 512;    // 4 atoms per 128 rows of B
  for (int i = threadIdx.x; i < (kA + kB) / 4; i += blockDim.x) {
    uint32_t h = static_cast<uint32_t>(i) * 2654435761u + blockIdx.x;
    h ^= h >> 13;
    reinterpret_cast<uint32_t*>(smem)[i] = h * 0x9E3779B1u;
  }
  for (int i = threadIdx.x; i < (4 + 4 * kNRB) * 512; i += blockDim.x) sfa[i] = 0x38;  // E4M3 1.0
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic writes -> tensor-core reads
  __syncthreads();
  if (warp == 0) {
    tmem_alloc(&s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  if (warp == 1 && lane == 0) {
    const uint32_t sfa_t = tmem + kProbeN, sfb_t = sfa_t + 16;
    for (int a = 0; a < 4; ++a) tc_cp_sf_atom(sfa_t + a * 4, smem_desc_sf(smem_u32(sfa + a * 512)));
    for (int rb = 0; rb < kNRB; ++rb)
      for (int a = 0; a < 4; ++a)
        tc_cp_sf_atom(sfb_t + (a * kNRB + rb) * 4, smem_desc_sf(smem_u32(sfb + (rb * 4 + a) * 512)));
    const uint64_t adesc = smem_desc_sw128(smem_u32(smem));
    const uint64_t bdesc = smem_desc_sw128(smem_u32(smem + kA));
    const uint32_t idesc = mma_idesc(kProbeN, false, 0, 0, 128);
    const unsigned long long c0 = clock64();
    for (int it = 0; it < iters; ++it)
      for (int k = 0; k < 4; ++k)
        tc_mma_nvfp4(tmem, adesc + 2 * k, bdesc + 2 * k, idesc, sfa_t + k * 4, sfb_t + k * kNRB * 4,
                     (it > 0 || k > 0) ? 1u : 0u);
    tc_commit(&bar);
    volatile int no_abort = 0;
    if (!mbar_wait(&bar, 0, &no_abort)) atomicOr(status, kStatusTimeout);
    cycles[blockIdx.x] = clock64() - c0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

cudaError_t launch_mma_peak(int iters, int grid, unsigned long long* cycles, unsigned* status, cudaStream_t st) {
  // more than half an SM's shared memory: one CTA per SM
  const int smem = 120 * 1024;
  cudaError_t e = cudaFuncSetAttribute(mma_peak_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  mma_peak_kernel<<<grid, 128, smem, st>>>(iters, cycles, status);
  return cudaGetLastError();
}

}  // namespace fp4
