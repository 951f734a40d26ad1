// fp4_internal.h -- declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <algorithm>
#include <cstdint>

namespace fp4 {

constexpr int kMaxGroups = 1024;      // grouped quantize / GEMM
constexpr int kAmaxMaxBlocks = 1024;  // partial maxima held in the quantize workspace
constexpr size_t kQuantWorkspaceBytes = (2 + kAmaxMaxBlocks) * sizeof(uint32_t);

// Production E2M1 encoder: the hardware conversion (cvt.rn.satfinite.e2m1x2.f32) when
// true, the threshold-count encoder when false.  Both are checked against the CPU
// definition over every float32 bit pattern by the encoder test.
#ifndef FP4_E2M1_HW
#define FP4_E2M1_HW 1
#endif
constexpr bool kE2M1Hardware = FP4_E2M1_HW != 0;

int num_sms();  // SM count of the current device (cached per device)

// rht != 0: the maximum of the 16-point Hadamard transform (sign bits `signs`) of x.
cudaError_t launch_amax(const void* x, int64_t n, int bf16, uint32_t* ws, float* amax_out, float* g_out,
                        unsigned* status, cudaStream_t st, int rht = 0, uint32_t signs = 0);
// Quantizer variants of the 1-D kernel (see fp4_quantize.cu).
enum { kQuantPlain = 0, kQuantMxFloor = 1, kQuantSR = 2, kQuantRHT = 3, kQuantFp8 = 4 };
cudaError_t launch_quantize_1d(const void* x, int64_t rows, int64_t cols, int bf16, int mx, uint8_t* codes,
                               uint8_t* scales, const float* g, const int32_t* offsets, int num_groups,
                               unsigned* status, cudaStream_t st, int variant = kQuantPlain,
                               const uint32_t* rbits = nullptr, uint32_t signs = 0);
// Small tensors (see quantize_small_fits): amax, global scale and 1-D quantize in one
// launch of one thread-block cluster; the scale buffer is zero-filled and written.
constexpr int kSmallCtas = 8, kSmallThreads = 512;
bool quantize_small_fits(int64_t rows, int64_t cols, int bf16, int mx);
cudaError_t launch_quantize_small(const void* x, int64_t rows, int64_t cols, int bf16, int mx, uint8_t* codes,
                                  uint8_t* scales, const float* g_in, float* g_out, unsigned* status,
                                  cudaStream_t st);
cudaError_t launch_quantize_2d(const void* x, int64_t rows, int64_t cols, int bf16, uint8_t* codes,
                               uint8_t* scales, uint8_t* codesT, uint8_t* scalesT, const float* g,
                               unsigned* status, cudaStream_t st);
cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* scales, const float* g, int64_t rows,
                              int64_t cols, int mx, float* out, cudaStream_t st);
cudaError_t launch_set_value(float* p, float v, cudaStream_t st);
// g = amax / (6 * 448), 1 when amax is 0; a non-finite amax latches kStatusNonFinite.
cudaError_t launch_global_scale(const float* amax, float* g, unsigned* status, cudaStream_t st);
cudaError_t launch_debug_encode(const float* in, int64_t n, int which, uint8_t* out, cudaStream_t st);
cudaError_t launch_mma_peak(int iters, int grid, unsigned long long* cycles, unsigned* status, cudaStream_t st);

// GEMM problem as the host API sees it (see fp4.h for the meaning of each field).
struct GemmProblem {
  int mx;
  const uint8_t *A, *sA, *B, *sB;
  const float *gA, *gB;
  int64_t M, N, K;
  void* D;
  int out_bf16;
  void* ws;
  size_t ws_bytes;
  int weights_ready;         // B was not written by the kernel just before this call
  // grouped
  int num_groups;            // 0: plain GEMM
  const int32_t* offsets;
  // epilogue after the scale: bias [N], activation (0 none, 1 ReLU), and an NVFP4 copy
  // of the result (codes [M, N/2], swizzled scales of [M, N/16], caller's global scale)
  const float* bias;
  int act;
  uint8_t *q_codes, *q_scales;
  const float* q_g;
  float* amax_out;  // max |result| (written; zeroed by the entry point), or null
};

size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int mx, bool fp4_out = false);

size_t gemm_bf16a_workspace_bytes(int64_t M, int64_t N, int64_t K);

// Encoded 2-D TMA map of a [rows, inner_bytes] uint8 matrix, boxes of box_rows x 128
// bytes with the 128-byte swizzle (cached per address and shape).
bool make_tensor_map_u8(CUtensorMap* m, const void* base, uint64_t inner_bytes, uint64_t rows, uint32_t box_rows);

// Decode-shaped NVFP4 GEMM (1 <= M <= 32): D [M, N] = gX gW (X_hat . W_hat^T), with the
// activations either pre-quantized (Xq / Xs / gX) or BF16 (X, quantized inside the
// kernel into Xq_out / Xs_out / gX_out).
struct DecodeProblem {
  const uint8_t *W, *sW;
  const float* gW;
  const uint8_t *Xq, *Xs;
  const float* gX;
  const void* X;
  uint8_t *Xq_out, *Xs_out;
  float* gX_out;
  int64_t M, N, K;
  void* D;
  int out_bf16;
  void* ws;
  size_t ws_bytes;
  int weights_ready;
  const float* bias;  // [N] or null
  int act;            // 0 none, 1 ReLU
  int stall_plus1;    // test hook: CTA stall_plus1 - 1 never publishes its amax share (0: none)
};
bool decode_eligible(int64_t M, int64_t N, int64_t K);
size_t decode_workspace_bytes(int64_t M, int64_t N);
int launch_decode(const DecodeProblem& q, unsigned* status, cudaStream_t st, const char** why, cudaError_t* err);
// Returns 0 on success, 1 on an unsupported shape / too-small workspace (message in
// *why), or 2 on a CUDA error (code in *err).
int launch_gemm(const GemmProblem& p, unsigned* status, cudaStream_t st, const char** why, cudaError_t* err);
// D = A B^T with A and B each MXFP4 (a_fp8 / b_fp8 = 0) or MXFP8 (1), kind::mxf8f6f4 MMAs;
// K % 128 == 0, A and B 32-byte aligned.  Uses g.A, g.sA, g.B, g.sB, g.M, g.N, g.K, g.D,
// g.out_bf16.
int launch_gemm_mixed(const GemmProblem& g, int a_fp8, int b_fp8, unsigned* status, cudaStream_t st,
                      const char** why, cudaError_t* err);

}  // namespace fp4
