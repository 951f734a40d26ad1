// fp4_api.cu -- the extern "C" entry points declared in include/fp4.h: argument
// checks, workspace sizing, the per-device status word, and kernel launches.
#include <cuda_runtime.h>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include "fp4.h"
#include "fp4_internal.h"
#include "fp4_ptx.cuh"

namespace fp4 {

// Latched device-side errors (kStatusNonFinite, kStatusTimeout); one word per device.
__device__ unsigned g_status_word;

static thread_local char g_err[256];

static fp4_status fail(fp4_status s, const char* msg) {
  snprintf(g_err, sizeof(g_err), "%s", msg);
  return s;
}

static fp4_status cuda_fail(cudaError_t e, const char* where) {
  snprintf(g_err, sizeof(g_err), "%s: %s", where, cudaGetErrorString(e));
  return FP4_ERR_CUDA;
}

constexpr int kMaxDevices = 64;

int num_sms() {
  static int cache[kMaxDevices] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= kMaxDevices) return 148;
  if (!cache[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}

// Address of this device's status word, and a check that the device is an sm_100.
static fp4_status device_state(unsigned** status) {
  static unsigned* addr[kMaxDevices] = {nullptr};
  static int ok[kMaxDevices] = {0};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(FP4_ERR_UNSUPPORTED, "device index out of range");
  std::lock_guard<std::mutex> lock(mu);
  if (!ok[dev]) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0) return fail(FP4_ERR_UNSUPPORTED, "libfp4 is built for sm_100a (B200) only");
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_status_word);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status)");
    addr[dev] = static_cast<unsigned*>(p);
    ok[dev] = 1;
  }
  *status = addr[dev];
  return FP4_OK;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Test hook (fp4_debug_stall_next_decode): the CTA whose amax share the next fused decode
// launch of this thread leaves unpublished, plus one (0: none).
static thread_local int g_stall_next_decode = 0;

}  // namespace fp4

using namespace fp4;

extern "C" {

const char* fp4_version(void) { return "libfp4 0.1 (sm_100a)"; }

const char* fp4_last_error(void) { return g_err; }

size_t fp4_scales_bytes(int64_t rows, int64_t cols, fp4_fmt fmt) {
  if (rows <= 0 || cols <= 0) return 0;
  const int64_t blk = fmt == FP4_MXFP4 || fmt == FP4_MXFP8 ? 32 : 16;
  const int64_t scols = (cols + blk - 1) / blk;
  return static_cast<size_t>(((rows + 127) / 128) * 128 * ((scols + 3) / 4) * 4);
}

size_t fp4_scales_bytes_grouped(int64_t total_rows, int num_groups, int64_t cols, fp4_fmt fmt) {
  if (total_rows < 0 || num_groups <= 0 || cols <= 0) return 0;
  const int64_t blk = fmt == FP4_MXFP4 ? 32 : 16;
  const int64_t scols = (cols + blk - 1) / blk;
  return static_cast<size_t>(((total_rows + 127) / 128 + num_groups) * 128 * ((scols + 3) / 4) * 4);
}

size_t fp4_quantize_workspace_size(void) { return kQuantWorkspaceBytes; }

fp4_status fp4_amax(const void* x, int64_t n, fp4_dtype in_dtype, float* amax_out, void* workspace,
                    size_t workspace_bytes, void* stream) {
  if (!x || !amax_out || !workspace) return fail(FP4_ERR_INVALID_ARG, "null pointer");
  if (n <= 0) return fail(FP4_ERR_INVALID_ARG, "n must be positive");
  if (in_dtype != FP4_F32 && in_dtype != FP4_BF16) return fail(FP4_ERR_INVALID_ARG, "in_dtype");
  if (!aligned16(x) || !aligned16(workspace)) return fail(FP4_ERR_INVALID_ARG, "x and workspace must be 16-byte aligned");
  if (workspace_bytes < kQuantWorkspaceBytes) return fail(FP4_ERR_INVALID_ARG, "workspace too small");
  unsigned* status;
  fp4_status s = device_state(&status);
  if (s != FP4_OK) return s;
  cudaError_t e = launch_amax(x, n, in_dtype == FP4_BF16, static_cast<uint32_t*>(workspace), amax_out, nullptr,
                              status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FP4_OK : cuda_fail(e, "amax launch");
}

static fp4_status quantize_common(const void* x, int64_t rows, int64_t cols, fp4_dtype in_dtype, fp4_fmt fmt,
                                  int block, uint8_t* codes, uint8_t* scales, float* gout, uint8_t* codesT,
                                  uint8_t* scalesT, const float* gin, void* ws, size_t ws_bytes, int num_groups,
                                  const int32_t* offsets, void* stream, int variant = kQuantPlain,
                                  const uint32_t* rbits = nullptr, uint32_t signs = 0) {
  if (!x || !codes || !scales) return fail(FP4_ERR_INVALID_ARG, "null pointer");
  if (rows <= 0 || cols <= 0) return fail(FP4_ERR_INVALID_ARG, "rows and cols must be positive");
  if (cols % 32 != 0) return fail(FP4_ERR_INVALID_ARG, "cols must be a multiple of 32");
  if (rows > (1ll << 31) - 256) return fail(FP4_ERR_UNSUPPORTED, "rows too large");  // row offsets are int32
  if (in_dtype != FP4_F32 && in_dtype != FP4_BF16) return fail(FP4_ERR_INVALID_ARG, "in_dtype");
  if (fmt != FP4_NVFP4 && fmt != FP4_MXFP4 && fmt != FP4_MXFP8) return fail(FP4_ERR_INVALID_ARG, "fmt");
  if (fmt == FP4_MXFP8) {
    if (block != 32) return fail(FP4_ERR_INVALID_ARG, "MXFP8 block must be 32");
    if (num_groups) return fail(FP4_ERR_UNSUPPORTED, "grouped MXFP8 quantization");
    if (variant != kQuantPlain) return fail(FP4_ERR_UNSUPPORTED, "quantizer variants are FP4 only");
    variant = kQuantFp8;
  }
  const bool two_d = block == 256;
  if (fmt == FP4_NVFP4 && block != 16 && block != 256) return fail(FP4_ERR_INVALID_ARG, "NVFP4 block must be 16 or 256");
  if (fmt == FP4_MXFP4 && block != 32) return fail(FP4_ERR_INVALID_ARG, "MXFP4 block must be 32");
  if (two_d && (!codesT || !scalesT)) return fail(FP4_ERR_INVALID_ARG, "block 256 needs codesT and scalesT");
  if (!two_d && (codesT || scalesT)) return fail(FP4_ERR_INVALID_ARG, "codesT/scalesT only for block 256");
  if (two_d && rows % 32 != 0) return fail(FP4_ERR_INVALID_ARG, "block 256 needs rows % 32 == 0");
  if (two_d && num_groups) return fail(FP4_ERR_UNSUPPORTED, "grouped 2-D quantization");
  if (fmt == FP4_NVFP4 && !gout) return fail(FP4_ERR_INVALID_ARG, "NVFP4 needs global_out");
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || (codesT && !aligned16(codesT)) ||
      (scalesT && !aligned16(scalesT)))
    return fail(FP4_ERR_INVALID_ARG, "x, codes and scales must be 16-byte aligned");
  if (num_groups && (num_groups > kMaxGroups || !offsets)) return fail(FP4_ERR_INVALID_ARG, "groups / offsets");
  if (variant != kQuantPlain && two_d) return fail(FP4_ERR_UNSUPPORTED, "quantizer variants are 1-D only");
  if (variant == kQuantMxFloor && fmt != FP4_MXFP4) return fail(FP4_ERR_INVALID_ARG, "the E8M0 floor is for MXFP4");
  if (variant == kQuantSR && (fmt != FP4_NVFP4 || !rbits || !aligned16(rbits)))
    return fail(FP4_ERR_INVALID_ARG, "stochastic rounding: NVFP4, 16-byte aligned random words");
  const bool need_amax = fmt == FP4_NVFP4 && !gin;
  if (need_amax && (!ws || ws_bytes < kQuantWorkspaceBytes || !aligned16(ws)))
    return fail(FP4_ERR_INVALID_ARG, "workspace too small or misaligned (fp4_quantize_workspace_size)");
  unsigned* status;
  fp4_status s = device_state(&status);
  if (s != FP4_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int bf16 = in_dtype == FP4_BF16;
  const int mx = fmt == FP4_MXFP4 || fmt == FP4_MXFP8;
  cudaError_t e = cudaSuccess;
  if (variant == kQuantPlain && !two_d && !num_groups && quantize_small_fits(rows, cols, bf16, mx)) {
    // one launch: amax, global scale and encode by one thread-block cluster
    e = launch_quantize_small(x, rows, cols, bf16, mx, codes, scales, mx ? nullptr : gin, gout, status, st);
    return e == cudaSuccess ? FP4_OK : cuda_fail(e, "quantize launch");
  }
  const float* g = nullptr;
  if (fmt == FP4_NVFP4) {
    if (need_amax) {
      e = launch_amax(x, rows * cols, bf16, static_cast<uint32_t*>(ws), nullptr, gout, status, st,
                      variant == kQuantRHT, signs);
      if (e != cudaSuccess) return cuda_fail(e, "amax launch");
      g = gout;
    } else {
      if (gout && gout != gin) {
        e = cudaMemcpyAsync(gout, gin, sizeof(float), cudaMemcpyDeviceToDevice, st);
        if (e != cudaSuccess) return cuda_fail(e, "global scale copy");
      }
      g = gin;
    }
  } else if (gout) {
    e = launch_set_value(gout, 1.0f, st);
    if (e != cudaSuccess) return cuda_fail(e, "global scale write");
  }
  if (two_d)
    e = launch_quantize_2d(x, rows, cols, bf16, codes, scales, codesT, scalesT, g, status, st);
  else
    e = launch_quantize_1d(x, rows, cols, bf16, mx, codes, scales, g, offsets, num_groups, status, st, variant, rbits,
                           signs);
  return e == cudaSuccess ? FP4_OK : cuda_fail(e, "quantize launch");
}

fp4_status fp4_quantize(const void* x, int64_t rows, int64_t cols, fp4_dtype in_dtype, fp4_fmt fmt, int block,
                        uint8_t* codes_out, uint8_t* scales_out, float* global_out, uint8_t* codesT_out,
                        uint8_t* scalesT_out, const float* global_in, void* workspace, size_t workspace_bytes,
                        void* stream) {
  return quantize_common(x, rows, cols, in_dtype, fmt, block, codes_out, scales_out, global_out, codesT_out,
                         scalesT_out, global_in, workspace, workspace_bytes, 0, nullptr, stream);
}

fp4_status fp4_quantize_ex(const void* x, int64_t rows, int64_t cols, fp4_dtype in_dtype, fp4_fmt fmt, int block,
                           unsigned flags, uint8_t* codes_out, uint8_t* scales_out, float* global_out,
                           uint8_t* codesT_out, uint8_t* scalesT_out, const float* global_in, void* workspace,
                           size_t workspace_bytes, void* stream) {
  if (flags & ~static_cast<unsigned>(FP4_QUANT_E8M0_FLOOR)) return fail(FP4_ERR_INVALID_ARG, "unknown flag");
  return quantize_common(x, rows, cols, in_dtype, fmt, block, codes_out, scales_out, global_out, codesT_out,
                         scalesT_out, global_in, workspace, workspace_bytes, 0, nullptr, stream,
                         (flags & FP4_QUANT_E8M0_FLOOR) ? kQuantMxFloor : kQuantPlain);
}

fp4_status fp4_quantize_sr(const void* x, int64_t rows, int64_t cols, fp4_dtype in_dtype, const uint32_t* rbits,
                           uint8_t* codes_out, uint8_t* scales_out, float* global_out, const float* global_in,
                           void* workspace, size_t workspace_bytes, void* stream) {
  return quantize_common(x, rows, cols, in_dtype, FP4_NVFP4, 16, codes_out, scales_out, global_out, nullptr, nullptr,
                         global_in, workspace, workspace_bytes, 0, nullptr, stream, kQuantSR, rbits, 0);
}

fp4_status fp4_quantize_rht(const void* x, int64_t rows, int64_t cols, fp4_dtype in_dtype, fp4_fmt fmt,
                            uint32_t signs, uint8_t* codes_out, uint8_t* scales_out, float* global_out,
                            const float* global_in, void* workspace, size_t workspace_bytes, void* stream) {
  if (signs > 0xFFFFu) return fail(FP4_ERR_INVALID_ARG, "signs: 16 bits");
  return quantize_common(x, rows, cols, in_dtype, fmt, fmt == FP4_MXFP4 ? 32 : 16, codes_out, scales_out, global_out,
                         nullptr, nullptr, global_in, workspace, workspace_bytes, 0, nullptr, stream, kQuantRHT,
                         nullptr, signs);
}

fp4_status fp4_global_scale(const float* amax, float* global_out, void* stream) {
  if (!amax || !global_out) return fail(FP4_ERR_INVALID_ARG, "null pointer");
  unsigned* status;
  fp4_status s = device_state(&status);
  if (s != FP4_OK) return s;
  const cudaError_t e = launch_global_scale(amax, global_out, status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FP4_OK : cuda_fail(e, "global scale launch");
}

fp4_status fp4_quantize_grouped(const void* x, int64_t rows, int64_t cols, fp4_dtype in_dtype, fp4_fmt fmt,
                                int num_groups, const int32_t* offsets, uint8_t* codes_out, uint8_t* scales_out,
                                float* global_out, const float* global_in, void* workspace,
                                size_t workspace_bytes, void* stream) {
  if (num_groups <= 0) return fail(FP4_ERR_INVALID_ARG, "num_groups must be positive");
  return quantize_common(x, rows, cols, in_dtype, fmt, fmt == FP4_NVFP4 ? 16 : 32, codes_out, scales_out,
                         global_out, nullptr, nullptr, global_in, workspace, workspace_bytes, num_groups, offsets,
                         stream);
}

fp4_status fp4_dequantize(const uint8_t* codes, const uint8_t* scales, const float* global, int64_t rows,
                          int64_t cols, fp4_fmt fmt, float* out, void* stream) {
  if (!codes || !scales || !out) return fail(FP4_ERR_INVALID_ARG, "null pointer");
  if (rows <= 0 || cols <= 0 || cols % 32 != 0) return fail(FP4_ERR_INVALID_ARG, "shape");
  if (fmt != FP4_NVFP4 && fmt != FP4_MXFP4) return fail(FP4_ERR_INVALID_ARG, "fmt");
  unsigned* status;
  fp4_status s = device_state(&status);
  if (s != FP4_OK) return s;
  cudaError_t e = launch_dequantize(codes, scales, fmt == FP4_NVFP4 ? global : nullptr, rows, cols,
                                    fmt == FP4_MXFP4, out, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FP4_OK : cuda_fail(e, "dequantize launch");
}

size_t fp4_gemm_workspace_size(int64_t M, int64_t N, int64_t K, fp4_fmt fmt) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  return gemm_workspace_bytes(M, N, K, fmt == FP4_MXFP4);
}

static fp4_status gemm_common(const GemmProblem& g, fp4_fmt fmt, fp4_dtype out_dtype, void* stream) {
  if (fmt != FP4_NVFP4 && fmt != FP4_MXFP4) return fail(FP4_ERR_INVALID_ARG, "fmt");
  if (out_dtype != FP4_F32 && out_dtype != FP4_BF16) return fail(FP4_ERR_INVALID_ARG, "out_dtype");
  if (!g.A || !g.B || !g.sA || !g.sB || (!g.D && !g.q_codes)) return fail(FP4_ERR_INVALID_ARG, "null pointer");
  if (g.M <= 0 || g.N <= 0 || g.K <= 0) return fail(FP4_ERR_INVALID_ARG, "M, N, K must be positive");
  if (g.K % 32 != 0) return fail(FP4_ERR_INVALID_ARG, "K must be a multiple of 32");
  if (g.M > (1ll << 31) - 256 || g.N > (1ll << 31) - 256) return fail(FP4_ERR_UNSUPPORTED, "dimension too large");
  if (!aligned16(g.A) || !aligned16(g.B) || !aligned16(g.sA) || !aligned16(g.sB) || (g.D && !aligned16(g.D)))
    return fail(FP4_ERR_INVALID_ARG, "A, B, scales and D must be 16-byte aligned");
  unsigned* status;
  fp4_status s = device_state(&status);
  if (s != FP4_OK) return s;
  const char* why = nullptr;
  cudaError_t err = cudaSuccess;
  const int rc = launch_gemm(g, status, static_cast<cudaStream_t>(stream), &why, &err);
  if (rc == 1) return fail(FP4_ERR_INVALID_ARG, why);
  if (rc == 2) return cuda_fail(err, "gemm launch");
  return FP4_OK;
}

static bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31) == 0; }

fp4_status fp4_gemm_mixed(fp4_fmt a_fmt, const uint8_t* A, const uint8_t* sA, fp4_fmt b_fmt, const uint8_t* B,
                          const uint8_t* sB, int64_t M, int64_t N, int64_t K, void* D, fp4_dtype out_dtype,
                          void* stream) {
  if ((a_fmt != FP4_MXFP4 && a_fmt != FP4_MXFP8) || (b_fmt != FP4_MXFP4 && b_fmt != FP4_MXFP8))
    return fail(FP4_ERR_INVALID_ARG, "a_fmt and b_fmt must each be FP4_MXFP4 or FP4_MXFP8");
  if (out_dtype != FP4_F32 && out_dtype != FP4_BF16) return fail(FP4_ERR_INVALID_ARG, "out_dtype");
  if (!A || !B || !sA || !sB || !D) return fail(FP4_ERR_INVALID_ARG, "null pointer");
  if (M <= 0 || N <= 0 || K <= 0) return fail(FP4_ERR_INVALID_ARG, "M, N, K must be positive");
  if (K % 128 != 0) return fail(FP4_ERR_INVALID_ARG, "K must be a multiple of 128");
  if (M > (1ll << 31) - 256 || N > (1ll << 31) - 256) return fail(FP4_ERR_UNSUPPORTED, "dimension too large");
  if (!aligned32(A) || !aligned32(B) || !aligned16(sA) || !aligned16(sB) || !aligned16(D))
    return fail(FP4_ERR_INVALID_ARG, "A and B must be 32-byte aligned, scales and D 16-byte aligned");
  unsigned* status;
  fp4_status s = device_state(&status);
  if (s != FP4_OK) return s;
  GemmProblem g{};
  g.mx = 1;
  g.A = A;
  g.sA = sA;
  g.B = B;
  g.sB = sB;
  g.M = M;
  g.N = N;
  g.K = K;
  g.D = D;
  g.out_bf16 = out_dtype == FP4_BF16;
  const char* why = nullptr;
  cudaError_t err = cudaSuccess;
  const int rc = launch_gemm_mixed(g, a_fmt == FP4_MXFP8, b_fmt == FP4_MXFP8, status, static_cast<cudaStream_t>(stream),
                                   &why, &err);
  if (rc == 1) return fail(FP4_ERR_INVALID_ARG, why);
  if (rc == 2) return cuda_fail(err, "gemm launch");
  return FP4_OK;
}

fp4_status fp4_gemm_ex(fp4_fmt fmt, const uint8_t* A, const uint8_t* sA, const float* gA, const uint8_t* B,
                       const uint8_t* sB, const float* gB, int64_t M, int64_t N, int64_t K, void* D,
                       fp4_dtype out_dtype, void* workspace, size_t workspace_bytes, unsigned flags,
                       void* stream) {
  if (flags & ~static_cast<unsigned>(FP4_GEMM_WEIGHTS_READY)) return fail(FP4_ERR_INVALID_ARG, "unknown flag");
  GemmProblem g{};
  g.mx = fmt == FP4_MXFP4;
  g.A = A;
  g.sA = sA;
  g.gA = gA;
  g.B = B;
  g.sB = sB;
  g.gB = gB;
  g.M = M;
  g.N = N;
  g.K = K;
  g.D = D;
  g.out_bf16 = out_dtype == FP4_BF16;
  g.ws = workspace;
  g.ws_bytes = workspace_bytes;
  g.weights_ready = (flags & FP4_GEMM_WEIGHTS_READY) ? 1 : 0;
  return gemm_common(g, fmt, out_dtype, stream);
}

fp4_status fp4_gemm(fp4_fmt fmt, const uint8_t* A, const uint8_t* sA, const float* gA, const uint8_t* B,
                    const uint8_t* sB, const float* gB, int64_t M, int64_t N, int64_t K, void* D, fp4_dtype out_dtype,
                    void* workspace, size_t workspace_bytes, void* stream) {
  return fp4_gemm_ex(fmt, A, sA, gA, B, sB, gB, M, N, K, D, out_dtype, workspace, workspace_bytes, 0u, stream);
}

fp4_status fp4_gemm_epilogue(fp4_fmt fmt, const uint8_t* A, const uint8_t* sA, const float* gA, const uint8_t* B,
                             const uint8_t* sB, const float* gB, int64_t M, int64_t N, int64_t K, const float* bias,
                             fp4_act act, void* D, fp4_dtype out_dtype, uint8_t* Dcodes, uint8_t* Dscales,
                             const float* gD, float* amax_out, void* workspace, size_t workspace_bytes,
                             void* stream) {
  if (act != FP4_ACT_NONE && act != FP4_ACT_RELU) return fail(FP4_ERR_INVALID_ARG, "act");
  if (!D && !Dcodes) return fail(FP4_ERR_INVALID_ARG, "no output: D and Dcodes are both NULL");
  if (Dcodes && (!Dscales || !gD)) return fail(FP4_ERR_INVALID_ARG, "FP4 output needs Dscales and gD");
  if (Dcodes && N % 32 != 0) return fail(FP4_ERR_INVALID_ARG, "FP4 output needs N % 32 == 0");
  if (Dcodes && (!aligned16(Dcodes) || !aligned16(Dscales))) return fail(FP4_ERR_INVALID_ARG, "Dcodes / Dscales alignment");
  if (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)) return fail(FP4_ERR_INVALID_ARG, "bias alignment");
  GemmProblem g{};
  g.mx = fmt == FP4_MXFP4;
  g.A = A;
  g.sA = sA;
  g.gA = gA;
  g.B = B;
  g.sB = sB;
  g.gB = gB;
  g.M = M;
  g.N = N;
  g.K = K;
  g.D = D;
  g.out_bf16 = out_dtype == FP4_BF16;
  g.ws = workspace;
  g.ws_bytes = workspace_bytes;
  g.bias = bias;
  g.act = act == FP4_ACT_RELU ? 1 : 0;
  g.q_codes = Dcodes;
  g.q_scales = Dscales;
  g.q_g = gD;
  g.amax_out = amax_out;
  if (amax_out) {
    if (reinterpret_cast<uintptr_t>(amax_out) & 3u) return fail(FP4_ERR_INVALID_ARG, "amax_out alignment");
    const cudaError_t e = cudaMemsetAsync(amax_out, 0, sizeof(float), static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "zeroing amax_out");
  }
  if (Dcodes && (M % 128 != 0 || (N / 16) % 4 != 0)) {
    // the kernel writes the scale bytes of real rows and blocks; the layout's pad bytes
    // (rows up to a multiple of 128, block columns up to a multiple of 4) must read as 0
    const cudaError_t e =
        cudaMemsetAsync(Dscales, 0, fp4_scales_bytes(M, N, FP4_NVFP4), static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "zero-filling the scale pads");
  }
  return gemm_common(g, fmt, out_dtype, stream);
}

size_t fp4_gemm_epilogue_workspace_size(int64_t M, int64_t N, int64_t K, fp4_fmt fmt, int rows_in_place) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  return gemm_workspace_bytes(M, N, K, fmt == FP4_MXFP4, rows_in_place != 0);
}

size_t fp4_gemm_bf16a_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  return gemm_bf16a_workspace_bytes(M, N, K);
}

fp4_status fp4_gemm_bf16a(const void* X, const uint8_t* B, const uint8_t* sB, const float* gB, int64_t M, int64_t N,
                          int64_t K, void* D, fp4_dtype out_dtype, uint8_t* Xcodes, uint8_t* Xscales, float* gX,
                          void* workspace, size_t workspace_bytes, unsigned flags, void* stream) {
  if (!X || !B || !sB || !D || !Xcodes || !Xscales || !gX || !workspace) return fail(FP4_ERR_INVALID_ARG, "null pointer");
  if (M <= 0 || N <= 0 || K <= 0 || K % 32 != 0) return fail(FP4_ERR_INVALID_ARG, "shape (K % 32 == 0)");
  if (out_dtype != FP4_F32 && out_dtype != FP4_BF16) return fail(FP4_ERR_INVALID_ARG, "out_dtype");
  if (flags & ~static_cast<unsigned>(FP4_GEMM_WEIGHTS_READY)) return fail(FP4_ERR_INVALID_ARG, "unknown flag");
  if (!aligned16(X) || !aligned16(B) || !aligned16(sB) || !aligned16(D) || !aligned16(Xcodes) || !aligned16(Xscales) ||
      !aligned16(workspace))
    return fail(FP4_ERR_INVALID_ARG, "buffers must be 16-byte aligned");
  if (workspace_bytes < gemm_bf16a_workspace_bytes(M, N, K))
    return fail(FP4_ERR_INVALID_ARG, "workspace too small (see fp4_gemm_bf16a_workspace_size)");
  const size_t qws = (kQuantWorkspaceBytes + 255) / 256 * 256;
  if (decode_eligible(M, N, K)) {
    // one launch: every CTA derives the activations' global scale and quantizes its K
    // segment of them itself while its weight stages stream in
    unsigned* status;
    const fp4_status ds = device_state(&status);
    if (ds != FP4_OK) return ds;
    DecodeProblem q{};
    q.W = B;
    q.sW = sB;
    q.gW = gB;
    q.X = X;
    q.Xq_out = Xcodes;
    q.Xs_out = Xscales;
    q.gX_out = gX;
    q.M = M;
    q.N = N;
    q.K = K;
    q.D = D;
    q.out_bf16 = out_dtype == FP4_BF16;
    q.ws = static_cast<uint8_t*>(workspace) + qws;
    q.ws_bytes = workspace_bytes - qws;
    q.weights_ready = (flags & FP4_GEMM_WEIGHTS_READY) ? 1 : 0;
    q.stall_plus1 = g_stall_next_decode;
    g_stall_next_decode = 0;
    const char* why = nullptr;
    cudaError_t err = cudaSuccess;
    const int rc = launch_decode(q, status, static_cast<cudaStream_t>(stream), &why, &err);
    if (rc == 1) return fail(FP4_ERR_INVALID_ARG, why);
    if (rc == 2) return cuda_fail(err, "decode GEMM launch");
    return FP4_OK;
  }
  // larger M: the activations' amax and codes, then the GEMM, chained by programmatic
  // dependent launch (FP4_GEMM_WEIGHTS_READY lets the GEMM stream the weights early)
  const fp4_status s = fp4_quantize(X, M, K, FP4_BF16, FP4_NVFP4, 16, Xcodes, Xscales, gX, nullptr, nullptr, nullptr, workspace,
                   kQuantWorkspaceBytes, stream);
  if (s != FP4_OK) return s;
  return fp4_gemm_ex(FP4_NVFP4, Xcodes, Xscales, gX, B, sB, gB, M, N, K, D, out_dtype,
                     static_cast<uint8_t*>(workspace) + qws, workspace_bytes - qws, flags, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------------
// Allocation-free GEMM.  Some callers cannot allocate device memory: a host (plugin
// runtime, embedded engine) that owns every device byte and hands this library no
// allocator.  They still need the split-K scratch that decode-sized GEMMs use, so this
// variant takes it from a fixed array compiled into the library instead of from the
// caller.
namespace fp4 {
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB on every device that loads the library
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the array on the current device.  The array's host-side name is
// only a stand-in; the device address comes from cudaGetSymbolAddress, done once per
// device with that device current (the first call on a device does it, so make that
// first call before any stream capture).
static fp4_status noalloc_scratch(void** out) {
  static void* addr[kMaxDevices] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(FP4_ERR_UNSUPPORTED, "device index out of range");
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
    addr[dev] = p;
  }
  *out = addr[dev];
  return FP4_OK;
}
}  // namespace fp4

extern "C" {

fp4_status fp4_gemm_noalloc(fp4_fmt fmt, const uint8_t* A, const uint8_t* sA, const float* gA, const uint8_t* B,
                            const uint8_t* sB, const float* gB, int64_t M, int64_t N, int64_t K, void* D,
                            fp4_dtype out_dtype, void* stream) {
  if (fmt != FP4_NVFP4 && fmt != FP4_MXFP4) return fail(FP4_ERR_INVALID_ARG, "fmt");
  const size_t need = (M > 0 && N > 0 && K > 0) ? gemm_workspace_bytes(M, N, K, fmt == FP4_MXFP4) : 0;
  if (need > kNoAllocScratchBytes) {
    snprintf(g_err, sizeof(g_err),
             "fp4_gemm_noalloc: this shape needs %zu bytes of scratch but the built-in array holds %zu "
             "(4 MiB); use fp4_gemm with a caller workspace",
             need, kNoAllocScratchBytes);
    return FP4_ERR_INVALID_ARG;
  }
  void* ws = nullptr;
  if (need) {
    fp4_status s = noalloc_scratch(&ws);
    if (s != FP4_OK) return s;
    // every call shares the array: clear the part this call accumulates into
    cudaError_t e = cudaMemsetAsync(ws, 0, need, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the no-alloc scratch");
  }
  return fp4_gemm(fmt, A, sA, gA, B, sB, gB, M, N, K, D, out_dtype, ws, need, stream);
}

fp4_status fp4_gemm_grouped(fp4_fmt fmt, int num_groups, const int32_t* offsets, const uint8_t* A,
                            const uint8_t* sA, const float* gA, const uint8_t* B, const uint8_t* sB,
                            const float* gB, int64_t total_rows, int64_t N, int64_t K, void* D,
                            fp4_dtype out_dtype, void* workspace, size_t workspace_bytes, void* stream) {
  if (num_groups <= 0 || num_groups > kMaxGroups || !offsets) return fail(FP4_ERR_INVALID_ARG, "groups / offsets");
  if (N % 128 != 0) return fail(FP4_ERR_INVALID_ARG, "grouped GEMM needs N % 128 == 0");
  if (total_rows <= 0) return fail(FP4_ERR_INVALID_ARG, "total_rows must be positive");
  GemmProblem g{};
  g.mx = fmt == FP4_MXFP4;
  g.A = A;
  g.sA = sA;
  g.gA = gA;
  g.B = B;
  g.sB = sB;
  g.gB = gB;
  g.M = total_rows;
  g.N = N;
  g.K = K;
  g.D = D;
  g.out_bf16 = out_dtype == FP4_BF16;
  g.ws = workspace;
  g.ws_bytes = workspace_bytes;
  g.num_groups = num_groups;
  g.offsets = offsets;
  return gemm_common(g, fmt, out_dtype, stream);
}

fp4_status fp4_get_status(void* stream) {
  unsigned* status;
  fp4_status s = device_state(&status);
  if (s != FP4_OK) return s;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  unsigned v = 0;
  e = cudaMemcpyFromSymbol(&v, g_status_word, sizeof(v));
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  const unsigned zero = 0;
  e = cudaMemcpyToSymbol(g_status_word, &zero, sizeof(zero));
  if (e != cudaSuccess) return cuda_fail(e, "status clear");
  if (v & kStatusTimeout) return fail(FP4_ERR_TIMEOUT, "a device-side wait timed out");
  if (v & kStatusNonFinite) return fail(FP4_ERR_NONFINITE, "non-finite input element");
  return FP4_OK;
}

fp4_status fp4_mma_peak(int iters, int grid, unsigned long long* cycles, void* stream) {
  if (!cycles || iters <= 0 || iters > (1 << 24) || grid <= 0 || grid > 4 * num_sms())
    return fail(FP4_ERR_INVALID_ARG, "iters in 1..2^24, grid in 1..4 x SMs, cycles non-null");
  unsigned* status;
  fp4_status s = device_state(&status);
  if (s != FP4_OK) return s;
  const cudaError_t e = launch_mma_peak(iters, grid, cycles, status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FP4_OK : cuda_fail(e, "MMA peak launch");
}

fp4_status fp4_debug_stall_next_decode(int cta) {
  if (cta < 0) return fail(FP4_ERR_INVALID_ARG, "cta must be >= 0");
  g_stall_next_decode = cta + 1;
  return FP4_OK;
}

fp4_status fp4_debug_encode(const float* in, int64_t n, int which, uint8_t* out, void* stream) {
  if (!in || !out) return fail(FP4_ERR_INVALID_ARG, "null pointer");
  if (n <= 0 || which < 0 || which > 4) return fail(FP4_ERR_INVALID_ARG, "n / which");
  unsigned* status;
  fp4_status s = device_state(&status);
  if (s != FP4_OK) return s;
  cudaError_t e = launch_debug_encode(in, n, which, out, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FP4_OK : cuda_fail(e, "debug encode launch");
}

}  // extern "C"
