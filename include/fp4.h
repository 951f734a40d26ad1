/*
 * fp4.h -- C ABI of libfp4: block-scaled 4-bit floating point (NVFP4, MXFP4)
 * quantization and the FP4 GEMM that consumes it, for NVIDIA B200 (sm_100a).
 *
 * Value format (all entry points): E2M1 -- 1 sign, 2 exponent (bias 1), 1 mantissa
 * bit; the only values are 0, +-0.5, +-1, +-1.5, +-2, +-3, +-4, +-6, no inf, no NaN
 * ("FP4" glossary entry, ultralytics.com, opening paragraph; "Rubin FP4 GEMM
 * overview", yfxerp.com, section 3.1 for the bit split).
 *
 * Block formats ("FP4" glossary entry, "How FP4 works"; "MXFP4 / NVFP4 video
 * transcript", prism.simon-ai.net, the MXFP4 and NVFP4 passages):
 *   NVFP4: 16 consecutive values share one E4M3 scale byte; the tensor carries one
 *          FP32 global scale g = amax(|x|) / (6 * 448) (g = 1 for an all-zero tensor).
 *   MXFP4: 32 consecutive values share one E8M0 (power-of-two) scale byte; g = 1.
 *
 * Data layouts (shared by every entry point):
 *   codes   row-major [rows, cols/2] bytes; element 2j of a row in the low nibble of
 *           byte j, element 2j+1 in the high nibble ("Rubin FP4 GEMM overview" 5.2
 *           says nibble order is an API convention; this is ours).
 *   scales  the row-major [rows, cols/block] matrix of scale bytes stored as 128x4
 *           atoms of 512 bytes: rows padded to a multiple of 128, scale columns to a
 *           multiple of 4 (pad bytes are written as 0).  Entry (r, c) lives at byte
 *             ((r/128) * (Cpad/4) + c/4) * 512 + (r%32) * 16 + ((r%128)/32) * 4 + c%4
 *           with Cpad = ceil(cols/block, 4).  This is the layout the tensor cores read
 *           scale factors in ("Rubin FP4 GEMM overview" 4.2: the scale layout must be
 *           tile-loadable together with the matrix).  fp4_scales_bytes() gives the size.
 *   grouped scales (MoE activations): each group's rows start a fresh 128-row block;
 *           group e's first block is sum_{e'<e} ceil(rows_e'/128).
 *   GEMM    A [M, K] and B [N, K], both K-major (the contraction dimension
 *           contiguous), D [M, N] row-major, D = (A_hat . B_hat^T) where the hats
 *           are the dequantized operands ("Rubin FP4 GEMM overview" 3.1, 3.2: FP4
 *           inputs, FP32 accumulation, block scales re-applied, global scales in the
 *           epilogue per 4.2).
 *
 * Ownership and streams: every pointer named *_dev or documented "device" is
 * caller-owned device memory; the library allocates no device memory in any call.
 * All work is enqueued on the caller's stream (cudaStream_t passed as void*; NULL is
 * the legacy default stream); no call synchronizes the host except
 * fp4_get_status().  Global scales stay on the device (no host round trip).
 *
 * Errors: argument checks happen before anything is enqueued and return
 * FP4_ERR_INVALID_ARG / FP4_ERR_UNSUPPORTED; a failed launch returns FP4_ERR_CUDA.
 * Errors found on the device (a non-finite input element, a bounded wait that ran
 * out) are latched in a per-device status word that fp4_get_status() reads and
 * clears.  Outputs of a call that latched an error are unspecified.
 */
#ifndef FP4_H_
#define FP4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* FP4_MXFP8: E4M3 elements (one byte each) with an E8M0 scale per 32 -- the FP8 operand of
 * fp4_gemm_mixed ("Rubin FP4 GEMM overview" 3.4: an FP4 operand opposite an FP8 one; 3.1
 * names MXFP8 beside MXFP4 among the OCP microscaling formats). */
typedef enum { FP4_NVFP4 = 0, FP4_MXFP4 = 1, FP4_MXFP8 = 2 } fp4_fmt;
typedef enum { FP4_F32 = 0, FP4_BF16 = 1 } fp4_dtype;
typedef enum {
  FP4_OK = 0,
  FP4_ERR_INVALID_ARG = 1, /* null pointer, bad size or alignment, too-small workspace */
  FP4_ERR_UNSUPPORTED = 2, /* legal but not implemented combination, or no sm_100 device */
  FP4_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
  FP4_ERR_TIMEOUT = 4,     /* a device-side bounded wait gave up (latched) */
  FP4_ERR_NONFINITE = 5    /* an input element was inf or NaN (latched) */
} fp4_status;

/* Library version string and the last host-side error message of this thread. */
const char* fp4_version(void);
const char* fp4_last_error(void);

/* Bytes of the swizzled scale-factor buffer for a [rows, cols] tensor in fmt
 * (block 16 for NVFP4, 32 for MXFP4): ceil(rows,128) * ceil(cols/block, 4). */
size_t fp4_scales_bytes(int64_t rows, int64_t cols, fp4_fmt fmt);

/* Upper bound of the grouped scale-factor buffer for total_rows rows split into
 * num_groups groups: (ceil(total_rows/128) + num_groups) * 128 * Cpad. */
size_t fp4_scales_bytes_grouped(int64_t total_rows, int num_groups, int64_t cols, fp4_fmt fmt);

/* Device workspace that fp4_quantize / fp4_quantize_grouped / fp4_amax need (for
 * the tensor-amax reduction).  It must be zero-filled before its first use; every
 * call leaves it zero-filled again.  Calls sharing one workspace must not overlap. */
size_t fp4_quantize_workspace_size(void);

/* Tensor amax ("MXFP4 / NVFP4 video transcript", NVFP4 passage: the FP32 tensor scale
 * covers the tensor's global range): amax_out_dev[0] = max_i |x_i| over n elements of
 * in_dtype.  A non-finite element latches FP4_ERR_NONFINITE.  x 16-byte aligned. */
fp4_status fp4_amax(const void* x_dev, int64_t n, fp4_dtype in_dtype, float* amax_out_dev,
                    void* workspace_dev, size_t workspace_bytes, void* stream);

/* Block-scaled quantization of a row-major [rows, cols] tensor ("FP4" glossary entry,
 * "How FP4 works": the block scale maps the block's largest magnitude to 6; values
 * round to the nearest E2M1 grid point, ties to the even mantissa; packed two per byte).
 *   fmt/block: (FP4_NVFP4, 16) 1-D blocks along cols; (FP4_MXFP4, 32) 1-D blocks;
 *              (FP4_NVFP4, 256) 16x16 2-D blocks for weights ("MXFP4 / NVFP4 video
 *              transcript", training-recipe passage: W and W^T share one quantization);
 *              (FP4_MXFP8, 32) E4M3 elements in 1-D blocks (not grouped).
 *   codes_out_dev  [rows, cols/2] ([rows, cols] for MXFP8); scales_out_dev
 *              fp4_scales_bytes(rows, cols, fmt).
 *   global_out_dev 1 float: g (NVFP4) or 1.0 (MXFP4).  May be NULL for MXFP4.
 *   codesT_out_dev / scalesT_out_dev: block 256 only -- W^T's codes [cols, rows/2] and
 *              scales fp4_scales_bytes(cols, rows, NVFP4); NULL otherwise.
 *   global_in_dev: NULL -> compute amax and g on the device (two passes over x);
 *              else the caller's g (one pass; e.g. a calibrated scale).
 * Requires cols % 32 == 0, 1 <= rows <= 2^31 - 256 (else FP4_ERR_UNSUPPORTED); block 256
 * also rows % 32 == 0; x, codes and scales 16-byte aligned.  NVFP4 block scale:
 * sb = E4M3_rn_sat((amax_b / 6) / g); elements x * (1 / (dec(sb) * g)) in FP32.  MXFP4:
 * sb = E8M0 nearest power of two of amax_b / 6 (a midpoint goes up); elements
 * x * 2^(127 - sb).  MXFP8: sb = E8M0 nearest power of two of amax_b / 448 (the sources
 * cited above fix no rule for MXFP8; 448 is E4M3's largest value as 6 is E2M1's); elements
 * E4M3_rn_sat(x * 2^(127 - sb)), sign in bit 7. */
fp4_status fp4_quantize(const void* x_dev, int64_t rows, int64_t cols, fp4_dtype in_dtype,
                        fp4_fmt fmt, int block, uint8_t* codes_out_dev, uint8_t* scales_out_dev,
                        float* global_out_dev, uint8_t* codesT_out_dev, uint8_t* scalesT_out_dev,
                        const float* global_in_dev, void* workspace_dev, size_t workspace_bytes,
                        void* stream);

/* As fp4_quantize (1-D blocks) for MoE activations whose rows are grouped by expert:
 * offsets_dev[num_groups + 1] (device int32, nondecreasing, offsets[0] = 0,
 * offsets[num_groups] = rows) delimit the groups; scales are written in the grouped
 * layout (size <= fp4_scales_bytes_grouped(rows, num_groups, cols, fmt); the bytes
 * up to that bound are written, pads 0).  For NVFP4 one g covers all groups. */
fp4_status fp4_quantize_grouped(const void* x_dev, int64_t rows, int64_t cols, fp4_dtype in_dtype,
                                fp4_fmt fmt, int num_groups, const int32_t* offsets_dev,
                                uint8_t* codes_out_dev, uint8_t* scales_out_dev,
                                float* global_out_dev, const float* global_in_dev,
                                void* workspace_dev, size_t workspace_bytes, void* stream);

/* fp4_quantize with options ("MXFP4 / NVFP4 video transcript", MXFP4 passage: a scale
 * that is not a power of two must be rounded to one, 70 to 64 or 128).  flags:
 *   FP4_QUANT_E8M0_FLOOR  (MXFP4 only) round the block scale down instead of to nearest:
 *       sb = 2^(floor(log2 amax_b) - 2), the largest power of two not above amax_b divided
 *       by 4 (E2M1's largest power of two), code clamped to [0, 254].  The block's largest
 *       element then scales into [4, 8); values from 6 up saturate to 6.
 * Other arguments and errors as fp4_quantize; unknown bits return FP4_ERR_INVALID_ARG. */
#define FP4_QUANT_E8M0_FLOOR 1u
fp4_status fp4_quantize_ex(const void* x_dev, int64_t rows, int64_t cols, fp4_dtype in_dtype, fp4_fmt fmt,
                           int block, unsigned flags, uint8_t* codes_out_dev, uint8_t* scales_out_dev,
                           float* global_out_dev, uint8_t* codesT_out_dev, uint8_t* scalesT_out_dev,
                           const float* global_in_dev, void* workspace_dev, size_t workspace_bytes,
                           void* stream);

/* NVFP4 1-D quantization with stochastic rounding of the elements ("MXFP4 / NVFP4 video
 * transcript", training-recipe passage: 0.3 between 0 and 1 becomes 1 with probability
 * 0.3, so that the expected value is kept; used for gradients).  The global and block
 * scales are fp4_quantize's; only the element rounding changes: a scaled magnitude a
 * between grid neighbours lo < a < hi becomes hi iff u < (a - lo) / (hi - lo), with
 * u = (rbits[i] >> 8) * 2^-24; grid values stay, a >= 6 saturates, the sign is kept.
 *   rbits_dev  one uint32 random word per element, row-major [rows, cols], 16-byte
 *              aligned (the caller draws them).
 * Other arguments and errors as fp4_quantize (block 16). */
fp4_status fp4_quantize_sr(const void* x_dev, int64_t rows, int64_t cols, fp4_dtype in_dtype,
                           const uint32_t* rbits_dev, uint8_t* codes_out_dev, uint8_t* scales_out_dev,
                           float* global_out_dev, const float* global_in_dev, void* workspace_dev,
                           size_t workspace_bytes, void* stream);

/* Quantization after a 16-point random Hadamard transform ("MXFP4 / NVFP4 video
 * transcript", training-recipe passage; "FP4" glossary entry, "Inference and training in
 * FP4": outliers are spread over their block before quantizing).  Every 16-element block
 * b along cols becomes (1/4) H16 diag(s) b, H16 the Sylvester Hadamard matrix and
 * s_j = -1 where bit j of `signs` (16 bits) is set, computed in FP32 as the signs, the
 * butterfly stages of half-width 1, 2, 4, 8, then the factor 1/4; the transformed tensor
 * is then quantized as fp4_quantize does (NVFP4 block 16, g from the transformed tensor's
 * amax unless global_in_dev is given; or MXFP4 block 32).  Both operands of a GEMM
 * transformed with the same signs keep their products: Q is orthogonal. */
fp4_status fp4_quantize_rht(const void* x_dev, int64_t rows, int64_t cols, fp4_dtype in_dtype, fp4_fmt fmt,
                            uint32_t signs, uint8_t* codes_out_dev, uint8_t* scales_out_dev,
                            float* global_out_dev, const float* global_in_dev, void* workspace_dev,
                            size_t workspace_bytes, void* stream);

/* NVFP4 global scale from a tensor amax already on the device ("MXFP4 / NVFP4 video
 * transcript", NVFP4 passage): global_out_dev[0] = amax / (6 * 448), or 1 for amax = 0.
 * For tensors split over ranks: each rank's fp4_amax, one all-reduce (MAX) of that float,
 * then this call gives every rank the g of the whole tensor, and fp4_quantize with
 * global_in_dev = g quantizes each shard exactly as the whole tensor would be.  A
 * non-finite amax latches FP4_ERR_NONFINITE. */
fp4_status fp4_global_scale(const float* amax_dev, float* global_out_dev, void* stream);

/* Dequantize (debug / tests): out_dev[r, k] = E2M1(code) * dec(scale) * g as FP32, for a
 * [rows, cols] tensor in the layouts above; global_dev may be NULL (g = 1). */
fp4_status fp4_dequantize(const uint8_t* codes_dev, const uint8_t* scales_dev,
                          const float* global_dev, int64_t rows, int64_t cols, fp4_fmt fmt,
                          float* out_dev, void* stream);

/* Device workspace bytes fp4_gemm needs for this shape (0 if none).  It must be
 * zero-filled before first use; every call leaves it zero-filled again.  After a call
 * that latched FP4_ERR_TIMEOUT its contents are undefined: zero it again. */
size_t fp4_gemm_workspace_size(int64_t M, int64_t N, int64_t K, fp4_fmt fmt);

/* Block-scaled FP4 GEMM on the 5th-generation tensor cores ("Rubin FP4 GEMM overview"
 * 3.1-3.2 and 4.2): D[m, n] = gA * gB * sum_k dec(sA[m, k/blk]) dec(sB[n, k/blk])
 *                             * e2m1(A[m, k]) * e2m1(B[n, k]), FP32 accumulation.
 *   A_dev [M, K/2] codes, sA_dev scales (fp4_scales_bytes(M, K, fmt)), gA_dev 1 float
 *   (NULL -> 1.0); B_dev [N, K/2], sB_dev, gB_dev likewise; D_dev [M, N] row-major,
 *   out_dtype FP4_BF16 (round to nearest even) or FP4_F32.
 * Requires K % 32 == 0, M, N >= 1, 16-byte aligned A, B, sA, sB and D.  Small M
 * (decode) runs with A and B swapped on the tensor cores and a split over K, which
 * uses the workspace. */
fp4_status fp4_gemm(fp4_fmt fmt, const uint8_t* A_dev, const uint8_t* sA_dev, const float* gA_dev,
                    const uint8_t* B_dev, const uint8_t* sB_dev, const float* gB_dev,
                    int64_t M, int64_t N, int64_t K, void* D_dev, fp4_dtype out_dtype,
                    void* workspace_dev, size_t workspace_bytes, void* stream);

/* fp4_gemm with options.  flags is a bitwise OR of:
 *   FP4_GEMM_WEIGHTS_READY  B, sB and gB were written before the kernel that runs just
 *       before this call on `stream` (for example pre-quantized weights).  The GEMM may
 *       then start streaming B while that kernel (typically the activation quantize)
 *       is still running; A and its scales are read only after it has finished.  Setting
 *       the flag when B is produced by the immediately preceding kernel is a data race.
 * Unknown bits return FP4_ERR_INVALID_ARG. */
#define FP4_GEMM_WEIGHTS_READY 1u
fp4_status fp4_gemm_ex(fp4_fmt fmt, const uint8_t* A_dev, const uint8_t* sA_dev, const float* gA_dev,
                       const uint8_t* B_dev, const uint8_t* sB_dev, const float* gB_dev,
                       int64_t M, int64_t N, int64_t K, void* D_dev, fp4_dtype out_dtype,
                       void* workspace_dev, size_t workspace_bytes, unsigned flags, void* stream);

/* GEMM with the epilogue that follows the scale ("Rubin FP4 GEMM overview" 3.2: the FP32
 * result is multiplied by the scale factors, the bias is added, the activation applied,
 * then it is converted to the output format, FP4 included; 4.2: C = (A.B)(sA.sB) + bias):
 *   t[m, n] = act(gA gB sum_k ... + bias[n])      (FP32: product, then + bias, then act)
 *   D_dev   [M, N] in out_dtype (BF16 round to nearest even, or FP32), or NULL;
 *   Dcodes_dev / Dscales_dev: or an NVFP4 copy of t (or both): 16-element blocks along n,
 *           codes [M, N/2], scales fp4_scales_bytes(M, N, FP4_NVFP4) in the swizzled
 *           layout, quantized exactly as fp4_quantize would quantize the FP32 t with
 *           global_in = gD_dev (the caller's global scale: t's amax is not known until
 *           the whole product is, so it cannot be computed here).  The layout's pad
 *           bytes are written as 0, as fp4_quantize writes them.  The result can feed
 *           the next fp4_gemm as its A operand directly.  Needs N % 32 == 0.
 *   bias_dev [N] FP32 or NULL; act FP4_ACT_NONE or FP4_ACT_RELU.
 *   amax_out_dev: 1 float, or NULL: max |t| over the whole result (zeroed, then written
 *           by this call), so that the next quantization of t (fp4_global_scale, then
 *           fp4_quantize with global_in) needs no separate amax pass over it.
 * workspace: fp4_gemm_epilogue_workspace_size(M, N, K, fmt, rows_in_place) bytes with
 * rows_in_place = (Dcodes_dev != NULL || amax_out_dev != NULL), zero-filled before first
 * use (left zero-filled).  Plain (not grouped) problems only. */
/* Mixed-format GEMM ("Rubin FP4 GEMM overview" 3.4: weights in FP4 where they tolerate it,
 * activations kept in FP8, or the other way round): D[M, N] = A[M, K] B[N, K]^T with each
 * operand FP4_MXFP4 (E2M1 codes [rows, K/2], E8M0 scales per 32) or FP4_MXFP8 (E4M3
 * codes [rows, K], E8M0 scales per 32), as fp4_quantize writes them; scales in the
 * swizzled layout, fp4_scales_bytes(rows, K, fmt) bytes.  FP32 accumulation of the
 * block-scaled products on the tensor cores (tcgen05 kind::mxf8f6f4: an FP4 operand is
 * widened to one byte per element in shared memory by the tensor copy).  D row-major,
 * FP32 or BF16.  Requires K % 128 == 0 (the limit of CUDA's 4-bit tensor-copy type), A
 * and B 32-byte aligned, scales and D 16-byte aligned; no workspace.  Errors:
 * FP4_ERR_INVALID_ARG before any launch. */
fp4_status fp4_gemm_mixed(fp4_fmt a_fmt, const uint8_t* A_dev, const uint8_t* sA_dev, fp4_fmt b_fmt,
                          const uint8_t* B_dev, const uint8_t* sB_dev, int64_t M, int64_t N, int64_t K,
                          void* D_dev, fp4_dtype out_dtype, void* stream);

typedef enum { FP4_ACT_NONE = 0, FP4_ACT_RELU = 1 } fp4_act;
size_t fp4_gemm_epilogue_workspace_size(int64_t M, int64_t N, int64_t K, fp4_fmt fmt, int rows_in_place);
fp4_status fp4_gemm_epilogue(fp4_fmt fmt, const uint8_t* A_dev, const uint8_t* sA_dev, const float* gA_dev,
                             const uint8_t* B_dev, const uint8_t* sB_dev, const float* gB_dev,
                             int64_t M, int64_t N, int64_t K, const float* bias_dev, fp4_act act,
                             void* D_dev, fp4_dtype out_dtype, uint8_t* Dcodes_dev, uint8_t* Dscales_dev,
                             const float* gD_dev, float* amax_out_dev, void* workspace_dev,
                             size_t workspace_bytes, void* stream);

/* BF16-activation GEMM (quantize-on-load): D = gX * gB * (Xq . Bq^T) where Xq is the
 * NVFP4 quantization of the bf16 activations X [M, K] (tensor amax -> gX, 16-blocks,
 * exactly as fp4_quantize) and B [N, K] holds pre-quantized NVFP4 weights.  The
 * activations' codes [M, K/2], scales (fp4_scales_bytes(M, K, NVFP4)) and gX are
 * written to Xcodes_dev / Xscales_dev / gX_dev as well.  ("Rubin FP4 GEMM overview"
 * 3.2: loads feed the tensor cores; the activations enter in BF16.)
 *   M <= 32 (decode): one cooperative launch.  Every CTA reduces a share of X, the
 *     shares meet through per-CTA slots in the workspace (bounded waits), and each CTA
 *     quantizes the K segment of X it needs straight into shared memory while its
 *     first weight stages stream in; split-K partial sums are reduced in the workspace
 *     and written out by the CTA that owns each tile.
 *   M > 32: fp4_quantize then fp4_gemm_ex, chained with programmatic dependent launch.
 * flags: FP4_GEMM_WEIGHTS_READY as for fp4_gemm_ex.  workspace: at least
 * fp4_gemm_bf16a_workspace_size(M, N, K) bytes, zero-filled before its first use; the
 * library keeps its contents consistent from call to call, so do not modify it between
 * calls, and calls sharing one workspace must not overlap. */
size_t fp4_gemm_bf16a_workspace_size(int64_t M, int64_t N, int64_t K);
fp4_status fp4_gemm_bf16a(const void* X_dev, const uint8_t* B_dev, const uint8_t* sB_dev, const float* gB_dev,
                          int64_t M, int64_t N, int64_t K, void* D_dev, fp4_dtype out_dtype,
                          uint8_t* Xcodes_dev, uint8_t* Xscales_dev, float* gX_dev,
                          void* workspace_dev, size_t workspace_bytes, unsigned flags, void* stream);

/* fp4_gemm for callers that cannot allocate device memory.  The sources cited above
 * have no counterpart to this entry point.  Some hosts own every byte of device memory and give
 * this library no allocator: plugin runtimes and embedded inference engines that carve
 * one arena out of the GPU at start-up and treat any later cudaMalloc as a failure.
 * Arguments as fp4_gemm minus the workspace.  The split-K scratch that decode-sized
 * problems need comes from a fixed 4 MiB array compiled into the library, which every
 * GPU that loads the library holds until the process exits; shapes whose scratch
 * (fp4_gemm_workspace_size) exceeds 4 MiB return FP4_ERR_INVALID_ARG.  The first call
 * on a device looks up the array's device address with cudaGetSymbolAddress, so make
 * that first call before any stream capture.  Every call clears the part of the array
 * it uses, and all calls on a device share the array: calls that overlap on the GPU
 * race.  Calls no cudaMalloc or cudaFree. */
fp4_status fp4_gemm_noalloc(fp4_fmt fmt, const uint8_t* A_dev, const uint8_t* sA_dev, const float* gA_dev,
                            const uint8_t* B_dev, const uint8_t* sB_dev, const float* gB_dev,
                            int64_t M, int64_t N, int64_t K, void* D_dev, fp4_dtype out_dtype,
                            void* stream);

/* Grouped (MoE) GEMM ("FP4" glossary entry, inference passage: MoE weights kept in
 * MXFP4): for each group e, rows [offsets[e], offsets[e+1]) of A times expert e's
 * weights B_dev + e*N*K/2 give the same rows of D:
 *   D[r, n] = gA * gB[e] * sum_k ...   (as fp4_gemm).
 *   A_dev [total_rows, K/2] with grouped scales sA_dev (fp4_quantize_grouped; the
 *   buffer holds fp4_scales_bytes_grouped(total_rows, num_groups, K, fmt) bytes);
 *   B_dev [num_groups, N, K/2], sB_dev num_groups consecutive fp4_scales_bytes(N, K)
 *   blocks; gB_dev [num_groups] floats or NULL; offsets_dev device int32 [groups+1]
 *   with offsets[num_groups] == total_rows.  D_dev [total_rows, N].
 * Requires K % 32 == 0, N % 128 == 0, num_groups <= 1024. */
fp4_status fp4_gemm_grouped(fp4_fmt fmt, int num_groups, const int32_t* offsets_dev,
                            const uint8_t* A_dev, const uint8_t* sA_dev, const float* gA_dev,
                            const uint8_t* B_dev, const uint8_t* sB_dev, const float* gB_dev,
                            int64_t total_rows, int64_t N, int64_t K, void* D_dev,
                            fp4_dtype out_dtype, void* workspace_dev, size_t workspace_bytes,
                            void* stream);

/* Reads and clears the device status word latched by earlier calls on this device
 * (after synchronizing `stream`).  Returns FP4_OK, FP4_ERR_NONFINITE or FP4_ERR_TIMEOUT
 * (the first error latched), or FP4_ERR_CUDA if the synchronization failed. */
fp4_status fp4_get_status(void* stream);

/* Measured peak of the block-scaled tensor-core MMA ("NVIDIA FP4" article, hardware table:
 * 9 PFLOP/s dense FP4 on B200 is the vendor's figure; this measures what the tensor pipe
 * sustains here).  grid CTAs (one per SM) each issue iters x 4 back-to-back
 * tcgen05.mma.kind::mxf4nvf4 of M = 128, N = 256, K = 64 from shared memory into TMEM,
 * with no loads and no epilogue, and write the loop's clock64 cycles to cycles_dev[cta].
 * Each CTA does 2 * 128 * 256 * 64 * 4 * iters FLOP; time the launch with events on
 * `stream` for FLOP/s.  iters <= 2^24. */
fp4_status fp4_mma_peak(int iters, int grid, unsigned long long* cycles_dev, void* stream);

/* Test hook for the device-side bounded waits (tests only): the next fp4_gemm_bf16a call
 * of this thread that takes the single-launch decode path runs with CTA `cta` never
 * publishing its share of the activations' tensor amax.  Every CTA's bounded wait for
 * that share then runs out (after about 2 s), the call latches FP4_ERR_TIMEOUT, every
 * CTA releases its resources and returns, and the outputs are unspecified.  Zero-fill
 * the workspace before its next use.  A cta beyond the grid has no effect. */
fp4_status fp4_debug_stall_next_decode(int cta);

/* Encoder check entry point (tests): out_dev[i] = the code the device encoders give
 * in_dev[i] (no scaling), i < n.  which = 0: E2M1 code (sign in bit 3) from the encoder
 * the quantize kernels use; 1: E4M3 scale byte of in_dev[i] >= 0; 2: E8M0 scale byte of
 * in_dev[i] >= 0; 3: E2M1 by threshold counting; 4: E2M1 by the hardware conversion. */
fp4_status fp4_debug_encode(const float* in_dev, int64_t n, int which, uint8_t* out_dev, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* FP4_H_ */
