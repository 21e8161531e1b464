/*
 * libvlaq — NVFP4 / FP8 quantize + linear for one NVIDIA B200 (sm_100a).
 *
 * The quantized linear projection of a VLA language backbone:
 *   1. dynamic per-token NVFP4 activation quantization, optionally after a
 *      fused RMSNorm and a block-64 Walsh-Hadamard rotation;
 *   2. a block-scaled FP4 GEMM against offline NVFP4 weights, BF16 output,
 *      optional fused residual add;
 *   3. an FP8 E4M3 W8A8 variant (per-row weight scale, per-token activation
 *      scale).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Device pointers are CUDA global-memory pointers of the current device;
 *   all of them must be 16-byte aligned (TMA and 128-bit accesses).
 *   "stream" is a cudaStream_t (NULL = legacy default stream).
 * - bf16 tensors are row-major with unit stride along K.
 * - The caller allocates every buffer (outputs and workspace).  The library
 *   never allocates device memory and keeps no state between calls except a
 *   thread-local error string and a device status word.
 * - Every call validates its arguments on the host first.  On any error it
 *   returns a non-zero vlaq_status, sets vlaq_last_error(), launches nothing
 *   and touches no output.  Otherwise the work is queued on `stream` and the
 *   call returns VLAQ_OK without synchronizing.
 * - A kernel whose bounded internal wait runs out records VLAQ_ERR_TIMEOUT
 *   in the device status word and returns; vlaq_check() reports it.
 *
 * Data formats
 * ------------
 * NVFP4 ("Feat/internvla n1 dualvln", NVFP4 loader and nibble-order commits;
 * "Alpamayo 2 Super NVFP4" test reflection, ModelOpt configuration):
 *   value = E2M1(code) * E4M3(block scale) * g       (block = 16 along K)
 *   g = amax / (6 * 448): one fp32 per token row for activations, one per
 *   tensor for weights.  Block scale = E4M3_rne_sat(a_b / (6 g)); code =
 *   E2M1_rne_sat(x / (E4M3(scale) * g)); all fp32 with correctly rounded
 *   division.  g == 0 gives zero scales and codes.
 *
 *   Packed codes: row r, element k lives in byte r * pitch + k / 2, in the
 *   low nibble when k is even.  pitch = vlaq_nvfp4_code_pitch(K) =
 *   ceil(K / 64) * 32 bytes (= K / 2 whenever K % 64 == 0); bytes past K / 2
 *   in a row are written as zero.
 *
 *   Block scales, 128x4 tiled (the layout the tensor cores read, so no
 *   second copy is ever needed): rows are padded to Rp = ceil(rows/128)*128,
 *   scale columns to Cp = ceil(K/64)*4.  The scale of row r, block j
 *   (j = k / 16) is the byte at
 *       ((r / 128) * (Cp / 4) + j / 4) * 512
 *       + (r % 32) * 16 + ((r % 128) / 32) * 4 + (j % 4).
 *   Total size vlaq_nvfp4_scale_bytes(rows, K) = Rp * Cp.  Padded columns
 *   (j >= K/16) of real rows are written as zero; padded rows are never
 *   written and never affect a stored output.
 *
 * FP8 E4M3 (per-row scale):  value = E4M3(code) * s,  s = amax / 448.
 *   Codes row-major [rows, K], one byte per element.
 *
 * Optional activation transforms (flags), applied before the amax:
 *   VLAQ_F_RMSNORM    y = (x * r) * gamma, r = 1 / sqrt(mean(x^2) + eps),
 *                     fp32; the sum of squares uses 32 lanes, lane l owning
 *                     the 8-element chunks l, l+32, ... in element order,
 *                     combined by an XOR butterfly 16, 8, 4, 2, 1
 *                     ("FoldQuant W8A8/W4A4 inference", SYCL commit).
 *   VLAQ_F_HADAMARD64 block-diagonal normalised Sylvester Walsh-Hadamard
 *                     transform, block 64 (same page, dequant commit); needs
 *                     K % 64 == 0.
 */
#ifndef VLAQ_H_
#define VLAQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define VLAQ_API __attribute__((visibility("default")))
#else
#define VLAQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  VLAQ_OK = 0,
  VLAQ_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad flag      */
  VLAQ_ERR_SHAPE = 2,       /* K not divisible by 16 (64 with Hadamard),  */
                            /* or a size beyond a documented limit        */
  VLAQ_ERR_ALIGN = 3,       /* a pointer not 16-byte aligned               */
  VLAQ_ERR_ARCH = 4,        /* current device is not sm_100               */
  VLAQ_ERR_CUDA = 5,        /* a CUDA runtime / driver call failed         */
  VLAQ_ERR_TIMEOUT = 6,     /* a device-side bounded wait ran out          */
  VLAQ_ERR_WORKSPACE = 7    /* workspace missing or smaller than needed    */
} vlaq_status;

enum {
  VLAQ_F_RMSNORM = 1u << 0,
  VLAQ_F_HADAMARD64 = 1u << 1,
  VLAQ_F_SMOOTH_AFTER = 1u << 2, /* smoothing after the rotation (default: before) */
  VLAQ_F_SMOOTH_MUL = 1u << 3    /* multiply by the smoothing factors (default: divide) */
};

/* Human-readable text of the last error on the calling thread ("" if
 * none).  A K that is not a multiple of 16 reports the division, e.g.
 * "... 3420 / 16 = 213.75 ..." ("Feat/internvla n1 dualvln", scheme gate).
 * The pointer stays valid until the next vlaq call on this thread. */
VLAQ_API const char* vlaq_last_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
VLAQ_API int vlaq_version(void);

/* Synchronizes `stream`, then reads and clears the device status word of
 * the current device.  Returns VLAQ_ERR_TIMEOUT if a kernel gave up a
 * bounded wait since the last check, VLAQ_ERR_CUDA on a CUDA error. */
VLAQ_API vlaq_status vlaq_check(void* stream);

/* Failure-path self test: launches one kernel whose bounded wait on an
 * mbarrier that nothing arrives on runs out after about 1 ms; it records
 * the timeout in the device status word exactly as the GEMM and quantizer
 * kernels do, so the next vlaq_check(stream) returns VLAQ_ERR_TIMEOUT and
 * the one after it VLAQ_OK.  No copy, MMA or tensor memory is involved; the
 * context stays usable. */
VLAQ_API vlaq_status vlaq_selftest_wait_timeout(void* stream);

/* ----------------------------------------------------------- size helpers */
VLAQ_API int64_t vlaq_nvfp4_code_pitch(int64_t K);               /* bytes per row   */
VLAQ_API int64_t vlaq_nvfp4_scale_bytes(int64_t rows, int64_t K);/* tiled scales    */

/* ------------------------------------------------------------------ NVFP4 */

/* Offline weight quantization, one global scale for the whole tensor.
 *   W       bf16 [N, K] (device)
 *   flags   0 or VLAQ_F_HADAMARD64 (rotate each row before quantizing)
 *   codes   out, vlaq_nvfp4_code_pitch(K) * N bytes
 *   scales  out, vlaq_nvfp4_scale_bytes(N, K) bytes (128x4 tiled)
 *   g_w     out, one fp32
 * Limits: 1 <= N, 16 <= K <= 32768, K % 16 == 0.
 * ("Alpamayo 2 Super NVFP4": max calibration, FP4 weights, block 16, FP8
 * block scales; "Feat/internvla n1 dualvln": float32 global scale.) */
VLAQ_API vlaq_status vlaq_quantize_weight_nvfp4(const void* W, int64_t N, int64_t K,
                                       uint32_t flags, uint8_t* codes,
                                       uint8_t* scales, float* g_w,
                                       void* stream);

/* Dynamic per-token activation quantization (the fused prologue).
 *   X       bf16 [M, K] (device)
 *   gamma   bf16 [K] RMSNorm gain (device), required with VLAQ_F_RMSNORM,
 *           else ignored (may be NULL)
 *   eps     RMSNorm epsilon (e.g. 1e-6)
 *   flags   any of VLAQ_F_RMSNORM | VLAQ_F_HADAMARD64
 *   codes   out, vlaq_nvfp4_code_pitch(K) * M bytes
 *   scales  out, vlaq_nvfp4_scale_bytes(M, K) bytes (128x4 tiled)
 *   g_x     out, M fp32 (one global scale per token)
 * M == 0 is a no-op.  Limits: 16 <= K <= 32768, K % 16 == 0.
 * ("NVIDIA/TensorRT-Edge-LLM PR #193": NVFP4 quantizes activations
 * dynamically; "FoldQuant W8A8/W4A4 inference": RMSNorm + butterfly + quant
 * prologue with per-token amax, round-half-even and clamp.) */
VLAQ_API vlaq_status vlaq_quantize_act_nvfp4(const void* X, int64_t M, int64_t K,
                                    const void* gamma, float eps,
                                    uint32_t flags, uint8_t* codes,
                                    uint8_t* scales, float* g_x,
                                    void* stream);

/* vlaq_quantize_act_nvfp4 with per-input-channel smoothing: after the
 * optional RMSNorm, every channel k is divided by smooth[k] (FoldQuant's
 * activation scale: "FoldQuant W8A8/W4A4 inference", dequant commit,
 * x' = R(x / a), or R(x) / a with VLAQ_F_SMOOTH_AFTER, R the block
 * rotation), or multiplied by it with VLAQ_F_SMOOTH_MUL (AWQ's
 * pre_quant_scale, which activations are multiplied by: "NVIDIA/TensorRT-
 * Edge-LLM PR #193", pre_quant_scale commit).  One correctly rounded fp32
 * operation per element; the weights must carry the inverse factor.
 *   smooth  fp32 [K] (device, 16-byte aligned), finite and non-zero
 *   flags   any of VLAQ_F_RMSNORM | VLAQ_F_HADAMARD64 | VLAQ_F_SMOOTH_AFTER
 *           | VLAQ_F_SMOOTH_MUL
 * Other arguments, outputs and limits as vlaq_quantize_act_nvfp4. */
VLAQ_API vlaq_status vlaq_quantize_act_nvfp4_smooth(const void* X, int64_t M, int64_t K,
                                            const void* gamma, const float* smooth,
                                            float eps, uint32_t flags, uint8_t* codes,
                                            uint8_t* scales, float* g_x, void* stream);

/* vlaq_quantize_act_nvfp4 with a static (calibrated) global scale instead
 * of the per-token amax: the fp32 input_scale that ModelOpt / TensorRT
 * NVFP4 checkpoints store beside weight_scale and weight_scale_2
 * ("NVIDIA/TensorRT-Edge-LLM PR #193", pre_quant_scale commit).  Every row
 * uses g = g_static; block scales and codes follow the same definitions
 * (block scale E4M3(max|y| / (6 g)), code E2M1(y / (E4M3 scale x g))), so
 * values beyond the calibrated range saturate at scale 448 and code 6.
 * g_x[m] receives g_static for every row, so vlaq_linear_nvfp4 consumes the
 * result unchanged.  The row-amax pass and its reduction are skipped.
 *   g_static  finite and > 0 (host value), else VLAQ_ERR_INVALID_ARG
 *   smooth    fp32 [K] (device, 16-byte aligned) or NULL; required when a
 *             smoothing flag is set (as vlaq_quantize_act_nvfp4_smooth)
 *   flags     any of VLAQ_F_RMSNORM | VLAQ_F_HADAMARD64 | VLAQ_F_SMOOTH_AFTER
 *             | VLAQ_F_SMOOTH_MUL (the smoothing flags only with smooth)
 * Other arguments, outputs and limits as vlaq_quantize_act_nvfp4.  Finite
 * inputs only. */
VLAQ_API vlaq_status vlaq_quantize_act_nvfp4_static(const void* X, int64_t M, int64_t K,
                                            const void* gamma, const float* smooth,
                                            float eps, uint32_t flags, float g_static,
                                            uint8_t* codes, uint8_t* scales, float* g_x,
                                            void* stream);

/* Block scales from the 128x4 tiled layout the GEMM reads (as written by
 * the NVFP4 quantizers, vlaq_nvfp4_scale_bytes(rows, K) bytes) to the
 * logical row-major layout: out[r * (K/16) + b] = E4M3 scale of row r,
 * 16-block b, for r < rows, b < K/16 (padding rows and columns dropped).
 *   in   device, 16-byte aligned;  out  device, rows * K/16 bytes
 * K % 16 != 0 is refused with the division in the message.  The layout
 * change itself is this library's: the pages store scales row-major
 * ("NVFP4 block scale per 16 values", [Recipes] NVFP4 loader commit), the
 * tensor cores read the tiled layout. */
VLAQ_API vlaq_status vlaq_scales_to_rowmajor(const uint8_t* in, uint8_t* out, int64_t rows, int64_t K,
                                             void* stream);

/* Bytes of workspace vlaq_linear_nvfp4 / _fp8 / _int8 need for the given
 * shape on the current device (0 when the shape runs without split-K).  The
 * workspace's first 1024 bytes hold the per-tile arrival counters of
 * split-K calls, the per-split partial sums (fp32, s32 for INT8) follow.  The counters must be
 * zero when a call starts: zero the workspace once after allocating it;
 * every call (of any shape, NVFP4 or FP8) leaves them zero again, so nothing
 * is cleared between calls.  After vlaq_check reports VLAQ_ERR_TIMEOUT, zero
 * the workspace again before reusing it.  Calls that share a workspace
 * must not overlap on the GPU. */
VLAQ_API size_t vlaq_linear_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* Y = bf16_rne( (sum_k dec(x)[m,k] * dec(w)[n,k]) + residual[m,n] )
 * with the product accumulated in fp32 on the tensor cores
 * (tcgen05 kind::mxf4nvf4, block-16 E4M3 scales) and the global scales
 * g_x[m] * g_w applied in the epilogue.  One or two token rows against a
 * weight of at most 2^25 elements run on the CUDA cores instead (weight
 * streaming; each 16-block dot product an exact integer, the block scaling
 * and the sum over blocks in fp32); those shapes need no workspace.
 *   xq, xs, g_x  activation codes / tiled scales / globals (M rows)
 *   wq, ws, g_w  weight codes / tiled scales / global (N rows)
 *   residual     bf16 [M, N] or NULL
 *   Y            out, bf16 [M, N]
 *   workspace    device buffer of ws_bytes >= vlaq_linear_workspace_bytes
 * M == 0 is a no-op.  Limits: 1 <= N, 16 <= K, K % 16 == 0, N % 8 == 0.
 * Stream order: the kernel is launched with programmatic dependent launch
 * and starts streaming the weight operand (wq, ws) before it waits for the
 * kernel launched just before it on the same stream; everything else
 * (activations, globals, residual, workspace, Y) is touched only after that
 * wait.  So wq and ws must not be written by the kernel launched
 * immediately before this call on the stream.  Every kernel two or more
 * launches back has completed by then (each library kernel lets its
 * successor start only after its own wait), so weights produced by
 * vlaq_quantize_weight_nvfp4 right before this call are safe: its codes and
 * scales come from its second-to-last kernel, its last kernel writes g_w
 * only, and g_w is read after the wait.
 * (Residual add in the o / down epilogues: "FoldQuant W8A8/W4A4 inference",
 * merge commit.) */
VLAQ_API vlaq_status vlaq_linear_nvfp4(const uint8_t* xq, const uint8_t* xs,
                              const float* g_x, const uint8_t* wq,
                              const uint8_t* ws, const float* g_w,
                              const void* residual, void* Y, int64_t M,
                              int64_t N, int64_t K, void* workspace,
                              size_t ws_bytes, void* stream);

/* Same computation, arguments and rules as vlaq_linear_nvfp4, for callers
 * that cannot allocate device memory (a host callback, a real-time control
 * loop that must not touch the allocator, an embedding whose arena owns all
 * device memory): no workspace argument, and the call never allocates.
 * The split-K partial sums of small-M shapes go to a 4 MiB array compiled
 * into the library, which every GPU that loads the library holds until the
 * process exits.  A shape whose split-K plan needs more than 4 MiB is refused
 * with VLAQ_ERR_WORKSPACE (use vlaq_linear_nvfp4 then).  The first call
 * that needs the array in a CUDA context (one per device; a new one after
 * cudaDeviceReset) looks its address up (cudaGetSymbolAddress) with that
 * device current and caches it beside the context's ID; make that first
 * call before any stream capture.  All calls on a
 * device share the array (zero when the library loads; each call leaves its
 * tile counters zero again, and vlaq_check clears the array when it
 * reports VLAQ_ERR_TIMEOUT); calls that overlap on the GPU, e.g. on two
 * streams, race on it and must be serialized by the caller.  The source pages have no counterpart of
 * this entry point. */
VLAQ_API vlaq_status vlaq_linear_nvfp4_noalloc(const uint8_t* xq, const uint8_t* xs,
                                      const float* g_x, const uint8_t* wq,
                                      const uint8_t* ws, const float* g_w,
                                      const void* residual, void* Y, int64_t M,
                                      int64_t N, int64_t K, void* stream);

/* ------------------------------------------------------------ FP8 W8A8 */

/* Per-row weight quantization: s_w[n] = max|w_n| / 448, codes E4M3.
 *   W bf16 [N, K]; flags 0 or VLAQ_F_HADAMARD64; codes out [N, K];
 *   s_w out, N fp32.  Limits: 16 <= K <= 32768, K % 16 == 0. */
VLAQ_API vlaq_status vlaq_quantize_weight_fp8(const void* W, int64_t N, int64_t K,
                                     uint32_t flags, uint8_t* codes,
                                     float* s_w, void* stream);

/* Per-token activation quantization with the same optional RMSNorm /
 * Hadamard prologue as the NVFP4 variant.  codes out [M, K]; s_x out, M
 * fp32.  ("Feat/internvla n1 dualvln": FP8 E4M3 weight + scale tensors.) */
VLAQ_API vlaq_status vlaq_quantize_act_fp8(const void* X, int64_t M, int64_t K,
                                  const void* gamma, float eps,
                                  uint32_t flags, uint8_t* codes, float* s_x,
                                  void* stream);

/* Y = bf16_rne( s_x[m] * s_w[n] * sum_k e4m3(x)[m,k] e4m3(w)[n,k]
 *               + residual[m,n] ), fp32 accumulation on the tensor cores
 * (tcgen05 kind::f8f6f4).  Same argument rules as vlaq_linear_nvfp4. */
VLAQ_API vlaq_status vlaq_linear_fp8(const uint8_t* xq, const float* s_x,
                            const uint8_t* wq, const float* s_w,
                            const void* residual, void* Y, int64_t M,
                            int64_t N, int64_t K, void* workspace,
                            size_t ws_bytes, void* stream);

/* ----------------------------------------------------------- INT8 W8A8 */
/* FoldQuant's 8-bit integer path ("FoldQuant W8A8/W4A4 inference and
 * FoldQuantVLA quantized-model converter", vla.cpp PR #33: INT8 codes with
 * per-row weight scales, activations quantized per token; its OpenVINO
 * commit: per-token amax scale, round-half-even, clamp).  Symmetric:
 * s = max|y| / 127 (fp32, correctly rounded), code = clamp(RNE(y / s), -127,
 * 127) with y / s correctly rounded in fp32; an all-zero row gets s = 0 and
 * zero codes.  Codes are two's-complement int8, row-major [rows, K]. */

/* Per-row weight quantization.  W bf16 [N, K]; flags 0 or
 * VLAQ_F_HADAMARD64; codes out [N, K]; s_w out, N fp32.
 * Limits: 16 <= K <= 32768, K % 16 == 0. */
VLAQ_API vlaq_status vlaq_quantize_weight_int8(const void* W, int64_t N, int64_t K,
                                      uint32_t flags, int8_t* codes,
                                      float* s_w, void* stream);

/* Per-token activation quantization with the same optional RMSNorm /
 * Hadamard prologue as the NVFP4 variant.  codes out [M, K]; s_x out, M
 * fp32. */
VLAQ_API vlaq_status vlaq_quantize_act_int8(const void* X, int64_t M, int64_t K,
                                   const void* gamma, float eps,
                                   uint32_t flags, int8_t* codes, float* s_x,
                                   void* stream);

/* Y[m, n] = bf16_rne( fp32( fp32(acc) * fp32(s_x[m] * s_w[n]) ) + residual )
 * with acc = sum_k x[m, k] w[n, k] exact in s32 on the tensor cores
 * (tcgen05 kind::i8; |acc| <= K 127^2 < 2^31) and each fp32 step rounded
 * once, the residual add included: the output has a single correct value,
 * independent of tiling and split-K (the integer partials are summed
 * exactly).  Same argument rules as vlaq_linear_nvfp4. */
VLAQ_API vlaq_status vlaq_linear_int8(const int8_t* xq, const float* s_x,
                             const int8_t* wq, const float* s_w,
                             const void* residual, void* Y, int64_t M,
                             int64_t N, int64_t K, void* workspace,
                             size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* VLAQ_H_ */
