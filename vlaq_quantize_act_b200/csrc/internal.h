// Internal launcher interface between the C-ABI layer (api.cu) and the
// kernels (quant.cu, gemm.cu).  Arguments are validated by the caller.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include <utility>

namespace vlaq {

// Device status word bits (read and cleared by vlaq_check).
enum : unsigned int { kStatusTimeout = 1u };

// Largest K of the row quantizers: two staged bf16 rows (2 x 64 KiB) per CTA.
constexpr int64_t kMaxQuantK = 32768;

// Clock-cycle limit of every bounded wait in the library kernels (~1 s).
constexpr long long kWaitBudgetCycles = 2000000000LL;

constexpr uint32_t kFlagRmsNorm = 1u;
constexpr uint32_t kFlagHadamard = 2u;
constexpr uint32_t kFlagSmoothAfter = 4u;  // smoothing after the rotation (default: before)
constexpr uint32_t kFlagSmoothMul = 8u;    // multiply by the smoothing factors (default: divide)

inline int64_t nvfp4_code_pitch(int64_t K) { return (K + 63) / 64 * 32; }
inline int64_t nvfp4_scale_cols_padded(int64_t K) { return (K + 63) / 64 * 4; }
inline int64_t nvfp4_rows_padded(int64_t rows) { return (rows + 127) / 128 * 128; }

// ---- prologue / quantizer kernels (quant.cu)
cudaError_t launch_quant_act_nvfp4(const void* X, int64_t M, int64_t K, const void* gamma, float eps,
                                   uint32_t flags, uint8_t* codes, uint8_t* scales, float* g_x,
                                   cudaStream_t s);
cudaError_t launch_quant_act_nvfp4_smooth(const void* X, int64_t M, int64_t K, const void* gamma,
                                          const float* smooth, float eps, uint32_t flags, uint8_t* codes,
                                          uint8_t* scales, float* g_x, cudaStream_t s);
cudaError_t launch_quant_act_nvfp4_static(const void* X, int64_t M, int64_t K, const void* gamma, const float* smooth,
                                          float eps, uint32_t flags, float g_static, uint8_t* codes, uint8_t* scales,
                                          float* g_x, cudaStream_t s);
cudaError_t launch_quant_weight_nvfp4(const void* W, int64_t N, int64_t K, uint32_t flags,
                                      uint8_t* codes, uint8_t* scales, float* g_w, cudaStream_t s);
cudaError_t launch_quant_fp8(const void* X, int64_t rows, int64_t K, const void* gamma, float eps,
                             uint32_t flags, uint8_t* codes, float* s_out, cudaStream_t s);
cudaError_t launch_quant_int8(const void* X, int64_t rows, int64_t K, const void* gamma, float eps,
                              uint32_t flags, int8_t* codes, float* s_out, cudaStream_t s);
cudaError_t launch_scales_to_rowmajor(const uint8_t* in, uint8_t* out, int64_t rows, int64_t K, cudaStream_t s);

// ---- GEMM (gemm.cu)
struct GemmPlan {
  int bn;            // tile width along N (0: the few-row CUDA-core kernel)
  int splits;        // split-K factor (1 = direct epilogue)
  int grid;          // persistent CTAs
  size_t ws_bytes;   // fp32 partials needed when splits > 1
  bool pair = false; // NVFP4: 256 x 256 tiles over CTA pairs (paired MMA)
};
GemmPlan plan_gemm(bool fp4, int64_t M, int64_t N, int64_t K, int num_sms);
// Split-K workspace layout: the NVFP4 per-tile arrival counters occupy the
// first kSplitCounterBytes (zero between calls, the same place for every
// shape, so no shape's partial sums ever overwrite them), the fp32 partial
// sums follow.  Split plans have at most num_sms / 2 tiles.
constexpr size_t kSplitCounterBytes = 1024;
// fp32 partial sums of a split-K plan, rounded up to 256 bytes.
inline size_t splitk_partial_bytes(int64_t splits, int64_t M, int64_t N) {
  return (static_cast<size_t>(splits) * M * N * sizeof(float) + 255) / 256 * 256;
}

cudaError_t launch_linear_int8(const int8_t* xq, const float* s_x, const int8_t* wq, const float* s_w,
                               const void* residual, void* Y, int64_t M, int64_t N, int64_t K, void* workspace,
                               const GemmPlan& plan, long long budget, cudaStream_t s);
// Few-row NVFP4 linear on the CUDA cores (gemv.cu): M <= kGemvMaxM, at most
// kGemvMaxWeights weight elements, and the expanded activation rows fit two
// CTAs per SM.
constexpr int kGemvMaxM = 2;
constexpr int64_t kGemvMaxWeights = int64_t(1) << 25;
constexpr size_t kGemvSmemBudget = 200 * 1024;
size_t gemv_smem_bytes(int64_t M, int64_t K);
bool gemv_supported(int64_t M, int64_t N, int64_t K);
cudaError_t launch_gemv_nvfp4(const uint8_t* xq, const uint8_t* xs, const float* xg, const uint8_t* wq,
                              const uint8_t* ws, const float* wg, const void* residual, void* Y, int64_t M, int64_t N,
                              int64_t K, cudaStream_t s);
cudaError_t launch_linear(bool fp4, const uint8_t* xq, const uint8_t* xs, const float* xg,
                          const uint8_t* wq, const uint8_t* ws, const float* wg,
                          const void* residual, void* Y, int64_t M, int64_t N, int64_t K,
                          void* workspace, size_t ws_bytes, const GemmPlan& plan,
                          long long wait_budget, cudaStream_t s);

// Device status word accessors (gemm.cu, quant.cu).
cudaError_t read_and_clear_status(unsigned int* out, cudaStream_t s);
cudaError_t read_and_clear_quant_status(unsigned int* out, cudaStream_t s);
cudaError_t launch_selftest_wait_timeout(cudaStream_t s);

// Kernel launch with the programmatic-stream-serialization attribute, so the
// kernel may start while the previous kernel on the stream drains; every
// library kernel calls griddep_wait() before it touches global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Current device's SM count (cached per device).
int device_sm_count();

// ---- static scratch for the allocation-free linear entry point (noalloc.cu)
constexpr size_t kNoallocScratchBytes = size_t(4) << 20;  // 4 MiB per device
constexpr int kMaxDevices = 64;
cudaError_t noalloc_scratch(void** out);
cudaError_t noalloc_clear(cudaStream_t s);

}  // namespace vlaq
