// C-ABI entry points of libvlaq (declared and documented in include/vlaq.h).
// Host-side validation happens before any launch: a refused call launches
// nothing, touches no output and leaves a message in vlaq_last_error().
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <string>

#include "../../include/vlaq.h"
#include "internal.h"

namespace {

thread_local std::string t_err;

vlaq_status fail(vlaq_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  t_err = buf;
  return st;
}

vlaq_status ok() {
  t_err.clear();
  return VLAQ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// "3420 / 16 = 213.75": the quotient printed exactly (d is a power of two,
// so the decimal expansion terminates).
std::string k_div(int64_t K, int64_t d) {
  std::string s = std::to_string(K) + " / " + std::to_string(d) + " = " + std::to_string(K / d);
  int64_t r = K % d;
  if (r) {
    s += '.';
    while (r) {
      r *= 10;
      s += static_cast<char>('0' + r / d);
      r %= d;
    }
  }
  return s;
}

vlaq_status check_k(const char* fn, int64_t K, uint32_t flags, bool nvfp4, int64_t kmax) {
  if (K <= 0) return fail(VLAQ_ERR_SHAPE, "%s: K must be positive (got %lld)", fn, (long long)K);
  if (K % 16 != 0)
    return fail(VLAQ_ERR_SHAPE,
                "%s: K = %lld is not divisible by the %s block of 16 (%s); refused before any work",
                fn, (long long)K, nvfp4 ? "NVFP4" : "FP8 tile", k_div(K, 16).c_str());
  if ((flags & VLAQ_F_HADAMARD64) && K % 64 != 0)
    return fail(VLAQ_ERR_SHAPE, "%s: the block-64 Hadamard rotation needs K %% 64 == 0 (%s)", fn,
                k_div(K, 64).c_str());
  if (kmax > 0 && K > kmax)
    return fail(VLAQ_ERR_SHAPE, "%s: K = %lld exceeds the supported maximum %lld", fn, (long long)K,
                (long long)kmax);
  return VLAQ_OK;
}

vlaq_status check_device(const char* fn) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(VLAQ_ERR_CUDA, "%s: no CUDA device (%s)", fn, cudaGetErrorString(e));
  static int cc_cache[64] = {0};
  int cc = dev < 64 ? cc_cache[dev] : 0;
  if (!cc) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cc = major * 10 + minor;
    if (dev < 64) cc_cache[dev] = cc;
  }
  if (cc != 100)
    return fail(VLAQ_ERR_ARCH, "%s: device %d has compute capability %d.%d; libvlaq is built for sm_100a only", fn,
                dev, cc / 10, cc % 10);
  return VLAQ_OK;
}

vlaq_status cuda_fail(const char* fn, cudaError_t e) {
  return fail(VLAQ_ERR_CUDA, "%s: CUDA error %s (%s)", fn, cudaGetErrorName(e), cudaGetErrorString(e));
}

#define VLAQ_NONNULL(fn, p)                                                        \
  do {                                                                             \
    if ((p) == nullptr) return fail(VLAQ_ERR_INVALID_ARG, "%s: %s is NULL", fn, #p); \
    if (!aligned16(p)) return fail(VLAQ_ERR_ALIGN, "%s: %s is not 16-byte aligned", fn, #p); \
  } while (0)

vlaq_status check_flags(const char* fn, uint32_t flags, uint32_t allowed) {
  if (flags & ~allowed) return fail(VLAQ_ERR_INVALID_ARG, "%s: unsupported flags 0x%x", fn, flags);
  return VLAQ_OK;
}


}  // namespace

extern "C" {

const char* vlaq_last_error(void) { return t_err.c_str(); }

int vlaq_version(void) { return 100; }

int64_t vlaq_nvfp4_code_pitch(int64_t K) { return K <= 0 ? 0 : vlaq::nvfp4_code_pitch(K); }

int64_t vlaq_nvfp4_scale_bytes(int64_t rows, int64_t K) {
  if (rows <= 0 || K <= 0) return 0;
  return vlaq::nvfp4_rows_padded(rows) * vlaq::nvfp4_scale_cols_padded(K);
}

vlaq_status vlaq_check(void* stream) {
  unsigned int st = 0;
  cudaError_t e = vlaq::read_and_clear_status(&st, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail("vlaq_check", e);
  unsigned int qst = 0;
  e = vlaq::read_and_clear_quant_status(&qst, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail("vlaq_check", e);
  st |= qst;
  if (st & vlaq::kStatusTimeout) {
    // a GEMM that gave up may have left split-K tile counters non-zero
    e = vlaq::noalloc_clear(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail("vlaq_check", e);
    return fail(VLAQ_ERR_TIMEOUT,
                "vlaq_check: a kernel gave up a bounded wait (device status 0x%x); zero any split-K workspace "
                "before reusing it", st);
  }
  return ok();
}

vlaq_status vlaq_selftest_wait_timeout(void* stream) {
  const char* fn = "vlaq_selftest_wait_timeout";
  vlaq_status st;
  if ((st = check_device(fn))) return st;
  cudaError_t e = vlaq::launch_selftest_wait_timeout(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(fn, e);
  return ok();
}

vlaq_status vlaq_quantize_act_nvfp4(const void* X, int64_t M, int64_t K, const void* gamma, float eps,
                                    uint32_t flags, uint8_t* codes, uint8_t* scales, float* g_x, void* stream) {
  const char* fn = "vlaq_quantize_act_nvfp4";
  vlaq_status st;
  if ((st = check_flags(fn, flags, VLAQ_F_RMSNORM | VLAQ_F_HADAMARD64))) return st;
  if ((st = check_k(fn, K, flags, true, vlaq::kMaxQuantK))) return st;
  if (M < 0) return fail(VLAQ_ERR_INVALID_ARG, "%s: M = %lld is negative", fn, (long long)M);
  if (M > 0x7FFFFFFF) return fail(VLAQ_ERR_SHAPE, "%s: M = %lld is too large", fn, (long long)M);
  if (M == 0) return ok();
  VLAQ_NONNULL(fn, X);
  VLAQ_NONNULL(fn, codes);
  VLAQ_NONNULL(fn, scales);
  VLAQ_NONNULL(fn, g_x);
  if (flags & VLAQ_F_RMSNORM) VLAQ_NONNULL(fn, gamma);
  if ((st = check_device(fn))) return st;
  cudaError_t e = vlaq::launch_quant_act_nvfp4(X, M, K, gamma, eps, flags, codes, scales, g_x,
                                               static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(fn, e);
  return ok();
}

vlaq_status vlaq_quantize_act_nvfp4_smooth(const void* X, int64_t M, int64_t K, const void* gamma,
                                           const float* smooth, float eps, uint32_t flags, uint8_t* codes,
                                           uint8_t* scales, float* g_x, void* stream) {
  const char* fn = "vlaq_quantize_act_nvfp4_smooth";
  vlaq_status st;
  if ((st = check_flags(fn, flags, VLAQ_F_RMSNORM | VLAQ_F_HADAMARD64 | VLAQ_F_SMOOTH_AFTER | VLAQ_F_SMOOTH_MUL)))
    return st;
  if ((st = check_k(fn, K, flags, true, vlaq::kMaxQuantK))) return st;
  if (M < 0) return fail(VLAQ_ERR_INVALID_ARG, "%s: M = %lld is negative", fn, (long long)M);
  if (M > 0x7FFFFFFF) return fail(VLAQ_ERR_SHAPE, "%s: M = %lld is too large", fn, (long long)M);
  if (M == 0) return ok();
  VLAQ_NONNULL(fn, X);
  VLAQ_NONNULL(fn, smooth);
  VLAQ_NONNULL(fn, codes);
  VLAQ_NONNULL(fn, scales);
  VLAQ_NONNULL(fn, g_x);
  if (flags & VLAQ_F_RMSNORM) VLAQ_NONNULL(fn, gamma);
  if ((st = check_device(fn))) return st;
  cudaError_t e = vlaq::launch_quant_act_nvfp4_smooth(X, M, K, gamma, smooth, eps, flags, codes, scales, g_x,
                                                      static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(fn, e);
  return ok();
}

vlaq_status vlaq_quantize_act_nvfp4_static(const void* X, int64_t M, int64_t K, const void* gamma,
                                           const float* smooth, float eps, uint32_t flags, float g_static,
                                           uint8_t* codes, uint8_t* scales, float* g_x, void* stream) {
  const char* fn = "vlaq_quantize_act_nvfp4_static";
  vlaq_status st;
  if ((st = check_flags(fn, flags, VLAQ_F_RMSNORM | VLAQ_F_HADAMARD64 | VLAQ_F_SMOOTH_AFTER | VLAQ_F_SMOOTH_MUL)))
    return st;
  if ((st = check_k(fn, K, flags, true, vlaq::kMaxQuantK))) return st;
  if (!(g_static > 0.0f) || !std::isfinite(g_static))
    return fail(VLAQ_ERR_INVALID_ARG, "%s: g_static = %g must be finite and positive", fn, (double)g_static);
  if ((flags & (VLAQ_F_SMOOTH_AFTER | VLAQ_F_SMOOTH_MUL)) && smooth == nullptr)
    return fail(VLAQ_ERR_INVALID_ARG, "%s: smoothing flags without smoothing factors", fn);
  if (M < 0) return fail(VLAQ_ERR_INVALID_ARG, "%s: M = %lld is negative", fn, (long long)M);
  if (M > 0x7FFFFFFF) return fail(VLAQ_ERR_SHAPE, "%s: M = %lld is too large", fn, (long long)M);
  if (M == 0) return ok();
  VLAQ_NONNULL(fn, X);
  VLAQ_NONNULL(fn, codes);
  VLAQ_NONNULL(fn, scales);
  VLAQ_NONNULL(fn, g_x);
  if (flags & VLAQ_F_RMSNORM) VLAQ_NONNULL(fn, gamma);
  if ((st = check_device(fn))) return st;
  cudaError_t e = vlaq::launch_quant_act_nvfp4_static(X, M, K, gamma, smooth, eps, flags, g_static, codes, scales,
                                                      g_x, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(fn, e);
  return ok();
}

vlaq_status vlaq_quantize_weight_nvfp4(const void* W, int64_t N, int64_t K, uint32_t flags, uint8_t* codes,
                                       uint8_t* scales, float* g_w, void* stream) {
  const char* fn = "vlaq_quantize_weight_nvfp4";
  vlaq_status st;
  if ((st = check_flags(fn, flags, VLAQ_F_HADAMARD64))) return st;
  if ((st = check_k(fn, K, flags, true, vlaq::kMaxQuantK))) return st;
  if (N <= 0 || N > 0x7FFFFFFF) return fail(VLAQ_ERR_SHAPE, "%s: N = %lld out of range", fn, (long long)N);
  VLAQ_NONNULL(fn, W);
  VLAQ_NONNULL(fn, codes);
  VLAQ_NONNULL(fn, scales);
  VLAQ_NONNULL(fn, g_w);
  if ((st = check_device(fn))) return st;
  cudaError_t e = vlaq::launch_quant_weight_nvfp4(W, N, K, flags, codes, scales, g_w,
                                                  static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(fn, e);
  return ok();
}

vlaq_status vlaq_scales_to_rowmajor(const uint8_t* in, uint8_t* out, int64_t rows, int64_t K, void* stream) {
  const char* fn = "vlaq_scales_to_rowmajor";
  vlaq_status st;
  if ((st = check_k(fn, K, 0, true, 0))) return st;
  if (rows < 0) return fail(VLAQ_ERR_INVALID_ARG, "%s: rows = %lld is negative", fn, (long long)rows);
  if (rows > 0x7FFFFFFF) return fail(VLAQ_ERR_SHAPE, "%s: rows = %lld is too large", fn, (long long)rows);
  if (rows == 0) return ok();
  VLAQ_NONNULL(fn, in);
  if (!out) return fail(VLAQ_ERR_INVALID_ARG, "%s: out is NULL", fn);
  if ((st = check_device(fn))) return st;
  cudaError_t e = vlaq::launch_scales_to_rowmajor(in, out, rows, K, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(fn, e);
  return ok();
}

vlaq_status vlaq_quantize_weight_fp8(const void* W, int64_t N, int64_t K, uint32_t flags, uint8_t* codes,
                                     float* s_w, void* stream) {
  const char* fn = "vlaq_quantize_weight_fp8";
  vlaq_status st;
  if ((st = check_flags(fn, flags, VLAQ_F_HADAMARD64))) return st;
  if ((st = check_k(fn, K, flags, false, vlaq::kMaxQuantK))) return st;
  if (N <= 0 || N > 0x7FFFFFFF) return fail(VLAQ_ERR_SHAPE, "%s: N = %lld out of range", fn, (long long)N);
  VLAQ_NONNULL(fn, W);
  VLAQ_NONNULL(fn, codes);
  VLAQ_NONNULL(fn, s_w);
  if ((st = check_device(fn))) return st;
  cudaError_t e = vlaq::launch_quant_fp8(W, N, K, nullptr, 0.0f, flags, codes, s_w, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(fn, e);
  return ok();
}

vlaq_status vlaq_quantize_act_fp8(const void* X, int64_t M, int64_t K, const void* gamma, float eps, uint32_t flags,
                                  uint8_t* codes, float* s_x, void* stream) {
  const char* fn = "vlaq_quantize_act_fp8";
  vlaq_status st;
  if ((st = check_flags(fn, flags, VLAQ_F_RMSNORM | VLAQ_F_HADAMARD64))) return st;
  if ((st = check_k(fn, K, flags, false, vlaq::kMaxQuantK))) return st;
  if (M < 0) return fail(VLAQ_ERR_INVALID_ARG, "%s: M = %lld is negative", fn, (long long)M);
  if (M > 0x7FFFFFFF) return fail(VLAQ_ERR_SHAPE, "%s: M = %lld is too large", fn, (long long)M);
  if (M == 0) return ok();
  VLAQ_NONNULL(fn, X);
  VLAQ_NONNULL(fn, codes);
  VLAQ_NONNULL(fn, s_x);
  if (flags & VLAQ_F_RMSNORM) VLAQ_NONNULL(fn, gamma);
  if ((st = check_device(fn))) return st;
  cudaError_t e = vlaq::launch_quant_fp8(X, M, K, gamma, eps, flags, codes, s_x, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(fn, e);
  return ok();
}

vlaq_status vlaq_quantize_weight_int8(const void* W, int64_t N, int64_t K, uint32_t flags, int8_t* codes,
                                      float* s_w, void* stream) {
  const char* fn = "vlaq_quantize_weight_int8";
  vlaq_status st;
  if ((st = check_flags(fn, flags, VLAQ_F_HADAMARD64))) return st;
  if ((st = check_k(fn, K, flags, false, vlaq::kMaxQuantK))) return st;
  if (N <= 0 || N > 0x7FFFFFFF) return fail(VLAQ_ERR_SHAPE, "%s: N = %lld out of range", fn, (long long)N);
  VLAQ_NONNULL(fn, W);
  VLAQ_NONNULL(fn, codes);
  VLAQ_NONNULL(fn, s_w);
  if ((st = check_device(fn))) return st;
  cudaError_t e = vlaq::launch_quant_int8(W, N, K, nullptr, 0.0f, flags, codes, s_w, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(fn, e);
  return ok();
}

vlaq_status vlaq_quantize_act_int8(const void* X, int64_t M, int64_t K, const void* gamma, float eps, uint32_t flags,
                                   int8_t* codes, float* s_x, void* stream) {
  const char* fn = "vlaq_quantize_act_int8";
  vlaq_status st;
  if ((st = check_flags(fn, flags, VLAQ_F_RMSNORM | VLAQ_F_HADAMARD64))) return st;
  if ((st = check_k(fn, K, flags, false, vlaq::kMaxQuantK))) return st;
  if (M < 0) return fail(VLAQ_ERR_INVALID_ARG, "%s: M = %lld is negative", fn, (long long)M);
  if (M > 0x7FFFFFFF) return fail(VLAQ_ERR_SHAPE, "%s: M = %lld is too large", fn, (long long)M);
  if (M == 0) return ok();
  VLAQ_NONNULL(fn, X);
  VLAQ_NONNULL(fn, codes);
  VLAQ_NONNULL(fn, s_x);
  if (flags & VLAQ_F_RMSNORM) VLAQ_NONNULL(fn, gamma);
  if ((st = check_device(fn))) return st;
  cudaError_t e = vlaq::launch_quant_int8(X, M, K, gamma, eps, flags, codes, s_x, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(fn, e);
  return ok();
}

size_t vlaq_linear_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  // the NVFP4 and 8-bit (FP8 / INT8) plans split differently; the larger
  const int sms = vlaq::device_sm_count();
  const size_t a = vlaq::plan_gemm(true, M, N, K, sms).ws_bytes;
  const size_t b = vlaq::plan_gemm(false, M, N, K, sms).ws_bytes;
  return a > b ? a : b;
}

enum LinearKind { kLinearNvfp4, kLinearFp8, kLinearInt8 };

// static_scratch: the split-K scratch is the library's static array
// (vlaq_linear_nvfp4_noalloc) instead of the caller's workspace.
static vlaq_status linear_common(const char* fn, LinearKind kind, const uint8_t* xq, const uint8_t* xs, const float* xg,
                                 const uint8_t* wq, const uint8_t* ws, const float* wg, const void* residual, void* Y,
                                 int64_t M, int64_t N, int64_t K, void* workspace, size_t ws_bytes, void* stream,
                                 bool static_scratch = false) {
  vlaq_status st;
  const bool fp4 = kind == kLinearNvfp4;
  if ((st = check_k(fn, K, 0, fp4, 0))) return st;
  if (M < 0) return fail(VLAQ_ERR_INVALID_ARG, "%s: M = %lld is negative", fn, (long long)M);
  if (N <= 0 || N % 8 != 0)
    return fail(VLAQ_ERR_SHAPE, "%s: N = %lld must be a positive multiple of 8", fn, (long long)N);
  if (M > 0x7FFFFFFF || N > 0x7FFFFFFF || K > 0x7FFFFFFF || M * N > (int64_t(1) << 40))
    return fail(VLAQ_ERR_SHAPE, "%s: shape %lld x %lld x %lld too large", fn, (long long)M, (long long)N,
                (long long)K);
  if (M == 0) return ok();
  VLAQ_NONNULL(fn, xq);
  VLAQ_NONNULL(fn, xg);
  VLAQ_NONNULL(fn, wq);
  VLAQ_NONNULL(fn, wg);
  VLAQ_NONNULL(fn, Y);
  if (fp4) {
    VLAQ_NONNULL(fn, xs);
    VLAQ_NONNULL(fn, ws);
  }
  if (residual && !aligned16(residual)) return fail(VLAQ_ERR_ALIGN, "%s: residual is not 16-byte aligned", fn);
  if ((st = check_device(fn))) return st;
  const vlaq::GemmPlan plan = vlaq::plan_gemm(fp4, M, N, K, vlaq::device_sm_count());
  if (static_scratch && plan.ws_bytes > 0) {
    if (plan.ws_bytes > vlaq::kNoallocScratchBytes)
      return fail(VLAQ_ERR_WORKSPACE,
                  "%s: shape %lld x %lld x %lld needs %zu bytes of split-K scratch, more than the %zu-byte static "
                  "scratch array; use vlaq_linear_nvfp4 with a caller-allocated workspace",
                  fn, (long long)M, (long long)N, (long long)K, plan.ws_bytes, vlaq::kNoallocScratchBytes);
    cudaError_t e = vlaq::noalloc_scratch(&workspace);
    if (e != cudaSuccess) return cuda_fail(fn, e);
    ws_bytes = vlaq::kNoallocScratchBytes;
  }
  if (plan.ws_bytes > 0) {
    if (!workspace || ws_bytes < plan.ws_bytes)
      return fail(VLAQ_ERR_WORKSPACE, "%s: this shape needs %zu bytes of workspace (got %zu%s)", fn, plan.ws_bytes,
                  ws_bytes, workspace ? "" : ", NULL pointer");
    if (!aligned16(workspace)) return fail(VLAQ_ERR_ALIGN, "%s: workspace is not 16-byte aligned", fn);
  }
  cudaError_t e =
      kind == kLinearInt8
          ? vlaq::launch_linear_int8(reinterpret_cast<const int8_t*>(xq), xg, reinterpret_cast<const int8_t*>(wq), wg,
                                     residual, Y, M, N, K, workspace, plan, vlaq::kWaitBudgetCycles,
                                     static_cast<cudaStream_t>(stream))
          : vlaq::launch_linear(fp4, xq, xs, xg, wq, ws, wg, residual, Y, M, N, K, workspace, ws_bytes, plan,
                                vlaq::kWaitBudgetCycles, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(fn, e);
  return ok();
}

vlaq_status vlaq_linear_nvfp4(const uint8_t* xq, const uint8_t* xs, const float* g_x, const uint8_t* wq,
                              const uint8_t* ws, const float* g_w, const void* residual, void* Y, int64_t M, int64_t N,
                              int64_t K, void* workspace, size_t ws_bytes, void* stream) {
  return linear_common("vlaq_linear_nvfp4", kLinearNvfp4, xq, xs, g_x, wq, ws, g_w, residual, Y, M, N, K, workspace,
                       ws_bytes, stream);
}

vlaq_status vlaq_linear_fp8(const uint8_t* xq, const float* s_x, const uint8_t* wq, const float* s_w,
                            const void* residual, void* Y, int64_t M, int64_t N, int64_t K, void* workspace,
                            size_t ws_bytes, void* stream) {
  return linear_common("vlaq_linear_fp8", kLinearFp8, xq, nullptr, s_x, wq, nullptr, s_w, residual, Y, M, N, K,
                       workspace, ws_bytes, stream);
}

vlaq_status vlaq_linear_int8(const int8_t* xq, const float* s_x, const int8_t* wq, const float* s_w,
                             const void* residual, void* Y, int64_t M, int64_t N, int64_t K, void* workspace,
                             size_t ws_bytes, void* stream) {
  return linear_common("vlaq_linear_int8", kLinearInt8, reinterpret_cast<const uint8_t*>(xq), nullptr, s_x,
                       reinterpret_cast<const uint8_t*>(wq), nullptr, s_w, residual, Y, M, N, K, workspace, ws_bytes,
                       stream);
}

vlaq_status vlaq_linear_nvfp4_noalloc(const uint8_t* xq, const uint8_t* xs, const float* g_x, const uint8_t* wq,
                                      const uint8_t* ws, const float* g_w, const void* residual, void* Y, int64_t M,
                                      int64_t N, int64_t K, void* stream) {
  // same validation and order as vlaq_linear_nvfp4; a split-K plan takes the
  // library's static scratch array (refused if it needs more)
  return linear_common("vlaq_linear_nvfp4_noalloc", kLinearNvfp4, xq, xs, g_x, wq, ws, g_w, residual, Y, M, N, K,
                       nullptr, 0, stream, true);
}

}  // extern "C"
