// Fused activation prologue and the offline weight quantizers.
//
// One CTA per row; thread b owns the 64-element block b of the row (the
// Hadamard block, four NVFP4 scale blocks, 32 packed code bytes and one
// 4-byte word of the 128x4 tiled scale layout).  The row is read once from
// HBM with 16-byte loads, optionally transformed in registers (RMSNorm,
// block-64 WHT), reduced to a per-row amax with warp shuffles, then
// quantized and written with 16-byte stores.  HBM-bound: 2 bytes in and
// 0.5625 (NVFP4) or 1 (FP8) bytes out per element.
//
// Arithmetic follows the format definitions stated in include/vlaq.h: every
// fp32 operation is an explicitly rounded intrinsic (no contraction),
// division and square root are correctly rounded, so codes and scales are
// bit-identical to any implementation that performs the same operations
// ("FoldQuant W8A8/W4A4 inference", SYCL commit: correctly rounded divide
// and sqrt, fixed reduction tree).
//
// Fast exact quotient: the code of x / S only depends on which side of the
// format's rounding decision points the correctly rounded quotient falls.
// Every decision point of E2M1 (the grid midpoints 0.25 ... 5) has its low
// 21 fp32 mantissa bits zero, and every decision point of E4M3 its low 19.
// q' = x * RN(1/S) is within 3 units in the last place of x / S, so when q'
// is more than 8 units away from any number with those low bits zero, q'
// and RN(x / S) give the same code; otherwise (a few per million elements,
// and values that sit exactly on grid-like numbers) the 16 values of the
// block are divided exactly.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace vlaq {
namespace {

enum { kNvfp4 = 0, kFp8 = 1 };
enum { kPerRow = 0, kTensorAmax = 1, kTensorQuant = 2 };

// XOR swizzle of 16-byte chunks in the staged row: both the per-thread
// writes (8 consecutive chunks) and the lane-strided tree reads hit 8
// distinct 16-byte bank groups.
__device__ __forceinline__ int swz_chunk(int c) { return c ^ ((c >> 3) & 7); }

__device__ __forceinline__ void unpack_bf16x8(const uint4& q, float* v) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    v[2 * j] = __uint_as_float(w[j] << 16);
    v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
  }
}

// max |x| of 16 bf16 values held in two 16-byte words (exact).
__device__ __forceinline__ float absmax_bf16x16(const uint4& a, const uint4& b) {
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  const uint32_t zero = 0u;
  __nv_bfloat162 m = *reinterpret_cast<const __nv_bfloat162*>(&zero);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t aw = w[j] & 0x7FFF7FFFu;  // |x| of both halves
    m = __hmax2(m, *reinterpret_cast<const __nv_bfloat162*>(&aw));
  }
  return fmaxf(__low2float(m), __high2float(m));
}

// Normalised Walsh-Hadamard transform of one 64-block, Sylvester order:
// butterfly stages h = 1, 2, ..., 32, then x 1/8 (exact).
__device__ __forceinline__ void wht64(float* v) {
#pragma unroll
  for (int h = 1; h < 64; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      if ((i & h) == 0) {
        const float a = v[i], b = v[i + h];
        v[i] = __fadd_rn(a, b);
        v[i + h] = __fsub_rn(a, b);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 64; ++i) v[i] = __fmul_rn(v[i], 0.125f);
}

// Max over the CTA; every thread gets the result.
__device__ __forceinline__ float block_max(float v, float* s_red) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) s_red[w] = v;
  __syncthreads();
  const int nw = blockDim.x >> 5;
  float r = (l < nw) ? s_red[l] : 0.0f;
#pragma unroll
  for (int o = 16; o; o >>= 1) r = fmaxf(r, __shfl_xor_sync(0xffffffffu, r, o));
  return r;
}

// Fast path of the quotient (see the file comment): approximate reciprocal
// (at most 2 units in the last place off, documented bound of
// rcp.approx.f32), one product per element, and a test that the product is
// at least 8 units in the last place away from every number whose low
// LOWBITS mantissa bits are zero.  t = (bits + 8) & (low mask without the
// last 4 bits) is zero exactly for products within [-8, +7] units of such a
// number (+-0 included, which merely takes the exact path).
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

template <int LOWBITS>
__device__ __forceinline__ uint32_t near_key(float q) {
  return (__float_as_uint(q) + 8u) & (((1u << LOWBITS) - 1u) & ~0xFu);
}

// The reciprocal shortcut needs 1/S to be a normal fp32 number.
__device__ __forceinline__ bool rcp_ok(float s) { return s >= 0x1p-125f && s <= 0x1p125f; }

// RN(v[i] / S) for 16 values, S > 0, as far as E2M1 (LOWBITS = 21) or E4M3
// (LOWBITS = 19) encoding can tell.  r = approximate 1/S, fast = rcp_ok(S).
template <int LOWBITS>
__device__ __forceinline__ void quotients16(const float* v, float S, float r, bool fast, float* q) {
  uint32_t key = fast ? 0xFFFFFFFFu : 0u;
  if (fast) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      q[i] = __fmul_rn(v[i], r);
      key = min(key, near_key<LOWBITS>(q[i]));
    }
  }
  if (key == 0u) {
#pragma unroll
    for (int i = 0; i < 16; ++i) q[i] = __fdiv_rn(v[i], S);
  }
}

// E4M3 byte of RN(a / d) (a >= 0, d > 0) with r_d = approximate 1/d.
__device__ __forceinline__ uint32_t e4m3_of_quotient(float a, float d, float r_d, bool fast) {
  float q = fast ? __fmul_rn(a, r_d) : 0.0f;
  if (!fast || near_key<19>(q) == 0u) q = __fdiv_rn(a, d);
  return cvt_e4m3x2(q, 0.0f) & 0xFFu;
}

// Scale byte and 16 codes (two words) of one NVFP4 block.
__device__ __forceinline__ uint32_t nvfp4_block(const float* v, float a16, float g, float six_g, float r6g,
                                                bool fast6g, uint32_t& w0, uint32_t& w1) {
  float q[16];
  uint32_t sb8 = 0;
  float S = 0.0f;
  if (g > 0.0f) {
    sb8 = e4m3_of_quotient(a16, six_g, r6g, fast6g);
    S = __fmul_rn(e4m3_to_f32(sb8), g);
  }
  if (S != 0.0f) {
    const bool fast = rcp_ok(S);
    quotients16<21>(v, S, fast ? rcp_approx(S) : 0.0f, fast, q);
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) q[i] = 0.0f;
  }
  w0 = cvt_e2m1x8(q);
  w1 = cvt_e2m1x8(q + 8);
  return sb8;
}

// 16 FP8 codes (four words) with the row scale s.
__device__ __forceinline__ void fp8_block(const float* v, float s, float r, bool fast, uint32_t* w) {
  float q[16];
  if (s != 0.0f) {
    quotients16<19>(v, s, r, fast, q);
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) q[i] = 0.0f;
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) w[j] = cvt_e4m3x2(q[4 * j], q[4 * j + 1]) | (cvt_e4m3x2(q[4 * j + 2], q[4 * j + 3]) << 16);
}

__device__ __forceinline__ void store_scale_word(uint8_t* scales, int64_t row, int b, int nblk, uint32_t word) {
  // 128x4 tiled scale layout: 512-byte atom per (128 rows, 4 blocks)
  const int64_t atom = (row >> 7) * nblk + b;
  const int64_t off = atom * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4;
  *reinterpret_cast<uint32_t*>(scales + off) = word;
}

struct RowArgs {
  const __nv_bfloat16* X;
  int K;
  const __nv_bfloat16* gamma;
  float eps;
  uint32_t flags;
  uint8_t* codes;
  int64_t pitch;
  uint8_t* scales;
  float* gout;
  unsigned int* amax_word;
};

// Global scale of the row (per-row modes) or of the tensor (quant pass).
template <int FMT, int MODE>
__device__ __forceinline__ float row_global(const RowArgs& a, float local, float* s_red, int64_t row) {
  if (MODE == kPerRow) {
    const float A = block_max(local, s_red);
    const float g = (FMT == kNvfp4) ? __fdiv_rn(A, 2688.0f) : __fdiv_rn(A, 448.0f);
    if (threadIdx.x == 0) a.gout[row] = g;
    return g;
  }
  return __fdiv_rn(__uint_as_float(*a.amax_word), 2688.0f);
}

// ---- rows without RMSNorm / Hadamard.  Thread t owns the elements
// [EPT t, EPT t + EPT) of the row (EPT = 16: one NVFP4 block, EPT = 64: one
// 64-block); the raw bf16 stays packed in registers.  Small EPT gives short
// rows many more warps in flight.  Threads past K / EPT (up to the next
// multiple of 64 elements) write the zero padding of codes and scales.
template <int FMT, int MODE, int EPT>
__global__ void __launch_bounds__(512, 1) quant_rows_plain_kernel(const RowArgs a) {
  constexpr int NB = EPT / 16;  // NVFP4 blocks per thread
  __shared__ float s_red[32];
  griddep_launch_dependents();
  griddep_wait();
  const int64_t row = blockIdx.x;
  const int t = threadIdx.x;
  const int K = a.K;
  const int nblk64 = (K + 63) >> 6;
  const int nel = max(0, min(EPT, K - EPT * t));         // real elements of this thread
  const bool writes = EPT * t < 64 * nblk64;             // inside the padded row

  const uint4* xr = reinterpret_cast<const uint4*>(a.X + row * static_cast<int64_t>(K));
  uint4 raw[2 * NB];
#pragma unroll
  for (int i = 0; i < 2 * NB; ++i)
    raw[i] = (8 * i < nel) ? __ldg(xr + (EPT / 8) * t + i) : make_uint4(0, 0, 0, 0);
  float a16[NB];
  float local = 0.0f;
#pragma unroll
  for (int q = 0; q < NB; ++q) {
    a16[q] = absmax_bf16x16(raw[2 * q], raw[2 * q + 1]);
    local = fmaxf(local, a16[q]);
  }

  if (MODE == kTensorAmax) {
    const float A = block_max(local, s_red);
    if (threadIdx.x == 0) atomicMax(a.amax_word, __float_as_uint(A));  // A >= 0: bit order = value order
    return;
  }
  const float g = row_global<FMT, MODE>(a, local, s_red, row);

  if (FMT == kNvfp4) {
    const float six_g = __fmul_rn(6.0f, g);
    const bool fast6g = rcp_ok(six_g);
    const float r6g = fast6g ? rcp_approx(six_g) : 0.0f;
    uint32_t sc_word = 0;
    uint32_t cw[2 * NB];
#pragma unroll
    for (int q = 0; q < NB; ++q) {
      cw[2 * q] = cw[2 * q + 1] = 0u;
      if (16 * q < nel) {
        float v[16];
        unpack_bf16x8(raw[2 * q], v);
        unpack_bf16x8(raw[2 * q + 1], v + 8);
        const uint32_t sb8 = nvfp4_block(v, a16[q], g, six_g, r6g, fast6g, cw[2 * q], cw[2 * q + 1]);
        sc_word |= sb8 << (8 * ((EPT == 16 ? t : q) & 3));
      }
    }
    if (EPT == 16) {
      // four neighbouring threads own the four bytes of one scale word
      sc_word |= __shfl_xor_sync(0xffffffffu, sc_word, 1);
      sc_word |= __shfl_xor_sync(0xffffffffu, sc_word, 2);
      if (writes) {
        *reinterpret_cast<uint2*>(a.codes + row * a.pitch + 8 * t) = make_uint2(cw[0], cw[1]);
        if ((t & 3) == 0) store_scale_word(a.scales, row, t >> 2, nblk64, sc_word);
      }
    } else if (writes) {
      uint4* crow = reinterpret_cast<uint4*>(a.codes + row * a.pitch + 32 * t);
      crow[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
      crow[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
      store_scale_word(a.scales, row, t, nblk64, sc_word);
    }
  } else {
    const bool fast = rcp_ok(g);
    const float r = fast ? rcp_approx(g) : 0.0f;
    uint4* crow = reinterpret_cast<uint4*>(a.codes + row * a.pitch + EPT * t);
#pragma unroll
    for (int q = 0; q < NB; ++q) {
      if (16 * q < nel) {
        float v[16];
        unpack_bf16x8(raw[2 * q], v);
        unpack_bf16x8(raw[2 * q + 1], v + 8);
        uint32_t w[4];
        fp8_block(v, g, r, fast, w);
        crow[q] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
}

// ---- rows with RMSNorm and / or the block-64 Hadamard rotation
template <int FMT, int MODE>
__global__ void __launch_bounds__(512, 1) quant_rows_xform_kernel(const RowArgs a) {
  extern __shared__ uint4 s_row[];
  __shared__ float s_red[32];
  __shared__ float s_r;
  griddep_launch_dependents();
  griddep_wait();

  const int64_t row = blockIdx.x;
  const int b = threadIdx.x;
  const int K = a.K;
  const int nblk = (K + 63) >> 6;
  const bool active = b < nblk;
  const int nel = active ? min(64, K - 64 * b) : 0;
  const bool do_norm = (MODE == kPerRow) && (a.flags & kFlagRmsNorm);
  const bool do_wht = (a.flags & kFlagHadamard) != 0;

  // ---- load the 64-block (bf16 -> fp32 is exact)
  const uint4* xr = reinterpret_cast<const uint4*>(a.X + row * static_cast<int64_t>(K));
  float v[64];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (8 * i < nel) {
      const uint4 q = __ldg(xr + 8 * b + i);
      unpack_bf16x8(q, v + 8 * i);
      if (do_norm) s_row[swz_chunk(8 * b + i)] = q;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[8 * i + j] = 0.0f;
    }
  }

  // ---- RMSNorm: fixed 32-lane tree over the staged row, then y = (x r) g
  if (do_norm) {
    __syncthreads();
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      float acc = 0.0f;
      const int nchunk = K >> 3;
      for (int c = lane; c < nchunk; c += 32) {
        float t[8];
        unpack_bf16x8(s_row[swz_chunk(c)], t);
#pragma unroll
        for (int j = 0; j < 8; ++j) acc = __fmaf_rn(t[j], t[j], acc);
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, o));
      if (lane == 0) {
        const float mean = __fdiv_rn(acc, static_cast<float>(K));
        const float var = __fadd_rn(mean, a.eps);
        s_r = __fdiv_rn(1.0f, __fsqrt_rn(var));
      }
    }
    __syncthreads();
    const float r = s_r;
    const uint4* gr = reinterpret_cast<const uint4*>(a.gamma);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (8 * i < nel) {
        float gm[8];
        unpack_bf16x8(__ldg(gr + 8 * b + i), gm);
#pragma unroll
        for (int j = 0; j < 8; ++j) v[8 * i + j] = __fmul_rn(__fmul_rn(v[8 * i + j], r), gm[j]);
      }
    }
  }

  if (do_wht && active) wht64(v);

  // ---- amax: per 16-block and per row
  float a16[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(v[16 * q + i]));
    a16[q] = m;
  }
  const float local = fmaxf(fmaxf(a16[0], a16[1]), fmaxf(a16[2], a16[3]));

  if (MODE == kTensorAmax) {
    const float A = block_max(local, s_red);
    if (threadIdx.x == 0) atomicMax(a.amax_word, __float_as_uint(A));
    return;
  }
  const float g = row_global<FMT, MODE>(a, local, s_red, row);
  if (!active) return;

  if (FMT == kNvfp4) {
    const float six_g = __fmul_rn(6.0f, g);
    const bool fast6g = rcp_ok(six_g);
    const float r6g = fast6g ? rcp_approx(six_g) : 0.0f;
    uint32_t sc_word = 0;
    uint32_t cw[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t sb8 =
          (16 * q < nel) ? nvfp4_block(v + 16 * q, a16[q], g, six_g, r6g, fast6g, cw[2 * q], cw[2 * q + 1]) : 0u;
      if (16 * q >= nel) cw[2 * q] = cw[2 * q + 1] = 0u;
      sc_word |= sb8 << (8 * q);
    }
    uint4* crow = reinterpret_cast<uint4*>(a.codes + row * a.pitch + 32 * b);
    crow[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    crow[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
    store_scale_word(a.scales, row, b, nblk, sc_word);
  } else {
    const bool fast = rcp_ok(g);
    const float r = fast ? rcp_approx(g) : 0.0f;
    uint4* crow = reinterpret_cast<uint4*>(a.codes + row * a.pitch + 64 * b);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (16 * q < nel) {
        uint32_t w[4];
        fp8_block(v + 16 * q, g, r, fast, w);
        crow[q] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
}

__global__ void finalize_global_kernel(float* g) {
  griddep_launch_dependents();
  griddep_wait();
  g[0] = __fdiv_rn(__uint_as_float(*reinterpret_cast<unsigned int*>(g)), 2688.0f);
}

inline int threads_for(int64_t K) {
  const int64_t nblk = (K + 63) / 64;
  const int64_t t = (nblk + 31) / 32 * 32;
  return static_cast<int>(t < 32 ? 32 : t);
}

template <int FMT, int MODE>
cudaError_t launch_rows(const void* X, int64_t rows, int64_t K, const void* gamma, float eps, uint32_t flags,
                        uint8_t* codes, int64_t pitch, uint8_t* scales, float* gout, unsigned int* amax,
                        cudaStream_t s) {
  RowArgs a;
  a.X = static_cast<const __nv_bfloat16*>(X);
  a.K = static_cast<int>(K);
  a.gamma = static_cast<const __nv_bfloat16*>(gamma);
  a.eps = eps;
  a.flags = flags;
  a.codes = codes;
  a.pitch = pitch;
  a.scales = scales;
  a.gout = gout;
  a.amax_word = amax;
  const bool norm = (MODE == kPerRow) && (flags & kFlagRmsNorm);
  const bool xform = norm || (flags & kFlagHadamard);
  const unsigned int grid = static_cast<unsigned int>(rows);
  if (!xform) {
    // one NVFP4 block per thread while a row fits in 512 threads
    if (K <= 8192) {
      const int threads = static_cast<int>(((K + 63) / 64 * 4 + 31) / 32 * 32);
      return launch_pdl(quant_rows_plain_kernel<FMT, MODE, 16>, dim3(grid), dim3(threads), 0, s, a);
    }
    return launch_pdl(quant_rows_plain_kernel<FMT, MODE, 64>, dim3(grid), dim3(threads_for(K)), 0, s, a);
  }
  // staged bf16 row, rounded up to whole 64-element groups (the chunk
  // swizzle permutes within groups of 8 chunks)
  const size_t smem = norm ? static_cast<size_t>((K + 63) / 64) * 64 * 2 : 0;
  auto kern = quant_rows_xform_kernel<FMT, MODE>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(kern, dim3(grid), dim3(threads_for(K)), smem, s, a);
}

}  // namespace

cudaError_t launch_quant_act_nvfp4(const void* X, int64_t M, int64_t K, const void* gamma, float eps,
                                   uint32_t flags, uint8_t* codes, uint8_t* scales, float* g_x, cudaStream_t s) {
  return launch_rows<kNvfp4, kPerRow>(X, M, K, gamma, eps, flags, codes, nvfp4_code_pitch(K), scales, g_x, nullptr,
                                      s);
}

cudaError_t launch_quant_weight_nvfp4(const void* W, int64_t N, int64_t K, uint32_t flags, uint8_t* codes,
                                      uint8_t* scales, float* g_w, cudaStream_t s) {
  // Three steps, no scratch memory: the tensor amax is accumulated in g_w
  // (as fp32 bits), read by the quantizing pass, then turned into g.
  cudaError_t e = cudaMemsetAsync(g_w, 0, sizeof(float), s);
  if (e != cudaSuccess) return e;
  unsigned int* amax = reinterpret_cast<unsigned int*>(g_w);
  const uint32_t f = flags & kFlagHadamard;
  e = launch_rows<kNvfp4, kTensorAmax>(W, N, K, nullptr, 0.0f, f, nullptr, 0, nullptr, nullptr, amax, s);
  if (e != cudaSuccess) return e;
  e = launch_rows<kNvfp4, kTensorQuant>(W, N, K, nullptr, 0.0f, f, codes, nvfp4_code_pitch(K), scales, nullptr,
                                        amax, s);
  if (e != cudaSuccess) return e;
  return launch_pdl(finalize_global_kernel, dim3(1), dim3(1), 0, s, g_w);
}

cudaError_t launch_quant_fp8(const void* X, int64_t rows, int64_t K, const void* gamma, float eps, uint32_t flags,
                             uint8_t* codes, float* s_out, cudaStream_t s) {
  return launch_rows<kFp8, kPerRow>(X, rows, K, gamma, eps, flags, codes, K, nullptr, s_out, nullptr, s);
}

}  // namespace vlaq
