// Fused activation prologue and the offline weight quantizers.
//
// One CTA per row; thread b owns the 64-element block b of the row
// (the Hadamard block, four NVFP4 scale blocks, 32 packed code bytes and one
// 4-byte word of the 128x4 tiled scale layout).  The row is read once from
// HBM with 16-byte loads, transformed in registers (RMSNorm, block-64 WHT),
// reduced to a per-row amax with warp shuffles, then quantized and written
// with 16-byte stores.  HBM-bound: 2 bytes in and 0.5625 (NVFP4) or 1 (FP8)
// bytes out per element.
//
// Arithmetic follows the format definitions stated in include/vlaq.h:
// every fp32 operation is an explicitly rounded intrinsic (no contraction),
// division and square root are correctly rounded, so codes and scales are
// bit-identical to any implementation that performs the same operations
// ("FoldQuant W8A8/W4A4 inference", SYCL commit: correctly rounded divide
// and sqrt, fixed reduction tree).
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

template <int FMT, int MODE>
__global__ void __launch_bounds__(512)
quant_rows_kernel(const __nv_bfloat16* __restrict__ X, int K, const __nv_bfloat16* __restrict__ gamma,
                  float eps, uint32_t flags, uint8_t* __restrict__ codes, int64_t pitch,
                  uint8_t* __restrict__ scales, float* __restrict__ gout,
                  unsigned int* __restrict__ amax_word) {
  extern __shared__ uint4 s_row[];
  __shared__ float s_red[32];
  __shared__ float s_r;

  const int64_t row = blockIdx.x;
  const int b = threadIdx.x;
  const int nblk = (K + 63) >> 6;
  const bool active = b < nblk;
  const int nel = active ? min(64, K - 64 * b) : 0;
  const bool do_norm = (MODE == kPerRow) && (flags & kFlagRmsNorm);
  const bool do_wht = (flags & kFlagHadamard) != 0;

  // ---- load the 64-block (bf16 -> fp32 is exact)
  const uint4* xr = reinterpret_cast<const uint4*>(X + row * static_cast<int64_t>(K));
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
        const float var = __fadd_rn(mean, eps);
        s_r = __fdiv_rn(1.0f, __fsqrt_rn(var));
      }
    }
    __syncthreads();
    const float r = s_r;
    const uint4* gr = reinterpret_cast<const uint4*>(gamma);
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
    if (threadIdx.x == 0) atomicMax(amax_word, __float_as_uint(A));  // A >= 0: bits order = value order
    return;
  }

  float g;
  if (MODE == kPerRow) {
    const float A = block_max(local, s_red);
    g = (FMT == kNvfp4) ? __fdiv_rn(A, 2688.0f) : __fdiv_rn(A, 448.0f);
    if (threadIdx.x == 0) gout[row] = g;
  } else {
    g = __fdiv_rn(__uint_as_float(*amax_word), 2688.0f);
  }
  if (!active) return;

  if (FMT == kNvfp4) {
    // ---- two-level NVFP4: E4M3 block scale, E2M1 codes
    const float six_g = __fmul_rn(6.0f, g);
    uint32_t sc_word = 0;
    uint32_t cw[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float S = 0.0f;
      uint32_t sb8 = 0;
      if (g > 0.0f && 16 * q < nel) {
        const float sb = __fdiv_rn(a16[q], six_g);
        sb8 = cvt_e4m3x2(sb, 0.0f) & 0xFFu;
        S = __fmul_rn(e4m3_to_f32(sb8), g);
      }
      sc_word |= sb8 << (8 * q);
      float qv[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) qv[i] = (S != 0.0f) ? __fdiv_rn(v[16 * q + i], S) : 0.0f;
      cw[2 * q] = cvt_e2m1x8(qv);
      cw[2 * q + 1] = cvt_e2m1x8(qv + 8);
    }
    uint4* crow = reinterpret_cast<uint4*>(codes + row * pitch + 32 * b);
    crow[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    crow[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
    // 128x4 tiled scale layout: 512-byte atom per (128 rows, 4 blocks)
    const int64_t atom = (row >> 7) * nblk + b;
    const int64_t off = atom * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4;
    *reinterpret_cast<uint32_t*>(scales + off) = sc_word;
  } else {
    // ---- FP8 E4M3 codes with one fp32 scale per row
    uint32_t w[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      float q0, q1, q2, q3;
      if (g != 0.0f) {
        q0 = __fdiv_rn(v[4 * j], g);
        q1 = __fdiv_rn(v[4 * j + 1], g);
        q2 = __fdiv_rn(v[4 * j + 2], g);
        q3 = __fdiv_rn(v[4 * j + 3], g);
      } else {
        q0 = q1 = q2 = q3 = 0.0f;
      }
      w[j] = cvt_e4m3x2(q0, q1) | (cvt_e4m3x2(q2, q3) << 16);
    }
    uint4* crow = reinterpret_cast<uint4*>(codes + row * pitch + 64 * b);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (16 * i < nel) crow[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  }
}

__global__ void finalize_global_kernel(float* g) {
  g[0] = __fdiv_rn(__uint_as_float(*reinterpret_cast<unsigned int*>(g)), 2688.0f);
}

inline int threads_for(int64_t K) {
  const int64_t nblk = (K + 63) / 64;
  const int64_t t = (nblk + 31) / 32 * 32;
  return static_cast<int>(t < 32 ? 32 : t);
}

template <int FMT, int MODE>
cudaError_t launch_rows(const void* X, int64_t rows, int64_t K, const void* gamma, float eps,
                        uint32_t flags, uint8_t* codes, int64_t pitch, uint8_t* scales, float* gout,
                        unsigned int* amax, cudaStream_t s) {
  const bool norm = (MODE == kPerRow) && (flags & kFlagRmsNorm);
  // staged bf16 row, rounded up to whole 64-element groups (the chunk
  // swizzle permutes within groups of 8 chunks)
  const size_t smem = norm ? static_cast<size_t>((K + 63) / 64) * 64 * 2 : 0;
  auto kern = quant_rows_kernel<FMT, MODE>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  kern<<<static_cast<unsigned int>(rows), threads_for(K), smem, s>>>(
      static_cast<const __nv_bfloat16*>(X), static_cast<int>(K),
      static_cast<const __nv_bfloat16*>(gamma), eps, flags, codes, pitch, scales, gout, amax);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quant_act_nvfp4(const void* X, int64_t M, int64_t K, const void* gamma, float eps,
                                   uint32_t flags, uint8_t* codes, uint8_t* scales, float* g_x,
                                   cudaStream_t s) {
  return launch_rows<kNvfp4, kPerRow>(X, M, K, gamma, eps, flags, codes, nvfp4_code_pitch(K), scales,
                                      g_x, nullptr, s);
}

cudaError_t launch_quant_weight_nvfp4(const void* W, int64_t N, int64_t K, uint32_t flags,
                                      uint8_t* codes, uint8_t* scales, float* g_w, cudaStream_t s) {
  // Three steps, no scratch memory: the tensor amax is accumulated in g_w
  // (as fp32 bits), read by the quantizing pass, then turned into g.
  cudaError_t e = cudaMemsetAsync(g_w, 0, sizeof(float), s);
  if (e != cudaSuccess) return e;
  unsigned int* amax = reinterpret_cast<unsigned int*>(g_w);
  const uint32_t f = flags & kFlagHadamard;
  e = launch_rows<kNvfp4, kTensorAmax>(W, N, K, nullptr, 0.0f, f, nullptr, 0, nullptr, nullptr,
                                       amax, s);
  if (e != cudaSuccess) return e;
  e = launch_rows<kNvfp4, kTensorQuant>(W, N, K, nullptr, 0.0f, f, codes, nvfp4_code_pitch(K),
                                        scales, nullptr, amax, s);
  if (e != cudaSuccess) return e;
  finalize_global_kernel<<<1, 1, 0, s>>>(g_w);
  return cudaGetLastError();
}

cudaError_t launch_quant_fp8(const void* X, int64_t rows, int64_t K, const void* gamma, float eps,
                             uint32_t flags, uint8_t* codes, float* s_out, cudaStream_t s) {
  return launch_rows<kFp8, kPerRow>(X, rows, K, gamma, eps, flags, codes, K, nullptr, s_out,
                                    nullptr, s);
}

}  // namespace vlaq
