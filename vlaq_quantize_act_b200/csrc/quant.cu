// Fused activation prologue and the offline weight quantizers.
//
// Rows are held in registers.  A CTA of W warps owns one row at a time (4
// warps for rows of up to 4096 elements, 8 for longer rows); lane l of warp
// w holds the 16-element blocks 32 (W i + w) + l of the row, i = 0 .. BPL-1
// (2 blocks per lane for short rows, 5 or 8 for long ones), read with two
// coalesced 16-byte loads each (a warp reads 1 KiB of contiguous bf16 per
// block index).  Per row:
//   pass A  (transform and) per-16 block amax; the transformed values of
//           the fused variants (RMSNorm, rotation, smoothing) are kept in
//           shared memory so each is computed once; row amax by one warp
//           reduction and a cross-warp max -> global scale g;
//   pass B  E4M3 block scale and codes from the kept values (or the bf16
//           words still in registers), stored with coalesced 8- or 16-byte
//           stores.
// Four lanes hold one Hadamard block (stages h = 1, 2, 4, 8 inside a lane,
// 16 and 32 across lanes) and one 4-byte word of the 128x4 tiled scale
// layout; a warp writes 256 (NVFP4) or 512 (FP8, INT8) contiguous code
// bytes per block index.  HBM-bound: 2 bytes in and 0.5625 (NVFP4) or 1
// (FP8, INT8) bytes out per element.
//
// Arithmetic follows the format definitions stated in include/vlaq.h: every
// fp32 operation is an explicitly rounded intrinsic (no contraction),
// division and square root are correctly rounded, so codes and scales are
// bit-identical to any implementation that performs the same operations
// ("FoldQuant W8A8/W4A4 inference", SYCL commit: correctly rounded divide
// and sqrt, fixed reduction tree).  The RMSNorm sum of squares follows the
// fixed 32-lane tree (lane l accumulates the 8-element chunks l, l + 32, ...
// in order with fused multiply-adds, then an XOR butterfly), and the
// Hadamard butterfly keeps the sequential stage order h = 1, 2, ..., 32.
//
// Every quotient x / S is the correctly rounded one (Markstein's
// correction step after a product with the correctly rounded reciprocal,
// see quotients() below), so the codes equal those of a plain division.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace vlaq {

__device__ unsigned int g_vlaq_quant_status = 0;

namespace {

enum { kNvfp4 = 0, kFp8 = 1, kInt8 = 2 };
enum { kPerRow = 0, kTensorAmax = 1, kTensorQuant = 2, kStatic = 3 };

// Row-group shape: W warps per row, at most BPL 16-element blocks per lane
// (8 bf16 words each, kept in registers).
template <int W, int BPL>
struct RowCfg {
  static_assert(W >= 2, "a row group is a whole CTA");
  static constexpr int kMaxK = 16 * 32 * W * BPL;
  static constexpr int kWarps = W;  // warps per CTA (one row group)
  static constexpr int kThreads = 32 * kWarps;
  // kept transformed values of the fused variants: per warp BPL x 16 fp32
  // per lane
  static constexpr int kCacheBytesPerWarp = BPL * 16 * 4 * 32;
  // rows of up to 4096 elements: seven CTAs per SM (at most 72 registers),
  // so that the 1036 resident CTAs hold every row of a 1024-token input
  // (measured: the fused smoothing variant at 80 registers, six CTAs per SM,
  // ran 6% slower).  The untransformed static-scale variant stays below 72
  // registers without the bound and ran 4% slower under it.
  static constexpr int min_blocks(bool bounded) { return (W == 4 && BPL == 2 && bounded) ? 7 : 1; }
};

__device__ __forceinline__ void unpack_bf16x8(const uint4& q, float* v) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    v[2 * j] = __uint_as_float(w[j] << 16);
    v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
  }
}

// max |x| of 16 bf16 values (two 16-byte words), exact: kept packed as
// bf16 pairs, the max of bf16 values is one of them.
__device__ __forceinline__ float absmax_bf16x16(const uint4& a, const uint4& b) {
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  __nv_bfloat162 h[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t aw = w[j] & 0x7FFF7FFFu;  // |x| of both halves
    h[j] = *reinterpret_cast<const __nv_bfloat162*>(&aw);
  }
#pragma unroll
  for (int s = 4; s; s >>= 1)
#pragma unroll
    for (int j = 0; j < s; ++j) h[j] = __hmax2(h[j], h[j + s]);
  return fmaxf(__low2float(h[0]), __high2float(h[0]));
}

// Correctly rounded quotient without a divide per element: Markstein's
// correction step (P. Markstein, "IA-64 and Elementary Functions", 2000:
// with y = RN(1/S) and q0 = RN(x y), the residual x - q0 S is exact under a
// fused multiply-add and RN(q0 + (x - q0 S) y) = RN(x / S)).  The residual
// is formed negated, e' = q0 S - x, so that x = -0 still yields -0.  The
// reciprocal is CUDA's correctly rounded __frcp_rn, once per divisor.  Only
// divisors far from 1 (where the residual or 1/S could leave the normal
// range) and S = 0 take the slow path, behind a warp vote.
struct Divisor {
  float S, y;
  bool slow;  // S = 0 (quotients 0) or S outside [2^-64, 2^64]
};

__device__ __forceinline__ Divisor make_divisor(float S) {
  Divisor d;
  d.S = S;
  const bool ok = S >= 0x1p-64f && S <= 0x1p64f;
  d.y = ok ? __frcp_rn(S) : 0.0f;
  d.slow = !ok;
  return d;
}

__device__ __forceinline__ float markstein_quotient(float x, float S, float y) {
  const float q0 = __fmul_rn(x, y);
  const float e = __fmaf_rn(q0, S, -x);  // q0 S - x, exact
  return __fmaf_rn(-e, y, q0);
}

// RN(v[i] / S) for N values (0 when S = 0).  Executed by the whole warp.
template <int N>
__device__ __forceinline__ void quotients(const float* v, const Divisor& d, float* q) {
  static_assert(N % 2 == 0, "pairs");
  // the same three steps on packed pairs (sm_100a fp32x2 multiply and fused
  // multiply-add, each lane rounded once): q0 = x y, e = q0 S - x (x negated
  // exactly, so -0 stays -0), q = q0 + e (-y)
  const float2 yy = make_float2(d.y, d.y);
  const float2 ny = make_float2(-d.y, -d.y);
  const float2 ss = make_float2(d.S, d.S);
#pragma unroll
  for (int i = 0; i < N; i += 2) {
    const float2 x = make_float2(v[i], v[i + 1]);
    const float2 q0 = __fmul2_rn(x, yy);
    const float2 e = __ffma2_rn(q0, ss, make_float2(-x.x, -x.y));
    const float2 r = __ffma2_rn(e, ny, q0);
    q[i] = r.x;
    q[i + 1] = r.y;
  }
  if (__any_sync(0xffffffffu, d.slow)) {
    if (d.slow) {
#pragma unroll
      for (int i = 0; i < N; ++i) q[i] = (d.S == 0.0f) ? 0.0f : __fdiv_rn(v[i], d.S);
    }
  }
}

// The global scale of a row from its amax A >= 0: RN(A / 2688) (NVFP4),
// RN(A / 448) (FP8) or RN(A / 127) (INT8), by the correction step against
// the constant's correctly rounded reciprocal; rows whose amax is tiny
// (quotient near the subnormal range) take a divide.  Uniform per row.
template <int FMT>
__device__ __forceinline__ float row_global(float A) {
  constexpr float c = (FMT == 0) ? 2688.0f : (FMT == 1) ? 448.0f : 127.0f;
  if (A < 0x1p-64f) return __fdiv_rn(A, c);
  return markstein_quotient(A, c, __frcp_rn(c));
}

// E4M3 byte of RN(a / d) for a >= 0 (d is warp-uniform).
__device__ __forceinline__ uint32_t e4m3_of_quotient(float a, const Divisor& d) {
  const float q = d.slow ? __fdiv_rn(a, d.S) : markstein_quotient(a, d.S, d.y);
  return cvt_e4m3x2(q, 0.0f) & 0xFFu;
}

// Byte offset of (row, 64-block 0) in the 128x4 tiled scale layout
// (512-byte atom per 128 rows x 4 blocks; nblk = 64-blocks per row).
__device__ __forceinline__ int64_t scale_row_base(int64_t row, int nblk) {
  return (row >> 7) * nblk * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4;
}

struct RowArgs {
  const __nv_bfloat16* X;
  int K;
  const __nv_bfloat16* gamma;
  float eps;
  uint8_t* codes;
  int64_t pitch;
  uint8_t* scales;
  float* gout;
  unsigned int* amax_word;
  int64_t rows;
  const float* smooth;  // per-input-channel smoothing factors [K] (or null)
  uint32_t sflags;      // kFlagSmoothAfter | kFlagSmoothMul
  float g_static;       // calibrated global scale (kStatic)
};

// Normalised WHT of the 64-block spread over lanes 4 g .. 4 g + 3 (16 values
// each, element 16 (lane % 4) + j): stages h = 1, 2, 4, 8 inside the lane,
// h = 16, 32 across lanes (xor 1, 2), then x 1/8 (exact) -- the stages of the
// sequential butterfly in the same order.  Executed by the whole warp.
// Stages h >= 2 run two butterflies per packed fp32x2 instruction (each lane
// rounded once, so the values are those of the scalar steps): a + b, and
// a - b as fma(b, -1, a), a single rounding of the same exact difference
// (signed zeros included).  Across lanes the new value is p + s v with s = -1
// in the upper lane and +1 in the lower one, again one fused multiply-add.
__device__ __forceinline__ void wht64_lanes(float* v, int lane) {
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    const float a = v[i], b = v[i + 1];
    v[i] = __fadd_rn(a, b);
    v[i + 1] = __fsub_rn(a, b);
  }
  const float2 m1 = make_float2(-1.0f, -1.0f);
#pragma unroll
  for (int h = 2; h < 16; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
      if ((i & h) == 0) {
        const float2 a = make_float2(v[i], v[i + 1]), b = make_float2(v[i + h], v[i + h + 1]);
        const float2 sum = __fadd2_rn(a, b), dif = __ffma2_rn(b, m1, a);
        v[i] = sum.x;
        v[i + 1] = sum.y;
        v[i + h] = dif.x;
        v[i + h + 1] = dif.y;
      }
    }
  }
#pragma unroll
  for (int x = 1; x < 4; x <<= 1) {
    const float sg = (lane & x) != 0 ? -1.0f : 1.0f;
    const float2 s2 = make_float2(sg, sg);
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
      const float2 p = make_float2(__shfl_xor_sync(0xffffffffu, v[i], x), __shfl_xor_sync(0xffffffffu, v[i + 1], x));
      const float2 r = __ffma2_rn(make_float2(v[i], v[i + 1]), s2, p);
      v[i] = r.x;
      v[i + 1] = r.y;
    }
  }
  const float2 e8 = make_float2(0.125f, 0.125f);
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    const float2 r = __fmul2_rn(make_float2(v[i], v[i + 1]), e8);
    v[i] = r.x;
    v[i + 1] = r.y;
  }
}

// y_k / a_k or y_k * a_k for the 16 channels of block q (smoothing).
__device__ __forceinline__ void smooth_block(const RowArgs& a, int q, float* v) {
  const float4* s4 = reinterpret_cast<const float4*>(a.smooth) + 4 * q;
  const bool mul = (a.sflags & kFlagSmoothMul) != 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 f = __ldg(s4 + i);
    const float fs[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) v[4 * i + j] = mul ? __fmul_rn(v[4 * i + j], fs[j]) : __fdiv_rn(v[4 * i + j], fs[j]);
  }
}

// The 16 values of block q after the row transform (zeros past the row):
// y = (x r) gamma for RMSNorm, the smoothing divide (or multiply) before or
// after the block-64 WHT.  x is the block's two bf16 words (zero past the
// row).  Warp-uniform.
template <bool NORM, bool WHT, bool SMOOTH>
__device__ __forceinline__ void block_values(const RowArgs& a, const uint4& x0, const uint4& x1, int q, int nblk16,
                                             float r, int lane, float* v) {
  unpack_bf16x8(x0, v);
  unpack_bf16x8(x1, v + 8);
  if (q < nblk16) {
    if (NORM) {
      const uint4* gsrc = reinterpret_cast<const uint4*>(a.gamma) + 2 * q;
      float gm[16];
      unpack_bf16x8(__ldg(gsrc), gm);
      unpack_bf16x8(__ldg(gsrc + 1), gm + 8);
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = __fmul_rn(__fmul_rn(v[j], r), gm[j]);
    }
    if (SMOOTH && !(a.sflags & kFlagSmoothAfter)) smooth_block(a, q, v);
  }
  if (WHT) wht64_lanes(v, lane);
  if (SMOOTH && (a.sflags & kFlagSmoothAfter) && q < nblk16) smooth_block(a, q, v);
}

__device__ __forceinline__ float absmax16(const float* v) {
  float m = 0.0f;
#pragma unroll
  for (int j = 0; j < 16; ++j) m = fmaxf(m, fabsf(v[j]));
  return m;
}

// RMSNorm factor r = 1 / sqrt(mean(x^2) + eps) of a row: the warps put their
// blocks into a shared-memory copy of the row, and one warp walks it in the
// fixed tree's order (lane l: the 8-element chunks l, l + 32, ..., the
// chain's next chunk loaded before the current chunk's eight steps; then
// the XOR butterfly).
__device__ __forceinline__ float rms_factor_row(const uint4* x4, int K, float eps, int lane) {
  const int nch = K >> 3;
  float acc = 0.0f;
  uint4 cur = lane < nch ? x4[lane] : make_uint4(0, 0, 0, 0);
  for (int c = lane; c < nch; c += 32) {
    const uint4 nxt = c + 32 < nch ? x4[c + 32] : make_uint4(0, 0, 0, 0);
    float t[8];
    unpack_bf16x8(cur, t);
#pragma unroll
    for (int j = 0; j < 8; ++j) acc = __fmaf_rn(t[j], t[j], acc);
    cur = nxt;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, o));
  const float mean = __fdiv_rn(acc, static_cast<float>(K));
  return __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(mean, eps)));
}

// All rows of one launch: FMT (NVFP4 / FP8 / INT8), MODE (per-row scale,
// tensor amax pass, tensor quantize pass, static calibrated scale), NORM
// (RMSNorm, per-row and static modes), WHT (block-64 Hadamard), SMOOTH
// (per-channel smoothing), W warps per row.  Row group k of the grid takes
// rows k, k + groups, ... (one row per group at the workload sizes).
template <int FMT, int MODE, bool NORM, bool WHT, bool SMOOTH, int W, int BPL>
__global__ void __launch_bounds__(RowCfg<W, BPL>::kThreads,
                                  RowCfg<W, BPL>::min_blocks(NORM || WHT || SMOOTH || MODE != kStatic))
    quant_rows_kernel(const RowArgs a) {
  using C = RowCfg<W, BPL>;
  constexpr bool KEEP = NORM || WHT || SMOOTH;  // transformed values kept in shared memory
  // dynamic shared memory: [kept values][row copy]
  extern __shared__ __align__(16) float4 s_keep[];
  __shared__ float s_red[C::kWarps];
  __shared__ float s_r;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wr = warp;  // warp index inside the row group
  const int K = a.K;
  const int nblk16 = K >> 4;
  const int nblk64 = (K + 63) >> 6;
  const int nblk16_pad = 4 * nblk64;  // blocks up to the padded row end
  const int64_t gstride = gridDim.x;
  float4* keep = s_keep + static_cast<size_t>(warp) * BPL * 4 * 32;

  griddep_wait();
  griddep_launch_dependents();

  float g_tensor = 0.0f;
  if (MODE == kTensorQuant) g_tensor = __fdiv_rn(__uint_as_float(*a.amax_word), 2688.0f);
  if (MODE == kStatic) g_tensor = a.g_static;

  for (int64_t row = blockIdx.x; row < a.rows; row += gstride) {
    // ---- the row's blocks into registers (zero past the row end)
    const uint4* x4 = reinterpret_cast<const uint4*>(a.X + row * K);
    uint4 d[BPL][2];
#pragma unroll
    for (int i = 0; i < BPL; ++i) {
      const int q = (i * W + wr) * 32 + lane;
      if (q < nblk16) {
        d[i][0] = __ldg(x4 + 2 * q);
        d[i][1] = __ldg(x4 + 2 * q + 1);
      } else {
        d[i][0] = make_uint4(0, 0, 0, 0);
        d[i][1] = make_uint4(0, 0, 0, 0);
      }
    }

    // ---- RMSNorm factor, fixed 32-lane tree
    float r = 1.0f;
    if (NORM) {
      // the row's copy follows the kept values in shared memory
      uint4* srow4 = reinterpret_cast<uint4*>(s_keep + static_cast<size_t>(C::kWarps) * BPL * 4 * 32);
#pragma unroll
      for (int i = 0; i < BPL; ++i) {
        const int q = (i * W + wr) * 32 + lane;
        if (q < nblk16) {
          srow4[2 * q] = d[i][0];
          srow4[2 * q + 1] = d[i][1];
        }
      }
      __syncthreads();
      if (wr == 0) {
        const float rr = rms_factor_row(srow4, K, a.eps, lane);
        if (lane == 0) s_r = rr;
      }
      __syncthreads();
      r = s_r;
    }

    // ---- pass A: per-block amax (kept in registers), transformed values
    // kept in shared memory, row amax
    float a16r[BPL];
    float local = 0.0f;
#pragma unroll
    for (int i = 0; i < BPL; ++i) {
      a16r[i] = 0.0f;
      if ((i * W + wr) * 32 < nblk16_pad) {  // warp-uniform
        const int q = (i * W + wr) * 32 + lane;
        float m;
        if (KEEP) {
          float v[16];
          block_values<NORM, WHT, SMOOTH>(a, d[i][0], d[i][1], q, nblk16, r, lane, v);
          m = absmax16(v);
#pragma unroll
          for (int t = 0; t < 4; ++t)
            keep[(i * 4 + t) * 32 + lane] = make_float4(v[4 * t], v[4 * t + 1], v[4 * t + 2], v[4 * t + 3]);
        } else {
          m = absmax_bf16x16(d[i][0], d[i][1]);
        }
        a16r[i] = m;
        local = fmaxf(local, m);
      }
    }
    float g = g_tensor;
    if (MODE == kStatic && wr == 0 && lane == 0) a.gout[row] = g;
    if (MODE == kPerRow || MODE == kTensorAmax) {
      // non-negative floats order like their bit patterns: one warp reduction
      float A = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(local)));
      if (lane == 0) s_red[wr] = A;
      __syncthreads();
      A = s_red[0];
#pragma unroll
      for (int w = 1; w < W; ++w) A = fmaxf(A, s_red[w]);
      if (MODE == kTensorAmax) {
        if (wr == 0 && lane == 0) atomicMax(a.amax_word, __float_as_uint(A));  // A >= 0: bit order = value order
      } else {
        g = row_global<FMT>(A);
        if (wr == 0 && lane == 0) a.gout[row] = g;
      }
    }

    // ---- pass B: block scales and codes
    if (MODE != kTensorAmax) {
      uint8_t* crow = a.codes + row * a.pitch;
      if (FMT == kNvfp4) {
        uint8_t* srow = a.scales + scale_row_base(row, nblk64);
        const Divisor d6g = make_divisor(__fmul_rn(6.0f, g));
#pragma unroll
        for (int i = 0; i < BPL; ++i) {
          if ((i * W + wr) * 32 < nblk16_pad) {
            const int q = (i * W + wr) * 32 + lane;
            float v[16];
            if (KEEP) {
#pragma unroll
              for (int t = 0; t < 4; ++t) {
                const float4 f = keep[(i * 4 + t) * 32 + lane];
                v[4 * t] = f.x;
                v[4 * t + 1] = f.y;
                v[4 * t + 2] = f.z;
                v[4 * t + 3] = f.w;
              }
            } else {
              unpack_bf16x8(d[i][0], v);
              unpack_bf16x8(d[i][1], v + 8);
            }
            float a16 = a16r[i];
            uint32_t sb8 = 0;
            float S = 0.0f;
            if (g > 0.0f) {
              // A calibrated g bounds neither a16 / 6 g nor v / S: values
              // whose quotient would pass 512 (scale 448 either way) or 8
              // (code 6 either way) are clamped there (exact: powers of two),
              // so no quotient overflows, in the correction step or a divide.
              if (MODE == kStatic) a16 = fminf(a16, __fmul_rn(512.0f, d6g.S));
              sb8 = e4m3_of_quotient(a16, d6g);
              S = __fmul_rn(e4m3_to_f32(sb8), g);
            }
            const Divisor dv = make_divisor(S);
            if (MODE == kStatic) {
              const float b = __fmul_rn(8.0f, S);
#pragma unroll
              for (int j = 0; j < 16; ++j) v[j] = fminf(fmaxf(v[j], -b), b);
            }
            float qv[16];
            quotients<16>(v, dv, qv);
            const uint32_t w0 = cvt_e2m1x8(qv);
            const uint32_t w1 = cvt_e2m1x8(qv + 8);
            if (q < nblk16_pad) {
              *reinterpret_cast<uint2*>(crow + 8 * q) = make_uint2(w0, w1);
              srow[(q >> 2) * 512 + (q & 3)] = static_cast<uint8_t>(sb8);
            }
          }
        }
      } else {
        const Divisor dg = make_divisor(g);
#pragma unroll
        for (int i = 0; i < BPL; ++i) {
          if ((i * W + wr) * 32 < nblk16_pad) {
            const int q = (i * W + wr) * 32 + lane;
            float v[16];
            if (KEEP) {
#pragma unroll
              for (int t = 0; t < 4; ++t) {
                const float4 f = keep[(i * 4 + t) * 32 + lane];
                v[4 * t] = f.x;
                v[4 * t + 1] = f.y;
                v[4 * t + 2] = f.z;
                v[4 * t + 3] = f.w;
              }
            } else {
              unpack_bf16x8(d[i][0], v);
              unpack_bf16x8(d[i][1], v + 8);
            }
            float qv[16];
            quotients<16>(v, dg, qv);
            uint32_t w[4];
            if (FMT == kInt8) {
              // round half to even, clamp to [-127, 127], two's complement bytes
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                uint32_t word = 0;
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                  const int c = min(127, max(-127, __float2int_rn(qv[4 * j + t])));
                  word |= (static_cast<uint32_t>(c) & 0xFFu) << (8 * t);
                }
                w[j] = word;
              }
            } else {
#pragma unroll
              for (int j = 0; j < 4; ++j)
                w[j] = cvt_e4m3x2(qv[4 * j], qv[4 * j + 1]) | (cvt_e4m3x2(qv[4 * j + 2], qv[4 * j + 3]) << 16);
            }
            if (q < nblk16) *reinterpret_cast<uint4*>(crow + 16 * q) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    }
    // the next row reuses s_red / s_r
    __syncthreads();
  }
}

__global__ void finalize_global_kernel(float* g) {
  griddep_wait();
  griddep_launch_dependents();
  g[0] = __fdiv_rn(__uint_as_float(*reinterpret_cast<unsigned int*>(g)), 2688.0f);
}

template <int FMT, int MODE, bool NORM, bool WHT, bool SMOOTH, int W, int BPL>
cudaError_t launch_groups(const RowArgs& a, cudaStream_t s) {
  using C = RowCfg<W, BPL>;
  auto kern = quant_rows_kernel<FMT, MODE, NORM, WHT, SMOOTH, W, BPL>;
  const bool keep = NORM || WHT || SMOOTH;
  size_t smem = keep ? static_cast<size_t>(C::kWarps) * C::kCacheBytesPerWarp : 0;
  if (NORM) smem += static_cast<size_t>(2) * a.K;  // the row's copy for the tree
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  // one row per CTA while rows last; very tall inputs loop (at most 64
  // CTAs per SM are launched)
  const int64_t ctas = a.rows;
  const int64_t cap = static_cast<int64_t>(device_sm_count()) * 64;
  const unsigned int grid = static_cast<unsigned int>(ctas < cap ? ctas : cap);
  return launch_pdl(kern, dim3(grid), dim3(C::kThreads), smem, s, a);
}

template <int FMT, int MODE, bool NORM, bool WHT, bool SMOOTH = false>
cudaError_t launch_shape(const RowArgs& a, cudaStream_t s) {
  // measured on B200 (graph-timed launches over inputs larger than L2,
  // M = 1024): rows of up to 4096 elements run fastest with 4 warps per row
  // and 2 blocks per lane (against 1, 2 or 8 warps), rows of up to 20480
  // with 8 warps and 5 blocks per lane (against 4 or 16 warps); loading the
  // rows into registers beat staging them through a shared-memory ring of
  // bulk copies at both lengths
  if (a.K <= RowCfg<4, 2>::kMaxK) return launch_groups<FMT, MODE, NORM, WHT, SMOOTH, 4, 2>(a, s);
  if (a.K <= RowCfg<8, 5>::kMaxK) return launch_groups<FMT, MODE, NORM, WHT, SMOOTH, 8, 5>(a, s);
  return launch_groups<FMT, MODE, NORM, WHT, SMOOTH, 8, 8>(a, s);
}

template <int FMT, int MODE>
cudaError_t launch_rows(const void* X, int64_t rows, int64_t K, const void* gamma, float eps, uint32_t flags,
                        uint8_t* codes, int64_t pitch, uint8_t* scales, float* gout, unsigned int* amax,
                        cudaStream_t s, const float* smooth = nullptr, float g_static = 0.0f) {
  RowArgs a;
  a.X = static_cast<const __nv_bfloat16*>(X);
  a.K = static_cast<int>(K);
  a.gamma = static_cast<const __nv_bfloat16*>(gamma);
  a.eps = eps;
  a.codes = codes;
  a.pitch = pitch;
  a.scales = scales;
  a.gout = gout;
  a.amax_word = amax;
  a.rows = rows;
  a.smooth = smooth;
  a.sflags = flags & (kFlagSmoothAfter | kFlagSmoothMul);
  a.g_static = g_static;
  const bool wht = (flags & kFlagHadamard) != 0;
  if constexpr ((MODE == kPerRow || MODE == kStatic) && FMT == kNvfp4) {
    if (smooth) {
      if (flags & kFlagRmsNorm)
        return wht ? launch_shape<FMT, MODE, true, true, true>(a, s) : launch_shape<FMT, MODE, true, false, true>(a, s);
      return wht ? launch_shape<FMT, MODE, false, true, true>(a, s) : launch_shape<FMT, MODE, false, false, true>(a, s);
    }
  }
  if constexpr (MODE == kPerRow || MODE == kStatic) {
    if (flags & kFlagRmsNorm)
      return wht ? launch_shape<FMT, MODE, true, true>(a, s) : launch_shape<FMT, MODE, true, false>(a, s);
  }
  return wht ? launch_shape<FMT, MODE, false, true>(a, s) : launch_shape<FMT, MODE, false, false>(a, s);
}

}  // namespace

cudaError_t launch_quant_act_nvfp4(const void* X, int64_t M, int64_t K, const void* gamma, float eps,
                                   uint32_t flags, uint8_t* codes, uint8_t* scales, float* g_x, cudaStream_t s) {
  return launch_rows<kNvfp4, kPerRow>(X, M, K, gamma, eps, flags, codes, nvfp4_code_pitch(K), scales, g_x, nullptr,
                                      s);
}

cudaError_t launch_quant_act_nvfp4_smooth(const void* X, int64_t M, int64_t K, const void* gamma, const float* smooth,
                                          float eps, uint32_t flags, uint8_t* codes, uint8_t* scales, float* g_x,
                                          cudaStream_t s) {
  return launch_rows<kNvfp4, kPerRow>(X, M, K, gamma, eps, flags, codes, nvfp4_code_pitch(K), scales, g_x, nullptr,
                                      s, smooth);
}

cudaError_t launch_quant_act_nvfp4_static(const void* X, int64_t M, int64_t K, const void* gamma, const float* smooth,
                                          float eps, uint32_t flags, float g_static, uint8_t* codes, uint8_t* scales,
                                          float* g_x, cudaStream_t s) {
  return launch_rows<kNvfp4, kStatic>(X, M, K, gamma, eps, flags, codes, nvfp4_code_pitch(K), scales, g_x, nullptr,
                                      s, smooth, g_static);
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

cudaError_t launch_quant_int8(const void* X, int64_t rows, int64_t K, const void* gamma, float eps, uint32_t flags,
                              int8_t* codes, float* s_out, cudaStream_t s) {
  return launch_rows<kInt8, kPerRow>(X, rows, K, gamma, eps, flags, reinterpret_cast<uint8_t*>(codes), K, nullptr,
                                     s_out, nullptr, s);
}

namespace {
// Tiled (128x4, the layout the tensor cores read) -> row-major [rows, K/16]
// block scales: one thread per output word of four scale bytes (K/16 may
// not be a multiple of 4: the last word of a row is written byte-wise).
__global__ void scales_to_rowmajor_kernel(const uint8_t* __restrict__ in, uint8_t* __restrict__ out, int64_t rows,
                                          int cols, int nblk64) {
  griddep_wait();
  griddep_launch_dependents();
  const int words = (cols + 3) >> 2;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= rows * words) return;
  const int64_t r = i / words;
  const int j = static_cast<int>(i % words);  // 64-block j: scale columns 4j .. 4j + 3
  const uint32_t w = *reinterpret_cast<const uint32_t*>(in + ((r >> 7) * nblk64 + j) * 512 + (r & 31) * 16 +
                                                        ((r & 127) >> 5) * 4);
  uint8_t* dst = out + r * cols + 4 * j;
  for (int b = 0; b < 4 && 4 * j + b < cols; ++b) dst[b] = static_cast<uint8_t>(w >> (8 * b));
}
}  // namespace

cudaError_t launch_scales_to_rowmajor(const uint8_t* in, uint8_t* out, int64_t rows, int64_t K, cudaStream_t s) {
  const int cols = static_cast<int>(K / 16);
  const int nblk64 = static_cast<int>((K + 63) / 64);
  const int64_t total = rows * ((cols + 3) / 4);
  const int threads = 256;
  return launch_pdl(scales_to_rowmajor_kernel, dim3(static_cast<unsigned int>((total + threads - 1) / threads)),
                    dim3(threads), 0, s, in, out, rows, cols, nblk64);
}

namespace {
// Failure-path self test: a bounded wait on an mbarrier that nothing ever
// arrives on runs out and records the timeout like any library kernel.
__global__ void selftest_wait_kernel(long long budget) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, budget)) atomicOr(&g_vlaq_quant_status, kStatusTimeout);
}
}  // namespace

cudaError_t launch_selftest_wait_timeout(cudaStream_t s) {
  selftest_wait_kernel<<<1, 32, 0, s>>>(2000000LL);  // about 1 ms of SM clock
  return cudaGetLastError();
}

cudaError_t read_and_clear_quant_status(unsigned int* out, cudaStream_t s) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_vlaq_quant_status, sizeof(unsigned int), 0,
                                            cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return e;
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return e;
  const unsigned int zero = 0;
  e = cudaMemcpyToSymbolAsync(g_vlaq_quant_status, &zero, sizeof(unsigned int), 0, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return e;
  return cudaStreamSynchronize(s);
}

}  // namespace vlaq
