// Fused activation prologue and the offline weight quantizers.
//
// Persistent CTAs, several per SM, each keeping up to four rows in flight in
// a shared-memory ring: thread 0 fetches a whole bf16 row with one bulk copy
// (cp.async.bulk, completion on the slot's mbarrier) and the CTA quantizes
// the oldest staged row while the next ones stream in, so HBM sees a steady
// queue of large reads instead of one dependent load-reduce-store chain per
// row.  A staged row is read twice from shared memory:
//   pass A  (transform and) per-16 block amax, kept in registers; row amax
//           -> global scale g of the row;
//   pass B  transform again, E4M3 block scale, codes.
// Lane l of warp w owns the 16-element block 32 (W it + w) + l of the row (W
// warps per CTA): one NVFP4 scale byte and 8 code bytes, so four lanes hold
// one Hadamard block and one 4-byte word of the 128x4 tiled scale layout,
// and a warp writes 256 (NVFP4) or 512 (FP8) contiguous code bytes per step.
// HBM-bound: 2 bytes in and 0.5625 (NVFP4) or 1 (FP8) bytes out per element.
// Short rows (K <= 8192) run 8-warp CTAs, four per SM; long rows 16-warp
// CTAs, two per SM, so one row is spread over more lanes.
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

constexpr int kMaxRowBufs = 4;
constexpr int kMidRowK = 4096;    // many rows up to this length: 4-warp CTAs, 8 per SM
constexpr int kShortRowK = 8192;  // rows up to this length take the 8-warp CTAs

// CTA shape per row length: W warps, CTAs resident per SM, ring budget.
template <int W>
struct RowCfg {
  static constexpr int kThreads = 32 * W;
  static constexpr int kCtasPerSm = 1024 / kThreads;  // 32 warps per SM, 64 registers a thread
  static constexpr int kRingBytes = (W == 4) ? 26 * 1024 : (W == 8) ? 52 * 1024 : 110 * 1024;
  static constexpr int kMaxK = (W == 4) ? kMidRowK : (W == 8) ? kShortRowK : int(kMaxQuantK);
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
#pragma unroll
  for (int i = 0; i < N; i += 2) markstein_pair(v[i], v[i + 1], d.S, d.y, q[i], q[i + 1]);
  if (__any_sync(0xffffffffu, d.slow)) {
    if (d.slow) {
#pragma unroll
      for (int i = 0; i < N; ++i) q[i] = (d.S == 0.0f) ? 0.0f : __fdiv_rn(v[i], d.S);
    }
  }
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
  int nbuf;       // ring depth (rows in flight per CTA)
  int row_bytes;  // ring slot size (2 K rounded up to 128)
  long long budget;
};

// Normalised WHT of the 64-block spread over lanes 4 g .. 4 g + 3 (16 values
// each, element 16 (lane % 4) + j): stages h = 1, 2, 4, 8 inside the lane,
// h = 16, 32 across lanes (xor 1, 2), then x 1/8 (exact) -- the stages of the
// sequential butterfly in the same order.  Executed by the whole warp.
__device__ __forceinline__ void wht64_lanes(float* v, int lane) {
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if ((i & h) == 0) {
        const float a = v[i], b = v[i + h];
        v[i] = __fadd_rn(a, b);
        v[i + h] = __fsub_rn(a, b);
      }
    }
  }
#pragma unroll
  for (int x = 1; x < 4; x <<= 1) {
    const bool upper = (lane & x) != 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float p = __shfl_xor_sync(0xffffffffu, v[i], x);
      v[i] = upper ? __fsub_rn(p, v[i]) : __fadd_rn(v[i], p);
    }
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __fmul_rn(v[i], 0.125f);
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
// after the block-64 WHT.  Warp-uniform.
template <bool NORM, bool WHT, bool SMOOTH>
__device__ __forceinline__ void block_values(const RowArgs& a, const uint8_t* rs, int q, int nblk16, float r,
                                             int lane, float* v) {
  if (q < nblk16) {
    const uint4* src = reinterpret_cast<const uint4*>(rs) + 2 * q;
    unpack_bf16x8(src[0], v);
    unpack_bf16x8(src[1], v + 8);
    if (NORM) {
      const uint4* gsrc = reinterpret_cast<const uint4*>(a.gamma) + 2 * q;
      float gm[16];
      unpack_bf16x8(__ldg(gsrc), gm);
      unpack_bf16x8(__ldg(gsrc + 1), gm + 8);
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = __fmul_rn(__fmul_rn(v[j], r), gm[j]);
    }
    if (SMOOTH && !(a.sflags & kFlagSmoothAfter)) smooth_block(a, q, v);
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = 0.0f;
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

// All rows of one launch: FMT (NVFP4 / FP8), MODE (per-row scale, tensor
// amax pass, tensor quantize pass, static calibrated scale), NORM (RMSNorm,
// per-row and static modes), WHT (block-64 Hadamard), W warps per CTA.  Persistent grid: the CTA takes rows
// blockIdx.x + i gridDim.x, the ring slot of row i is i mod nbuf.
template <int FMT, int MODE, bool NORM, bool WHT, bool SMOOTH, int W>
__global__ void __launch_bounds__(RowCfg<W>::kThreads, RowCfg<W>::kCtasPerSm) quant_rows_kernel(const RowArgs a) {
  constexpr int T = RowCfg<W>::kThreads;
  constexpr int MAXIT = RowCfg<W>::kMaxK / 16 / T;  // blocks per lane, at most
  extern __shared__ __align__(128) uint8_t s_ring[];
  __shared__ __align__(8) uint64_t s_bar[kMaxRowBufs];
  __shared__ float s_red[W];
  __shared__ float s_r;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int K = a.K;
  const int nblk16 = K >> 4;
  const int nblk64 = (K + 63) >> 6;
  const int nblk16_pad = 4 * nblk64;  // blocks up to the padded row end
  const int iters = (nblk16_pad + T - 1) / T;
  const int nbuf = a.nbuf;
  const uint32_t row_tx = static_cast<uint32_t>(2 * K);
  const int64_t stride = gridDim.x;

  if (tid == 0) {
    for (int b = 0; b < nbuf; ++b) mbar_init(&s_bar[b], 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  griddep_wait();
  griddep_launch_dependents();

  if (tid == 0) {
    for (int b = 0; b < nbuf; ++b) {
      const int64_t row = blockIdx.x + b * stride;
      if (row >= a.rows) break;
      mbar_arrive_expect_tx(&s_bar[b], row_tx);
      bulk_load(s_ring + b * a.row_bytes, a.X + row * K, row_tx, &s_bar[b]);
    }
  }
  float g_tensor = 0.0f;
  if (MODE == kTensorQuant) g_tensor = __fdiv_rn(__uint_as_float(*a.amax_word), 2688.0f);
  if (MODE == kStatic) g_tensor = a.g_static;

  int slot = 0;
  uint32_t phase = 0;
  for (int64_t row = blockIdx.x; row < a.rows; row += stride) {
    const bool ok = __syncthreads_and(mbar_wait(&s_bar[slot], phase, a.budget));
    if (!ok) {
      // record it, let the copies still in flight land, and stop
      if (tid == 0) {
        atomicOr(&g_vlaq_quant_status, kStatusTimeout);
        for (int k = 0; k < nbuf && row + k * stride < a.rows; ++k) {
          const int sk = slot + k;
          mbar_wait(&s_bar[sk % nbuf], phase ^ (sk >= nbuf ? 1u : 0u), a.budget);
        }
      }
      break;
    }
    const uint8_t* rs = s_ring + slot * a.row_bytes;

    // ---- RMSNorm factor r = 1 / sqrt(mean(x^2) + eps), fixed 32-lane tree
    float r = 1.0f;
    if (NORM) {
      if (warp == 0) {
        // the chain of fused multiply-adds is fixed; the next chunk's load
        // is issued before the current chunk's eight steps
        const uint4* rs4 = reinterpret_cast<const uint4*>(rs);
        const int nch = K >> 3;
        float acc = 0.0f;
        uint4 cur = lane < nch ? rs4[lane] : make_uint4(0, 0, 0, 0);
        for (int c = lane; c < nch; c += 32) {
          const uint4 nxt = c + 32 < nch ? rs4[c + 32] : make_uint4(0, 0, 0, 0);
          float t[8];
          unpack_bf16x8(cur, t);
#pragma unroll
          for (int j = 0; j < 8; ++j) acc = __fmaf_rn(t[j], t[j], acc);
          cur = nxt;
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, o));
        if (lane == 0) {
          const float mean = __fdiv_rn(acc, static_cast<float>(K));
          s_r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(mean, a.eps)));
        }
      }
      __syncthreads();
      r = s_r;
    }

    // ---- pass A: per-block amax (kept in registers) and row amax
    float a16r[MAXIT];
    float g = g_tensor;
    if (MODE == kStatic && tid == 0) a.gout[row] = g;
    if (MODE == kPerRow || MODE == kTensorAmax) {
      float local = 0.0f;
#pragma unroll
      for (int it = 0; it < MAXIT; ++it) {
        a16r[it] = 0.0f;
        if (it < iters && (it * W + warp) * 32 < nblk16_pad) {
          const int q = (it * W + warp) * 32 + lane;
          float m = 0.0f;
          if (NORM || WHT || SMOOTH) {
            float v[16];
            block_values<NORM, WHT, SMOOTH>(a, rs, q, nblk16, r, lane, v);
            m = absmax16(v);
          } else if (q < nblk16) {
            const uint4* src = reinterpret_cast<const uint4*>(rs) + 2 * q;
            m = absmax_bf16x16(src[0], src[1]);
          }
          a16r[it] = m;
          local = fmaxf(local, m);
        }
      }
      // non-negative floats order like their bit patterns: one warp reduction
      local = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(local)));
      if (lane == 0) s_red[warp] = local;
      __syncthreads();
      float A = s_red[0];
#pragma unroll
      for (int w = 1; w < W; ++w) A = fmaxf(A, s_red[w]);
      if (MODE == kTensorAmax) {
        if (tid == 0) atomicMax(a.amax_word, __float_as_uint(A));  // A >= 0: bit order = value order
      } else {
        g = (FMT == kNvfp4) ? __fdiv_rn(A, 2688.0f) : __fdiv_rn(A, FMT == kFp8 ? 448.0f : 127.0f);
        if (tid == 0) a.gout[row] = g;
      }
    }

    // ---- pass B: block scales and codes
    if (MODE != kTensorAmax) {
      uint8_t* crow = a.codes + row * a.pitch;
      if (FMT == kNvfp4) {
        uint8_t* srow = a.scales + scale_row_base(row, nblk64);
        const Divisor d6g = make_divisor(__fmul_rn(6.0f, g));
#pragma unroll
        for (int it = 0; it < MAXIT; ++it) {
          if (it < iters && (it * W + warp) * 32 < nblk16_pad) {
            const int q = (it * W + warp) * 32 + lane;
            float v[16];
            block_values<NORM, WHT, SMOOTH>(a, rs, q, nblk16, r, lane, v);
            float a16 = (MODE == kPerRow) ? a16r[it] : absmax16(v);
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
        for (int it = 0; it < MAXIT; ++it) {
          if (it < iters && (it * W + warp) * 32 < nblk16_pad) {
            const int q = (it * W + warp) * 32 + lane;
            float v[16];
            block_values<NORM, WHT, SMOOTH>(a, rs, q, nblk16, r, lane, v);
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

    // ---- every thread is done with this slot: refill it with the row nbuf steps ahead
    __syncthreads();
    if (tid == 0) {
      const int64_t next = row + nbuf * stride;
      if (next < a.rows) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&s_bar[slot], row_tx);
        bulk_load(s_ring + slot * a.row_bytes, a.X + next * K, row_tx, &s_bar[slot]);
      }
    }
    if (++slot == nbuf) {
      slot = 0;
      phase ^= 1u;
    }
  }
}

__global__ void finalize_global_kernel(float* g) {
  griddep_wait();
  griddep_launch_dependents();
  g[0] = __fdiv_rn(__uint_as_float(*reinterpret_cast<unsigned int*>(g)), 2688.0f);
}

template <int FMT, int MODE, bool NORM, bool WHT, bool SMOOTH, int W>
cudaError_t launch_ring(RowArgs a, cudaStream_t s) {
  using C = RowCfg<W>;
  auto kern = quant_rows_kernel<FMT, MODE, NORM, WHT, SMOOTH, W>;
  const int fit = C::kRingBytes / a.row_bytes;
  a.nbuf = fit < 2 ? 2 : (fit > kMaxRowBufs ? kMaxRowBufs : fit);  // 2 x 64 KiB at the largest K
  const size_t smem = static_cast<size_t>(a.nbuf) * a.row_bytes;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  // resident CTAs per SM: the register limit, or fewer where the rings do
  // not fit (1 KiB per CTA is reserved by the SM)
  int per_sm = static_cast<int>(228 * 1024 / (smem + 2048));
  per_sm = per_sm < 1 ? 1 : (per_sm > C::kCtasPerSm ? C::kCtasPerSm : per_sm);
  const int64_t ctas = static_cast<int64_t>(device_sm_count()) * per_sm;
  const unsigned int grid = static_cast<unsigned int>(a.rows < ctas ? a.rows : ctas);
  return launch_pdl(kern, dim3(grid), dim3(C::kThreads), smem, s, a);
}

template <int FMT, int MODE, bool NORM, bool WHT, bool SMOOTH = false>
cudaError_t launch_shape(const RowArgs& a, cudaStream_t s) {
  // short rows and enough of them for every SM: one row per small CTA, so
  // more rows are worked on at once; few rows keep the 8-warp CTAs (shorter
  // per-row chains)
  if (a.K <= kMidRowK && a.rows >= 2 * device_sm_count()) return launch_ring<FMT, MODE, NORM, WHT, SMOOTH, 4>(a, s);
  if (a.K <= kShortRowK) return launch_ring<FMT, MODE, NORM, WHT, SMOOTH, 8>(a, s);
  return launch_ring<FMT, MODE, NORM, WHT, SMOOTH, 16>(a, s);
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
  a.nbuf = 0;
  a.row_bytes = static_cast<int>((2 * K + 127) / 128 * 128);
  a.budget = kWaitBudgetCycles;
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
