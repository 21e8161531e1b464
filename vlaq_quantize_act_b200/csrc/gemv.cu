// NVFP4 linear for one or two token rows against a small weight matrix: a
// weight-streaming kernel on the CUDA cores.
//
//   Y[m, n] = bf16_rne( g_x[m] g_w sum_b (sw[n, b] sx[m, b] / 4) D[m, n, b] + residual[m, n] )
//   D[m, n, b] = sum_{k in b} (2 e2m1(w[n, k])) (2 e2m1(x[m, k]))      (exact integers)
//
// At M <= 2 the projection moves 0.5625 weight bytes per multiply-add, so it
// is bound by HBM, and a 128-row tensor-core tile would be almost all
// padding.  For weights up to 2^25 elements (the q / k / v / o shapes) the
// fixed cost of the tensor-core kernel (one tile per SM, split-K partials)
// dominates and this kernel is faster; larger weights stream faster through
// the tensor-core kernel's TMA ring (measured), so the dispatcher keeps them
// there.  Twice an E2M1 value is an integer in [-12, 12], so every 16-block
// dot product is an exact integer sum: the weight codes are streamed with
// coalesced 16-byte loads into registers, expanded to bytes with a byte
// permute (magnitudes of the non-negative codes, then of the negative ones),
// and multiplied with the activation bytes four at a time (dp4a).  Only the
// per-block scaling and the sum over blocks are rounded (fp32).
//
// One warp owns one weight row at a time; lane l takes the 16-byte code
// chunks l, l + 32, ... (two chunks per step), and the loads of the next step
// -- also across rows -- are issued before the current step is computed.  The
// persistent grid strides over the rows; every CTA expands the activation
// rows once into shared memory (bytes plus per-block scales, laid out so
// that a warp's reads are consecutive).  The weight loads of a warp's first
// step are issued before the grid-dependency wait, so they overlap the kernel
// that produced the activations.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "ptx.cuh"

namespace vlaq {
namespace {

constexpr int kGemvWarps = 8;
constexpr int kGemvThreads = 32 * kGemvWarps;
constexpr int kGemvCtasPerSm = 4;
constexpr int kGemvUnroll = 2;  // 16-byte weight chunks per lane per step

// 2 |e2m1| for the magnitude index 0..7, one byte each (all below 0x80)
constexpr uint32_t kMagLo = 0x03020100u;  // 0, 1, 2, 3
constexpr uint32_t kMagHi = 0x0C080604u;  // 4, 6, 8, 12

struct GemvArgs {
  const uint8_t* xq;   // activation codes [M, pitch]
  const uint8_t* xs;   // activation block scales, 128x4 tiled
  const float* xg;     // g_x[M]
  const uint8_t* wq;   // weight codes [N, pitch]
  const uint8_t* ws;   // weight block scales, 128x4 tiled
  const float* wg;     // g_w[1]
  const __nv_bfloat16* residual;
  __nv_bfloat16* Y;
  int M, N;
  int pitch;           // bytes per code row = 32 nblk64
  int nblk64;          // 64-element groups per row
  int nchunk;          // 16-byte code chunks per row = pitch / 16
  int nchunk_pad;      // nchunk rounded up to 32
  int steps;           // steps per row = ceil(nchunk / (32 kGemvUnroll))
};

// Byte offset of (row, 16-block b) in the 128x4 tiled scale layout.
__device__ __forceinline__ int64_t tiled_scale_offset(int64_t row, int b, int nblk64) {
  return ((row >> 7) * nblk64 + (b >> 2)) * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4 + (b & 3);
}

// Byte i of the result = 2 |e2m1| of code nibble i of sel (nibbles 0..3) when
// that code is non-negative, 0 when it is negative (the selector's top bit
// asks for the sign of a table byte, and every table byte is positive).
__device__ __forceinline__ uint32_t mag4(uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(kMagLo), "r"(kMagHi), "r"(sel));
  return d;
}

// d += sum of the four products of unsigned bytes a and signed bytes b
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Eight codes (one word, low nibble first) -> non-negative and negative
// magnitudes, four bytes per word each.
struct Mags {
  uint32_t p[2], n[2];
};
__device__ __forceinline__ Mags expand8(uint32_t codes) {
  const uint32_t neg = codes ^ 0x88888888u;
  Mags r;
  r.p[0] = mag4(codes);
  r.p[1] = mag4(codes >> 16);
  r.n[0] = mag4(neg);
  r.n[1] = mag4(neg >> 16);
  return r;
}

// Shared-memory layout of the expanded activation rows: bytes 2 e2m1(x) as
// uint4 halves (half h of chunk c = block 2c + h), index
// m (2 nchunk_pad) + ((c / 32) 2 + h) 32 + c % 32, then one float2 per chunk
// holding sx / 4 of its two blocks, index m nchunk_pad + c.
__device__ __forceinline__ int xb_index(int m, int c, int h, int nchunk_pad) {
  return m * (2 * nchunk_pad) + ((c >> 5) * 2 + h) * 32 + (c & 31);
}

template <int M>
__global__ void __launch_bounds__(kGemvThreads, kGemvCtasPerSm) gemv_nvfp4_kernel(const GemvArgs a) {
  extern __shared__ __align__(16) uint4 s_xb[];
  const float2* s_xs = reinterpret_cast<const float2*>(s_xb + M * 2 * a.nchunk_pad);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row_stride = static_cast<int64_t>(gridDim.x) * kGemvWarps;

  uint4 wcur[kGemvUnroll], wnxt[kGemvUnroll];
  uint32_t scur[kGemvUnroll], snxt[kGemvUnroll];
  // chunks lane + 32 (U step + u) of row `row`; absent chunks read as zero
  auto load_step = [&](int64_t row, int step, uint4* wb, uint32_t* sb) {
    const uint8_t* wrow = a.wq + row * a.pitch;
    const uint8_t* srow = a.ws + tiled_scale_offset(row, 0, a.nblk64);
#pragma unroll
    for (int u = 0; u < kGemvUnroll; ++u) {
      const int c = lane + 32 * (kGemvUnroll * step + u);
      if (c < a.nchunk) {
        wb[u] = __ldg(reinterpret_cast<const uint4*>(wrow) + c);
        // blocks 2c, 2c + 1: bytes 2 (c % 2) and 2 (c % 2) + 1 of scale column c / 2
        sb[u] = __ldg(reinterpret_cast<const uint16_t*>(srow + (c >> 1) * 512 + 2 * (c & 1)));
      } else {
        wb[u] = make_uint4(0, 0, 0, 0);
        sb[u] = 0;
      }
    }
  };

  int64_t row = static_cast<int64_t>(blockIdx.x) * kGemvWarps + warp;
  int step = 0;
  if (row < a.N) load_step(row, 0, wcur, scur);

  griddep_wait();
  griddep_launch_dependents();

  // activation rows -> bytes 2 e2m1(x) and block scales / 4 (padding zero)
  for (int i = threadIdx.x; i < M * a.nchunk_pad * 2; i += kGemvThreads) {
    const int m = i / (a.nchunk_pad * 2);
    const int r = i - m * (a.nchunk_pad * 2);
    const int c = r >> 1, h = r & 1;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (c < a.nchunk) {
      const uint2 codes =
          *reinterpret_cast<const uint2*>(a.xq + static_cast<int64_t>(m) * a.pitch + 16 * c + 8 * h);
      const Mags lo = expand8(codes.x), hi = expand8(codes.y);
      v = make_uint4(__vsub4(lo.p[0], lo.n[0]), __vsub4(lo.p[1], lo.n[1]), __vsub4(hi.p[0], hi.n[0]),
                     __vsub4(hi.p[1], hi.n[1]));
    }
    s_xb[xb_index(m, c, h, a.nchunk_pad)] = v;
  }
  for (int i = threadIdx.x; i < M * a.nchunk_pad; i += kGemvThreads) {
    const int m = i / a.nchunk_pad;
    const int c = i - m * a.nchunk_pad;
    float2 sc = make_float2(0.0f, 0.0f);
    if (c < a.nchunk) {
      sc.x = 0.25f * e4m3_to_f32(a.xs[tiled_scale_offset(m, 2 * c, a.nblk64)]);
      sc.y = 0.25f * e4m3_to_f32(a.xs[tiled_scale_offset(m, 2 * c + 1, a.nblk64)]);
    }
    reinterpret_cast<float2*>(s_xb + M * 2 * a.nchunk_pad)[m * a.nchunk_pad + c] = sc;
  }
  __syncthreads();

  const float gw = a.wg[0];
  float acc[M];
#pragma unroll
  for (int m = 0; m < M; ++m) acc[m] = 0.0f;
  while (row < a.N) {
    // the next step (next row after the last one) is in flight while this one is computed
    int64_t nrow = row;
    int nstep = step + 1;
    if (nstep == a.steps) {
      nstep = 0;
      nrow += row_stride;
    }
    if (nrow < a.N) load_step(nrow, nstep, wnxt, snxt);
#pragma unroll
    for (int u = 0; u < kGemvUnroll; ++u) {
      const int c = lane + 32 * (kGemvUnroll * step + u);
      if (c < a.nchunk) {
        const uint32_t wv[4] = {wcur[u].x, wcur[u].y, wcur[u].z, wcur[u].w};
        Mags mg[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) mg[j] = expand8(wv[j]);
        const float sw0 = e4m3_to_f32(scur[u] & 0xFFu), sw1 = e4m3_to_f32((scur[u] >> 8) & 0xFFu);
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const uint4 x0 = s_xb[xb_index(m, c, 0, a.nchunk_pad)];
          const uint4 x1 = s_xb[xb_index(m, c, 1, a.nchunk_pad)];
          const float2 sx = s_xs[m * a.nchunk_pad + c];
          int p0 = dp4a_us(mg[0].p[0], x0.x, 0), n0 = dp4a_us(mg[0].n[0], x0.x, 0);
          p0 = dp4a_us(mg[0].p[1], x0.y, p0), n0 = dp4a_us(mg[0].n[1], x0.y, n0);
          p0 = dp4a_us(mg[1].p[0], x0.z, p0), n0 = dp4a_us(mg[1].n[0], x0.z, n0);
          p0 = dp4a_us(mg[1].p[1], x0.w, p0), n0 = dp4a_us(mg[1].n[1], x0.w, n0);
          int p1 = dp4a_us(mg[2].p[0], x1.x, 0), n1 = dp4a_us(mg[2].n[0], x1.x, 0);
          p1 = dp4a_us(mg[2].p[1], x1.y, p1), n1 = dp4a_us(mg[2].n[1], x1.y, n1);
          p1 = dp4a_us(mg[3].p[0], x1.z, p1), n1 = dp4a_us(mg[3].n[0], x1.z, n1);
          p1 = dp4a_us(mg[3].p[1], x1.w, p1), n1 = dp4a_us(mg[3].n[1], x1.w, n1);
          acc[m] = __fmaf_rn(static_cast<float>(p0 - n0), __fmul_rn(sw0, sx.x), acc[m]);
          acc[m] = __fmaf_rn(static_cast<float>(p1 - n1), __fmul_rn(sw1, sx.y), acc[m]);
        }
      }
    }
    if (nstep == 0) {
      // row done: add the lanes (fixed butterfly), scale, residual, store
#pragma unroll
      for (int m = 0; m < M; ++m) {
#pragma unroll
        for (int o = 16; o; o >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], o);
      }
      if (lane < M) {
        float v = acc[0];
#pragma unroll
        for (int m = 1; m < M; ++m)
          if (lane == m) v = acc[m];
        const int64_t o = static_cast<int64_t>(lane) * a.N + row;
        float y = v * (a.xg[lane] * gw);
        if (a.residual) y += __bfloat162float(a.residual[o]);
        a.Y[o] = __float2bfloat16_rn(y);
      }
#pragma unroll
      for (int m = 0; m < M; ++m) acc[m] = 0.0f;
    }
#pragma unroll
    for (int u = 0; u < kGemvUnroll; ++u) {
      wcur[u] = wnxt[u];
      scur[u] = snxt[u];
    }
    row = nrow;
    step = nstep;
  }
}

template <int M>
cudaError_t launch_gemv_m(const GemvArgs& a, size_t smem, int ctas, cudaStream_t s) {
  auto kern = gemv_nvfp4_kernel<M>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(kern, dim3(ctas), dim3(kGemvThreads), smem, s, a);
}

}  // namespace

size_t gemv_smem_bytes(int64_t M, int64_t K) {
  const int64_t nchunk = (K + 63) / 64 * 2;
  return static_cast<size_t>(M * ((nchunk + 31) / 32 * 32) * 40);  // 32 bytes + a float2 per chunk
}

bool gemv_supported(int64_t M, int64_t N, int64_t K) {
  return M >= 1 && M <= kGemvMaxM && N * K <= kGemvMaxWeights && gemv_smem_bytes(M, K) * 2 <= kGemvSmemBudget;
}

cudaError_t launch_gemv_nvfp4(const uint8_t* xq, const uint8_t* xs, const float* xg, const uint8_t* wq,
                              const uint8_t* ws, const float* wg, const void* residual, void* Y, int64_t M, int64_t N,
                              int64_t K, cudaStream_t s) {
  GemvArgs a;
  a.xq = xq;
  a.xs = xs;
  a.xg = xg;
  a.wq = wq;
  a.ws = ws;
  a.wg = wg;
  a.residual = static_cast<const __nv_bfloat16*>(residual);
  a.Y = static_cast<__nv_bfloat16*>(Y);
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.nblk64 = static_cast<int>((K + 63) / 64);
  a.pitch = 32 * a.nblk64;
  a.nchunk = a.pitch / 16;
  a.nchunk_pad = (a.nchunk + 31) / 32 * 32;
  a.steps = (a.nchunk + 32 * kGemvUnroll - 1) / (32 * kGemvUnroll);
  const size_t smem = gemv_smem_bytes(M, K);
  int per_sm = static_cast<int>(kGemvSmemBudget / smem);
  per_sm = per_sm > kGemvCtasPerSm ? kGemvCtasPerSm : per_sm;
  const int64_t rows_ctas = (N + kGemvWarps - 1) / kGemvWarps;
  const int64_t slots = static_cast<int64_t>(device_sm_count()) * per_sm;
  const int ctas = static_cast<int>(rows_ctas < slots ? rows_ctas : slots);
  static_assert(kGemvMaxM == 2, "instantiations below");
  return M == 1 ? launch_gemv_m<1>(a, smem, ctas, s) : launch_gemv_m<2>(a, smem, ctas, s);
}

}  // namespace vlaq
