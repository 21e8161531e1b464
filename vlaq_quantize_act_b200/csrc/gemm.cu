// Block-scaled FP4 (NVFP4), FP8 E4M3 and INT8 GEMM on the sm_100a tensor cores.
//
//   Y[m, n] = bf16_rne( acc[m, n] * scale(m, n) + residual[m, n] )
//   acc[m, n] = sum_b sx[m, b] sw[n, b] sum_{k in b} e2m1(x[m, k]) e2m1(w[n, k])   (NVFP4)
//             = sum_k e4m3(x[m, k]) e4m3(w[n, k])                                 (FP8)
//             = sum_k x[m, k] w[n, k], exact in s32                               (INT8)
//   scale = g_x[m] * g_w (NVFP4) or s_x[m] * s_w[n] (FP8, INT8)
// INT8 rounds each epilogue step once (fp32(acc), s_x s_w, product, residual
// add), so its output is exact: one value, whatever the split or order.
//
// Persistent, warp-specialised kernels, one CTA per SM, fed by TMA (2-D
// tiled loads of the packed codes with 128-byte swizzle) through a ring of
// shared-memory stages, accumulating in TMEM with tcgen05.mma issued from
// one thread:
//   gemm_fp4_sfw_kernel  NVFP4, 128 x 256 tiles, kind::mxf4nvf4 with block-16
//                        UE4M3 scale vectors that four warps write into TMEM;
//                        split-K (decode shapes) reduced in-kernel by the
//                        last split of each tile;
//   gemm_fp4_pair_kernel NVFP4, 256 x 256 tiles over the two CTAs of a
//                        cluster (paired MMA, cta_group::2): each SM streams
//                        half of the weight tile; prefill shapes;
//   gemm_fp8_kernel<BN, I8>  FP8 E4M3 (kind::f8f6f4, fp32 accumulators) or
//                        INT8 (kind::i8, s32), 128 x 256 or 128 x 128 tiles
//                        (double-buffered accumulator); split-K (decode
//                        shapes) reduced in-kernel by the last split;
//   gemm_fp8_pair_kernel<I8>  FP8 / INT8, 256 x 256 tiles over CTA pairs
//                        with two accumulators; prefill shapes.
// Epilogues: tcgen05.ld of the accumulator, scale, residual add, bf16 round,
// global stores.
//
// Every mbarrier wait is bounded (clock budget); a wait that runs out sets a
// shared abort flag and the device status word, the roles drain their own
// in-flight copies and MMAs, TMEM is freed and the kernel returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace vlaq {

__device__ unsigned int g_vlaq_status = 0;

namespace {

constexpr int kBM = 128;
constexpr int kTmemCols = 512;

// 8-bit kernel shape: tile 128 x BN, stages of K = 128 E4M3 (or INT8)
// elements.
template <int BN, bool I8 = false>
struct Fp8Cfg {
  static constexpr int A_BYTES = kBM * 128;
  static constexpr int B_BYTES = BN * 128;
  static constexpr int NRB = BN / 128;                  // 128-column halves of the tile
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (220 * 1024) / STAGE_BYTES > 8 ? 8 : (220 * 1024) / STAGE_BYTES;
  static constexpr int ACC_BUFS = (BN <= 128) ? 2 : 1;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024;
  // one epilogue warp per (TMEM sub-partition, 128-column half)
  static constexpr int EPI_WARPS = 4 * NRB;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static_assert(ACC_BUFS * BN <= kTmemCols, "TMEM budget");
  static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
  // instruction descriptor: kind::f8f6f4, E4M3 x E4M3, fp32 D (bits 4-5 =
  // 1), or kind::i8, signed x signed (bits 7-9, 10-12 = 1), s32 D (bits 4-5
  // = 2), no saturation; N = BN (bits 17-22, N / 8), M = 128 (bits 24-28, M / 16)
  static constexpr uint32_t IDESC = (I8 ? (2u << 4) | (1u << 7) | (1u << 10) : (1u << 4)) |
                                    (uint32_t(BN >> 3) << 17) | (uint32_t(kBM >> 4) << 24);
};

struct GemmArgs {
  const uint8_t* xs;            // activation tiled scales (NVFP4)
  const uint8_t* ws;            // weight tiled scales (NVFP4)
  const float* xg;              // g_x[M] or s_x[M]
  const float* wg;              // g_w[1] or s_w[N]
  const __nv_bfloat16* residual;
  __nv_bfloat16* Y;
  float* partial;               // [splits][M][N] when splits > 1
  int M, N, K;
  unsigned int* counters;       // per output tile: splits arrived (zero between calls)
  int k_steps;                  // MMA k-steps (64 fp4 or 32 fp8 elements each)
  int k_tiles;                  // stages of 4 k-steps
  int m_tiles, n_tiles, splits;
  int units;                    // m_tiles * n_tiles * splits
  int ka;                       // 512-byte scale atoms per 128-row block = ceil(K/64)
  int w_row_blocks;             // ceil(N/128)
  long long budget;             // cycles per bounded wait
};

struct Unit {
  int m, n, split, kt0, kt1;
};

__device__ __forceinline__ Unit decode_unit(const GemmArgs& a, int u) {
  Unit r;
  r.m = u % a.m_tiles;
  const int t = u / a.m_tiles;
  r.split = t % a.splits;
  r.n = t / a.splits;
  r.kt0 = static_cast<int>(static_cast<long long>(r.split) * a.k_tiles / a.splits);
  r.kt1 = static_cast<int>(static_cast<long long>(r.split + 1) * a.k_tiles / a.splits);
  return r;
}

__device__ __forceinline__ void raise_abort(volatile int* abort_flag) {
  *abort_flag = 1;
  atomicOr(&g_vlaq_status, kStatusTimeout);
}

// Bounded wait that also gives up as soon as another role aborted.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, long long budget,
                                              volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > budget) {
      raise_abort(abort_flag);
      return false;
    }
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Partial sums of one 32-column row segment (split-K): the accumulator bits
// as they are (fp32, or s32 for INT8).
__device__ __forceinline__ void store_partial(const GemmArgs& a, int split, int row, int col0,
                                              const uint32_t (&r)[32]) {
  float* dst = a.partial + (static_cast<size_t>(split) * a.M + row) * a.N + col0;
  if (col0 + 32 <= a.N) {
    if ((reinterpret_cast<uintptr_t>(dst) & 31u) == 0) {  // 32-byte stores need 32-byte alignment
#pragma unroll
      for (int j = 0; j < 4; ++j) st_global_v8(dst + 8 * j, r + 8 * j);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        reinterpret_cast<uint4*>(dst)[j] = make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
    }
  } else {
    uint32_t* dw = reinterpret_cast<uint32_t*>(dst);
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (col0 + j < a.N) dw[j] = r[j];
  }
}

// INT8 epilogue value before the residual: fp32(acc) * fp32(s_x s_w), each
// step rounded once (no contraction), the order the integer path defines.
__device__ __forceinline__ float int8_scaled(uint32_t acc_bits, float sx, float sw) {
  return __fmul_rn(__int2float_rn(static_cast<int>(acc_bits)), __fmul_rn(sx, sw));
}

// y + residual: one rounding for INT8 (exact output), free otherwise.
template <bool I8>
__device__ __forceinline__ float add_residual(float y, float r) {
  return I8 ? __fadd_rn(y, r) : y + r;
}

// Scaled, residual-added fp32 values of one 32-column row segment (row < M),
// in place: r holds the accumulator bits on entry and the values' fp32 bits
// on return (columns from N on are never stored).
template <bool FP4, bool I8 = false>
__device__ __forceinline__ void epilogue_values(const GemmArgs& a, int row, int col0, float rs, uint32_t (&r)[32]) {
  const bool full = col0 + 32 <= a.N;
  float* y = reinterpret_cast<float*>(r);
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    if constexpr (FP4) {
      y[j] = __uint_as_float(r[j]) * rs;  // rs = g_x[m] g_w (one global weight scale)
    } else {
      const float sw = (col0 + j < a.N) ? a.wg[col0 + j] : 0.0f;  // per-row weight scale
      y[j] = I8 ? int8_scaled(r[j], rs, sw) : __uint_as_float(r[j]) * (rs * sw);
    }
  }
  const size_t base = static_cast<size_t>(row) * a.N + col0;
  if (a.residual) {
    if (full) {
      const uint4* rp = reinterpret_cast<const uint4*>(a.residual + base);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 v = __ldg(rp + j);
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          y[8 * j + 2 * t] = add_residual<I8>(y[8 * j + 2 * t], __uint_as_float(wv[t] << 16));
          y[8 * j + 2 * t + 1] = add_residual<I8>(y[8 * j + 2 * t + 1], __uint_as_float(wv[t] & 0xFFFF0000u));
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col0 + j < a.N) y[j] = add_residual<I8>(y[j], __bfloat162float(a.residual[base + j]));
    }
  }
}

// Scale, residual add, bf16 round and store of one 32-column row segment
// (r is overwritten).
template <bool FP4, bool I8 = false>
__device__ __forceinline__ void store_output(const GemmArgs& a, int row, int col0, float rs, uint32_t (&r)[32]) {
  const bool full = col0 + 32 <= a.N;
  epilogue_values<FP4, I8>(a, row, col0, rs, r);
  const float* y = reinterpret_cast<const float*>(r);
  const size_t base = static_cast<size_t>(row) * a.N + col0;
  if (full) {
    // two 32-byte stores: each thread writes whole sectors of its row
    uint32_t pk[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) pk[j] = pack_bf16x2(y[2 * j], y[2 * j + 1]);
    __nv_bfloat16* yp = a.Y + base;
    if ((reinterpret_cast<uintptr_t>(yp) & 31u) == 0) {  // 32-byte stores need 32-byte alignment
      st_global_v8(yp, pk);
      st_global_v8(yp + 16, pk + 8);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        reinterpret_cast<uint4*>(yp)[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (col0 + j < a.N) a.Y[base + j] = __float2bfloat16_rn(y[j]);
  }
}

// Barrier `id` over the first `n` threads' warps that reach it (n a
// multiple of 32); id 0 is __syncthreads.
__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Last split of an 8-bit tile: the splits' partials summed in split order
// (INT8: exact s32 sums; FP8: fp32 from 0, absent splits of a batch read as
// -0, the exact identity of the addition), then the direct epilogue's
// steps: FP8 acc * (s_x[m] s_w[n]), INT8 fp32(acc) * fp32(s_x s_w) with each
// step rounded once, + residual, bf16.  Outputs in 4-column groups over
// `nthreads` threads, up to 16 splits' loads in flight per group.
template <bool I8>
__device__ __forceinline__ void splitk_finish_tile_8bit(const GemmArgs& a, int m_tile, int n_tile, int bn, int tid,
                                                        int nthreads) {
  constexpr int kLoads = 16;
  const int r0 = m_tile * kBM, c0 = n_tile * bn;
  const int rows = min(kBM, a.M - r0), cols = min(bn, a.N - c0);
  const int groups = cols >> 2;  // N % 8 == 0
  const size_t split_stride = static_cast<size_t>(a.M) * a.N;
  for (int item = tid; item < rows * groups; item += nthreads) {
    const int row = r0 + item / groups;
    const int col = c0 + 4 * (item % groups);
    const float* src = a.partial + static_cast<size_t>(row) * a.N + col;
    float y[4];
    if constexpr (I8) {
      int acc[4] = {0, 0, 0, 0};
      for (int sp = 0; sp < a.splits; sp += kLoads) {
        int4 v[kLoads];
#pragma unroll
        for (int t = 0; t < kLoads; ++t)
          v[t] = sp + t < a.splits ? __ldcg(reinterpret_cast<const int4*>(src + (sp + t) * split_stride))
                                   : make_int4(0, 0, 0, 0);
#pragma unroll
        for (int t = 0; t < kLoads; ++t) {
          acc[0] += v[t].x;
          acc[1] += v[t].y;
          acc[2] += v[t].z;
          acc[3] += v[t].w;
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) y[j] = int8_scaled(static_cast<uint32_t>(acc[j]), a.xg[row], a.wg[col + j]);
    } else {
      float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      const float4 nz = make_float4(-0.0f, -0.0f, -0.0f, -0.0f);
      for (int sp = 0; sp < a.splits; sp += kLoads) {
        float4 v[kLoads];
#pragma unroll
        for (int t = 0; t < kLoads; ++t)
          v[t] = sp + t < a.splits ? __ldcg(reinterpret_cast<const float4*>(src + (sp + t) * split_stride)) : nz;
#pragma unroll
        for (int t = 0; t < kLoads; ++t) {
          acc[0] += v[t].x;
          acc[1] += v[t].y;
          acc[2] += v[t].z;
          acc[3] += v[t].w;
        }
      }
      const float rs = a.xg[row];
#pragma unroll
      for (int j = 0; j < 4; ++j) y[j] = acc[j] * (rs * a.wg[col + j]);
    }
    const size_t o = static_cast<size_t>(row) * a.N + col;
    if (a.residual) {
      const uint2 rv = __ldg(reinterpret_cast<const uint2*>(a.residual + o));
      y[0] = add_residual<I8>(y[0], __uint_as_float(rv.x << 16));
      y[1] = add_residual<I8>(y[1], __uint_as_float(rv.x & 0xFFFF0000u));
      y[2] = add_residual<I8>(y[2], __uint_as_float(rv.y << 16));
      y[3] = add_residual<I8>(y[3], __uint_as_float(rv.y & 0xFFFF0000u));
    }
    *reinterpret_cast<uint2*>(a.Y + o) = make_uint2(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]));
  }
}

// 8-bit W8A8 GEMM, FP8 E4M3 (kind::f8f6f4, fp32 accumulators) or INT8
// (I8: kind::i8, exact s32 accumulators): 64 + 32 EPI_WARPS threads, warp 0
// TMA producer, warp 1 TMEM allocator and MMA issuer, the rest epilogue
// warps; the last split of a tile adds the split-K partials in-kernel.
template <int BN, bool I8>
__global__ void __launch_bounds__(Fp8Cfg<BN, I8>::THREADS, 1)
gemm_fp8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const GemmArgs args) {
  using C = Fp8Cfg<BN, I8>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[C::STAGES];
  __shared__ __align__(8) uint64_t empty_bar[C::STAGES];
  __shared__ __align__(8) uint64_t accf_bar[C::ACC_BUFS];
  __shared__ __align__(8) uint64_t acce_bar[C::ACC_BUFS];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t s_tmem_base;
  __shared__ volatile int s_abort;
  __shared__ int s_last;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < C::ACC_BUFS; ++i) {
      mbar_init(&accf_bar[i], 1);
      mbar_init(&acce_bar[i], C::EPI_WARPS);
    }
    mbar_init(&drain_bar, 1);
    s_abort = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem_base;
  // barrier setup, TMEM allocation and descriptor prefetch above overlap the
  // previous kernel's tail; global memory is touched only after this wait
  griddep_wait();
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_phase = 0;  // per-stage bitmask / last armed parity
      bool ok = true;
      for (int u = blockIdx.x; u < args.units && ok; u += gridDim.x) {
        const Unit w = decode_unit(args, u);
        for (int kt = w.kt0; kt < w.kt1; ++kt) {
          if (!wait_or_abort(&empty_bar[stage], phase ^ 1u, args.budget, &s_abort)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * C::STAGE_BYTES;
          uint8_t* sb = sa + C::A_BYTES;
          mbar_arrive_expect_tx(&full_bar[stage], C::A_BYTES + C::B_BYTES);
          armed |= 1u << stage;
          armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
          tma_load_2d(sa, &tmA, &full_bar[stage], kt * 128, w.m * kBM);
          tma_load_2d(sb, &tmB, &full_bar[stage], kt * 128, w.n * BN);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // drain: let every load this thread issued land before teardown
        for (int i = 0; i < C::STAGES; ++i)
          if (armed & (1u << i)) {
            const long long t0 = clock64();
            while (!mbar_try_wait(&full_bar[i], (armed_phase >> i) & 1u) &&
                   clock64() - t0 < args.budget) {
            }
          }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < args.units && ok; u += gridDim.x) {
        const Unit w = decode_unit(args, u);
        if (!wait_or_abort(&acce_bar[acc], acc_phase ^ 1u, args.budget, &s_abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc * BN);
        for (int kt = w.kt0; kt < w.kt1; ++kt) {
          if (!wait_or_abort(&full_bar[stage], phase, args.budget, &s_abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint8_t* sa = smem + stage * C::STAGE_BYTES;
          uint8_t* sb = sa + C::A_BYTES;
          const int steps = min(4, args.k_steps - 4 * kt);
          const uint32_t a0 = smem_u32(sa), b0 = smem_u32(sb);
          for (int j = 0; j < steps; ++j) {
            const uint64_t ad = sdesc_kmajor_sw128(a0 + 32 * j), bd = sdesc_kmajor_sw128(b0 + 32 * j);
            const uint32_t accum = (kt > w.kt0 || j > 0) ? 1u : 0u;
            if constexpr (I8)
              mma_i8(d_tmem, ad, bd, C::IDESC, accum);
            else
              mma_f8f6f4(d_tmem, ad, bd, C::IDESC, accum);
          }
          umma_commit(&empty_bar[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&accf_bar[acc]);
        if (++acc == C::ACC_BUFS) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // drain: every tcgen05 op issued by this thread completes before TMEM
      // is released
      umma_commit(&drain_bar);
      const long long t0 = clock64();
      while (!mbar_try_wait(&drain_bar, 0) && clock64() - t0 < 4 * args.budget + 1000000) {
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Warp e handles TMEM sub-partition (warp % 4) and columns
    // [128 h, 128 h + 128), h = e / 4.  It copies its 128 accumulator
    // columns to registers, hands the TMEM buffer back to the MMA issuer at
    // once, then scales, adds the residual and stores while the next tile's
    // MMAs run.
    const int e = warp - 2;
    const int q = warp & 3;
    const int h = e >> 2;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int u = blockIdx.x; u < args.units; u += gridDim.x) {
      const Unit w = decode_unit(args, u);
      if (!wait_or_abort(&accf_bar[acc], acc_phase, args.budget, &s_abort)) break;
      tc_fence_after();
      const int row = w.m * kBM + 32 * q + lane;
      const bool row_ok = row < args.M;
      const uint32_t tbase = tmem + (static_cast<uint32_t>(32 * q) << 16) +
                             static_cast<uint32_t>(acc * BN + 128 * h);
      __syncwarp();
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(tbase + 32 * c, r[c]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce_bar[acc]);
      if (++acc == C::ACC_BUFS) {
        acc = 0;
        acc_phase ^= 1u;
      }
      float rs = 0.0f;
      if (row_ok && args.splits == 1) rs = args.xg[row];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int col0 = w.n * BN + 128 * h + 32 * c;
        if (row_ok && col0 < args.N) {
          if (args.splits > 1)
            store_partial(args, w.split, row, col0, r[c]);
          else
            store_output<false, I8>(args, row, col0, rs, r[c]);
        }
      }
      if (args.splits > 1) {
        // Split-K: the split that arrives last at the tile's counter adds
        // the partials in split order and writes the output, then puts the
        // counter back to zero for the next call (as in the NVFP4 kernel).
        __threadfence();
        named_bar_sync(1, 32 * C::EPI_WARPS);
        if (e == 0 && lane == 0) {
          unsigned int* cnt = args.counters + (w.n * args.m_tiles + w.m);
          const unsigned int done = atomicAdd(cnt, 1u);
          s_last = (done == static_cast<unsigned int>(args.splits - 1));
          if (s_last) *cnt = 0u;
        }
        named_bar_sync(1, 32 * C::EPI_WARPS);
        if (s_last) {
          __threadfence();
          splitk_finish_tile_8bit<I8>(args, w.m, w.n, BN, e * 32 + lane, 32 * C::EPI_WARPS);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ----------------------------------------------------------------------------
// NVFP4 GEMM with dedicated scale-factor writers (prefill shapes, BN = 256).
//
// The block scales reach TMEM through registers (tcgen05.st) from four
// "scale writer" warps, one per TMEM sub-partition, into NSF rotating TMEM
// buffers, instead of tcgen05.cp issued by the MMA thread: the single MMA
// issuer then only waits, issues four MMAs per stage and commits.  Layout of
// one scale buffer is the one the block-scaled MMA reads (per k-step, 4
// columns of A scales and 8 of B scales; lane r0 + 32 q of column c holds
// the four block scales of row r0 + 32 c, replicated in every q).
//   warps 0-3   (warpgroup 0): TMA producer (warp 0), TMEM allocator + MMA
//               issuer (warp 1), warps 2-3 idle;
//   warps 4-11  (warpgroups 1, 2): epilogue, registers raised to 168;
//   warps 12-15 (warpgroup 3): scale writers, registers lowered to 48.
// The warpgroup register budgets add up to the launch allocation:
// 128 + 168 + 168 + 48 = 4 x 128 per thread (the build checks that ptxas
// allocates 128 registers at entry).
// Last split of a tile: output = bf16(sum of the splits' fp32 partials, in
// split order) * g_x[m] g_w + residual.  The tile's valid outputs are spread
// over `nthreads` threads in 4-column groups (a decode tile of one row still
// occupies 64 threads), and each thread issues the partial loads of up to
// kSplitLoads splits at once, so the reduction costs one L2 round trip per
// kSplitLoads splits.
constexpr int kSplitLoads = 16;
__device__ __forceinline__ void splitk_finish_tile(const GemmArgs& a, int m_tile, int n_tile, int bn, int tid,
                                                   int nthreads) {
  const int r0 = m_tile * kBM, c0 = n_tile * bn;
  const int rows = min(kBM, a.M - r0), cols = min(bn, a.N - c0);
  const int groups = cols >> 2;  // N % 8 == 0
  const size_t split_stride = static_cast<size_t>(a.M) * a.N;
  for (int item = tid; item < rows * groups; item += nthreads) {
    const int row = r0 + item / groups;
    const int col = c0 + 4 * (item % groups);
    const float* src = a.partial + static_cast<size_t>(row) * a.N + col;
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    // absent splits of the last batch read as -0, the exact identity of
    // the addition: the sums equal the plain split-order sums bit for bit
    const float4 nz = make_float4(-0.0f, -0.0f, -0.0f, -0.0f);
    for (int sp = 0; sp < a.splits; sp += kSplitLoads) {
      float4 v[kSplitLoads];
#pragma unroll
      for (int t = 0; t < kSplitLoads; ++t)
        v[t] = sp + t < a.splits ? __ldcg(reinterpret_cast<const float4*>(src + (sp + t) * split_stride)) : nz;
#pragma unroll
      for (int t = 0; t < kSplitLoads; ++t) {
        acc[0] += v[t].x;
        acc[1] += v[t].y;
        acc[2] += v[t].z;
        acc[3] += v[t].w;
      }
    }
    const float rs = a.xg[row] * a.wg[0];
    float y[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) y[j] = acc[j] * rs;
    const size_t o = static_cast<size_t>(row) * a.N + col;
    if (a.residual) {
      const uint2 rv = __ldg(reinterpret_cast<const uint2*>(a.residual + o));
      y[0] += __uint_as_float(rv.x << 16);
      y[1] += __uint_as_float(rv.x & 0xFFFF0000u);
      y[2] += __uint_as_float(rv.y << 16);
      y[3] += __uint_as_float(rv.y & 0xFFFF0000u);
    }
    *reinterpret_cast<uint2*>(a.Y + o) = make_uint2(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]));
  }
}

// Barrier over the eight epilogue warps (warps 4-11) of the scale-writer
// kernel; id 0 is __syncthreads.
__device__ __forceinline__ void epilogue_bar_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

struct SfwCfg {
  static constexpr int BN = 256;
  static constexpr int NRB = 2;
  static constexpr int A_BYTES = kBM * 128;
  static constexpr int B_BYTES = BN * 128;
  static constexpr int SFA_BYTES = 4 * 512;
  static constexpr int SFB_BYTES = NRB * 4 * 512;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // operand tiles of one stage
  static constexpr int STAGES = 4;
  static constexpr int SF_STAGE_BYTES = SFA_BYTES + SFB_BYTES;  // scale atoms of one stage
  static constexpr int SF_STAGES = 4;
  static constexpr int NSF = 4;                       // TMEM scale buffers
  static constexpr int SF_COLS = 16 + 16 * NRB;        // per buffer: 16 (A) + 32 (B)
  static constexpr int SF_COL0 = BN;                   // after the accumulator
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + SF_STAGES * SF_STAGE_BYTES + 1024;
  static constexpr int THREADS = 512;
  static constexpr int EPI_WARPS = 8;
  static constexpr uint32_t IDESC =
      (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) | (uint32_t(kBM >> 4) << 24);
  static_assert(SF_COL0 + NSF * SF_COLS <= kTmemCols, "TMEM budget");
  static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

__global__ void __launch_bounds__(SfwCfg::THREADS, 1)
gemm_fp4_sfw_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const GemmArgs args) {
  using C = SfwCfg;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[C::STAGES];
  __shared__ __align__(8) uint64_t empty_bar[C::STAGES];
  __shared__ __align__(8) uint64_t sff_bar[C::NSF];
  __shared__ __align__(8) uint64_t sfe_bar[C::NSF];
  __shared__ __align__(8) uint64_t sfsf_bar[C::SF_STAGES];  // scale atoms landed
  __shared__ __align__(8) uint64_t sfse_bar[C::SF_STAGES];  // scale atoms copied to TMEM
  __shared__ __align__(8) uint64_t accf_bar;
  __shared__ __align__(8) uint64_t acce_bar;
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t s_tmem_base;
  __shared__ volatile int s_abort;
  __shared__ int s_last;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int wg = warp >> 2;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < C::NSF; ++i) {
      mbar_init(&sff_bar[i], 4);
      mbar_init(&sfe_bar[i], 1);
    }
    for (int i = 0; i < C::SF_STAGES; ++i) {
      mbar_init(&sfsf_bar[i], 1);
      mbar_init(&sfse_bar[i], 4);
    }
    mbar_init(&accf_bar, 1);
    mbar_init(&acce_bar, C::EPI_WARPS);
    mbar_init(&drain_bar, 1);
    s_abort = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem_base;

  // Two producers, two rings.  Operand tiles (warp 0): the weight half (B)
  // and the activation half (A) of a stage complete on its full barrier.
  // Scale atoms (warp 2): the weight scales (SFB) and activation scales
  // (SFA) of a stage land in a ring of their own, which the scale writers
  // release as soon as the atoms are in TMEM, so the scale factors of the
  // next stages are in place before their operand tiles land.
  uint8_t* sf_ring = smem + C::STAGES * C::STAGE_BYTES;
  auto stage_steps = [&](int kt) { return min(4, args.k_steps - 4 * kt); };
  auto sf_bytes = [&](const Unit& w, int kt) -> uint32_t {
    const int nrb = min(C::NRB, args.w_row_blocks - w.n * C::NRB);
    return static_cast<uint32_t>(stage_steps(kt) * 512 * (1 + nrb));
  };
  auto issue_weights = [&](int stage, const Unit& w, int kt) {
    tma_load_2d(smem + stage * C::STAGE_BYTES + C::A_BYTES, &tmB, &full_bar[stage], kt * 128, w.n * C::BN);
  };
  auto issue_acts = [&](int stage, const Unit& w, int kt) {
    tma_load_2d(smem + stage * C::STAGE_BYTES, &tmA, &full_bar[stage], kt * 128, w.m * kBM);
  };
  auto issue_weight_scales = [&](int slot, const Unit& w, int kt) {
    uint8_t* ssfb = sf_ring + slot * C::SF_STAGE_BYTES + C::SFA_BYTES;
    const int nrb = min(C::NRB, args.w_row_blocks - w.n * C::NRB);
    for (int rb = 0; rb < nrb; ++rb)
      bulk_load(ssfb + rb * 2048, args.ws + (static_cast<size_t>(w.n * C::NRB + rb) * args.ka + 4 * kt) * 512,
                stage_steps(kt) * 512, &sfsf_bar[slot]);
  };
  auto issue_act_scales = [&](int slot, const Unit& w, int kt) {
    bulk_load(sf_ring + slot * C::SF_STAGE_BYTES, args.xs + (static_cast<size_t>(w.m) * args.ka + 4 * kt) * 512,
              stage_steps(kt) * 512, &sfsf_bar[slot]);
  };

  // Weights do not depend on the previous kernel on the stream (every
  // library kernel triggers its dependents only after its own dependency
  // wait, so all kernels two or more launches back, the weight quantizer
  // among them, have completed): the first stages' weight tiles and weight
  // scales stream in while the previous kernel (the activation quantizer)
  // still runs.
  int pre = 0, sf_pre = 0;
  uint32_t armed = 0, sf_armed = 0;
  if (warp == 0 && lane == 0) {
    for (int u = blockIdx.x; u < args.units && pre < C::STAGES; u += gridDim.x) {
      const Unit w = decode_unit(args, u);
      for (int kt = w.kt0; kt < w.kt1 && pre < C::STAGES; ++kt, ++pre) {
        mbar_arrive_expect_tx(&full_bar[pre], C::A_BYTES + C::B_BYTES);
        armed |= 1u << pre;
        issue_weights(pre, w, kt);
      }
    }
  }
  if (warp == 2 && lane == 0) {
    for (int u = blockIdx.x; u < args.units && sf_pre < C::SF_STAGES; u += gridDim.x) {
      const Unit w = decode_unit(args, u);
      for (int kt = w.kt0; kt < w.kt1 && sf_pre < C::SF_STAGES; ++kt, ++sf_pre) {
        mbar_arrive_expect_tx(&sfsf_bar[sf_pre], sf_bytes(w, kt));
        sf_armed |= 1u << sf_pre;
        issue_weight_scales(sf_pre, w, kt);
      }
    }
  }
  griddep_wait();
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed_phase = 0;
      int it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < args.units && ok; u += gridDim.x) {
        const Unit w = decode_unit(args, u);
        for (int kt = w.kt0; kt < w.kt1; ++kt, ++it) {
          if (it >= pre) {
            if (!wait_or_abort(&empty_bar[stage], phase ^ 1u, args.budget, &s_abort)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full_bar[stage], C::A_BYTES + C::B_BYTES);
            armed |= 1u << stage;
            armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
            issue_weights(stage, w, kt);
          }
          issue_acts(stage, w, kt);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        for (int i = 0; i < C::STAGES; ++i)
          if (armed & (1u << i)) {
            const long long t0 = clock64();
            while (!mbar_try_wait(&full_bar[i], (armed_phase >> i) & 1u) && clock64() - t0 < args.budget) {
            }
          }
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------ scale-atom producer
    if (lane == 0) {
      int slot = 0;
      uint32_t phase = 0;
      uint32_t armed_phase = 0;
      int it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < args.units && ok; u += gridDim.x) {
        const Unit w = decode_unit(args, u);
        for (int kt = w.kt0; kt < w.kt1; ++kt, ++it) {
          if (it >= sf_pre) {
            if (!wait_or_abort(&sfse_bar[slot], phase ^ 1u, args.budget, &s_abort)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&sfsf_bar[slot], sf_bytes(w, kt));
            sf_armed |= 1u << slot;
            armed_phase = (armed_phase & ~(1u << slot)) | (phase << slot);
            issue_weight_scales(slot, w, kt);
          }
          issue_act_scales(slot, w, kt);
          if (++slot == C::SF_STAGES) {
            slot = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        for (int i = 0; i < C::SF_STAGES; ++i)
          if (sf_armed & (1u << i)) {
            const long long t0 = clock64();
            while (!mbar_try_wait(&sfsf_bar[i], (armed_phase >> i) & 1u) && clock64() - t0 < args.budget) {
            }
          }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int sfb = 0;
      uint32_t sf_phase = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < args.units && ok; u += gridDim.x) {
        const Unit w = decode_unit(args, u);
        if (!wait_or_abort(&acce_bar, acc_phase ^ 1u, args.budget, &s_abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kt = w.kt0; kt < w.kt1; ++kt) {
          if (!wait_or_abort(&full_bar[stage], phase, args.budget, &s_abort) ||
              !wait_or_abort(&sff_bar[sfb], sf_phase, args.budget, &s_abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint8_t* sa = smem + stage * C::STAGE_BYTES;
          const uint32_t a0 = smem_u32(sa), b0 = smem_u32(sa + C::A_BYTES);
          const uint32_t sf = tmem + C::SF_COL0 + sfb * C::SF_COLS;
          const int steps = min(4, args.k_steps - 4 * kt);
          for (int j = 0; j < steps; ++j)
            mma_mxf4nvf4(tmem, sdesc_kmajor_sw128(a0 + 32 * j), sdesc_kmajor_sw128(b0 + 32 * j), C::IDESC,
                         sf + 4 * j, sf + 16 + 8 * j, (kt > w.kt0 || j > 0) ? 1u : 0u);
          umma_commit(&empty_bar[stage]);
          umma_commit(&sfe_bar[sfb]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
          if (++sfb == C::NSF) {
            sfb = 0;
            sf_phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&accf_bar);
        acc_phase ^= 1u;
      }
      umma_commit(&drain_bar);
      const long long t0 = clock64();
      while (!mbar_try_wait(&drain_bar, 0) && clock64() - t0 < 4 * args.budget + 1000000) {
      }
    }
  } else if (wg == 3) {
    // ------------------------------------------------------ scale writers
    regs_dec<48>();
    const int q = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    int slot = 0;
    uint32_t phase = 0;
    int sfb = 0;
    uint32_t sf_phase = 0;
    for (int u = blockIdx.x; u < args.units; u += gridDim.x) {
      const Unit w = decode_unit(args, u);
      bool ok = true;
      for (int kt = w.kt0; kt < w.kt1; ++kt) {
        if (!wait_or_abort(&sfsf_bar[slot], phase, args.budget, &s_abort) ||
            !wait_or_abort(&sfe_bar[sfb], sf_phase ^ 1u, args.budget, &s_abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ssfa = smem_u32(sf_ring + slot * C::SF_STAGE_BYTES);
        const uint32_t ssfb = ssfa + C::SFA_BYTES;
        const uint32_t dst = tmem + lane_base + C::SF_COL0 + sfb * C::SF_COLS;
        const int steps = min(4, args.k_steps - 4 * kt);
        for (int j = 0; j < steps; ++j) {
          tmem_st_32x32b_x4(dst + 4 * j, ld_shared_v4(ssfa + 512 * j + 16 * lane));
#pragma unroll
          for (int rb = 0; rb < C::NRB; ++rb)
            tmem_st_32x32b_x4(dst + 16 + 8 * j + 4 * rb, ld_shared_v4(ssfb + rb * 2048 + 512 * j + 16 * lane));
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sff_bar[sfb]);
          mbar_arrive(&sfse_bar[slot]);  // the atoms are in TMEM: the slot may be refilled
        }
        if (++slot == C::SF_STAGES) {
          slot = 0;
          phase ^= 1u;
        }
        if (++sfb == C::NSF) {
          sfb = 0;
          sf_phase ^= 1u;
        }
      }
      if (!ok) break;
    }
    tmem_st_wait();
  } else if (wg == 1 || wg == 2) {
    // ------------------------------------------------------------ epilogue
    regs_inc<168>();
    const int e = warp - 4;
    const int q = warp & 3;
    const int h = e >> 2;
    uint32_t acc_phase = 0;
    for (int u = blockIdx.x; u < args.units; u += gridDim.x) {
      const Unit w = decode_unit(args, u);
      if (!wait_or_abort(&accf_bar, acc_phase, args.budget, &s_abort)) break;
      tc_fence_after();
      const int row = w.m * kBM + 32 * q + lane;
      const bool row_ok = row < args.M;
      const uint32_t tbase = tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(128 * h);
      __syncwarp();
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(tbase + 32 * c, r[c]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce_bar);
      acc_phase ^= 1u;
      const float rs = row_ok ? args.xg[row] * args.wg[0] : 0.0f;
      if (args.splits == 1) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int col0 = w.n * C::BN + 128 * h + 32 * c;
          if (row_ok && col0 < args.N) store_output<true>(args, row, col0, rs, r[c]);
        }
        continue;
      }
      // Split-K: store this split's fp32 partial sums; the split that
      // arrives last at the tile's counter adds all partials in split order
      // and writes the output (deterministic, no second kernel), and puts
      // the counter back to zero for the next call.  Nothing clears the
      // counters between calls: the next GEMM on the stream reaches its
      // epilogue only after this grid has completed (every library kernel
      // triggers its dependents after its own dependency wait).
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int col0 = w.n * C::BN + 128 * h + 32 * c;
        if (row_ok && col0 < args.N) store_partial(args, w.split, row, col0, r[c]);
      }
      __threadfence();
      epilogue_bar_sync();
      if (e == 0 && lane == 0) {
        unsigned int* cnt = args.counters + (w.n * args.m_tiles + w.m);
        const unsigned int done = atomicAdd(cnt, 1u);
        s_last = (done == static_cast<unsigned int>(args.splits - 1));
        if (s_last) *cnt = 0u;  // every split of this call has arrived
      }
      epilogue_bar_sync();
      if (s_last) {
        __threadfence();
        splitk_finish_tile(args, w.m, w.n, C::BN, e * 32 + lane, 256);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// NVFP4 GEMM over CTA pairs: 256 x 256 tiles computed by the paired MMA
// (tcgen05.mma.cta_group::2) across the two CTAs of a cluster.  CTA r of the
// pair loads rows [128 r, 128 r + 128) of the A tile and of the B tile, so
// each SM streams half of the weight tile: 256 operand rows per 128 x 256
// outputs instead of 384 on one SM.  Each CTA writes the scale factors of
// its own 128 A rows and of all 256 B rows into its own TMEM (the layout
// of the single-CTA kernel), reads its own 128 accumulator rows and stores
// them through shared memory with TMA tile stores.  The leader (even CTA)
// issues the MMAs.  The issuing thread waits once and commits once per stage
// (an MMA issue returns only about when the tensor core takes it, so every
// barrier operation of that thread is idle tensor-core time): the leader's
// full barrier of a stage completes on the operand bytes of both CTAs and
// the arrivals of both CTAs' scale writers, and one commit to the stage's
// empty barrier in both CTAs frees the operand stage and the stage's TMEM
// scale buffer.  Direct epilogue only (used when the output tiles already
// fill the GPU).
// CH: 128-byte K-chunks per stage.  CH = 2 (K = 512 per stage) loads each
// row's two chunks with one 3-D TMA box; the TMA engine moves about twice
// the bytes per load instruction, and the MMA thread's one wait and one
// commit cover eight MMAs.  It needs rows of whole chunks (K % 256 == 0);
// other K run CH = 1 with 2-D boxes.  CH = 1 stages the output for TMA
// stores; CH = 2 has no shared memory left for that and stores rows directly.
template <int CH>
struct PairCfg {
  static constexpr int BM = 256;                 // tile rows over the pair
  static constexpr int BN = 256;
  static constexpr int CHUNK_BYTES = 128 * 128;  // one K-chunk of this CTA's 128 rows
  static constexpr int A_BYTES = CH * CHUNK_BYTES;
  static constexpr int B_BYTES = CH * CHUNK_BYTES;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STEPS = 4 * CH;           // MMAs (K = 64) per stage
  static constexpr int STAGES = CH == 1 ? 5 : 3;
  static constexpr int SFA_BYTES = STEPS * 512;
  static constexpr int SFB_ROW_BYTES = STEPS * 512;  // one 128-row block of the B tile
  static constexpr int SFB_BYTES = 2 * SFB_ROW_BYTES;
  static constexpr int SF_STAGE_BYTES = SFA_BYTES + SFB_BYTES;
  static constexpr int SF_STAGES = CH == 1 ? 4 : 2;
  static constexpr int NSF = CH == 1 ? 4 : 2;   // TMEM scale buffers (fewer than STAGES)
  static constexpr int SFB_COL = 4 * STEPS;      // B scale columns after the A ones
  static constexpr int SF_COLS = 12 * STEPS;     // per buffer: 4 (A) + 8 (B) per MMA
  static constexpr int SF_COL0 = BN;             // after the accumulator
  static constexpr int EPI_WARPS = 8;
  static constexpr bool TMA_STORE = CH == 1;
  static constexpr int OUT_BOX_COLS = 64;        // output store box: 32 rows x 64 bf16 (128-byte rows)
  static constexpr int OUT_BYTES = 32 * OUT_BOX_COLS * 2;  // one box per epilogue warp
  static constexpr int OUT_OFFSET = STAGES * STAGE_BYTES + SF_STAGES * SF_STAGE_BYTES;
  static constexpr int SMEM_BYTES = OUT_OFFSET + (TMA_STORE ? EPI_WARPS * OUT_BYTES : 0) + 1024;
  static constexpr int THREADS = 512;
  static constexpr uint32_t IDESC =
      (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);
  static_assert(OUT_OFFSET % 1024 == 0 && OUT_BYTES % 1024 == 0, "128-byte swizzle atoms of the output boxes");
  static_assert(SF_COL0 + NSF * SF_COLS <= kTmemCols, "TMEM budget");
  // a scale buffer is rewritten for stage i once stage i - NSF is consumed;
  // with NSF < STAGES that empty phase cannot be overtaken before it is
  // waited on, and the writers' arrival for stage i lands in stage i's phase
  static_assert(NSF < STAGES, "scale buffers recycle on the operand stages' empty barriers");
  static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

// Bounded wait for the pair kernel: gives up when either CTA of the pair
// aborted, and on running out raises the abort flag of both.
__device__ __forceinline__ bool pair_wait(uint64_t* bar, uint32_t parity, long long budget, volatile int* abort_flag,
                                          uint32_t peer_abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > budget) {
      raise_abort(abort_flag);
      st_shared_cluster_u32(peer_abort, 1u);
      return false;
    }
  }
}

template <int CH>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg<CH>::THREADS, 1)
gemm_fp4_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmY, const GemmArgs args) {
  using C = PairCfg<CH>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[C::STAGES];     // leader: operands and scale factors of both CTAs
  __shared__ __align__(8) uint64_t empty_bar[C::STAGES];    // stage consumed (leader's commit)
  __shared__ __align__(8) uint64_t sfsf_bar[C::SF_STAGES];  // scale atoms landed
  __shared__ __align__(8) uint64_t sfse_bar[C::SF_STAGES];  // scale atoms copied to TMEM
  __shared__ __align__(8) uint64_t accf_bar;                // accumulator complete (leader's commit)
  __shared__ __align__(8) uint64_t acce_bar;                // leader: both CTAs' accumulators read
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t s_tmem_base;
  __shared__ volatile int s_abort;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int wg = warp >> 2;
  const uint32_t rank = cluster_ctarank();
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int pairs = static_cast<int>(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full_bar[i], 1 + 8);  // the leader's producer + four scale writers per CTA
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < C::SF_STAGES; ++i) {
      mbar_init(&sfsf_bar[i], 1);
      mbar_init(&sfse_bar[i], 4);
    }
    mbar_init(&accf_bar, 1);
    mbar_init(&acce_bar, 2 * C::EPI_WARPS);
    mbar_init(&drain_bar, 1);
    s_abort = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    prefetch_tensormap(&tmY);
  }
  if (warp == 1) {
    tmem_alloc_pair(&s_tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync();  // both CTAs' barriers are initialised before either CTA signals the other's
  tc_fence_after();
  const uint32_t tmem = s_tmem_base;
  const uint32_t peer_abort = mapa_shared(smem_u32(const_cast<int*>(&s_abort)), rank ^ 1u);
  auto leader_bar = [&](uint64_t* bar) { return mapa_shared(smem_u32(bar), 0u); };

  uint8_t* sf_ring = smem + C::STAGES * C::STAGE_BYTES;
  const int x_row_blocks = (args.M + 127) / 128;
  auto stage_steps = [&](int kt) { return min(C::STEPS, args.k_steps - C::STEPS * kt); };
  auto own_a_block = [&](const Unit& w) { return 2 * w.m + static_cast<int>(rank); };
  auto sf_bytes = [&](const Unit& w, int kt) -> uint32_t {
    const int nrb = min(2, args.w_row_blocks - 2 * w.n);
    const int has_a = own_a_block(w) < x_row_blocks ? 1 : 0;
    return static_cast<uint32_t>(stage_steps(kt) * 512 * (has_a + nrb));
  };
  auto load = [&](uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int kt, int row) {
    if constexpr (CH == 1)
      tma_load_2d_pair(dst, map, leader_bar(bar), kt * 128, row);
    else
      tma_load_3d_pair(dst, map, leader_bar(bar), 0, row, kt * CH);
  };
  auto issue_weights = [&](int stage, const Unit& w, int kt) {
    load(smem + stage * C::STAGE_BYTES + C::A_BYTES, &tmB, &full_bar[stage], kt,
         w.n * C::BN + 128 * static_cast<int>(rank));
  };
  auto issue_acts = [&](int stage, const Unit& w, int kt) {
    load(smem + stage * C::STAGE_BYTES, &tmA, &full_bar[stage], kt, w.m * C::BM + 128 * static_cast<int>(rank));
  };
  auto issue_weight_scales = [&](int slot, const Unit& w, int kt) {
    uint8_t* ssfb = sf_ring + slot * C::SF_STAGE_BYTES + C::SFA_BYTES;
    const int nrb = min(2, args.w_row_blocks - 2 * w.n);
    for (int rb = 0; rb < nrb; ++rb)
      bulk_load(ssfb + rb * C::SFB_ROW_BYTES,
                args.ws + (static_cast<size_t>(2 * w.n + rb) * args.ka + C::STEPS * kt) * 512, stage_steps(kt) * 512,
                &sfsf_bar[slot]);
  };
  auto issue_act_scales = [&](int slot, const Unit& w, int kt) {
    const int ab = own_a_block(w);
    if (ab < x_row_blocks)
      bulk_load(sf_ring + slot * C::SF_STAGE_BYTES,
                args.xs + (static_cast<size_t>(ab) * args.ka + C::STEPS * kt) * 512, stage_steps(kt) * 512,
                &sfsf_bar[slot]);
  };

  // Weights (and their scale atoms) do not depend on the previous kernel on
  // the stream: the first stages stream in before the dependency wait.
  int pre = 0, sf_pre = 0;
  uint32_t armed = 0, sf_armed = 0;
  if (warp == 0 && lane == 0) {
    for (int u = pair; u < args.units && pre < C::STAGES; u += pairs) {
      const Unit w = decode_unit(args, u);
      for (int kt = w.kt0; kt < w.kt1 && pre < C::STAGES; ++kt, ++pre) {
        if (rank == 0) mbar_arrive_expect_tx(&full_bar[pre], 2 * C::STAGE_BYTES);
        armed |= 1u << pre;
        issue_weights(pre, w, kt);
      }
    }
  }
  if (warp == 2 && lane == 0) {
    for (int u = pair; u < args.units && sf_pre < C::SF_STAGES; u += pairs) {
      const Unit w = decode_unit(args, u);
      for (int kt = w.kt0; kt < w.kt1 && sf_pre < C::SF_STAGES; ++kt, ++sf_pre) {
        mbar_arrive_expect_tx(&sfsf_bar[sf_pre], sf_bytes(w, kt));
        sf_armed |= 1u << sf_pre;
        issue_weight_scales(sf_pre, w, kt);
      }
    }
  }
  griddep_wait();
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------- operand producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed_phase = 0;
      int it = 0;
      bool ok = true;
      for (int u = pair; u < args.units && ok; u += pairs) {
        const Unit w = decode_unit(args, u);
        for (int kt = w.kt0; kt < w.kt1; ++kt, ++it) {
          if (it >= pre) {
            if (!pair_wait(&empty_bar[stage], phase ^ 1u, args.budget, &s_abort, peer_abort)) {
              ok = false;
              break;
            }
            if (rank == 0) mbar_arrive_expect_tx(&full_bar[stage], 2 * C::STAGE_BYTES);
            armed |= 1u << stage;
            armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
            issue_weights(stage, w, kt);
          }
          issue_acts(stage, w, kt);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (ok) {
        // every stage released: the leader's last commits to this CTA have landed
        for (int i = 0; i < C::STAGES && ok; ++i) {
          ok = pair_wait(&empty_bar[stage], phase ^ 1u, args.budget, &s_abort, peer_abort);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      } else if (rank == 0) {
        for (int i = 0; i < C::STAGES; ++i)
          if (armed & (1u << i)) {
            const long long t0 = clock64();
            while (!mbar_try_wait(&full_bar[i], (armed_phase >> i) & 1u) && clock64() - t0 < args.budget) {
            }
          }
      } else {
        // the peer cannot observe the leader's barriers: give its copies in
        // flight time to land before the pair's final barrier
        const long long t0 = clock64();
        while (clock64() - t0 < (1ll << 21)) {
        }
      }
    }
  } else if (warp == 2) {
    // ------------------------------------- scale-atom producer (both CTAs)
    if (lane == 0) {
      int slot = 0;
      uint32_t phase = 0;
      uint32_t armed_phase = 0;
      int it = 0;
      bool ok = true;
      for (int u = pair; u < args.units && ok; u += pairs) {
        const Unit w = decode_unit(args, u);
        for (int kt = w.kt0; kt < w.kt1; ++kt, ++it) {
          if (it >= sf_pre) {
            if (!pair_wait(&sfse_bar[slot], phase ^ 1u, args.budget, &s_abort, peer_abort)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&sfsf_bar[slot], sf_bytes(w, kt));
            sf_armed |= 1u << slot;
            armed_phase = (armed_phase & ~(1u << slot)) | (phase << slot);
            issue_weight_scales(slot, w, kt);
          }
          issue_act_scales(slot, w, kt);
          if (++slot == C::SF_STAGES) {
            slot = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        for (int i = 0; i < C::SF_STAGES; ++i)
          if (sf_armed & (1u << i)) {
            const long long t0 = clock64();
            while (!mbar_try_wait(&sfsf_bar[i], (armed_phase >> i) & 1u) && clock64() - t0 < args.budget) {
            }
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (leader)
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int sfb = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int u = pair; u < args.units && ok; u += pairs) {
        const Unit w = decode_unit(args, u);
        if (!pair_wait(&acce_bar, acc_phase ^ 1u, args.budget, &s_abort, peer_abort)) break;
        tc_fence_after();
        for (int kt = w.kt0; kt < w.kt1; ++kt) {
          if (!pair_wait(&full_bar[stage], phase, args.budget, &s_abort, peer_abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint8_t* sa = smem + stage * C::STAGE_BYTES;
          const uint32_t a0 = smem_u32(sa), b0 = smem_u32(sa + C::A_BYTES);
          const uint32_t sf = tmem + C::SF_COL0 + sfb * C::SF_COLS;
          const int steps = stage_steps(kt);
          for (int j = 0; j < steps; ++j) {
            const uint32_t off = (j >> 2) * C::CHUNK_BYTES + 32 * (j & 3);  // chunk, then 64 K within it
            mma_mxf4nvf4_pair(tmem, sdesc_kmajor_sw128(a0 + off), sdesc_kmajor_sw128(b0 + off), C::IDESC, sf + 4 * j,
                              sf + C::SFB_COL + 8 * j, (kt > w.kt0 || j > 0) ? 1u : 0u);
          }
          umma_commit_pair(&empty_bar[stage], 0x3);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
          if (++sfb == C::NSF) sfb = 0;
        }
        if (!ok) break;
        umma_commit_pair(&accf_bar, 0x3);
        acc_phase ^= 1u;
      }
      umma_commit_pair(&drain_bar, 0x1);
      const long long t0 = clock64();
      while (!mbar_try_wait(&drain_bar, 0) && clock64() - t0 < 4 * args.budget + 1000000) {
      }
    }
  } else if (wg == 3) {
    // ----------------------------------------- scale writers (both CTAs)
    // Stage i (counted over this pair's tiles) goes to TMEM scale buffer
    // i % NSF once stage i - NSF is consumed; the writers then arrive on the
    // leader's full barrier of stage i.
    regs_dec<48>();
    const int q = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    int slot = 0;
    uint32_t phase = 0;
    int i = 0;
    bool ok = true;
    for (int u = pair; u < args.units && ok; u += pairs) {
      const Unit w = decode_unit(args, u);
      for (int kt = w.kt0; kt < w.kt1; ++kt, ++i) {
        const int prev = i - C::NSF;
        if (!pair_wait(&sfsf_bar[slot], phase, args.budget, &s_abort, peer_abort) ||
            (prev >= 0 && !pair_wait(&empty_bar[prev % C::STAGES], static_cast<uint32_t>(prev / C::STAGES) & 1u,
                                     args.budget, &s_abort, peer_abort))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ssfa = smem_u32(sf_ring + slot * C::SF_STAGE_BYTES);
        const uint32_t ssfb = ssfa + C::SFA_BYTES;
        const uint32_t dst = tmem + lane_base + C::SF_COL0 + (i % C::NSF) * C::SF_COLS;
        const int steps = stage_steps(kt);
        for (int j = 0; j < steps; ++j) {
          tmem_st_32x32b_x4(dst + 4 * j, ld_shared_v4(ssfa + 512 * j + 16 * lane));
#pragma unroll
          for (int rb = 0; rb < 2; ++rb)
            tmem_st_32x32b_x4(dst + C::SFB_COL + 8 * j + 4 * rb,
                              ld_shared_v4(ssfb + rb * C::SFB_ROW_BYTES + 512 * j + 16 * lane));
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive_cluster(leader_bar(&full_bar[i % C::STAGES]));
          mbar_arrive(&sfse_bar[slot]);
        }
        if (++slot == C::SF_STAGES) {
          slot = 0;
          phase ^= 1u;
        }
      }
    }
    tmem_st_wait();
  } else if (wg == 1 || wg == 2) {
    // ------------------------------------------------- epilogue (both CTAs)
    // Warp (q, h) owns TMEM lanes 32q..32q+31 (tile rows) and columns
    // 128h..128h+127; each 64-column box is scaled, rounded to bf16, written
    // to the warp's staging box in the 128-byte swizzle layout and stored
    // with one TMA tile store (rows from M and columns from N are clipped).
    regs_inc<168>();
    const int e = warp - 4;
    const int q = warp & 3;
    const int h = e >> 2;
    const uint32_t box = smem_u32(smem + C::OUT_OFFSET + e * C::OUT_BYTES);
    uint32_t acc_phase = 0;
    for (int u = pair; u < args.units; u += pairs) {
      const Unit w = decode_unit(args, u);
      if (!pair_wait(&accf_bar, acc_phase, args.budget, &s_abort, peer_abort)) break;
      tc_fence_after();
      const int row0 = w.m * C::BM + 128 * static_cast<int>(rank) + 32 * q;
      const int row = row0 + lane;
      const bool row_ok = row < args.M;
      const uint32_t tbase = tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(128 * h);
      __syncwarp();
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(tbase + 32 * c, r[c]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_bar(&acce_bar));
      acc_phase ^= 1u;
      const float rs = row_ok ? args.xg[row] * args.wg[0] : 0.0f;
      if constexpr (!C::TMA_STORE) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int col0 = w.n * C::BN + 128 * h + 32 * c;
          if (row_ok && col0 < args.N) store_output<true>(args, row, col0, rs, r[c]);
        }
      } else {
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          const int col0 = w.n * C::BN + 128 * h + C::OUT_BOX_COLS * b;
          if (col0 >= args.N || row0 >= args.M) continue;  // box wholly outside the output (warp-uniform)
          if (lane == 0) bulk_wait_group_read0();          // the previous store has read the staging box
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            if (row_ok) epilogue_values<true>(args, row, col0 + 32 * c, rs, r[2 * b + c]);
            const float* y = reinterpret_cast<const float*>(r[2 * b + c]);  // rows from M on: clipped by the store
#pragma unroll
            for (int j = 0; j < 4; ++j) {  // 16-byte chunk 4c + j of this row, swizzled by row % 8
              const uint32_t chunk = static_cast<uint32_t>((4 * c + j) ^ (lane & 7));
              st_shared_v4(box + 128 * lane + 16 * chunk, pack_bf16x2(y[8 * j], y[8 * j + 1]),
                           pack_bf16x2(y[8 * j + 2], y[8 * j + 3]), pack_bf16x2(y[8 * j + 4], y[8 * j + 5]),
                           pack_bf16x2(y[8 * j + 6], y[8 * j + 7]));
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmY, smem + C::OUT_OFFSET + e * C::OUT_BYTES, col0, row0);
            bulk_commit_group();
          }
        }
      }
    }
    if (C::TMA_STORE && lane == 0) bulk_wait_group0();
  }

  // Neither CTA leaves (or frees its TMEM) while the other may still signal
  // it or the paired MMAs may still touch its shared memory or TMEM.
  tc_fence_before();
  __syncwarp();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------ host side --
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D byte tensor [rows, row_bytes] with the given pitch, box 128 x box_rows,
// 128-byte swizzle, zero fill out of bounds.
// 8-bit GEMM over CTA pairs (prefill shapes): FP8 E4M3 (kind::f8f6f4, fp32
// accumulators) or INT8 (I8: kind::i8, exact s32), 256 x 256 tiles of the
// paired MMA (tcgen05.mma.cta_group::2) across the two CTAs of a cluster.
// Without block scales the whole TMEM is accumulator: two 256-column
// buffers, so the epilogue of one tile runs while the next tile's MMAs
// accumulate.  CTA r of the pair loads rows [128 r, 128 r + 128) of the A
// and B tiles, two 128-byte K-chunks (K = 256) per stage through 3-D boxes
// (K % 256 == 0), and the leader's full barrier completes on both CTAs'
// bytes.  The leader (even CTA) issues the MMAs and commits each stage to
// both CTAs' empty barriers; each CTA reads its own 128 accumulator rows and
// stores them directly (per-row activation scale, per-column weight scale,
// residual).  Weight tiles of the first stages are loaded before the
// dependency wait.
//   warps 0, 10, 11: operand producers (both CTAs), one per stage slot;
//   warp 1: TMEM allocator (both) and MMA issuer (leader); warps 2-9:
//   epilogue, warp e = w - 2 owns TMEM lanes 32 (w % 4) .. + 31 and
//   columns 128 (e / 4) .. + 127.
template <bool I8>
struct Fp8PairCfg {
  static constexpr int BM = 256;
  static constexpr int BN = 256;
  static constexpr int CH = 2;
  static constexpr int CHUNK_BYTES = 128 * 128;
  static constexpr int A_BYTES = CH * CHUNK_BYTES;
  static constexpr int B_BYTES = CH * CHUNK_BYTES;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STEPS = 4 * CH;  // MMAs (K = 32) per stage
  static constexpr int STAGES = 3;
  static constexpr int ACC_BUFS = 2;
  static constexpr int EPI_WARPS = 8;
  static constexpr int PRODUCERS = STAGES;  // one producer warp per stage slot
  static constexpr int THREADS = 64 + 32 * EPI_WARPS + 32 * (PRODUCERS - 1);
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024;
  static constexpr uint32_t IDESC = (I8 ? (2u << 4) | (1u << 7) | (1u << 10) : (1u << 4)) |
                                    (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);
  static_assert(ACC_BUFS * BN <= kTmemCols, "TMEM budget");
  static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

template <bool I8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Fp8PairCfg<I8>::THREADS, 1)
gemm_fp8_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const GemmArgs args) {
  using C = Fp8PairCfg<I8>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[C::STAGES];      // leader: operands of both CTAs
  __shared__ __align__(8) uint64_t empty_bar[C::STAGES];     // stage consumed (leader's commit)
  __shared__ __align__(8) uint64_t accf_bar[C::ACC_BUFS];    // accumulator complete (leader's commit)
  __shared__ __align__(8) uint64_t acce_bar[C::ACC_BUFS];    // leader: both CTAs' accumulators read
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t s_tmem_base;
  __shared__ volatile int s_abort;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int pairs = static_cast<int>(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < C::ACC_BUFS; ++i) {
      mbar_init(&accf_bar[i], 1);
      mbar_init(&acce_bar[i], 2 * C::EPI_WARPS);
    }
    mbar_init(&drain_bar, 1);
    s_abort = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(&s_tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync();  // both CTAs' barriers are initialised before either CTA signals the other's
  tc_fence_after();
  const uint32_t tmem = s_tmem_base;
  const uint32_t peer_abort = mapa_shared(smem_u32(const_cast<int*>(&s_abort)), rank ^ 1u);
  auto leader_bar = [&](uint64_t* bar) { return mapa_shared(smem_u32(bar), 0u); };
  auto stage_steps = [&](int kt) { return min(C::STEPS, args.k_steps - C::STEPS * kt); };
  auto issue_weights = [&](int stage, const Unit& w, int kt) {
    tma_load_3d_pair(smem + stage * C::STAGE_BYTES + C::A_BYTES, &tmB, leader_bar(&full_bar[stage]), 0,
                     w.n * C::BN + 128 * static_cast<int>(rank), kt * C::CH);
  };
  auto issue_acts = [&](int stage, const Unit& w, int kt) {
    tma_load_3d_pair(smem + stage * C::STAGE_BYTES, &tmA, leader_bar(&full_bar[stage]), 0,
                     w.m * C::BM + 128 * static_cast<int>(rank), kt * C::CH);
  };

  // Producer p (warp 0, then warps 2 + EPI_WARPS ...) owns stage slot p: it
  // issues the loads of stages p, p + STAGES, p + 2 STAGES, ... so that
  // several threads keep TMA copies in flight.  Weights do not depend on the
  // previous kernel on the stream: each producer's first weight tile
  // streams in before the dependency wait.
  const int prod = warp == 0 ? 0 : (warp >= 2 + C::EPI_WARPS ? warp - (1 + C::EPI_WARPS) : -1);
  bool armed = false;
  uint32_t armed_phase = 0;
  if (prod >= 0 && lane == 0) {
    int it = 0;
    for (int u = pair; u < args.units && it <= prod; u += pairs) {
      const Unit w = decode_unit(args, u);
      for (int kt = w.kt0; kt < w.kt1 && it <= prod; ++kt, ++it) {
        if (it != prod) continue;
        if (rank == 0) mbar_arrive_expect_tx(&full_bar[prod], 2 * C::STAGE_BYTES);
        armed = true;
        issue_weights(prod, w, kt);
      }
    }
  }
  griddep_wait();
  griddep_launch_dependents();

  if (prod >= 0) {
    // ------------------------------------------- operand producers (both CTAs)
    if (lane == 0) {
      int it = 0, uses = 0;
      bool ok = true;
      for (int u = pair; u < args.units && ok; u += pairs) {
        const Unit w = decode_unit(args, u);
        for (int kt = w.kt0; kt < w.kt1; ++kt, ++it) {
          if (it % C::STAGES != prod) continue;
          const uint32_t phase = static_cast<uint32_t>(uses) & 1u;
          if (it >= C::STAGES) {
            if (!pair_wait(&empty_bar[prod], phase ^ 1u, args.budget, &s_abort, peer_abort)) {
              ok = false;
              break;
            }
            if (rank == 0) mbar_arrive_expect_tx(&full_bar[prod], 2 * C::STAGE_BYTES);
            armed = true;
            armed_phase = phase;
            issue_weights(prod, w, kt);
          }
          issue_acts(prod, w, kt);
          ++uses;
        }
      }
      if (ok) {
        // the slot released after its last use: the leader's last commit to
        // this CTA has landed
        if (uses > 0) pair_wait(&empty_bar[prod], (static_cast<uint32_t>(uses) & 1u) ^ 1u, args.budget, &s_abort, peer_abort);
      } else if (rank == 0) {
        if (armed) {
          const long long t0 = clock64();
          while (!mbar_try_wait(&full_bar[prod], armed_phase) && clock64() - t0 < args.budget) {
          }
        }
      } else {
        // the peer cannot observe the leader's barriers: give its copies in
        // flight time to land before the pair's final barrier
        const long long t0 = clock64();
        while (clock64() - t0 < (1ll << 21)) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (leader)
    if (lane == 0 && rank == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int u = pair; u < args.units && ok; u += pairs) {
        const Unit w = decode_unit(args, u);
        if (!pair_wait(&acce_bar[acc], acc_phase ^ 1u, args.budget, &s_abort, peer_abort)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc * C::BN);
        for (int kt = w.kt0; kt < w.kt1; ++kt) {
          if (!pair_wait(&full_bar[stage], phase, args.budget, &s_abort, peer_abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * C::STAGE_BYTES), b0 = a0 + C::A_BYTES;
          const int steps = stage_steps(kt);
          for (int j = 0; j < steps; ++j) {
            const uint32_t off = (j >> 2) * C::CHUNK_BYTES + 32 * (j & 3);  // chunk, then 32 K within it
            const uint64_t ad = sdesc_kmajor_sw128(a0 + off), bd = sdesc_kmajor_sw128(b0 + off);
            const uint32_t accum = (kt > w.kt0 || j > 0) ? 1u : 0u;
            if constexpr (I8)
              mma_i8_pair(d_tmem, ad, bd, C::IDESC, accum);
            else
              mma_f8f6f4_pair(d_tmem, ad, bd, C::IDESC, accum);
          }
          umma_commit_pair(&empty_bar[stage], 0x3);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair(&accf_bar[acc], 0x3);
        if (++acc == C::ACC_BUFS) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      umma_commit_pair(&drain_bar, 0x1);
      const long long t0 = clock64();
      while (!mbar_try_wait(&drain_bar, 0) && clock64() - t0 < 4 * args.budget + 1000000) {
      }
    }
  } else if (warp >= 2) {
    // ------------------------------------------------- epilogue (both CTAs)
    const int e = warp - 2;
    const int q = warp & 3;
    const int h = e >> 2;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int u = pair; u < args.units; u += pairs) {
      const Unit w = decode_unit(args, u);
      if (!pair_wait(&accf_bar[acc], acc_phase, args.budget, &s_abort, peer_abort)) break;
      tc_fence_after();
      const int row = w.m * C::BM + 128 * static_cast<int>(rank) + 32 * q + lane;
      const bool row_ok = row < args.M;
      const uint32_t tbase =
          tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(acc * C::BN + 128 * h);
      __syncwarp();
      const float rs = row_ok ? args.xg[row] : 0.0f;
      // 64 columns at a time (the other accumulator buffer keeps the MMAs
      // busy meanwhile); the buffer is handed back after the last load
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        uint32_t r[2][32];
#pragma unroll
        for (int c = 0; c < 2; ++c) tmem_ld_32x32b_x32(tbase + 64 * g + 32 * c, r[c]);
        tmem_ld_wait();
        if (g == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(leader_bar(&acce_bar[acc]));
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int col0 = w.n * C::BN + 128 * h + 64 * g + 32 * c;
          if (row_ok && col0 < args.N) store_output<false, I8>(args, row, col0, rs, r[c]);
        }
      }
      if (++acc == C::ACC_BUFS) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  // Neither CTA leaves (or frees its TMEM) while the other may still signal
  // it or the paired MMAs may still touch its shared memory or TMEM.
  tc_fence_before();
  __syncwarp();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

bool make_map(CUtensorMap* map, const void* base, uint64_t row_bytes, uint64_t rows, uint64_t pitch,
              uint32_t box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {row_bytes, rows};
  const cuuint64_t strides[1] = {pitch};
  const cuuint32_t box[2] = {128, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 output [rows, cols] for TMA tile stores: box 64 columns x 32 rows
// (128-byte rows), 128-byte swizzle.  Needs a 16-byte aligned base and
// cols % 8 == 0.
bool make_out_map(CUtensorMap* map, void* base, uint64_t cols, uint64_t rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, 32};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Packed codes [rows, pitch bytes] viewed as [pitch / 128 chunks][rows][128
// bytes] for 3-D boxes of 128 bytes x box_rows x box_chunks, 128-byte swizzle
// (each chunk of the box lands as its own swizzled block).  pitch % 128 == 0.
bool make_chunk_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t pitch, uint32_t box_rows,
                    uint32_t box_chunks) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc || pitch % 128 != 0) return false;
  const cuuint64_t dims[3] = {128, rows, pitch / 128};
  const cuuint64_t strides[2] = {pitch, 128};
  const cuuint32_t box[3] = {128, box_rows, box_chunks};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Launch arguments shared by both GEMM kernels (BN: tile width).
GemmArgs make_args(bool fp4, int BN, const uint8_t* xs, const float* xg, const uint8_t* ws, const float* wg,
                   const void* residual, void* Y, int64_t M, int64_t N, int64_t K, void* workspace,
                   const GemmPlan& plan, long long budget) {
  GemmArgs a;
  a.xs = xs;
  a.ws = ws;
  a.xg = xg;
  a.wg = wg;
  a.residual = static_cast<const __nv_bfloat16*>(residual);
  a.Y = static_cast<__nv_bfloat16*>(Y);
  // split-K workspace: tile counters first (NVFP4), then the partial sums
  a.partial = plan.splits > 1 ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kSplitCounterBytes)
                              : nullptr;
  a.counters = plan.splits > 1 ? static_cast<unsigned int*>(workspace) : nullptr;
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.k_steps = static_cast<int>(fp4 ? (K + 63) / 64 : (K + 31) / 32);
  a.k_tiles = (a.k_steps + 3) / 4;
  a.m_tiles = static_cast<int>((M + kBM - 1) / kBM);
  a.n_tiles = static_cast<int>((N + BN - 1) / BN);
  a.splits = plan.splits;
  a.units = a.m_tiles * a.n_tiles * a.splits;
  a.ka = static_cast<int>((K + 63) / 64);
  a.w_row_blocks = static_cast<int>((N + 127) / 128);
  a.budget = budget;
  return a;
}

// NVFP4: the scale-writer kernel; split-K partials are reduced in-kernel.
cudaError_t run_fp4(const uint8_t* xq, const uint8_t* xs, const float* xg, const uint8_t* wq, const uint8_t* ws,
                    const float* wg, const void* residual, void* Y, int64_t M, int64_t N, int64_t K,
                    void* workspace, const GemmPlan& plan, long long budget, cudaStream_t s) {
  const int64_t pitch = nvfp4_code_pitch(K);
  CUtensorMap ta, tb;
  if (!make_map(&ta, xq, static_cast<uint64_t>(pitch), static_cast<uint64_t>(M), static_cast<uint64_t>(pitch), kBM) ||
      !make_map(&tb, wq, static_cast<uint64_t>(pitch), static_cast<uint64_t>(N), static_cast<uint64_t>(pitch),
                SfwCfg::BN))
    return cudaErrorInvalidValue;
  const GemmArgs a = make_args(true, SfwCfg::BN, xs, xg, ws, wg, residual, Y, M, N, K, workspace, plan, budget);
  const int grid = plan.grid < a.units ? plan.grid : a.units;
  cudaError_t e =
      cudaFuncSetAttribute(gemm_fp4_sfw_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SfwCfg::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  return launch_pdl(gemm_fp4_sfw_kernel, dim3(grid), dim3(SfwCfg::THREADS), SfwCfg::SMEM_BYTES, s, ta, tb, a);
}

// Clusters of gemm_fp4_pair_kernel<CH> that fit on the device at once
// (cached per device; half the SMs when the query fails).
template <int CH>
int pair_clusters_resident() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return device_sm_count() / 2;
  static int cache[64] = {0};
  if (dev < 64 && cache[dev]) return cache[dev];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned int>(device_sm_count()));
  cfg.blockDim = dim3(PairCfg<CH>::THREADS);
  cfg.dynamicSmemBytes = PairCfg<CH>::SMEM_BYTES;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_fp4_pair_kernel<CH>, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = device_sm_count() / 2;
  }
  if (dev < 64) cache[dev] = n;
  return n;
}

template <int CH>
cudaError_t launch_pair(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& ty, GemmArgs a,
                        const GemmPlan& plan, cudaStream_t s) {
  using C = PairCfg<CH>;
  a.k_tiles = (a.k_steps + C::STEPS - 1) / C::STEPS;
  cudaError_t e = cudaFuncSetAttribute(gemm_fp4_pair_kernel<CH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  int pairs = pair_clusters_resident<CH>();
  if (plan.grid / 2 < pairs) pairs = plan.grid / 2;
  if (a.units < pairs) pairs = a.units;
  if (pairs < 1) pairs = 1;
  return launch_pdl(gemm_fp4_pair_kernel<CH>, dim3(static_cast<unsigned int>(2 * pairs)), dim3(C::THREADS),
                    C::SMEM_BYTES, s, ta, tb, ty, a);
}

// NVFP4 over CTA pairs: 256 x 256 tiles, direct epilogue.  Rows of whole
// 128-byte chunks (K % 256 == 0) take two chunks per stage through 3-D
// boxes; other K one chunk per stage with TMA stores of the output, and an
// output the store map cannot describe (base not 16-byte aligned) the
// single-CTA kernel.
cudaError_t run_fp4_pair(const uint8_t* xq, const uint8_t* xs, const float* xg, const uint8_t* wq, const uint8_t* ws,
                         const float* wg, const void* residual, void* Y, int64_t M, int64_t N, int64_t K,
                         void* workspace, const GemmPlan& plan, long long budget, cudaStream_t s) {
  const int64_t pitch = nvfp4_code_pitch(K);
  GemmArgs a = make_args(true, PairCfg<1>::BN, xs, xg, ws, wg, residual, Y, M, N, K, nullptr, plan, budget);
  a.m_tiles = static_cast<int>((M + PairCfg<1>::BM - 1) / PairCfg<1>::BM);
  a.splits = 1;
  a.units = a.m_tiles * a.n_tiles;
  CUtensorMap ta, tb, ty;
  if (K % 256 == 0) {
    if (!make_chunk_map(&ta, xq, static_cast<uint64_t>(M), static_cast<uint64_t>(pitch), 128, 2) ||
        !make_chunk_map(&tb, wq, static_cast<uint64_t>(N), static_cast<uint64_t>(pitch), 128, 2))
      return cudaErrorInvalidValue;
    ty = tb;  // not read: this variant stores rows directly
    return launch_pair<2>(ta, tb, ty, a, plan, s);
  }
  if (!make_out_map(&ty, Y, static_cast<uint64_t>(N), static_cast<uint64_t>(M)))
    return run_fp4(xq, xs, xg, wq, ws, wg, residual, Y, M, N, K, workspace, plan, budget, s);
  if (!make_map(&ta, xq, static_cast<uint64_t>(pitch), static_cast<uint64_t>(M), static_cast<uint64_t>(pitch), 128) ||
      !make_map(&tb, wq, static_cast<uint64_t>(pitch), static_cast<uint64_t>(N), static_cast<uint64_t>(pitch), 128))
    return cudaErrorInvalidValue;
  return launch_pair<1>(ta, tb, ty, a, plan, s);
}

// Clusters of gemm_fp8_pair_kernel<I8> that fit on the device at once
// (cached per device; half the SMs when the query fails).
template <bool I8>
int fp8_pair_clusters_resident() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return device_sm_count() / 2;
  static int cache[64] = {0};
  if (dev < 64 && cache[dev]) return cache[dev];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned int>(device_sm_count()));
  cfg.blockDim = dim3(Fp8PairCfg<I8>::THREADS);
  cfg.dynamicSmemBytes = Fp8PairCfg<I8>::SMEM_BYTES;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_fp8_pair_kernel<I8>, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = device_sm_count() / 2;
  }
  if (dev < 64) cache[dev] = n;
  return n;
}

// FP8 / INT8 over CTA pairs: 256 x 256 tiles, two K-chunks per stage (K %
// 256 == 0), direct epilogue, no split.
template <bool I8>
cudaError_t run_fp8_pair(const uint8_t* xq, const float* xg, const uint8_t* wq, const float* wg,
                         const void* residual, void* Y, int64_t M, int64_t N, int64_t K, const GemmPlan& plan,
                         long long budget, cudaStream_t s) {
  using C = Fp8PairCfg<I8>;
  CUtensorMap ta, tb;
  if (!make_chunk_map(&ta, xq, static_cast<uint64_t>(M), static_cast<uint64_t>(K), 128, C::CH) ||
      !make_chunk_map(&tb, wq, static_cast<uint64_t>(N), static_cast<uint64_t>(K), 128, C::CH))
    return cudaErrorInvalidValue;
  GemmArgs a = make_args(false, C::BN, nullptr, xg, nullptr, wg, residual, Y, M, N, K, nullptr, plan, budget);
  a.m_tiles = static_cast<int>((M + C::BM - 1) / C::BM);
  a.splits = 1;
  a.units = a.m_tiles * a.n_tiles;
  a.k_tiles = (a.k_steps + C::STEPS - 1) / C::STEPS;
  auto kern = gemm_fp8_pair_kernel<I8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  int pairs = fp8_pair_clusters_resident<I8>();
  if (plan.grid / 2 < pairs) pairs = plan.grid / 2;
  if (a.units < pairs) pairs = a.units;
  if (pairs < 1) pairs = 1;
  return launch_pdl(kern, dim3(static_cast<unsigned int>(2 * pairs)), dim3(C::THREADS), C::SMEM_BYTES, s, ta, tb, a);
}

// FP8 / INT8: gemm_fp8_kernel<BN, I8>, then the ordered split-K reduction
// when split.
template <int BN, bool I8>
cudaError_t run_fp8(const uint8_t* xq, const float* xg, const uint8_t* wq, const float* wg, const void* residual,
                    void* Y, int64_t M, int64_t N, int64_t K, void* workspace, const GemmPlan& plan,
                    long long budget, cudaStream_t s) {
  using C = Fp8Cfg<BN, I8>;
  CUtensorMap ta, tb;
  if (!make_map(&ta, xq, static_cast<uint64_t>(K), static_cast<uint64_t>(M), static_cast<uint64_t>(K), kBM) ||
      !make_map(&tb, wq, static_cast<uint64_t>(K), static_cast<uint64_t>(N), static_cast<uint64_t>(K), BN))
    return cudaErrorInvalidValue;
  const GemmArgs a = make_args(false, BN, nullptr, xg, nullptr, wg, residual, Y, M, N, K, workspace, plan, budget);
  const int grid = plan.grid < a.units ? plan.grid : a.units;
  auto kern = gemm_fp8_kernel<BN, I8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, s, ta, tb, a);
}

}  // namespace

GemmPlan plan_gemm(bool fp4, int64_t M, int64_t N, int64_t K, int num_sms) {
  GemmPlan p;
  const int64_t k_steps = fp4 ? (K + 63) / 64 : (K + 31) / 32;
  const int64_t k_tiles = (k_steps + 3) / 4;
  const int64_t m_tiles = (M + kBM - 1) / kBM;
  if (fp4 && gemv_supported(M, N, K)) {
    // one or two token rows, small weights: the weight-streaming kernel on the CUDA cores
    p.bn = 0;
    p.splits = 1;
    p.grid = 0;
    p.ws_bytes = 0;
    return p;
  }
  if (fp4) {
    // NVFP4: the 128 x 256 scale-writer kernel; few output tiles
    // (decode) are split along K so every SM streams weights, and the last
    // split of each tile reduces in-kernel (per-tile counters after the
    // partials, zero between calls).
    p.bn = 256;
    const int64_t tiles = m_tiles * ((N + 255) / 256);
    int64_t splits = 1;
    if (tiles * 2 <= num_sms && tiles * sizeof(unsigned int) <= kSplitCounterBytes) {
      // at least two K-stages per split (measured: one-stage splits of o at
      // M = 4 / 8 took 8.0 / 9.0 us, two-stage ones 7.6 / 8.5)
      splits = num_sms / tiles;
      if (splits > k_tiles / 2) splits = k_tiles / 2;
      if (splits < 1) splits = 1;
    }
    p.splits = static_cast<int>(splits);
    const int64_t units = tiles * splits;
    p.grid = static_cast<int>(units < num_sms ? units : num_sms);
    p.ws_bytes = splits > 1 ? kSplitCounterBytes + splitk_partial_bytes(splits, M, N) : 0;
    // Tiles that fill the GPU and more than 128 rows: 256 x 256 tiles over
    // CTA pairs, each SM streaming half of the weight tile.
    if (splits == 1 && M > kBM) {
      const int64_t pair_units = ((M + 255) / 256) * ((N + 255) / 256);
      const int64_t pairs = num_sms / 2;
      p.pair = true;
      p.grid = static_cast<int>(2 * (pair_units < pairs ? pair_units : pairs));
    }
    return p;
  }
  // Wide tiles halve the scale-factor copies per FLOP and the A re-reads;
  // they are used whenever they still give every SM work.
  const int64_t tiles256 = m_tiles * ((N + 255) / 256);
  if (tiles256 * 2 > num_sms) {
    p.bn = 256;
    p.splits = 1;
    p.grid = static_cast<int>(tiles256 < num_sms ? tiles256 : num_sms);
    p.ws_bytes = 0;
    // more than 128 rows and rows of whole 256-byte K-chunks: 256 x 256
    // tiles over CTA pairs
    if (M > kBM && K % 256 == 0) {
      const int64_t pair_units = ((M + 255) / 256) * ((N + 255) / 256);
      const int64_t pairs = num_sms / 2;
      p.pair = true;
      p.grid = static_cast<int>(2 * (pair_units < pairs ? pair_units : pairs));
    }
    return p;
  }
  // Few output tiles (decode): narrow tiles and split-K over the SMs.
  p.bn = 128;
  const int64_t tiles = m_tiles * ((N + 127) / 128);
  int64_t splits = 1;
  if (tiles * 2 <= num_sms) {
    splits = num_sms / tiles;
    if (splits > k_tiles / 2) splits = k_tiles / 2;
    if (splits < 1) splits = 1;
  }
  p.splits = static_cast<int>(splits);
  const int64_t units = tiles * splits;
  p.grid = static_cast<int>(units < num_sms ? units : num_sms);
  p.ws_bytes = splits > 1 ? kSplitCounterBytes + splitk_partial_bytes(splits, M, N) : 0;
  return p;
}

cudaError_t launch_linear(bool fp4, const uint8_t* xq, const uint8_t* xs, const float* xg, const uint8_t* wq,
                          const uint8_t* ws, const float* wg, const void* residual, void* Y, int64_t M, int64_t N,
                          int64_t K, void* workspace, size_t ws_bytes, const GemmPlan& plan, long long budget,
                          cudaStream_t s) {
  (void)ws_bytes;
  if (fp4 && plan.bn == 0) return launch_gemv_nvfp4(xq, xs, xg, wq, ws, wg, residual, Y, M, N, K, s);
  if (fp4 && plan.pair)
    return run_fp4_pair(xq, xs, xg, wq, ws, wg, residual, Y, M, N, K, workspace, plan, budget, s);
  if (fp4) return run_fp4(xq, xs, xg, wq, ws, wg, residual, Y, M, N, K, workspace, plan, budget, s);
  if (plan.pair) return run_fp8_pair<false>(xq, xg, wq, wg, residual, Y, M, N, K, plan, budget, s);
  if (plan.bn == 256) return run_fp8<256, false>(xq, xg, wq, wg, residual, Y, M, N, K, workspace, plan, budget, s);
  return run_fp8<128, false>(xq, xg, wq, wg, residual, Y, M, N, K, workspace, plan, budget, s);
}

cudaError_t launch_linear_int8(const int8_t* xq, const float* s_x, const int8_t* wq, const float* s_w,
                               const void* residual, void* Y, int64_t M, int64_t N, int64_t K, void* workspace,
                               const GemmPlan& plan, long long budget, cudaStream_t s) {
  const uint8_t* x8 = reinterpret_cast<const uint8_t*>(xq);
  const uint8_t* w8 = reinterpret_cast<const uint8_t*>(wq);
  if (plan.pair) return run_fp8_pair<true>(x8, s_x, w8, s_w, residual, Y, M, N, K, plan, budget, s);
  if (plan.bn == 256) return run_fp8<256, true>(x8, s_x, w8, s_w, residual, Y, M, N, K, workspace, plan, budget, s);
  return run_fp8<128, true>(x8, s_x, w8, s_w, residual, Y, M, N, K, workspace, plan, budget, s);
}

cudaError_t read_and_clear_status(unsigned int* out, cudaStream_t s) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_vlaq_status, sizeof(unsigned int), 0,
                                            cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return e;
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return e;
  const unsigned int zero = 0;
  e = cudaMemcpyToSymbolAsync(g_vlaq_status, &zero, sizeof(unsigned int), 0, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return e;
  return cudaStreamSynchronize(s);
}

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  static int cache[64] = {0};
  if (dev < 64 && cache[dev]) return cache[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  if (dev < 64) cache[dev] = n;
  return n;
}

}  // namespace vlaq
