/*
 * vlaq oracle: a plain, slow, obviously correct CPU statement of what the
 * NVFP4 / FP8 / INT8 quantize + linear path computes.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file.  It shares no code, header, table or constant generator
 * with the CUDA path.  Only tests/, the smoke check and the benchmark's
 * cpu_baseline / reference leg use it.
 *
 * Sources (page title, then the passage):
 *  - "Feat/internvla n1 dualvln" (model-quantization-recipes PR #2), the
 *    NVFP4 loader commit: two E2M1 values per byte, one FP8 (E4M3) scale per
 *    16 values, one float32 global scale; the nibble-order commit: the low
 *    nibble holds the first element.
 *  - same page, scheme-gate commits: NVFP4 needs K divisible by 16
 *    (3420 / 16 = 213.75 is refused).
 *  - "Alpamayo 2 Super NVFP4: full test reflection", the ModelOpt paragraph:
 *    max-based calibration, FP4 weights and input activations, block 16,
 *    FP8 block scales.
 *  - "FoldQuant W8A8/W4A4 inference ..." (vla.cpp PR #33): the activation
 *    node is RMSNorm with the folded gain, the block rotation by the
 *    normalised Sylvester-Hadamard butterfly (symmetric, orthonormal),
 *    per-token amax scale, round-half-even and clamp (OpenVINO commit); the
 *    SYCL commit fixes the reduction tree (lane l of a 32-wide group owns
 *    chunks l, l+32, ...) and demands correctly rounded divide and sqrt with
 *    no contraction; the residual add sits in the o / down epilogues.
 *  - "NVIDIA/TensorRT-Edge-LLM PR #193", results section: NVFP4 quantizes
 *    activations dynamically (no static input scale).
 *  - FP8 E4M3 W8A8 with per-row weight scale and per-token activation
 *    scale (the FP8 recipe commit of PR #2 uses per-tensor scales; the
 *    per-row / per-token granularity is the stated workload's choice).
 *  - "FoldQuant W8A8/W4A4 inference ...", the INT8 path: INT8 codes with
 *    per-row weight scales, activations quantized per token, integer GEMMs
 *    whose sums are exact in any order (SYCL commit).
 *  - same page, dequant commit: per-input-channel smoothing x' = R(x / a)
 *    or R(x) / a; "NVIDIA/TensorRT-Edge-LLM PR #193", pre_quant_scale
 *    commit: the AWQ pre_quant_scale multiplies the activations, and an
 *    NVFP4 linear carries input_scale (a static activation global scale)
 *    beside weight_scale and weight_scale_2.
 *
 * Floating point: quantization runs in IEEE fp32 with every operation
 * rounded once (build with -ffp-contract=off, no -ffast-math); the GEMM
 * decodes both operands exactly and sums in fp64 in k order.
 *
 * Readings where the pages are silent (each one is listed in the design
 * notes): the two-level NVFP4 scale g = amax / (6 * 448); block scale by
 * round-to-nearest-even with saturation; x / S as a correctly rounded
 * divide; negative values that round to zero keep their sign (code 0x8);
 * an all-zero scope (g == 0) gives zero scales and zero codes; RMSNorm in
 * fp32 with the 32-lane tree below; block-64 Walsh-Hadamard in Sylvester
 * natural order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define VO_F_RMSNORM 1u
#define VO_F_HADAMARD64 2u
#define VO_F_SMOOTH_AFTER 4u  /* smoothing after the rotation (default before) */
#define VO_F_SMOOTH_MUL 8u    /* multiply by the smoothing vector (default divide) */

/* ---------------------------------------------------------------- bf16 -- */

float vo_bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* ---------------------------------------------------------------- E2M1 -- */
/*
 * E2M1: 1 sign bit, 2 exponent bits, 1 mantissa bit.  Magnitude codes 0..7
 * stand for 0, 0.5, 1, 1.5, 2, 3, 4, 6.  Encoding is round to nearest with
 * ties going to the code whose least significant bit is 0 (the "even"
 * neighbour), and magnitudes above 6 saturate to 6.  The midpoints between
 * neighbours are 0.25, 0.75, 1.25, 1.75, 2.5, 3.5 and 5; at each midpoint
 * the tie picks the even code, which is what the <= / < pattern below says.
 */
uint8_t vo_e2m1_encode(float v) {
  uint8_t s = signbit(v) ? 0x8 : 0x0;
  float a = fabsf(v);
  uint8_t m;
  if (a <= 0.25f)      m = 0; /* tie at 0.25 -> code 0 (even) */
  else if (a < 0.75f)  m = 1; /* tie at 0.75 -> code 2 (even) */
  else if (a <= 1.25f) m = 2; /* tie at 1.25 -> code 2 */
  else if (a < 1.75f)  m = 3; /* tie at 1.75 -> code 4 */
  else if (a <= 2.5f)  m = 4; /* tie at 2.5  -> code 4 */
  else if (a < 3.5f)   m = 5; /* tie at 3.5  -> code 6 */
  else if (a <= 5.0f)  m = 6; /* tie at 5    -> code 6 */
  else                 m = 7; /* saturate at 6 */
  return (uint8_t)(s | m);
}

double vo_e2m1_decode(uint8_t code) {
  static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  double v = mag[code & 7];
  return (code & 8) ? -v : v;
}

/* ---------------------------------------------------------------- E4M3 -- */
/*
 * E4M3 ("fn" variant): bias 7, 3 mantissa bits, no infinities, 0x7F / 0xFF
 * are NaN, largest finite magnitude 448 (0x7E), subnormals are m * 2^-9.
 * Encoding: exact round to nearest even on the E4M3 grid of the fp32 value,
 * magnitudes at or above 448 saturate to 448.
 */
uint8_t vo_e4m3_encode(float v) {
  uint8_t s = signbit(v) ? 0x80 : 0x00;
  double a = fabs((double)v);
  if (a >= 448.0) return (uint8_t)(s | 0x7E);
  if (a < ldexp(1.0, -6)) {
    /* subnormal range: grid step 2^-9 */
    double q = nearbyint(a / ldexp(1.0, -9)); /* default mode: ties to even */
    if (q >= 8.0) return (uint8_t)(s | 0x08); /* rounds up to 2^-6 */
    return (uint8_t)(s | (uint8_t)q);
  }
  int e;
  (void)frexp(a, &e);      /* a = f * 2^e, f in [0.5, 1) */
  e -= 1;                  /* a in [2^e, 2^(e+1)) */
  double step = ldexp(1.0, e - 3);
  double q = nearbyint(a / step); /* in [8, 16]; exact division by 2^k */
  if (q >= 16.0) { q = 8.0; e += 1; }
  int be = e + 7;          /* 1 .. 15 */
  return (uint8_t)(s | (uint8_t)(be << 3) | (uint8_t)((int)q - 8));
}

double vo_e4m3_decode(uint8_t code) {
  int be = (code >> 3) & 0xF;
  int m = code & 7;
  double v;
  if (be == 0xF && m == 7) return NAN;
  if (be == 0) v = ldexp((double)m, -9);
  else v = ldexp(1.0 + m / 8.0, be - 7);
  return (code & 0x80) ? -v : v;
}

/* ------------------------------------------------------------- RMSNorm -- */
/*
 * Sum of squares in the fixed tree: 32 lanes, lane l owns the 8-element
 * chunks l, l+32, l+64, ... and accumulates them in element order with a
 * fused multiply-add; the 32 partial sums are then combined by the XOR
 * butterfly with offsets 16, 8, 4, 2, 1 and lane 0's value is the sum.
 * K must be a multiple of 8.
 */
float vo_sumsq_tree(const float* x, int64_t K) {
  float lane[32];
  int64_t nchunk = K / 8;
  for (int l = 0; l < 32; ++l) {
    float acc = 0.0f;
    for (int64_t c = l; c < nchunk; c += 32)
      for (int e = 0; e < 8; ++e) acc = fmaf(x[8 * c + e], x[8 * c + e], acc);
    lane[l] = acc;
  }
  for (int off = 16; off >= 1; off >>= 1) {
    float nxt[32];
    for (int l = 0; l < 32; ++l) nxt[l] = lane[l] + lane[l ^ off];
    memcpy(lane, nxt, sizeof lane);
  }
  return lane[0];
}

/* y_k = (x_k * r) * gamma_k with r = 1 / sqrt(mean(x^2) + eps), all fp32. */
void vo_rmsnorm_row(const float* x, int64_t K, const float* gamma, float eps,
                    float* y) {
  float ss = vo_sumsq_tree(x, K);
  float mean = ss / (float)K;
  float v = mean + eps;
  float r = 1.0f / sqrtf(v);
  for (int64_t k = 0; k < K; ++k) y[k] = (x[k] * r) * gamma[k];
}

/* ------------------------------------------------------- Hadamard (64) -- */
/*
 * Block-diagonal normalised Walsh-Hadamard transform, block 64, Sylvester
 * natural order: for each 64-block, butterfly stages h = 1, 2, ..., 32 map
 * (y_i, y_{i+h}) to (y_i + y_{i+h}, y_i - y_{i+h}) for every i with
 * (i & h) == 0, then every value is multiplied by 1/8 (exact).  The
 * resulting matrix is H[i][j] = (-1)^popcount(i & j) / 8: symmetric and
 * orthonormal.  K must be a multiple of 64.
 */
void vo_wht64_inplace(float* y, int64_t K) {
  for (int64_t b = 0; b < K; b += 64) {
    float* blk = y + b;
    for (int h = 1; h < 64; h <<= 1) {
      for (int i = 0; i < 64; ++i) {
        if (i & h) continue;
        float u = blk[i] + blk[i + h];
        float w = blk[i] - blk[i + h];
        blk[i] = u;
        blk[i + h] = w;
      }
    }
    for (int i = 0; i < 64; ++i) blk[i] = blk[i] * 0.125f;
  }
}

/* bf16 row -> fp32, optional RMSNorm (gain gamma, bf16), optional WHT-64. */
/*
 * Per-input-channel smoothing (one fp32 factor a_k per channel), applied to
 * the normalised row: y_k / a_k (FoldQuant's activation scale divide:
 * "FoldQuant W8A8/W4A4 inference ...", dequant commit, x' = R(x / a) when
 * folded before the rotation R, R(x) / a when folded after; OpenVINO commit:
 * RMSNorm with the folded gain, then the divide, then the rotation) or
 * y_k * a_k (AWQ's pre_quant_scale, which the activations are multiplied by:
 * "NVIDIA/TensorRT-Edge-LLM PR #193", the pre_quant_scale commit, and
 * "Alpamayo 2 Super NVFP4 ...", the AWQ paragraph).  One fp32 operation per
 * element, correctly rounded.
 */
static void smooth_row(float* y, int64_t K, const float* a, unsigned flags) {
  for (int64_t k = 0; k < K; ++k) y[k] = (flags & VO_F_SMOOTH_MUL) ? y[k] * a[k] : y[k] / a[k];
}

static void transform_row(const uint16_t* x, int64_t K, const uint16_t* gamma, float eps, unsigned flags,
                          const float* smooth, float* y) {
  for (int64_t k = 0; k < K; ++k) y[k] = vo_bf16_to_f32(x[k]);
  if (flags & VO_F_RMSNORM) {
    float* g = (float*)malloc(sizeof(float) * (size_t)K);
    float* t = (float*)malloc(sizeof(float) * (size_t)K);
    for (int64_t k = 0; k < K; ++k) g[k] = vo_bf16_to_f32(gamma[k]);
    vo_rmsnorm_row(y, K, g, eps, t);
    memcpy(y, t, sizeof(float) * (size_t)K);
    free(t);
    free(g);
  }
  if (smooth && !(flags & VO_F_SMOOTH_AFTER)) smooth_row(y, K, smooth, flags);
  if (flags & VO_F_HADAMARD64) vo_wht64_inplace(y, K);
  if (smooth && (flags & VO_F_SMOOTH_AFTER)) smooth_row(y, K, smooth, flags);
}

void vo_transform_row(const uint16_t* x, int64_t K, const uint16_t* gamma,
                      float eps, unsigned flags, float* y) {
  transform_row(x, K, gamma, eps, flags, NULL, y);
}

/* The row transform with a smoothing vector (NULL: none). */
void vo_transform_row_smooth(const uint16_t* x, int64_t K, const uint16_t* gamma, float eps, unsigned flags,
                             const float* smooth, float* y) {
  transform_row(x, K, gamma, eps, flags, smooth, y);
}

/* --------------------------------------------------------------- NVFP4 -- */
/*
 * Two-level NVFP4 quantization of one scope (a token row, or a whole weight
 * tensor) given its fp32 values y:
 *   A   = max |y| over the scope (exact)
 *   g   = A / (6 * 448)                        fp32 global scale
 *   per 16-block b: a_b = max |y| in the block,
 *   s_b = a_b / (6 * g)  -> E4M3 (RNE, saturate) = sb8
 *   S_b = E4M3(sb8) * g                        fp32
 *   code_i = E2M1(y_i / S_b)   (0 when S_b == 0)
 * Decoded value: E2M1(code) * E4M3(sb8) * g.  g == 0 (all-zero scope, or a
 * scope so small that A / 2688 underflows) gives zero scales and codes.
 */
float vo_nvfp4_global(float amax) { return amax / 2688.0f; }

static void quant_block16(const float* y, int n, float g, uint8_t* sb8_out,
                          uint8_t* code_out /* n codes, one per byte */) {
  if (g == 0.0f) {
    *sb8_out = 0;
    for (int i = 0; i < n; ++i) code_out[i] = 0;
    return;
  }
  float ab = 0.0f;
  for (int i = 0; i < n; ++i) ab = fmaxf(ab, fabsf(y[i]));
  float sb = ab / (6.0f * g);
  uint8_t sb8 = vo_e4m3_encode(sb);
  float S = (float)vo_e4m3_decode(sb8) * g;
  *sb8_out = sb8;
  for (int i = 0; i < n; ++i)
    code_out[i] = (S == 0.0f) ? 0 : vo_e2m1_encode(y[i] / S);
}

/*
 * X: bf16 [rows, K] row-major.  per_tensor = 0: one global scale per row
 * (activations, g has rows entries); per_tensor = 1: one global scale for
 * the whole tensor (weights, g has 1 entry).
 * codes: [rows, K/2] row-major, element k in byte k/2, low nibble first.
 * scales: [rows, K/16] row-major (logical layout).
 * Returns 0, or -1 when K is not a multiple of 16 (64 with the Hadamard
 * flag) or a gamma is missing for RMSNorm.
 */
static int quantize_nvfp4(const uint16_t* X, int64_t rows, int64_t K, const uint16_t* gamma, float eps,
                          unsigned flags, const float* smooth, int per_tensor, const float* g_static,
                          uint8_t* codes, uint8_t* scales, float* g);

int vo_quantize_nvfp4(const uint16_t* X, int64_t rows, int64_t K,
                      const uint16_t* gamma, float eps, unsigned flags,
                      int per_tensor, uint8_t* codes, uint8_t* scales,
                      float* g) {
  return quantize_nvfp4(X, rows, K, gamma, eps, flags, NULL, per_tensor, NULL, codes, scales, g);
}

/* Per-token NVFP4 quantization of activations smoothed per input channel
 * (smooth: fp32 [K], non-NULL). */
int vo_quantize_nvfp4_smooth(const uint16_t* X, int64_t rows, int64_t K, const uint16_t* gamma, float eps,
                             unsigned flags, const float* smooth, uint8_t* codes, uint8_t* scales, float* g) {
  if (smooth == NULL) return -1;
  return quantize_nvfp4(X, rows, K, gamma, eps, flags, smooth, 0, NULL, codes, scales, g);
}

/* Activations with a static (calibrated) global scale instead of the
 * per-token amax: the ModelOpt / TensorRT NVFP4 linear carries an fp32
 * input_scale ("NVIDIA/TensorRT-Edge-LLM PR #193", the pre_quant_scale
 * commit lists weight, weight_scale, weight_scale_2 and input_scale).  Every
 * row uses g = g_static; blocks and codes follow the same definitions, so
 * values beyond the calibrated range saturate (E4M3 at 448, E2M1 at 6).  g
 * receives g_static per row.  smooth may be NULL. */
int vo_quantize_nvfp4_static(const uint16_t* X, int64_t rows, int64_t K, const uint16_t* gamma, float eps,
                             unsigned flags, const float* smooth, float g_static, uint8_t* codes,
                             uint8_t* scales, float* g) {
  return quantize_nvfp4(X, rows, K, gamma, eps, flags, smooth, 0, &g_static, codes, scales, g);
}

static int quantize_nvfp4(const uint16_t* X, int64_t rows, int64_t K, const uint16_t* gamma, float eps,
                          unsigned flags, const float* smooth, int per_tensor, const float* g_static,
                          uint8_t* codes, uint8_t* scales, float* g) {
  if (K <= 0 || K % 16 != 0) return -1;
  if ((flags & VO_F_HADAMARD64) && K % 64 != 0) return -1;
  if ((flags & VO_F_RMSNORM) && gamma == NULL) return -1;
  float* Y = (float*)malloc(sizeof(float) * (size_t)(rows * K));
  for (int64_t r = 0; r < rows; ++r)
    transform_row(X + r * K, K, gamma, eps, flags, smooth, Y + r * K);
  float gt = 0.0f;
  if (per_tensor) {
    float A = 0.0f;
    for (int64_t i = 0; i < rows * K; ++i) A = fmaxf(A, fabsf(Y[i]));
    gt = vo_nvfp4_global(A);
    g[0] = gt;
  }
  for (int64_t r = 0; r < rows; ++r) {
    const float* y = Y + r * K;
    float gr = gt;
    if (g_static) {
      gr = *g_static;
      g[r] = gr;
    } else if (!per_tensor) {
      float A = 0.0f;
      for (int64_t k = 0; k < K; ++k) A = fmaxf(A, fabsf(y[k]));
      gr = vo_nvfp4_global(A);
      g[r] = gr;
    }
    for (int64_t b = 0; b < K / 16; ++b) {
      uint8_t c[16];
      quant_block16(y + 16 * b, 16, gr, scales + r * (K / 16) + b, c);
      for (int i = 0; i < 16; i += 2)
        codes[r * (K / 2) + 8 * b + i / 2] = (uint8_t)(c[i] | (c[i + 1] << 4));
    }
  }
  free(Y);
  return 0;
}

/* Decode NVFP4 (logical layouts as produced above) to fp64 [rows, K]. */
void vo_decode_nvfp4(const uint8_t* codes, const uint8_t* scales,
                     const float* g, int64_t rows, int64_t K, int per_tensor,
                     double* out) {
  for (int64_t r = 0; r < rows; ++r) {
    double gr = per_tensor ? (double)g[0] : (double)g[r];
    for (int64_t k = 0; k < K; ++k) {
      uint8_t byte = codes[r * (K / 2) + k / 2];
      uint8_t c = (k & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
      double s = vo_e4m3_decode(scales[r * (K / 16) + k / 16]);
      out[r * K + k] = vo_e2m1_decode(c) * s * gr;
    }
  }
}

/* ----------------------------------------------------------------- FP8 -- */
/*
 * FP8 E4M3 per-row quantization: s = max|y| / 448 (fp32),
 * code = E4M3(y / s) (RNE, saturate), or 0 when s == 0.
 * Decoded value: E4M3(code) * s.
 */
int vo_quantize_fp8(const uint16_t* X, int64_t rows, int64_t K,
                    const uint16_t* gamma, float eps, unsigned flags,
                    uint8_t* codes, float* s) {
  if (K <= 0 || K % 16 != 0) return -1;
  if ((flags & VO_F_HADAMARD64) && K % 64 != 0) return -1;
  if ((flags & VO_F_RMSNORM) && gamma == NULL) return -1;
  float* y = (float*)malloc(sizeof(float) * (size_t)K);
  for (int64_t r = 0; r < rows; ++r) {
    vo_transform_row(X + r * K, K, gamma, eps, flags, y);
    float A = 0.0f;
    for (int64_t k = 0; k < K; ++k) A = fmaxf(A, fabsf(y[k]));
    float sr = A / 448.0f;
    s[r] = sr;
    for (int64_t k = 0; k < K; ++k)
      codes[r * K + k] = (sr == 0.0f) ? 0 : vo_e4m3_encode(y[k] / sr);
  }
  free(y);
  return 0;
}

void vo_decode_fp8(const uint8_t* codes, const float* s, int64_t rows,
                   int64_t K, double* out) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t k = 0; k < K; ++k)
      out[r * K + k] = vo_e4m3_decode(codes[r * K + k]) * (double)s[r];
}

/* ---------------------------------------------------------------- INT8 -- */
/*
 * INT8 symmetric per-row quantization ("FoldQuant W8A8/W4A4 inference ...":
 * INT8 codes with per-row weight scales, activations quantized per token;
 * its OpenVINO commit lists per-token amax scale, round-half-even, clamp):
 * s = max|y| / 127 (fp32), code = clamp(RNE(fp32(y / s)), -127, 127), or 0
 * when s == 0.  Decoded value: code * s.
 */
static int8_t int8_code(float q) {
  float r = nearbyintf(q); /* default rounding mode: half to even */
  if (r > 127.0f) r = 127.0f;
  if (r < -127.0f) r = -127.0f;
  return (int8_t)r;
}

int vo_quantize_int8(const uint16_t* X, int64_t rows, int64_t K, const uint16_t* gamma, float eps,
                     unsigned flags, int8_t* codes, float* s) {
  if (K <= 0 || K % 16 != 0) return -1;
  if ((flags & VO_F_HADAMARD64) && K % 64 != 0) return -1;
  if ((flags & VO_F_RMSNORM) && gamma == NULL) return -1;
  float* y = (float*)malloc(sizeof(float) * (size_t)K);
  for (int64_t r = 0; r < rows; ++r) {
    vo_transform_row(X + r * K, K, gamma, eps, flags, y);
    float A = 0.0f;
    for (int64_t k = 0; k < K; ++k) A = fmaxf(A, fabsf(y[k]));
    float sr = A / 127.0f;
    s[r] = sr;
    for (int64_t k = 0; k < K; ++k) codes[r * K + k] = (sr == 0.0f) ? 0 : int8_code(y[k] / sr);
  }
  free(y);
  return 0;
}

void vo_decode_int8(const int8_t* codes, const float* s, int64_t rows, int64_t K, double* out) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t k = 0; k < K; ++k) out[r * K + k] = (double)codes[r * K + k] * (double)s[r];
}

/* fp32 -> bf16, round to nearest even on the bit pattern (finite inputs). */
static uint16_t f32_to_bf16_rne(float v) {
  uint32_t u;
  memcpy(&u, &v, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/*
 * INT8 GEMM and its epilogue.  The integer sum is exact in any order (the
 * FoldQuant SYCL commit relies on that), so the output has one value:
 * acc = sum_k cx[m, k] cw[n, k] (int64), t = fp32(acc), c = fp32(s_x[m]
 * s_w[n]), y = fp32(t c), y = fp32(y + residual[m, n]) when a residual is
 * given, out = bf16(y) (round to nearest even).  Rows row_idx (all M when
 * NULL; nrows must then equal M).  acc_out (int64 [nrows, N]) may be NULL.
 */
void vo_linear_int8(const int8_t* cx, const float* sx, const int8_t* cw, const float* sw, const uint16_t* residual,
                    int64_t M, int64_t N, int64_t K, const int64_t* row_idx, int64_t nrows, uint16_t* Y,
                    int64_t* acc_out) {
  (void)M;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < nrows; ++i) {
    int64_t m = row_idx ? row_idx[i] : i;
    const int8_t* x = cx + m * K;
    for (int64_t n = 0; n < N; ++n) {
      const int8_t* w = cw + n * K;
      int64_t acc = 0;
      for (int64_t k = 0; k < K; ++k) acc += (int64_t)x[k] * (int64_t)w[k];
      if (acc_out) acc_out[i * N + n] = acc;
      float t = (float)acc;
      float c = sx[m] * sw[n];
      float y = t * c;
      if (residual) y = y + vo_bf16_to_f32(residual[m * N + n]);
      Y[i * N + n] = f32_to_bf16_rne(y);
    }
  }
}

/* ---------------------------------------------------------------- GEMM -- */
/*
 * Y[i, n] = sum_k Xd[row_i, k] * Wd[n, k] + residual[row_i, n], fp64, k in
 * order, for the selected rows row_i = row_idx[i] (all rows when row_idx is
 * NULL; then nrows must equal M).  residual is bf16 [M, N] or NULL.
 */
void vo_linear_f64(const double* Xd, const double* Wd, const uint16_t* residual,
                   int64_t M, int64_t N, int64_t K, const int64_t* row_idx,
                   int64_t nrows, double* Y) {
  (void)M;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < nrows; ++i) {
    int64_t m = row_idx ? row_idx[i] : i;
    const double* x = Xd + m * K;
    for (int64_t n = 0; n < N; ++n) {
      const double* w = Wd + n * K;
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) acc += x[k] * w[k];
      if (residual) acc += (double)vo_bf16_to_f32(residual[m * N + n]);
      Y[i * N + n] = acc;
    }
  }
}

/* Number of OpenMP threads the GEMM above will use (1 without OpenMP). */
int vo_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}
