/*
 * oracle.c -- plain, slow, obviously correct CPU oracle for group-wise 4-bit
 * weight-only quantization (INT4 asymmetric / symmetric and NVFP4) and the
 * quantized Linear Y = X * dequant(Wq)^T.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or helper
 * with the CUDA library; it is written directly from the formulas on the
 * pages it cites.
 *
 * Sources (page title, section):
 *  [P4] "quantization primer" (xingyuwang.me), section 2 "Symmetric 与
 *       Asymmetric Quantization": q = round(x/s) + z, x_hat = (q - z) s, with
 *       clipping to the integer range; symmetric q = round(x/s), x_hat = q s.
 *       Section 3 "Quantization Granularity": per-group scales (32/64/128).
 *       Section 12 "FP8 与 FP4": E4M3 = 1 sign + 4 exponent + 3 mantissa.
 *  [P1] "Lance-Quant" (zingnex.cn), section "量化应用": AWQ grid search over an
 *       activation-aware scale, group-wise INT4 packing; NVFP4 = E2M1 codes
 *       with one FP8-E4M3 scale per 16 elements; min-max fallback when a layer
 *       has no calibration activations (section "校准阶段").
 *  [P2] "OmniQuant" tutorial (cyqw.cn), section 2.1 (scale and zero point)
 *       and section 2.2.2 (equivalence transform Y = (X s)(W / s)).
 *  [P4] section 6 "GPTQ": quantize, estimate the error with second-order
 *       information, adjust the remaining weights, continue.
 *  Where the pages are silent the readings used here are listed next to the
 *  code that takes them (min-max range, 1e-5 scale floor, fp16 scale,
 *  LSB-first nibble order, NVFP4 per-tensor scale amax/(6*448), E2M1 ties to
 *  even code, AWQ loss and alpha grid).
 *
 * Precision: every quantization DECISION (scale, zero, code) is taken in
 * IEEE fp32 with round-to-nearest-even division and rint(), the precision the
 * GPU kernels use, so both sides produce identical codes.  Everything
 * real-valued (dequantized weights, matrix products, AWQ losses) is fp64.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fopenmp -shared -fPIC.
 * -ffp-contract=off keeps a*b+c from fusing, so every fp32 step rounds once.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1

/* ------------------------------------------------------------------ */
/* Scalar codecs                                                        */
/* ------------------------------------------------------------------ */

/* bf16 is the upper half of an IEEE binary32. */
static float bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

double oracle_bf16_to_f64(uint16_t b) { return (double)bf16_to_f32(b); }

/* IEEE binary16 value of a bit pattern (1 sign, 5 exponent bias 15, 10 mantissa). */
double oracle_f16_to_f64(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1F;
  int m = h & 0x3FF;
  double v;
  if (e == 0)
    v = ldexp((double)m, -24); /* subnormal: m * 2^-14 / 1024 */
  else if (e == 31)
    v = m ? NAN : INFINITY;
  else
    v = ldexp(1024.0 + m, e - 25); /* (1 + m/1024) * 2^(e-15) */
  return sign ? -v : v;
}

/* binary16 round-to-nearest-even of a finite fp32 value, saturating at the
 * largest finite half (65504).  Written from the binary16 definition: find
 * the quantum of the binade that holds |x|, round |x|/quantum to an integer
 * with ties to even (exact in fp64), and encode. */
uint16_t oracle_f32_to_f16_rne_sat(float x) {
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  double a = fabs((double)x);
  if (a == 0.0) return sign;
  if (a >= 65504.0) return sign | 0x7BFF;
  int E;
  frexp(a, &E);  /* a = f * 2^E, f in [0.5, 1) -> binade exponent E-1 */
  int e = E - 1;
  if (e < -14) { /* subnormal range: quantum 2^-24 */
    double r = rint(a / ldexp(1.0, -24));
    /* r == 1024 is the smallest normal, whose encoding is also 0x0400 */
    return sign | (uint16_t)r;
  }
  double r = rint(a / ldexp(1.0, e - 10)); /* in [1024, 2048] */
  if (r == 2048.0) { e += 1; r = 1024.0; }
  if (e > 15) return sign | 0x7BFF;
  return sign | (uint16_t)(((e + 15) << 10) | ((int)r - 1024));
}

/* FP8 E4M3 ("FP8 与 FP4": 1 sign, 4 exponent, 3 mantissa).  Bias 7, no
 * infinities, S.1111.111 is NaN, largest finite 448, subnormals m/8 * 2^-6. */
double oracle_e4m3_decode(uint8_t b) {
  int sign = b >> 7;
  int e = (b >> 3) & 0xF;
  int m = b & 7;
  double v;
  if (e == 15 && m == 7)
    v = NAN;
  else if (e == 0)
    v = ldexp((double)m, -9);
  else
    v = ldexp(8.0 + m, e - 10); /* (1 + m/8) * 2^(e-7) */
  return sign ? -v : v;
}

/* Nearest non-negative finite E4M3 code to v >= 0 by exhaustive search over
 * all 127 codes, ties to the even code (even mantissa), saturating: any v
 * above 448 maps to 448.  This is round-to-nearest-even with satfinite. */
uint8_t oracle_e4m3_encode_sat(float v) {
  double x = (double)v;
  int best = 0;
  double bestd = INFINITY;
  for (int c = 0; c <= 0x7E; ++c) {
    double d = fabs(x - oracle_e4m3_decode((uint8_t)c));
    if (d < bestd || (d == bestd && (c & 1) == 0 && (best & 1) == 1)) {
      best = c;
      bestd = d;
    }
  }
  return (uint8_t)best;
}

/* E2M1 (FP4): 1 sign, 2 exponent, 1 mantissa.  Magnitudes by code 0..7:
 * 0, 0.5, 1, 1.5, 2, 3, 4, 6 (the NVFP4 code set). */
double oracle_e2m1_decode(uint8_t code) {
  static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  double v = mag[code & 7];
  return (code & 8) ? -v : v;
}

/* Nearest E2M1 magnitude to |v| by exhaustive search, ties to the even code,
 * saturating at 6; the sign bit copies the sign bit of v (so a negative value
 * that rounds to zero is encoded 0x8). */
uint8_t oracle_e2m1_encode(float v) {
  double a = fabs((double)v);
  int best = 0;
  double bestd = INFINITY;
  for (int c = 0; c < 8; ++c) {
    double d = fabs(a - oracle_e2m1_decode((uint8_t)c));
    if (d < bestd || (d == bestd && (c & 1) == 0 && (best & 1) == 1)) {
      best = c;
      bestd = d;
    }
  }
  return (uint8_t)(best | (signbit(v) ? 8 : 0));
}

/* ------------------------------------------------------------------ */
/* INT4 group-wise quantization ([P4] section 2 and 3)                 */
/* ------------------------------------------------------------------ */

/* w' = W (bf16) optionally times the per-input-channel AWQ scale s[k], one
 * fp32 multiply. */
static float wprime(const uint16_t* W, const float* s, int64_t K, int64_t n, int64_t k) {
  float w = bf16_to_f32(W[n * K + k]);
  return s ? w * s[k] : w;
}

/* Scale of one group, from the fp32 range r (asymmetric: max-min over 15
 * levels; symmetric: max|w| over 7 levels).  Reading of the pages: min-max
 * range ("simple min-max", Lance-Quant), a 1e-5 floor for degenerate
 * groups, stored as fp16 (round to nearest even, saturating).  Returns the
 * fp16 bits; *sc gets its value as fp32. */
static uint16_t group_scale(float r, float levels, float* sc) {
  float sc32 = r / levels;
  if (!(sc32 >= 1e-5f)) sc32 = 1e-5f;
  if (sc32 > 65504.0f) sc32 = 65504.0f;
  uint16_t h = oracle_f32_to_f16_rne_sat(sc32);
  *sc = (float)oracle_f16_to_f64(h);
  return h;
}

static float clampf(float v, float lo, float hi) { return v < lo ? lo : (v > hi ? hi : v); }

/* INT4 quantize-and-pack of W [N, K] (row n = output channel, K = input).
 *   asymmetric (zero_point=1): sc = fp16(max((mx-mn)/15, 1e-5)),
 *     z = clamp(rint(-mn/sc), 0, 15), q = clamp(rint(w'/sc) + z, 0, 15)
 *   symmetric  (zero_point=0): sc = fp16(max(max|w'|/7, 1e-5)),
 *     q = clamp(rint(w'/sc), -7, 7) + 8 (stored offset-8, no zeros)
 * rint() rounds half to even.  Packing (pages silent; chosen LSB-first):
 *   qweight[n][k/8] nibble k%8 = q(n,k)          (uint32, N x K/8)
 *   scales[n][g] = fp16 bits                       (uint16, N x K/G)
 *   zeros[n][g/8] nibble g%8 = z(n,g), pad = 0     (uint32, N x ceil(K/G/8))
 */
int oracle_quantize_int4(const uint16_t* W, int64_t N, int64_t K, int bits, int group_size,
                         int zero_point, const float* s, uint32_t* qweight, uint16_t* scales,
                         uint32_t* zeros) {
  if (bits != 4 || N <= 0 || K <= 0 || group_size <= 0 || K % group_size || K % 8) return ORACLE_ERR_ARG;
  if (zero_point && !zeros) return ORACLE_ERR_ARG;
  const int64_t G = group_size, ng = K / G, nzw = (ng + 7) / 8;
  memset(qweight, 0, (size_t)(N * (K / 8)) * sizeof(uint32_t));
  if (zero_point) memset(zeros, 0, (size_t)(N * nzw) * sizeof(uint32_t));
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t g = 0; g < ng; ++g) {
      float mn = INFINITY, mx = -INFINITY, amax = 0.0f;
      for (int64_t k = g * G; k < (g + 1) * G; ++k) {
        float w = wprime(W, s, K, n, k);
        if (w < mn) mn = w;
        if (w > mx) mx = w;
        if (fabsf(w) > amax) amax = fabsf(w);
      }
      float sc;
      float z = 0.0f;
      if (zero_point) {
        scales[n * ng + g] = group_scale(mx - mn, 15.0f, &sc);
        z = clampf(rintf(-mn / sc), 0.0f, 15.0f);
        zeros[n * nzw + g / 8] |= (uint32_t)z << (4 * (g % 8));
      } else {
        scales[n * ng + g] = group_scale(amax, 7.0f, &sc);
      }
      for (int64_t k = g * G; k < (g + 1) * G; ++k) {
        float w = wprime(W, s, K, n, k);
        float q = zero_point ? clampf(rintf(w / sc) + z, 0.0f, 15.0f)
                             : clampf(rintf(w / sc), -7.0f, 7.0f) + 8.0f;
        qweight[n * (K / 8) + k / 8] |= (uint32_t)q << (4 * (k % 8));
      }
    }
  }
  return ORACLE_OK;
}

/* Unpack one INT4 code. */
static int int4_code(const uint32_t* qweight, int64_t K, int64_t n, int64_t k) {
  return (qweight[n * (K / 8) + k / 8] >> (4 * (k % 8))) & 0xF;
}

/* Dequantize rows `rows[0..nrows)` (or all N rows if rows == NULL) of an INT4
 * pack: w_hat = (q - z) * sc in fp64 ([P4] section 2).  out is nrows x K. */
void oracle_dequant_int4(const uint32_t* qweight, const uint16_t* scales, const uint32_t* zeros,
                         int64_t N, int64_t K, int group_size, int zero_point, const int64_t* rows,
                         int64_t nrows, double* out) {
  const int64_t G = group_size, ng = K / G, nzw = (ng + 7) / 8;
  if (!rows) nrows = N;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < nrows; ++i) {
    int64_t n = rows ? rows[i] : i;
    for (int64_t k = 0; k < K; ++k) {
      int64_t g = k / G;
      double sc = oracle_f16_to_f64(scales[n * ng + g]);
      int z = zero_point ? (int)((zeros[n * nzw + g / 8] >> (4 * (g % 8))) & 0xF) : 8;
      out[i * K + k] = (double)(int4_code(qweight, K, n, k) - z) * sc;
    }
  }
}

/* ------------------------------------------------------------------ */
/* NVFP4 ([P1] "nvfp4_apply.py"; [P4] section 12)                       */
/* ------------------------------------------------------------------ */

/* NVFP4 quantize of A [R, C] (weights: R = N, C = K; activations: R = M).
 *   g   = amax(|A'|) / (6 * 448) in fp32 (1 if the tensor is all zero)
 *   per 16 consecutive elements of a row: sb = E4M3_satfinite((amax_b / 6) / g)
 *   code = E2M1(A' / (dec(sb) * g)), all codes 0 when dec(sb) == 0
 * Reading of the pages: the fp32 per-tensor scale and its formula are not on
 * the pages (only "E2M1 + FP8 E4M3 per 16"); this is the plainest choice that
 * makes the largest block scale land on the E4M3 maximum.
 * Packing: codes[r][c/2], low nibble = even c; bscale[r][c/16]; *g_out = g.
 * s (optional, length C) multiplies column c before quantization. */
int oracle_quantize_nvfp4(const uint16_t* A, int64_t R, int64_t C, const float* s, uint8_t* codes,
                          uint8_t* bscale, float* g_out) {
  if (R <= 0 || C <= 0 || C % 16) return ORACLE_ERR_ARG;
  float amax = 0.0f;
  for (int64_t r = 0; r < R; ++r)
    for (int64_t c = 0; c < C; ++c) {
      float a = fabsf(wprime(A, s, C, r, c));
      if (a > amax) amax = a;
    }
  const float g = amax > 0.0f ? amax / 2688.0f : 1.0f;
  *g_out = g;
  memset(codes, 0, (size_t)(R * C / 2));
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < R; ++r) {
    for (int64_t b = 0; b < C / 16; ++b) {
      float ab = 0.0f;
      for (int64_t c = b * 16; c < b * 16 + 16; ++c) {
        float a = fabsf(wprime(A, s, C, r, c));
        if (a > ab) ab = a;
      }
      float t = (ab / 6.0f) / g;
      uint8_t sb = oracle_e4m3_encode_sat(t);
      bscale[r * (C / 16) + b] = sb;
      float d = (float)oracle_e4m3_decode(sb);
      if (d == 0.0f) continue; /* codes stay 0 */
      float denom = d * g;
      for (int64_t c = b * 16; c < b * 16 + 16; ++c) {
        float v = wprime(A, s, C, r, c) / denom;
        uint8_t code = oracle_e2m1_encode(v);
        codes[r * (C / 2) + c / 2] |= (uint8_t)(code << (4 * (c % 2)));
      }
    }
  }
  return ORACLE_OK;
}

/* NVFP4 dequantize: e2m1(code) * dec(sb) * g in fp64; rows as for INT4. */
void oracle_dequant_nvfp4(const uint8_t* codes, const uint8_t* bscale, float g, int64_t R, int64_t C,
                          const int64_t* rows, int64_t nrows, double* out) {
  if (!rows) nrows = R;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < nrows; ++i) {
    int64_t r = rows ? rows[i] : i;
    for (int64_t c = 0; c < C; ++c) {
      uint8_t code = (codes[r * (C / 2) + c / 2] >> (4 * (c % 2))) & 0xF;
      out[i * C + c] = oracle_e2m1_decode(code) * oracle_e4m3_decode(bscale[r * (C / 16) + c / 16]) * (double)g;
    }
  }
}

/* ------------------------------------------------------------------ */
/* Linear ([P4] section 4 "W4A16": weights 4-bit, activations 16-bit)   */
/* ------------------------------------------------------------------ */

/* bf16 activations [M, K] to fp64, each column optionally times inv_s[k]
 * (the AWQ transform (X / s)(W s)^T, [P2] section 2.2.2). */
void oracle_activations_f64(const uint16_t* X, int64_t M, int64_t K, const float* inv_s, double* out) {
  for (int64_t m = 0; m < M; ++m)
    for (int64_t k = 0; k < K; ++k) {
      double x = oracle_bf16_to_f64(X[m * K + k]);
      out[m * K + k] = inv_s ? x * (double)inv_s[k] : x;
    }
}

/* Y [M, N] = A [M, K] * B [N, K]^T, textbook fp64 dot products. */
void oracle_matmul_abT(const double* A, int64_t M, int64_t K, const double* B, int64_t N, double* Y) {
#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) acc += A[m * K + k] * B[n * K + k];
      Y[m * N + n] = acc;
    }
}

/* ------------------------------------------------------------------ */
/* AWQ grid search ([P1] "awq_apply.py"; [P4] section 7 AWQ)           */
/* ------------------------------------------------------------------ */

/* Delta = W - dequant(Q(W s)) / s in fp64 for one AWQ scale s (asymmetric
 * INT4, group_size): the weight error the AWQ loss measures.  out is N x K. */
int oracle_awq_delta(const uint16_t* W, int64_t N, int64_t K, const float* s, int group_size, double* out) {
  if (N <= 0 || K <= 0 || K % group_size || !s) return ORACLE_ERR_ARG;
  const int64_t ng = K / group_size, nzw = (ng + 7) / 8;
  uint32_t* qw = malloc(sizeof(uint32_t) * N * (K / 8));
  uint16_t* sc = malloc(sizeof(uint16_t) * N * ng);
  uint32_t* zr = malloc(sizeof(uint32_t) * N * nzw);
  oracle_quantize_int4(W, N, K, 4, group_size, 1, s, qw, sc, zr);
  oracle_dequant_int4(qw, sc, zr, N, K, group_size, 1, NULL, 0, out);
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) out[n * K + k] = oracle_bf16_to_f64(W[n * K + k]) - out[n * K + k] / (double)s[k];
  free(qw); free(sc); free(zr);
  return ORACLE_OK;
}

/* For each alpha_i: s_k = fp32(a_k ^ alpha_i) with a_k = max(mean_t |X_tk|, 1e-4)
 * (or the given act_mean when X is NULL), W' = Q(W s) by the INT4 rule above
 * (asymmetric, group_size G), Delta = W - dequant(W') / s, and
 *   L(alpha) = || X Delta^T ||_F^2                     (X given)
 *   L(alpha) = sum_{n,k} (a_k Delta_nk)^2              (X NULL: only mean |x|
 *                                                       is known, as in Lance's
 *                                                       saved statistics)
 * best = first argmin; s_out = the s of best.  All of L in fp64.
 * Readings: the loss form and the grid are not on the pages (only "grid
 * search" over an activation-aware scale); the diagonal proxy is the plainest
 * loss computable from mean |activation| alone. */
int oracle_awq_search(const uint16_t* W, int64_t N, int64_t K, const uint16_t* X, int64_t T,
                      const float* act_mean, const float* alphas, int n_alpha, int group_size,
                      float* s_out, double* loss_out, int* best_out) {
  if (N <= 0 || K <= 0 || n_alpha <= 0 || K % group_size) return ORACLE_ERR_ARG;
  if (X && T <= 0) return ORACLE_ERR_ARG;
  if (!X && !act_mean) return ORACLE_ERR_ARG;
  double* a = malloc(sizeof(double) * K);
  float* s = malloc(sizeof(float) * K);
  double* delta = malloc(sizeof(double) * N * K);
  double* xd = X ? malloc(sizeof(double) * T * K) : NULL;
  double* y = X ? malloc(sizeof(double) * T * N) : NULL;
  for (int64_t k = 0; k < K; ++k) {
    double m = 0.0;
    if (X) {
      for (int64_t t = 0; t < T; ++t) m += fabs(oracle_bf16_to_f64(X[t * K + k]));
      m /= (double)T;
    } else {
      m = (double)act_mean[k];
    }
    a[k] = m > 1e-4 ? m : 1e-4;
  }
  if (X) oracle_activations_f64(X, T, K, NULL, xd);
  int best = 0;
  for (int i = 0; i < n_alpha; ++i) {
    for (int64_t k = 0; k < K; ++k) s[k] = (float)pow(a[k], (double)alphas[i]);
    oracle_awq_delta(W, N, K, s, group_size, delta);
    double L = 0.0;
    if (X) {
      oracle_matmul_abT(xd, T, K, delta, N, y);
      for (int64_t j = 0; j < T * N; ++j) L += y[j] * y[j];
    } else {
      for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
          double v = a[k] * delta[n * K + k];
          L += v * v;
        }
    }
    loss_out[i] = L;
    if (L < loss_out[best]) best = i;
  }
  for (int64_t k = 0; k < K; ++k) s_out[k] = (float)pow(a[k], (double)alphas[best]);
  *best_out = best;
  free(a); free(s); free(delta); free(xd); free(y);
  return ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* GPTQ ([P4] section 6 "GPTQ")                                          */
/* ------------------------------------------------------------------ */

/* GPTQ INT4 quantize-and-pack.  The page gives the loop only: quantize a
 * weight, estimate its error with approximate second-order information,
 * adjust the weights not yet quantized, continue; 4-bit weights, calibration
 * data, group size 128 and no activation reordering in its example.
 * Readings taken here:
 *  - the second-order information is the upper Cholesky factor U of the
 *    damped inverse Hessian of the calibration activations (U^T U =
 *    (2 X^T X + lambda I)^-1), given by the caller in fp32;
 *  - columns are quantized in order k = 0..K-1, every row on its own;
 *  - a group's scale and zero point come from the plain quantizer's min-max
 *    rule applied to the group's weights as they stand when its first column
 *    is reached (after the adjustments from earlier columns);
 *  - the error of column k is e_k = (w_k - dequant(q_k)) / U[k][k], and every
 *    later column j is adjusted by w_j = w_j - e_k * U[k][j], k in increasing
 *    order; the arithmetic is fp32 (the precision in which the codes, an
 *    integer decision, are taken), each +, -, *, / rounded on its own (IEEE
 *    round-to-nearest-even; this file is compiled without contraction into
 *    fused multiply-adds).
 * In exact arithmetic this gives W - dequant(Q) = E U row by row, which the
 * tests check.  err (optional, fp32 [N, K]) receives the e_k. */
int oracle_gptq_int4(const uint16_t* W, int64_t N, int64_t K, const float* U, int group_size, int zero_point,
                     uint32_t* qweight, uint16_t* scales, uint32_t* zeros, float* err) {
  if (N <= 0 || K <= 0 || group_size <= 0 || K % group_size || K % 8 || !U) return ORACLE_ERR_ARG;
  if (zero_point && !zeros) return ORACLE_ERR_ARG;
  const int64_t G = group_size, ng = K / G, nzw = (ng + 7) / 8;
  memset(qweight, 0, (size_t)(N * (K / 8)) * sizeof(uint32_t));
  if (zero_point) memset(zeros, 0, (size_t)(N * nzw) * sizeof(uint32_t));
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t n = 0; n < N; ++n) {
    float* w = (float*)malloc((size_t)K * sizeof(float));
    if (!w) {
#pragma omp atomic write
      bad = 1;
      continue;
    }
    for (int64_t k = 0; k < K; ++k) w[k] = bf16_to_f32(W[n * K + k]);
    float sc = 1.0f, z = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      if (k % G == 0) {  /* the group's scale and zero point from its current weights */
        const int64_t g = k / G;
        float mn = INFINITY, mx = -INFINITY, amax = 0.0f;
        for (int64_t i = k; i < k + G; ++i) {
          if (w[i] < mn) mn = w[i];
          if (w[i] > mx) mx = w[i];
          if (fabsf(w[i]) > amax) amax = fabsf(w[i]);
        }
        if (zero_point) {
          scales[n * ng + g] = group_scale(mx - mn, 15.0f, &sc);
          z = clampf(rintf(-mn / sc), 0.0f, 15.0f);
          zeros[n * nzw + g / 8] |= (uint32_t)z << (4 * (g % 8));
        } else {
          scales[n * ng + g] = group_scale(amax, 7.0f, &sc);
          z = 8.0f;
        }
      }
      /* quantize the weight */
      const float q = zero_point ? clampf(rintf(w[k] / sc) + z, 0.0f, 15.0f)
                                 : clampf(rintf(w[k] / sc), -7.0f, 7.0f) + 8.0f;
      qweight[n * (K / 8) + k / 8] |= (uint32_t)q << (4 * (k % 8));
      /* estimate its error, scaled by the second-order information */
      const float deq = (q - z) * sc; /* exact: |q - z| <= 15, sc has 11 significant bits */
      const float e = (w[k] - deq) / U[k * K + k];
      if (err) err[n * K + k] = e;
      /* adjust the weights not yet quantized */
      for (int64_t j = k + 1; j < K; ++j) w[j] = w[j] - e * U[k * K + j];
    }
    free(w);
  }
  return bad ? ORACLE_ERR_ARG : ORACLE_OK;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
