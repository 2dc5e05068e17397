// awq.cuh -- AWQ grid search of the per-input-channel scale.
//
// "Lance-Quant", section "量化应用": awq_apply.py grid-searches an AWQ scale
// equalization per layer before group-wise INT4 packing; section "校准阶段":
// the calibration statistic is the mean absolute activation per input
// channel.  "quantization primer", section 7 (AWQ): salient channels are
// found from activation magnitudes and protected by scaling.
//
// For every alpha of the grid:
//   s_k   = fp32(a_k ^ alpha),  a_k = max(mean_t |X[t,k]|, 1e-4)
//   Delta = W - dequant(Q(W s)) / s           (asymmetric INT4, group G)
//   L     = || X Delta^T ||_F^2               (tcgen05 GEMM, sum-of-squares epilogue)
//   or, with no calibration tokens, L = sum_{n,k} (a_k Delta[n,k])^2.
// Delta is stored as two bf16 planes (hi = bf16(Delta), lo = bf16(Delta - hi))
// side by side, [N, 2K], so the loss GEMM X [T, K] x [hi | lo]^T over a
// reduction of 2K keeps ~16 significant bits of Delta with bf16 tensor cores.
// Every partial sum is written to its own slot and summed in a fixed order
// in fp64: the losses are bit-reproducible run to run.
#pragma once

#include "quant.cuh"
#include "wq_common.cuh"

namespace wq {

// a[k] = max(mean_t |X[t, k]|, 1e-4) (fp64), or max(act_mean[k], 1e-4).
__global__ void __launch_bounds__(256) awq_act_mean_kernel(const uint16_t* __restrict__ X, int64_t T, int64_t K,
                                                           const float* __restrict__ act_mean, double* __restrict__ a) {
  const int64_t k = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (k >= K) return;
  double m;
  if (X) {
    double acc = 0.0;
    for (int64_t t = 0; t < T; ++t) acc += fabs(double(bf16_bits_to_f32(X[t * K + k])));
    m = acc / double(T);
  } else {
    m = double(act_mean[k]);
  }
  a[k] = m > 1e-4 ? m : 1e-4;
}

// s[k] = fp32(a[k] ^ alpha), alpha read from device memory.
__global__ void __launch_bounds__(256) awq_scale_kernel(const double* __restrict__ a, const float* __restrict__ alpha,
                                                        int64_t K, float* __restrict__ s) {
  const int64_t k = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (k < K) s[k] = float(pow(a[k], double(*alpha)));
}

// Delta of one INT4 quantization round trip at scale s, same decisions as
// quantize_int4_kernel (asymmetric).  grid = (ceil(K/2048), N).
//   D != null: write Delta as bf16 hi at D[n, k] and lo at D[n, K + k].
//   D == null: partials[cta] = sum over the CTA of (a_k * Delta[n,k])^2.
template <int G>
__global__ void __launch_bounds__(kQuantThreads) awq_delta_kernel(const uint16_t* __restrict__ W,
                                                                  const float* __restrict__ s, int64_t N, int64_t K,
                                                                  uint16_t* __restrict__ D,
                                                                  const double* __restrict__ a,
                                                                  double* __restrict__ partials) {
  constexpr int LPG = G / 8;
  const int64_t n = blockIdx.y;
  const int64_t words = K / 8;
  const int64_t u = int64_t(blockIdx.x) * kQuantThreads + threadIdx.x;
  const bool active = u < words;
  const int64_t k = u * 8;
  float w[8], wp[8];
  float mn = INFINITY, mx = -INFINITY;
  if (active) {
    load_wprime8(W, nullptr, K, n, k, w);
    load_wprime8(W, s, K, n, k, wp);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      mn = fminf(mn, wp[j]);
      mx = fmaxf(mx, wp[j]);
    }
  }
#pragma unroll
  for (int off = 1; off < LPG; off <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  }
  float sc;
  group_scale_f16_fast(__fsub_rn(mx, mn), 15.0f, 1.0f / 15.0f, &sc);
  // z = rint(-mn / sc) and q = rint(w' / sc) as the quantizer takes them: through the
  // reciprocal, with the IEEE division (in a branch of its own) where the product
  // lies within 2^-21 |t| of a half-integer
  const float rsc = __frcp_rn(sc);
  const float tz = __fmul_rn(-mn, rsc);
  float zr = rintf(tz);
  if (__builtin_expect(__fsub_rn(0.5f, fabsf(__fsub_rn(tz, zr))) <= fabsf(tz) * 0x1p-21f, 0))
    zr = rintf(__fdiv_rn(-mn, sc));
  const float z = fminf(fmaxf(zr, 0.0f), 15.0f);
  double sq = 0.0;
  if (active) {
    float sv[8];
    {
      const float4 s0 = __ldg(reinterpret_cast<const float4*>(s + k));
      const float4 s1 = __ldg(reinterpret_cast<const float4*>(s + k + 4));
      sv[0] = s0.x; sv[1] = s0.y; sv[2] = s0.z; sv[3] = s0.w;
      sv[4] = s1.x; sv[5] = s1.y; sv[6] = s1.z; sv[7] = s1.w;
    }
    float qr[8];
    uint32_t slow = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float t = __fmul_rn(wp[j], rsc);
      qr[j] = rintf(t);
      if (__fsub_rn(0.5f, fabsf(__fsub_rn(t, qr[j]))) <= fabsf(t) * 0x1p-21f) slow |= 1u << j;
    }
    if (__builtin_expect(slow != 0, 0)) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (slow & (1u << j)) qr[j] = rintf(__fdiv_rn(wp[j], sc));
    }
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float q = fminf(fmaxf(__fadd_rn(qr[j], z), 0.0f), 15.0f);
      const float deq = __fmul_rn(__fsub_rn(q, z), sc);  // exact: |q - z| <= 15, sc has 11 bits
      // W - dequant / s, the quotient through the correctly rounded reciprocal of s
      // (within an ulp of the division; Delta then travels as a bf16 hi + lo pair)
      const float dl = __fsub_rn(w[j], __fmul_rn(deq, __frcp_rn(sv[j])));
      if (D) {
        const uint32_t h = f32_to_bf16_bits(dl);
        const uint32_t l = f32_to_bf16_bits(__fsub_rn(dl, bf16_bits_to_f32(h)));
        if (j & 1) { hi[j >> 1] |= h << 16; lo[j >> 1] |= l << 16; }
        else { hi[j >> 1] = h; lo[j >> 1] = l; }
      } else {
        const double v = a[k + j] * double(dl);
        sq += v * v;
      }
    }
    if (D) {
      *reinterpret_cast<uint4*>(D + n * 2 * K + k) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(D + n * 2 * K + K + k) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
  }
  if (!D) {
    // fixed-order block reduction -> one partial per CTA
    __shared__ double red[kQuantThreads / 32];
#pragma unroll
    for (int off = 16; off; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = sq;
    __syncthreads();
    if (threadIdx.x == 0) {
      double t = 0.0;
      for (int i = 0; i < kQuantThreads / 32; ++i) t += red[i];
      partials[int64_t(blockIdx.y) * gridDim.x + blockIdx.x] = t;
    }
  }
}

// ------------------------------------------------------------------ diagonal proxy, all alphas at once
// Without calibration tokens the loss of alpha_i is sum_{n,k} (a_k Delta_i[n,k])^2
// and needs W only: one pass over W evaluates every alpha.  A CTA keeps 4 rows x
// 1024 k of W in registers and loops over the alphas (s and 1/s per alpha from a
// small table that stays in L2), so W is read from HBM once instead of once per
// alpha.  The codes take the quantizer's decisions: rint(w'/scale) through a
// reciprocal, with the IEEE division where the product lies near a rounding tie.
// Delta = w - deq * (1/s) in fp32 and the squares are summed per thread in fp32,
// then in fp64 across the CTA in a fixed order, one partial per (alpha, CTA).
constexpr int kAwqProxyRows = 4;
constexpr int kAwqProxyThreads = 128;   // 128 x 8 = 1024 k per CTA
constexpr int kAwqProxyMaxAlphas = 32;

// tab[i][k] = s = fp32(a_k ^ alpha_i), tab[n_alpha + i][k] = fp32 1 / s, tab[2 n_alpha][k] = fp32(a_k).
__global__ void __launch_bounds__(256) awq_proxy_table_kernel(const double* __restrict__ a,
                                                              const float* __restrict__ alphas, int n_alpha,
                                                              int64_t K, float* __restrict__ tab) {
  const int64_t k = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const int i = blockIdx.y;
  if (k >= K) return;
  if (i < n_alpha) {
    const float sv = float(pow(a[k], double(alphas[i])));
    tab[int64_t(i) * K + k] = sv;
    tab[int64_t(n_alpha + i) * K + k] = __frcp_rn(sv);
  } else {
    tab[int64_t(2 * n_alpha) * K + k] = float(a[k]);
  }
}

// grid = (ceil(K / 1024), ceil(N / 4)); partials[i * P + p0 + blockIdx.y * gridDim.x + blockIdx.x].
template <int G>
__global__ void __launch_bounds__(kAwqProxyThreads) awq_proxy_kernel(const uint16_t* __restrict__ W, int64_t N,
                                                                     int64_t K, const float* __restrict__ tab,
                                                                     int n_alpha, double* __restrict__ partials,
                                                                     int64_t P, int64_t p0) {
  constexpr int LPG = G / 8;
  __shared__ double red[kAwqProxyThreads / 32][kAwqProxyMaxAlphas];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t k = (int64_t(blockIdx.x) * kAwqProxyThreads + threadIdx.x) * 8;
  const bool kin = k < K;
  const int64_t row0 = int64_t(blockIdx.y) * kAwqProxyRows;
  uint4 wr[kAwqProxyRows];
  bool rin[kAwqProxyRows];
#pragma unroll
  for (int r = 0; r < kAwqProxyRows; ++r) {
    rin[r] = kin && row0 + r < N;
    wr[r] = rin[r] ? ldg_stream_v4(W + (row0 + r) * K + k) : make_uint4(0, 0, 0, 0);
  }
  float av[8];
  if (kin) {
    const float4 a0 = __ldg(reinterpret_cast<const float4*>(tab + int64_t(2 * n_alpha) * K + k));
    const float4 a1 = __ldg(reinterpret_cast<const float4*>(tab + int64_t(2 * n_alpha) * K + k + 4));
    av[0] = a0.x; av[1] = a0.y; av[2] = a0.z; av[3] = a0.w; av[4] = a1.x; av[5] = a1.y; av[6] = a1.z; av[7] = a1.w;
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) av[j] = 0.f;
  }
  for (int i = 0; i < n_alpha; ++i) {
    float sv[8], rv[8];
    if (kin) {
      const float* st = tab + int64_t(i) * K + k;
      const float* rt = tab + int64_t(n_alpha + i) * K + k;
      const float4 s0 = __ldg(reinterpret_cast<const float4*>(st)), s1 = __ldg(reinterpret_cast<const float4*>(st + 4));
      const float4 r0 = __ldg(reinterpret_cast<const float4*>(rt)), r1 = __ldg(reinterpret_cast<const float4*>(rt + 4));
      sv[0] = s0.x; sv[1] = s0.y; sv[2] = s0.z; sv[3] = s0.w; sv[4] = s1.x; sv[5] = s1.y; sv[6] = s1.z; sv[7] = s1.w;
      rv[0] = r0.x; rv[1] = r0.y; rv[2] = r0.z; rv[3] = r0.w; rv[4] = r1.x; rv[5] = r1.y; rv[6] = r1.z; rv[7] = r1.w;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) sv[j] = rv[j] = 1.f;
    }
    float sq = 0.f;
#pragma unroll
    for (int r = 0; r < kAwqProxyRows; ++r) {
      const uint32_t u[4] = {wr[r].x, wr[r].y, wr[r].z, wr[r].w};
      float w[8], wp[8];
      float mn = INFINITY, mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        w[j] = __uint_as_float((j & 1) ? (u[j >> 1] & 0xFFFF0000u) : (u[j >> 1] << 16));
        wp[j] = __fmul_rn(w[j], sv[j]);
        mn = fminf(mn, wp[j]);
        mx = fmaxf(mx, wp[j]);
      }
#pragma unroll
      for (int off = 1; off < LPG; off <<= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      }
      if (!rin[r]) continue;  // whole groups share rin (a group never straddles rows or K)
      float sc;
      group_scale_f16_fast(__fsub_rn(mx, mn), 15.0f, 1.0f / 15.0f, &sc);
      const float rsc = __frcp_rn(sc);
      // z = rint(-mn / sc) and q = rint(wp / sc) through the reciprocal: |t - x / sc|
      // <= ~2^-22 |t| with |t| <= ~16, so rint(t) is the quotient's rint unless t lies
      // within 1e-5 of a half-integer; those few take the division in a branch of
      // their own (not issued, predicated off, for every weight)
      const float tz = __fmul_rn(-mn, rsc);
      float zr = rintf(tz);
      float qr[8];
      uint32_t slow = __fsub_rn(0.5f, fabsf(__fsub_rn(tz, zr))) < 1e-5f ? 0x100u : 0u;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float t = __fmul_rn(wp[j], rsc);
        qr[j] = rintf(t);
        if (__fsub_rn(0.5f, fabsf(__fsub_rn(t, qr[j]))) < 1e-5f) slow |= 1u << j;  // |t - rint(t)| <= 0.5
      }
      if (__builtin_expect(slow != 0, 0)) {
        if (slow & 0x100u) zr = rintf(__fdiv_rn(-mn, sc));
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (slow & (1u << j)) qr[j] = rintf(__fdiv_rn(wp[j], sc));
      }
      // q - z = clamp(rint + z, 0, 15) - z = clamp(rint, -z, 15 - z), exactly (small integers)
      const float z = fminf(fmaxf(zr, 0.0f), 15.0f), lo_q = -z, hi_q = __fsub_rn(15.0f, z);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float deq = __fmul_rn(fminf(fmaxf(qr[j], lo_q), hi_q), sc);
        const float v = __fmul_rn(av[j], __fsub_rn(w[j], __fmul_rn(deq, rv[j])));
        sq = __fmaf_rn(v, v, sq);
      }
    }
    double d = double(sq);
#pragma unroll
    for (int off = 16; off; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
    if (lane == 0) red[warp][i] = d;
  }
  __syncthreads();
  if (int(threadIdx.x) < n_alpha) {
    double t = 0.0;
#pragma unroll
    for (int w2 = 0; w2 < kAwqProxyThreads / 32; ++w2) t += red[w2][threadIdx.x];
    partials[int64_t(threadIdx.x) * P + p0 + int64_t(blockIdx.y) * gridDim.x + blockIdx.x] = t;
  }
}

// loss[i] = sum of partials[i*P .. i*P+P) (fp64, fixed order), best = first
// argmin, s_out = fp32(a ^ alphas[best]).  One CTA of 256 threads.
__global__ void __launch_bounds__(256) awq_finalize_kernel(const double* __restrict__ partials, int64_t P, int n_alpha,
                                                           const double* __restrict__ a,
                                                           const float* __restrict__ alphas, int64_t K,
                                                           float* __restrict__ loss_out, int* __restrict__ best_out,
                                                           float* __restrict__ s_out) {
  __shared__ double losses[1024];
  __shared__ int best_sh;
  // one warp per alpha: lane-strided sums, then a butterfly over the lanes (a fixed
  // order for a given P, so the losses are reproducible)
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int i = warp; i < n_alpha; i += nwarps) {
    double t = 0.0;
    for (int64_t j = lane; j < P; j += 32) t += partials[int64_t(i) * P + j];
#pragma unroll
    for (int off = 16; off; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
    if (lane == 0) {
      losses[i] = t;
      loss_out[i] = float(t);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int b = 0;
    for (int i = 1; i < n_alpha; ++i)
      if (losses[i] < losses[b]) b = i;
    best_sh = b;
    *best_out = b;
  }
  __syncthreads();
  const double al = double(alphas[best_sh]);
  for (int64_t k = threadIdx.x; k < K; k += blockDim.x) s_out[k] = float(pow(a[k], al));
}

}  // namespace wq
