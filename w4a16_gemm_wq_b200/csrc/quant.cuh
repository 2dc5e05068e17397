// quant.cuh -- stage 1 kernels: group-wise INT4 quantize+pack and NVFP4 pack.
//
// INT4 rule ("quantization primer", sections 2-3; "OmniQuant" section 2.1):
// q = clamp(round(w'/scale) + z, 0, 15) per group of G consecutive k with a
// min-max scale and zero point.  NVFP4 ("Lance-Quant", section "量化应用";
// "quantization primer", section 12): E2M1 codes, one E4M3 scale per 16 k,
// one fp32 scale per tensor.  Every decision is taken in fp32 with IEEE
// round-to-nearest-even arithmetic (__fdiv_rn / __fmul_rn, never fused) so
// the packed bytes are bit-exact and reproducible.
//
// Both kernels are HBM-bound streaming passes: each thread reads 16 bytes
// (8 bf16) with one 128-bit load and writes one 32-bit word of codes.
#pragma once

#include <cuda_fp16.h>

#include "wq_common.cuh"

namespace wq {

// ------------------------------------------------------------------ INT4
constexpr int kQuantThreads = 256;  // one row chunk of 256 * 8 = 2048 k per CTA

// Loads 8 consecutive bf16 weights of row n starting at k (k % 8 == 0) and
// applies the optional per-channel AWQ scale (one fp32 multiply each).
__device__ __forceinline__ void load_wprime8(const uint16_t* __restrict__ W, const float* __restrict__ s,
                                             int64_t K, int64_t n, int64_t k, float w[8]) {
  const uint4 v = ldg_stream_v4(W + n * K + k);
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    w[2 * j] = __uint_as_float(u[j] << 16);
    w[2 * j + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
  }
  if (s) {
    const float4 s0 = __ldg(reinterpret_cast<const float4*>(s + k));
    const float4 s1 = __ldg(reinterpret_cast<const float4*>(s + k + 4));
    const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) w[j] = __fmul_rn(w[j], sv[j]);
  }
}

// fp16 scale of a group from its fp32 range: clamp(r / levels, 1e-5, 65504),
// rounded to nearest even.  Returns the fp16 bits; *sc is its value.
__device__ __forceinline__ uint16_t group_scale_f16(float r, float levels, float* sc) {
  float sc32 = __fdiv_rn(r, levels);
  if (!(sc32 >= 1e-5f)) sc32 = 1e-5f;
  if (sc32 > 65504.0f) sc32 = 65504.0f;
  const __half h = __float2half_rn(sc32);
  *sc = __half2float(h);
  return __half_as_ushort(h);
}

// The same fp16 scale without the division where it is not needed: t = r *
// fp32(1 / levels) is within 2^-23 (relative) of the fp32 quotient, and the
// clamp-then-round map is monotonic, so when t (1 - 2^-19) and t (1 + 2^-19)
// map to the same fp16 that is the quotient's; otherwise (rare) the division.
__device__ __forceinline__ uint16_t group_scale_f16_fast(float r, float levels, float rlevels, float* sc) {
  const auto map = [](float x) {
    if (!(x >= 1e-5f)) x = 1e-5f;
    if (x > 65504.0f) x = 65504.0f;
    return __half_as_ushort(__float2half_rn(x));
  };
  const float t = __fmul_rn(r, rlevels);
  const uint16_t lo = map(__fmul_rn(t, 1.0f - 0x1p-19f)), hi = map(__fmul_rn(t, 1.0f + 0x1p-19f));
  if (__builtin_expect(lo != hi, 0)) return group_scale_f16(r, levels, sc);
  *sc = __half2float(__ushort_as_half(lo));
  return lo;
}

// rint(x / sc) through the correctly rounded reciprocal rsc = 1 / sc: the product
// is within 2^-23 (relative) of the IEEE quotient, so its rint is the quotient's
// unless it lies within 2^-21 of a half-integer (relative), where the division
// is taken (a branch of its own: rare).
__device__ __forceinline__ float rint_quotient(float x, float sc, float rsc) {
  const float t = __fmul_rn(x, rsc);
  const float r = rintf(t);
  if (__builtin_expect(__fsub_rn(0.5f, fabsf(__fsub_rn(t, r))) <= fabsf(t) * 0x1p-21f, 0)) return rintf(__fdiv_rn(x, sc));
  return r;
}

// grid = (ceil(K/2048), N); thread t of CTA (c, n) owns word u = c*256 + t of
// row n, i.e. k in [8u, 8u+8).  A group is G/8 consecutive lanes of one warp.
template <int G, bool ASYM>
__global__ void __launch_bounds__(kQuantThreads) quantize_int4_kernel(
    const uint16_t* __restrict__ W, const float* __restrict__ s, int64_t N, int64_t K,
    uint32_t* __restrict__ qweight, uint16_t* __restrict__ scales, uint32_t* __restrict__ zeros) {
  constexpr int LPG = G / 8;  // lanes per group
  __shared__ uint8_t zsh[kQuantThreads / LPG];
  const int64_t n = blockIdx.y;
  const int64_t words = K / 8;
  const int64_t u = int64_t(blockIdx.x) * kQuantThreads + threadIdx.x;
  const bool active = u < words;
  const int64_t k = u * 8;

  float w[8];
  float mn = INFINITY, mx = -INFINITY, amax = 0.f;
  if (active) {
    load_wprime8(W, s, K, n, k, w);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      mn = fminf(mn, w[j]);
      mx = fmaxf(mx, w[j]);
      amax = fmaxf(amax, fabsf(w[j]));
    }
  }
  // groups never straddle a warp (LPG divides 32, rows hold whole groups)
#pragma unroll
  for (int off = 1; off < LPG; off <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  }
  const int64_t ng = K / G;
  const int64_t g = k / G;
  float sc, z = 0.f;
  uint16_t hbits;
  if (ASYM) {
    hbits = group_scale_f16_fast(__fsub_rn(mx, mn), 15.0f, 1.0f / 15.0f, &sc);
    z = fminf(fmaxf(rint_quotient(-mn, sc, __frcp_rn(sc)), 0.0f), 15.0f);
  } else {
    hbits = group_scale_f16_fast(amax, 7.0f, 1.0f / 7.0f, &sc);
  }
  if (active) {
    uint32_t word = 0;
    // rint(w / sc) through the correctly rounded reciprocal: t = w * (1 / sc) is
    // within 2^-23 |t| of the IEEE quotient, so its rint is the quotient's unless t
    // lies within 2^-21 |t| of a half-integer, where the division itself is taken.
    // Those (rare) weights are flagged and divided in a branch of their own, so
    // the division sequence is not issued, predicated off, for every weight.
    const float rsc = __frcp_rn(sc);
    float r[8];
    uint32_t slow = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float t = __fmul_rn(w[j], rsc);
      r[j] = rintf(t);
      if (fabsf(0.5f - fabsf(__fsub_rn(t, r[j]))) <= fabsf(t) * 0x1p-21f) slow |= 1u << j;
    }
    if (__builtin_expect(slow != 0, 0)) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (slow & (1u << j)) r[j] = rintf(__fdiv_rn(w[j], sc));
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float q = ASYM ? fminf(fmaxf(__fadd_rn(r[j], z), 0.0f), 15.0f)
                           : __fadd_rn(fminf(fmaxf(r[j], -7.0f), 7.0f), 8.0f);
      word |= uint32_t(q) << (4 * j);
    }
    qweight[n * words + u] = word;
    if ((threadIdx.x % LPG) == 0) scales[n * ng + g] = hbits;
  }
  if (ASYM) {
    // Pack 8 group zero points per word.  A CTA covers 2048 k of one row,
    // a whole number of zero words (8*G divides 2048), so no word is shared.
    if ((threadIdx.x % LPG) == 0) zsh[threadIdx.x / LPG] = active ? uint8_t(z) : uint8_t(0);
    __syncthreads();
    constexpr int GROUPS_PER_CTA = kQuantThreads / LPG;
    const int64_t nzw = (ng + 7) / 8;
    const int64_t g0 = int64_t(blockIdx.x) * GROUPS_PER_CTA;
    if (threadIdx.x < GROUPS_PER_CTA / 8) {
      const int64_t zw = g0 / 8 + threadIdx.x;
      if (zw < nzw) {
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int64_t gg = zw * 8 + j;
          if (gg < ng) word |= uint32_t(zsh[threadIdx.x * 8 + j] & 0xF) << (4 * j);
        }
        zeros[n * nzw + zw] = word;
      }
    }
  }
}

// 8 consecutive elements at flat index e of a row-major [R, C] bf16 tensor as
// fp32, times s[e % C] when an AWQ scale is given (the column is only needed then).
__device__ __forceinline__ void load_flat8(const uint16_t* __restrict__ A, const float* __restrict__ s, int64_t C,
                                           int64_t e, float w[8]) {
  const uint4 v = ldg_stream_v4(A + e);
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    w[2 * j] = __uint_as_float(u[j] << 16);
    w[2 * j + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
  }
  if (s) {
    const int64_t c = e % C;
    const float4 s0 = __ldg(reinterpret_cast<const float4*>(s + c));
    const float4 s1 = __ldg(reinterpret_cast<const float4*>(s + c + 4));
    const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) w[j] = __fmul_rn(w[j], sv[j]);
  }
}

// ------------------------------------------------------------------ NVFP4
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Pass 1: amax over the tensor, atomically max-ed into *amax_out (which the
// host zeroed).  Non-negative floats order like their bit patterns.  Without
// an AWQ scale the magnitudes are the bf16 bit patterns with the sign cleared,
// compared as unsigned 16-bit pairs (one SIMD max per two elements, eight
// 16-byte loads in flight per thread); a thread that saw a NaN pattern
// (above 0x7F80) redoes its elements with fmaxf, which skips NaNs.
__global__ void __launch_bounds__(256) nvfp4_amax_kernel(const uint16_t* __restrict__ A, const float* __restrict__ s,
                                                         int64_t R, int64_t C, float* amax_out,
                                                         float* __restrict__ block_max) {
  const int64_t words = R * C / 8;
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  const int64_t t0 = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  float m = 0.f;
  bool fp32_path = s != nullptr;
  if (!fp32_path) {
    uint32_t mi = 0;
    for (int64_t u0 = t0; u0 < words; u0 += 8 * stride) {
      uint4 v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int64_t u = u0 + q * stride;
        v[q] = u < words ? ldg_stream_v4(A + u * 8) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        mi = max_u16x2(mi, v[q].x & 0x7FFF7FFFu);
        mi = max_u16x2(mi, v[q].y & 0x7FFF7FFFu);
        mi = max_u16x2(mi, v[q].z & 0x7FFF7FFFu);
        mi = max_u16x2(mi, v[q].w & 0x7FFF7FFFu);
      }
    }
    const uint32_t top = max(mi & 0xFFFFu, mi >> 16);
    if (top > 0x7F80u) fp32_path = true;  // a NaN: take the fmaxf pass below for this thread
    else m = __uint_as_float(top << 16);
  }
  if (fp32_path) {
    // four independent 16-byte loads in flight per thread per iteration
    for (int64_t u0 = t0; u0 < words; u0 += 4 * stride) {
      float w[4][8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int64_t u = u0 + q * stride;
        if (u < words) {
          load_flat8(A, s, C, u * 8, w[q]);
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) w[q][j] = 0.f;
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(w[q][j]));
    }
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  __shared__ float red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < int(blockDim.x >> 5); ++i) m = fmaxf(m, red[i]);
    if (block_max)
      block_max[blockIdx.x] = m;  // the pack pass takes the maximum of these (no zeroing, no atomics)
    else
      atomicMax(reinterpret_cast<unsigned int*>(amax_out), __float_as_uint(m));
  }
}

// amax from the amax pass's per-CTA maxima (n of them), the same value in every thread
__device__ __forceinline__ float nvfp4_amax_of_blocks(const float* __restrict__ block_max, int n) {
  __shared__ float red[8];
  float m = 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) m = fmaxf(m, block_max[i]);
#pragma unroll
  for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  m = red[0];
  for (int i = 1; i < int(blockDim.x >> 5); ++i) m = fmaxf(m, red[i]);
  return m;
}

// Hardware conversions: round to nearest with ties to the even mantissa (for
// E2M1 that is the even code), saturating at the largest finite value, sign
// kept -- the readings of the pages' "E2M1 + E4M3" packing; the bit-exact pack
// tests hold them to the oracle's table-driven encoders, exact ties and both
// signs included.
// Two fp32 -> E2M1 codes, `lo` in bits 0-3 and `hi` in bits 4-7.
__device__ __forceinline__ uint32_t e2m1x2_rn_sat(float lo, float hi) {
  uint32_t d;
  asm("{ .reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %1, %2; cvt.u32.u8 %0, t; }" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}
// One non-negative fp32 -> E4M3 code (satfinite: 448 for anything larger).
__device__ __forceinline__ uint32_t e4m3_rn_sat(float t) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(0.0f), "f"(t));
  return uint32_t(d) & 0xFFu;
}

__device__ __forceinline__ float nvfp4_global_from_amax(float amax) {
  return amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f;  // 6 * 448
}

// Pass 2: one thread per block of 16 consecutive elements (flat order), so
// block-scale bytes and 8-byte code groups are written coalesced.
__global__ void __launch_bounds__(256) nvfp4_pack_kernel(const uint16_t* __restrict__ A, const float* __restrict__ s,
                                                         int64_t R, int64_t C, const float* __restrict__ amax_in,
                                                         uint8_t* __restrict__ codes, uint8_t* __restrict__ bscale,
                                                         float* __restrict__ g_out, const float* __restrict__ block_max,
                                                         int n_block_max) {
  const int64_t nblk = R * C / 16;
  // the tensor's amax: accumulated by the amax pass, or its per-CTA maxima reduced here
  const float g = nvfp4_global_from_amax(block_max ? nvfp4_amax_of_blocks(block_max, n_block_max) : *amax_in);
  const float rg = __frcp_rn(g);
  const bool rg_ok = __float_as_uint(rg) < 0x7F800000u;  // not for a subnormal g (amax below ~3e-35)
  if (g_out && blockIdx.x == 0 && threadIdx.x == 0) *g_out = g;  // amax lives elsewhere: no finalize pass
  for (int64_t b = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; b < nblk; b += int64_t(gridDim.x) * blockDim.x) {
    float w[16];
    load_flat8(A, s, C, b * 16, w);
    load_flat8(A, s, C, b * 16 + 8, w + 8);
    float ab = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) ab = fmaxf(ab, fabsf(w[j]));
    // E4M3 block scale of the IEEE quotient (ab / 6) / g.  t = ab * fp32(1/6) *
    // fp32(1/g) is within ~6 2^-24 (relative) of it, so the product by 1 - 2^-19
    // and by 1 + 2^-19 bracket the quotient: when both convert to the same code
    // (conversion is monotonic) that is its code; else the divisions are taken.
    // The bracket needs normal intermediates: blocks with ab < 2^-120 (zero blocks
    // among them) and a g whose reciprocal overflows take the divisions.
    uint32_t sb;
    {
      const float t = __fmul_rn(__fmul_rn(ab, 1.0f / 6.0f), rg);
      const uint32_t sl = e4m3_rn_sat(__fmul_rn(t, 1.0f - 0x1p-19f)), sh = e4m3_rn_sat(__fmul_rn(t, 1.0f + 0x1p-19f));
      sb = sl;
      if (__builtin_expect(sl != sh || !(ab >= 0x1p-120f) || !rg_ok, 0))
        sb = e4m3_rn_sat(__fdiv_rn(__fdiv_rn(ab, 6.0f), g));
    }
    const float d = e4m3_decode_pos(sb);
    uint32_t lo = 0, hi = 0;
    if (d != 0.0f) {
      const float denom = __fmul_rn(d, g);
      const float rcp = __frcp_rn(denom);
      // Codes of the IEEE quotients w / denom, two per conversion.  w * rcp is
      // within 2^-22 (relative) of the quotient, so w * (rcp (1 - 2^-19)) and
      // w * (rcp (1 + 2^-19)) bracket it: when they convert to the same pair of
      // codes, so does every value between them (rounding is monotonic), the
      // quotient included.  Only pairs near a rounding boundary take the
      // divisions, flagged and converted in a branch of their own (rare), so the
      // divisions are not issued, predicated off, for all.  A denominator below
      // 2^-128 (tensors with amax under ~1e-33) has no finite reciprocal: then
      // every pair takes the divisions.
      const float rlo = __fmul_rn(rcp, 1.0f - 0x1p-19f), rhi = __fmul_rn(rcp, 1.0f + 0x1p-19f);
      const bool rcp_ok = __float_as_uint(rhi) < 0x7F800000u;
      uint32_t pairs[8];
      uint32_t slow = 0;
#pragma unroll
      for (int j = 0; j < 16; j += 2) {
        const uint32_t cl = e2m1x2_rn_sat(__fmul_rn(w[j], rlo), __fmul_rn(w[j + 1], rlo));
        const uint32_t ch = e2m1x2_rn_sat(__fmul_rn(w[j], rhi), __fmul_rn(w[j + 1], rhi));
        pairs[j >> 1] = cl;
        if (!(rcp_ok && cl == ch)) slow |= 1u << (j >> 1);
      }
      if (__builtin_expect(slow != 0, 0)) {
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (slow & (1u << q)) pairs[q] = e2m1x2_rn_sat(__fdiv_rn(w[2 * q], denom), __fdiv_rn(w[2 * q + 1], denom));
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        lo |= pairs[q] << (8 * q);
        hi |= pairs[4 + q] << (8 * q);
      }
    }
    reinterpret_cast<uint2*>(codes)[b] = make_uint2(lo, hi);
    bscale[b] = uint8_t(sb);
  }
}

// Pass 3: replace the amax in *gs by the per-tensor scale g.
__global__ void nvfp4_finalize_kernel(float* gs) { *gs = nvfp4_global_from_amax(*gs); }

}  // namespace wq
