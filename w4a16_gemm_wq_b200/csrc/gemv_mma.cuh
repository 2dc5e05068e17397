// gemv_mma.cuh -- decode GEMV for 3..16 activation rows on the tensor cores
// (mma.sync m16n8k16), reading every packed weight once.
//
// Y[m, n] = sum_k x'[m, k] w_hat[n, k] for M up to 16 ("quantization primer"
// section 13: decode stays memory-bound as long as the weights are read once
// per step; a CUDA-core GEMV would need 16 multiply-adds per weight here,
// several times the HBM time of the weight).
//
// Grid: CTA (bx, s) owns the row blocks 8 bx .. 8 bx + 7 (16 weight rows each,
// one per warp) over the K slice s; the S slices of a row-block group form a
// thread-block cluster; each CTA of the cluster sums a share of the outputs
// over the slices' partials through distributed shared memory, in rank order
// (deterministic, no workspace).
// Step: 16 rows x 128 k.  Lane (g, c) (g = lane / 4, c = lane % 4) loads 16
// code bytes of rows g and g + 8 at k = 128 j + 32 c (64-byte runs per row).
// A lane's 32 codes always lie in one quantization group (G >= 32), so it
// dequantizes them in registers with its own scale and zero point:
//   INT4  bf16 {128 + q_i, 128 + q_{i+4}} by one LOP3 per pair (exponent-bias
//         trick), minus {128 + z} (exact), times the fp16 scale in bf16 (one
//         rounding; bf16 keeps any fp16 scale times 15 in range);
//   NVFP4 e2m1x2 -> f16x2 in hardware times the E4M3 block scale in f16
//         (exact: at most 6 significant bits, |v| <= 6 * 448).
// A word's codes feed two mma (the k order inside an mma is free; B follows
// the same order).  B = the activations of rows 8 t .. 8 t + 7 of n8 tile t,
// staged once per CTA for its K slice in shared memory, as bf16 (INT4, order
// {x0, x4} {x1, x5} {x2, x6} {x3, x7} per 8 k) or f16 (NVFP4, natural pairs),
// times act_inv_s, with a 16-byte row pad so a warp's fragment loads are
// conflict-free.  fp32 accumulation in the mma; the NVFP4 tensor scale
// multiplies the sum.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "gemm_tcgen05.cuh"
#include "gemv.cuh"
#include "gemv_tc.cuh"
#include "wq_common.cuh"

namespace wq {

constexpr int kMmaWarps = 8;        // row blocks (of 16 rows) per CTA
constexpr int kMmaStepK = 128;
constexpr int kMmaDepth = 4;        // steps in flight per warp
constexpr int kMmaMaxSplits = 8;    // portable cluster size
constexpr int kMmaMaxSliceSteps = 24;  // staged K slice: 16 rows x 3072 k x 2 bytes = 96 KB at most

struct GemvMmaArgs {
  const uint16_t* X;       // bf16 [M, K]
  const float* inv_s;      // fp32 [K] or null
  const uint8_t* packed;   // INT4 qweight / NVFP4 codes, K/2 bytes per row
  const uint16_t* scales;  // INT4 fp16 [N, K/G]
  const uint32_t* zeros;   // INT4 [N, ceil(K/G/8)] or null (symmetric, z = 8)
  const uint8_t* bscale;   // NVFP4 E4M3 [N, K/16]
  const float* gscale;     // NVFP4 fp32 [1]
  uint16_t* Y;             // bf16 [M, N]
  int M, N, K;
  int log2g;
  int slice_steps;         // steps of 128 k per K slice (gridDim.y slices)
};

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t bf2_sub(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hsub2(*reinterpret_cast<__nv_bfloat162*>(&a), *reinterpret_cast<__nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t bf2_mul(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&a), *reinterpret_cast<__nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t h2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t e2m1x2_f16x2(uint32_t byte) {
  uint32_t h;
  asm("{ .reg .b8 q; cvt.u8.u32 q, %1; cvt.rn.f16x2.e2m1x2 %0, q; }" : "=r"(h) : "r"(byte));
  return h;
}

// One word of 8 codes (k0..k7) of one row -> the A registers of two mma:
// r[0], r[1] = k-pairs of the first mma, r[2], r[3] of the second (INT4:
// {k0,k4} {k1,k5} | {k2,k6} {k3,k7}; NVFP4: {k0,k1} {k2,k3} | {k4,k5} {k6,k7}).
template <int FMT>
__device__ __forceinline__ void mma_dequant_word(uint32_t w, uint32_t zoff2, uint32_t sc2, uint32_t (&r)[4]) {
  if (FMT == FMT_INT4) {
    r[0] = bf2_mul(bf2_sub(lop3_and_or(w, 0x000F000Fu, 0x43004300u), zoff2), sc2);
    r[1] = bf2_mul(bf2_sub(lop3_and_or(w >> 4, 0x000F000Fu, 0x43004300u), zoff2), sc2);
    r[2] = bf2_mul(bf2_sub(lop3_and_or(w >> 8, 0x000F000Fu, 0x43004300u), zoff2), sc2);
    r[3] = bf2_mul(bf2_sub(lop3_and_or(w >> 12, 0x000F000Fu, 0x43004300u), zoff2), sc2);
  } else {
    r[0] = h2_mul(e2m1x2_f16x2(w), sc2);
    r[1] = h2_mul(e2m1x2_f16x2(w >> 8), sc2);
    r[2] = h2_mul(e2m1x2_f16x2(w >> 16), sc2);
    r[3] = h2_mul(e2m1x2_f16x2(w >> 24), sc2);
  }
}

// NT: n8 tiles of activation rows (1 for M <= 8, 2 for M <= 16).
template <int FMT, int NT>
__global__ void __launch_bounds__(kMmaWarps * 32) gemv_mma_kernel(const GemvMmaArgs a) {
  extern __shared__ __align__(16) uint8_t mma_smem[];
  __shared__ float part[kMmaWarps][16][NT * 8];  // this CTA's partial sums of its row blocks
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int K = a.K, N = a.N;
  const int nsteps = K / kMmaStepK;
  const int j0 = blockIdx.y * a.slice_steps, j1 = min(nsteps, j0 + a.slice_steps);
  const int slice_k = (j1 - j0) * kMmaStepK;
  const int xstride = a.slice_steps * kMmaStepK * 2 + 16;  // bytes per staged row (+16 against bank conflicts)
  const int rb = blockIdx.x * kMmaWarps + warp;
  const int nlo = min(rb * 16 + g, N - 1), nhi = min(rb * 16 + g + 8, N - 1);
  const int64_t rbytes = K >> 1;
  const uint8_t* clo = a.packed + int64_t(nlo) * rbytes + 16 * c;
  const uint8_t* chi = a.packed + int64_t(nhi) * rbytes + 16 * c;
  const int ng = K >> a.log2g, zw = (ng + 7) >> 3;

  // ---- this lane's codes and metadata of step j, kMmaDepth steps in flight
  struct Entry {
    uint4 lo, hi;
    uint32_t mlo, mhi;  // INT4: fp16 scale; NVFP4: the two E4M3 bytes of the lane's blocks
    uint32_t zlo, zhi;  // INT4: the packed zero-point words holding this step's group (decoded at use)
  };
  const auto load = [&](int j, Entry& e) {
    e.lo = tc_ld_stream(clo + 64 * j);
    e.hi = tc_ld_stream(chi + 64 * j);
    const int k = j * kMmaStepK + 32 * c;
    if (FMT == FMT_INT4) {
      const int grp = k >> a.log2g;
      e.zlo = a.zeros ? __ldg(a.zeros + int64_t(nlo) * zw + (grp >> 3)) : 0x88888888u;
      e.zhi = a.zeros ? __ldg(a.zeros + int64_t(nhi) * zw + (grp >> 3)) : 0x88888888u;
      e.mlo = __ldg(a.scales + int64_t(nlo) * ng + grp);
      e.mhi = __ldg(a.scales + int64_t(nhi) * ng + grp);
    } else {
      e.mlo = __ldg(reinterpret_cast<const uint16_t*>(a.bscale + int64_t(nlo) * (K >> 4) + (k >> 4)));
      e.mhi = __ldg(reinterpret_cast<const uint16_t*>(a.bscale + int64_t(nhi) * (K >> 4) + (k >> 4)));
    }
  };
  // warm L2 with the first steps' codes while the previous kernel drains (a
  // prefetch never yields stale data), then wait for the previous kernel's writes
  // before any load: the weights themselves may have just been written
#pragma unroll
  for (int u = 0; u < kMmaDepth; ++u)
    if (j0 + u < j1) {
      asm volatile("prefetch.global.L2 [%0];" ::"l"(clo + 64 * (j0 + u)));
      asm volatile("prefetch.global.L2 [%0];" ::"l"(chi + 64 * (j0 + u)));
    }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  Entry R[kMmaDepth];
#pragma unroll
  for (int u = 0; u < kMmaDepth; ++u)
    if (j0 + u < j1) load(j0 + u, R[u]);

  // ---- stage the activation slice: rows 0..8 NT - 1 (zero past M), times inv_s
  for (int e = threadIdx.x; e < NT * 8 * (slice_k / 8); e += blockDim.x) {
    const int m = e / (slice_k / 8), ch = e - m * (slice_k / 8);
    const int k = j0 * kMmaStepK + 8 * ch;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (m < a.M) {
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(a.X + int64_t(m) * K + k));
      const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
      float f[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        f[2 * q] = __uint_as_float(wv[q] << 16);
        f[2 * q + 1] = __uint_as_float(wv[q] & 0xFFFF0000u);
      }
      if (a.inv_s) {
        const float4 i0 = __ldg(reinterpret_cast<const float4*>(a.inv_s + k));
        const float4 i1 = __ldg(reinterpret_cast<const float4*>(a.inv_s + k) + 1);
        f[0] *= i0.x; f[1] *= i0.y; f[2] *= i0.z; f[3] *= i0.w;
        f[4] *= i1.x; f[5] *= i1.y; f[6] *= i1.z; f[7] *= i1.w;
      }
      if (FMT == FMT_INT4) {  // bf16 pairs {x0, x4} {x1, x5} {x2, x6} {x3, x7}
        v.x = f32_to_bf16_bits(f[0]) | (f32_to_bf16_bits(f[4]) << 16);
        v.y = f32_to_bf16_bits(f[1]) | (f32_to_bf16_bits(f[5]) << 16);
        v.z = f32_to_bf16_bits(f[2]) | (f32_to_bf16_bits(f[6]) << 16);
        v.w = f32_to_bf16_bits(f[3]) | (f32_to_bf16_bits(f[7]) << 16);
      } else {  // f16 natural pairs
        __half2 h[4] = {__floats2half2_rn(f[0], f[1]), __floats2half2_rn(f[2], f[3]), __floats2half2_rn(f[4], f[5]),
                        __floats2half2_rn(f[6], f[7])};
        v = *reinterpret_cast<const uint4*>(h);
      }
    }
    *reinterpret_cast<uint4*>(mma_smem + m * xstride + 16 * ch) = v;
  }
  __syncthreads();

  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
  for (int base = j0; base < j1; base += kMmaDepth) {
#pragma unroll
    for (int u = 0; u < kMmaDepth; ++u) {
      const int j = base + u;
      if (j >= j1) break;
      const Entry e = R[u];
      if (j + kMmaDepth < j1) load(j + kMmaDepth, R[u]);
      uint32_t sl, sh, zl2 = 0, zh2 = 0;
      if (FMT == FMT_INT4) {
        const float fl = __half2float(__ushort_as_half(uint16_t(e.mlo))), fh = __half2float(__ushort_as_half(uint16_t(e.mhi)));
        sl = pack_bf16x2(fl, fl);
        sh = pack_bf16x2(fh, fh);
        const int zsh = 4 * (((j * kMmaStepK + 32 * c) >> a.log2g) & 7);  // this step's group in its zero word
        const uint32_t zbl = 0x4300u | ((e.zlo >> zsh) & 0xFu), zbh = 0x4300u | ((e.zhi >> zsh) & 0xFu);  // bf16(128 + z)
        zl2 = zbl | (zbl << 16);
        zh2 = zbh | (zbh << 16);
      } else {
        sl = tc_e4m3x2(e.mlo);  // {block 2c, block 2c + 1} of row g as f16x2
        sh = tc_e4m3x2(e.mhi);
      }
      const uint32_t wl[4] = {e.lo.x, e.lo.y, e.lo.z, e.lo.w}, wh[4] = {e.hi.x, e.hi.y, e.hi.z, e.hi.w};
      const uint8_t* xrow = mma_smem + (j - j0) * (kMmaStepK * 2) + 64 * c;  // this lane's 32 k of the step
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        uint32_t al[4], ah[4];
        if (FMT == FMT_INT4) {
          mma_dequant_word<FMT>(wl[w], zl2, sl, al);
          mma_dequant_word<FMT>(wh[w], zh2, sh, ah);
        } else {  // words 0-1: block 2c, words 2-3: block 2c + 1
          const uint32_t bl = __byte_perm(sl, 0, w < 2 ? 0x1010 : 0x3232);
          const uint32_t bh = __byte_perm(sh, 0, w < 2 ? 0x1010 : 0x3232);
          mma_dequant_word<FMT>(wl[w], 0, bl, al);
          mma_dequant_word<FMT>(wh[w], 0, bh, ah);
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const uint4 b = *reinterpret_cast<const uint4*>(xrow + (8 * t + g) * xstride + 16 * w);
          if (FMT == FMT_INT4) {
            mma_bf16_16816(acc[t], al[0], ah[0], al[1], ah[1], b.x, b.y);
            mma_bf16_16816(acc[t], al[2], ah[2], al[3], ah[3], b.z, b.w);
          } else {
            mma_f16_16816(acc[t], al[0], ah[0], al[1], ah[1], b.x, b.y);
            mma_f16_16816(acc[t], al[2], ah[2], al[3], ah[3], b.z, b.w);
          }
        }
      }
    }
  }
  // acc[t]: rows g (0, 1) and g + 8 (2, 3), columns m = 8 t + 2 c (+1)
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    part[warp][g][8 * t + 2 * c] = acc[t][0];
    part[warp][g][8 * t + 2 * c + 1] = acc[t][1];
    part[warp][g + 8][8 * t + 2 * c] = acc[t][2];
    part[warp][g + 8][8 * t + 2 * c + 1] = acc[t][3];
  }
  const float gmul = (FMT == FMT_NVFP4) ? __ldg(a.gscale) : 1.0f;
  constexpr int PARTS = kMmaWarps * 16 * NT * 8;
  const int nsplit = gridDim.y;
  if (nsplit > 1) {
    cluster_sync();  // every CTA of the cluster has its partials in shared memory
    // rank r sums outputs [r PARTS / S, (r + 1) PARTS / S): the S partials of an output
    // are fetched at once and added in rank order (the result does not depend on timing)
    const int rank = int(cluster_ctarank());
    const int i0 = rank * PARTS / nsplit, i1 = (rank + 1) * PARTS / nsplit;
    for (int i = i0 + threadIdx.x; i < i1; i += blockDim.x) {
      const uint32_t saddr = smem_u32(&part[0][0][0] + i);
      float pv[kMmaMaxSplits];
#pragma unroll
      for (int rk = 0; rk < kMmaMaxSplits; ++rk) {
        pv[rk] = 0.f;
        if (rk < nsplit) {
          const uint32_t ra = map_shared_rank(saddr, uint32_t(rk));
          asm("ld.shared::cluster.f32 %0, [%1];" : "=f"(pv[rk]) : "r"(ra));
        }
      }
      float v = 0.f;
#pragma unroll
      for (int rk = 0; rk < kMmaMaxSplits; ++rk) v += pv[rk];
      const int wr = i / (16 * NT * 8), r = (i / (NT * 8)) % 16, m = i % (NT * 8);
      const int n = (blockIdx.x * kMmaWarps + wr) * 16 + r;
      if (n < N && m < a.M) a.Y[int64_t(m) * N + n] = uint16_t(f32_to_bf16_bits(v * gmul));
    }
    cluster_sync();  // keep every CTA's shared memory alive until all ranks have read it
  } else {
    __syncthreads();
    for (int i = threadIdx.x; i < PARTS; i += blockDim.x) {
      const int wr = i / (16 * NT * 8), r = (i / (NT * 8)) % 16, m = i % (NT * 8);
      const int n = (blockIdx.x * kMmaWarps + wr) * 16 + r;
      if (n < N && m < a.M) a.Y[int64_t(m) * N + n] = uint16_t(f32_to_bf16_bits((&part[0][0][0])[i] * gmul));
    }
  }
}

}  // namespace wq
