// gemv.cuh -- split-K decode GEMV for the quantized Linear at small M (M <= 16).
//
// Y[m, n] = sum_k x'[m, k] * w_hat[n, k], x' = x * act_inv_s (W4A16: weights
// 4-bit, activations 16-bit, "quantization primer" section 4).  At decode
// batch sizes the op reads every packed weight once and does a handful of
// flops per byte, so it is HBM-bound ("quantization primer" section 13:
// "Memory-bound Decode" benefits from 4x fewer weight bytes).
//
// Mapping (one warp = R rows x one K slice):
//   * lane l of iteration `it` owns k in [1024*it + 32*l, +32): one 128-bit
//     load of packed weights per row (32 codes), coalesced across the warp
//     (512 contiguous bytes per row);
//   * the lane's 32 activations are loaded once per iteration and reused for
//     the R rows of the warp;
//   * nibbles are unpacked in registers: INT4 codes become the bf16 value
//     1 + q/16 with one shift + one LOP3 per pair (exponent-bias trick), and
//     multiply bf16 activations with an fp32-accumulating mixed-precision FMA;
//     the group's scale and zero point are applied once per 32 weights:
//         sum_k (q_k - z) x_k s = s * (16 * sum_k (1 + q_k/16) x_k - (16 + z) sum_k x_k)
//     NVFP4 codes are converted in hardware (e2m1x2 -> f16x2) against fp16
//     activations; the E4M3 block scale multiplies each 16-element partial
//     sum and the per-tensor scale multiplies the result;
//   * lanes reduce with warp shuffles; the S split-K CTAs of a row block form
//     one thread-block cluster and CTA rank 0 sums their partials through
//     distributed shared memory in rank order (deterministic, no workspace).
#pragma once

#include <cuda_fp16.h>

#include "wq_common.cuh"

namespace wq {

constexpr int kGemvWarps = 8;
constexpr int kGemvRows = 4;          // rows per warp
constexpr int kGemvKPerIter = 1024;   // 32 lanes x 32 k
constexpr int kGemvMaxSplits = 8;     // portable cluster size

enum { FMT_INT4 = 0, FMT_NVFP4 = 1 };

struct GemvArgs {
  const uint16_t* X;       // bf16 [M, K]
  const float* inv_s;      // fp32 [K] or null
  const void* wq;          // INT4 qweight u32 [N, K/8] | NVFP4 codes u8 [N, K/2]
  const uint16_t* scales;  // INT4 fp16 [N, K/G]
  const uint32_t* zeros;   // INT4 u32 [N, ceil(K/G/8)], null = symmetric (z = 8)
  const uint8_t* bscale;   // NVFP4 e4m3 [N, K/16]
  const float* gscale;     // NVFP4 fp32 [1]
  uint16_t* Y;             // bf16 [M, N]
  int M, N, K;
  int log2g;               // INT4 log2(group_size)
  int iters_per_split;
};

// acc += a.lo * b.lo + a.hi * b.hi, bf16 inputs, fp32 accumulation.
__device__ __forceinline__ void fma2_bf16(float& acc, uint32_t a, uint32_t b) {
  asm("{ .reg .b16 a0, a1, b0, b1;\n\t"
      "mov.b32 {a0, a1}, %1;\n\t"
      "mov.b32 {b0, b1}, %2;\n\t"
      "fma.rn.f32.bf16 %0, a0, b0, %0;\n\t"
      "fma.rn.f32.bf16 %0, a1, b1, %0; }"
      : "+f"(acc)
      : "r"(a), "r"(b));
}

// acc += e2m1(byte k of c).lo * x.lo + .hi * x.hi with the code byte converted
// to f16x2 in hardware (low nibble -> low half); fp32 accumulation.
template <int BYTE>
__device__ __forceinline__ void fma2_e2m1(float& acc, uint32_t c, uint32_t x) {
  static_assert(BYTE >= 0 && BYTE < 4, "byte");
  if (BYTE == 0)
    asm("{ .reg .b8 q0, q1, q2, q3; .reg .b32 h; .reg .b16 h0, h1, x0, x1;\n\t"
        "mov.b32 {q0, q1, q2, q3}, %1;\n\t cvt.rn.f16x2.e2m1x2 h, q0;\n\t"
        "mov.b32 {h0, h1}, h;\n\t mov.b32 {x0, x1}, %2;\n\t"
        "fma.rn.f32.f16 %0, h0, x0, %0;\n\t fma.rn.f32.f16 %0, h1, x1, %0; }"
        : "+f"(acc) : "r"(c), "r"(x));
  else if (BYTE == 1)
    asm("{ .reg .b8 q0, q1, q2, q3; .reg .b32 h; .reg .b16 h0, h1, x0, x1;\n\t"
        "mov.b32 {q0, q1, q2, q3}, %1;\n\t cvt.rn.f16x2.e2m1x2 h, q1;\n\t"
        "mov.b32 {h0, h1}, h;\n\t mov.b32 {x0, x1}, %2;\n\t"
        "fma.rn.f32.f16 %0, h0, x0, %0;\n\t fma.rn.f32.f16 %0, h1, x1, %0; }"
        : "+f"(acc) : "r"(c), "r"(x));
  else if (BYTE == 2)
    asm("{ .reg .b8 q0, q1, q2, q3; .reg .b32 h; .reg .b16 h0, h1, x0, x1;\n\t"
        "mov.b32 {q0, q1, q2, q3}, %1;\n\t cvt.rn.f16x2.e2m1x2 h, q2;\n\t"
        "mov.b32 {h0, h1}, h;\n\t mov.b32 {x0, x1}, %2;\n\t"
        "fma.rn.f32.f16 %0, h0, x0, %0;\n\t fma.rn.f32.f16 %0, h1, x1, %0; }"
        : "+f"(acc) : "r"(c), "r"(x));
  else
    asm("{ .reg .b8 q0, q1, q2, q3; .reg .b32 h; .reg .b16 h0, h1, x0, x1;\n\t"
        "mov.b32 {q0, q1, q2, q3}, %1;\n\t cvt.rn.f16x2.e2m1x2 h, q3;\n\t"
        "mov.b32 {h0, h1}, h;\n\t mov.b32 {x0, x1}, %2;\n\t"
        "fma.rn.f32.f16 %0, h0, x0, %0;\n\t fma.rn.f32.f16 %0, h1, x1, %0; }"
        : "+f"(acc) : "r"(c), "r"(x));
}

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t mask, uint32_t bits) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(bits));  // (a & b) | c
  return d;
}

// INT4 nibbles i and i+4 of word w as bf16x2 {1 + q_i/16, 1 + q_{i+4}/16}.
template <int I>
__device__ __forceinline__ uint32_t int4_pair_bf16(uint32_t w) {
  const uint32_t t = (I == 0) ? (w << 3) : (w >> (4 * I - 3));
  return lop3_and_or(t, 0x00780078u, 0x3F803F80u);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Activations of one lane for one iteration: 32 consecutive k of row m,
// optionally times inv_s, as 16 pairs.  INT4 wants bf16 pairs ordered
// {x_{8j+i}, x_{8j+i+4}} (matching int4_pair_bf16); NVFP4 wants natural
// f16 pairs {x_{2b}, x_{2b+1}}.  *sum gets sum_k x'_k (INT4 zero-point fold).
template <int FMT>
__device__ __forceinline__ void load_x32(const uint16_t* __restrict__ xrow, const float* __restrict__ inv_s, int kb,
                                         uint32_t xp[16], float* sum) {
  uint32_t raw[16];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 v = ldg_v4(xrow + kb + 8 * q);
    raw[4 * q + 0] = v.x; raw[4 * q + 1] = v.y; raw[4 * q + 2] = v.z; raw[4 * q + 3] = v.w;
  }
  float s = 0.f;
  if (inv_s || FMT == FMT_NVFP4) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      float4 iv = make_float4(1.f, 1.f, 1.f, 1.f);
      if (inv_s) iv = __ldg(reinterpret_cast<const float4*>(inv_s + kb) + q);
      float f0 = __uint_as_float(raw[2 * q] << 16) * iv.x;
      float f1 = __uint_as_float(raw[2 * q] & 0xFFFF0000u) * iv.y;
      float f2 = __uint_as_float(raw[2 * q + 1] << 16) * iv.z;
      float f3 = __uint_as_float(raw[2 * q + 1] & 0xFFFF0000u) * iv.w;
      if (FMT == FMT_NVFP4) {
        __half2 h01 = __floats2half2_rn(f0, f1), h23 = __floats2half2_rn(f2, f3);
        raw[2 * q] = *reinterpret_cast<uint32_t*>(&h01);
        raw[2 * q + 1] = *reinterpret_cast<uint32_t*>(&h23);
      } else {
        raw[2 * q] = f32_to_bf16_bits(f0) | (f32_to_bf16_bits(f1) << 16);
        raw[2 * q + 1] = f32_to_bf16_bits(f2) | (f32_to_bf16_bits(f3) << 16);
      }
    }
  }
  if (FMT == FMT_INT4) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t a = raw[4 * j], b = raw[4 * j + 1], c = raw[4 * j + 2], d = raw[4 * j + 3];
      xp[4 * j + 0] = prmt(a, c, 0x5410);  // {x0, x4}
      xp[4 * j + 1] = prmt(a, c, 0x7632);  // {x1, x5}
      xp[4 * j + 2] = prmt(b, d, 0x5410);  // {x2, x6}
      xp[4 * j + 3] = prmt(b, d, 0x7632);  // {x3, x7}
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t r = raw[4 * j + e];
        s += __uint_as_float(r << 16) + __uint_as_float(r & 0xFFFF0000u);
      }
    }
  } else {
#pragma unroll
    for (int q = 0; q < 16; ++q) xp[q] = raw[q];
  }
  *sum = s;
}

// R: weight rows per warp (4; 2 gives small-N problems twice the CTAs).
template <int FMT, int MT, int R = kGemvRows>
__global__ void __launch_bounds__(kGemvWarps * 32) gemv_kernel(const GemvArgs a) {
  __shared__ float part[kGemvWarps * R * MT];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n0 = (blockIdx.x * kGemvWarps + warp) * R;
  const int m0 = blockIdx.z * MT;
  const int K = a.K, N = a.N;
  const int iters = (K + kGemvKPerIter - 1) / kGemvKPerIter;
  const int it0 = blockIdx.y * a.iters_per_split;
  const int it1 = min(iters, it0 + a.iters_per_split);

  float acc[R][MT];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[r][m] = 0.f;

  // Packed weights of iteration `it` for the warp's R rows (zero past N or K).
  auto load_w = [&](int it, uint4 (&wv)[R]) {
    const int kb = it * kGemvKPerIter + lane * 32;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int n = n0 + r;
      if (n < N && it < it1 && kb < K) {
        if (FMT == FMT_INT4)
          wv[r] = ldg_stream_v4(static_cast<const uint32_t*>(a.wq) + int64_t(n) * (K / 8) + kb / 8);
        else
          wv[r] = ldg_stream_v4(static_cast<const uint8_t*>(a.wq) + int64_t(n) * (K / 2) + kb / 2);
      } else {
        wv[r] = make_uint4(0, 0, 0, 0);
      }
    }
  };

  // Warm L2 with this warp's first weights while the previous kernel drains (L2
  // is the point of coherence, so a prefetch never yields stale data), let the
  // next kernel launch, and wait for the previous kernel's writes to become
  // visible before any load: the weights themselves may have just been written.
  {
    const int kb = it0 * kGemvKPerIter + lane * 32;
    if (it0 < it1 && kb < K) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int n = min(n0 + r, N - 1);
        const size_t off = FMT == FMT_INT4 ? size_t(n) * (K / 8) * 4 + size_t(kb) / 2 : size_t(n) * (K / 2) + kb / 2;
        asm volatile("prefetch.global.L2 [%0];" ::"l"(static_cast<const uint8_t*>(a.wq) + off));
      }
    }
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  uint4 wnext[R];
  load_w(it0, wnext);

  for (int it = it0; it < it1; ++it) {
    uint4 wv[R];
#pragma unroll
    for (int r = 0; r < R; ++r) wv[r] = wnext[r];
    load_w(it + 1, wnext);  // register double buffering: next iteration in flight
    const int kb = it * kGemvKPerIter + lane * 32;
    if (kb >= K) continue;  // K % 32 == 0: a lane's 32 k are all in or all out
    // per-row metadata for this lane's 32 k
    float msc[R], mzf[R], md1[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int n = min(n0 + r, N - 1);
      if (FMT == FMT_INT4) {
        const int ng = K >> a.log2g;
        const int g = kb >> a.log2g;
        msc[r] = __half2float(__ushort_as_half(__ldg(a.scales + int64_t(n) * ng + g)));
        int z = 8;
        if (a.zeros) z = (__ldg(a.zeros + int64_t(n) * ((ng + 7) >> 3) + (g >> 3)) >> (4 * (g & 7))) & 0xF;
        mzf[r] = float(16 + z);
        md1[r] = 0.f;
      } else {
        const uint16_t sb2 = __ldg(reinterpret_cast<const uint16_t*>(a.bscale + int64_t(n) * (K / 16) + kb / 16));
        msc[r] = e4m3_decode_pos(sb2 & 0x7F);  // block scales are non-negative
        md1[r] = e4m3_decode_pos((sb2 >> 8) & 0x7F);
        mzf[r] = 0.f;
      }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (m0 + m >= a.M) break;
      uint32_t xp[16];
      float sx;
      load_x32<FMT>(a.X + int64_t(m0 + m) * K, a.inv_s, kb, xp, &sx);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const uint32_t w4[4] = {wv[r].x, wv[r].y, wv[r].z, wv[r].w};
        if (FMT == FMT_INT4) {
          float d0 = 0.f, d1 = 0.f;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            fma2_bf16(d0, int4_pair_bf16<0>(w4[j]), xp[4 * j + 0]);
            fma2_bf16(d1, int4_pair_bf16<1>(w4[j]), xp[4 * j + 1]);
            fma2_bf16(d0, int4_pair_bf16<2>(w4[j]), xp[4 * j + 2]);
            fma2_bf16(d1, int4_pair_bf16<3>(w4[j]), xp[4 * j + 3]);
          }
          acc[r][m] += msc[r] * (16.f * (d0 + d1) - mzf[r] * sx);
        } else {
          float b0 = 0.f, b1 = 0.f;
#pragma unroll
          for (int j = 0; j < 2; ++j) {  // words 0,1 = block 0 (k 0..15)
            fma2_e2m1<0>(b0, w4[j], xp[4 * j + 0]);
            fma2_e2m1<1>(b0, w4[j], xp[4 * j + 1]);
            fma2_e2m1<2>(b0, w4[j], xp[4 * j + 2]);
            fma2_e2m1<3>(b0, w4[j], xp[4 * j + 3]);
          }
#pragma unroll
          for (int j = 2; j < 4; ++j) {  // words 2,3 = block 1 (k 16..31)
            fma2_e2m1<0>(b1, w4[j], xp[4 * j + 0]);
            fma2_e2m1<1>(b1, w4[j], xp[4 * j + 1]);
            fma2_e2m1<2>(b1, w4[j], xp[4 * j + 2]);
            fma2_e2m1<3>(b1, w4[j], xp[4 * j + 3]);
          }
          acc[r][m] += msc[r] * b0 + md1[r] * b1;
        }
      }
    }
  }

  // warp reduction over lanes
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      float v = acc[r][m];
#pragma unroll
      for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      acc[r][m] = v;
    }
  if (lane == 0) {
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) part[(warp * R + r) * MT + m] = acc[r][m];
  }

  const float gmul = (FMT == FMT_NVFP4) ? __ldg(a.gscale) : 1.0f;
  const int nsplit = gridDim.y;
  if (nsplit > 1) {
    cluster_sync();  // partials of every CTA of the cluster are in shared memory
    if (cluster_ctarank() == 0) {
      for (int t = threadIdx.x; t < kGemvWarps * R * MT; t += blockDim.x) {
        const uint32_t saddr = smem_u32(&part[t]);
        float v = 0.f;
        for (int rk = 0; rk < nsplit; ++rk) v += ld_shared_cluster_f32(map_shared_rank(saddr, rk));
        const int row = blockIdx.x * kGemvWarps * R + t / MT, m = m0 + t % MT;
        if (row < N && m < a.M) a.Y[int64_t(m) * N + row] = uint16_t(f32_to_bf16_bits(v * gmul));
      }
    }
    cluster_sync();  // keep every CTA's shared memory alive until rank 0 has read it
  } else {
    __syncthreads();
    for (int t = threadIdx.x; t < kGemvWarps * R * MT; t += blockDim.x) {
      const int row = blockIdx.x * kGemvWarps * R + t / MT, m = m0 + t % MT;
      if (row < N && m < a.M) a.Y[int64_t(m) * N + row] = uint16_t(f32_to_bf16_bits(part[t] * gmul));
    }
  }
}

}  // namespace wq
