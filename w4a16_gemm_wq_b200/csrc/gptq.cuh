// gptq.cuh -- GPTQ INT4 quantize-and-pack with second-order error feedback
// ("quantization primer" section 6 "GPTQ": quantize a weight, estimate its
// error with approximate second-order information, adjust the weights not yet
// quantized, continue; the ms-swift page: Hessian from 128-512 calibration
// samples, group size 128, no activation reordering).
//
// Input: the caller's upper Cholesky factor U of the damped inverse Hessian
// (U^T U = (2 X^T X + lambda I)^-1, fp32 [K, K]).  For every row, columns in
// order k = 0..K-1:
//   k % G == 0:  the group's fp16 scale and zero point from the weights
//                [k, k + G) as they stand now (the plain quantizer's min-max rule)
//   q_k = quant(w_k),  e_k = (w_k - (q_k - z) sc) / U[k][k]
//   w_j = w_j - e_k U[k][j]  for every j > k
// in fp32, every operation rounded on its own (no fused multiply-add).  Every
// w_j sees exactly the chain of w_j - e_k U[k][j] for k = 0, 1, .., j - 1 in
// that order, whatever the schedule below, so the codes are bit-identical to
// the sequential definition.
//
// Schedule: a CTA takes R rows at a time (their working weights fp32 in shared
// memory) and walks the K columns in blocks of G (one group each):
//   1. the block's diagonal tile of U goes to shared memory;
//   2. warp r runs row r's block sequentially from registers: group min/max by
//      warp shuffles, then per column the owning lane quantizes and divides the
//      error by the diagonal, the error is broadcast, and every lane adjusts its
//      later columns of the block; the codes are packed, the scale and zero point
//      written;
//   3. all threads apply the block's G errors to the columns after the block:
//      thread j streams U[b..b+G)[j] (coalesced, shared by the R rows) and runs
//      each row's chain of adjustments in k order.
// The sequential part is latency-bound (~G steps per block); the update part
// is bound by reading U (K^2/2 floats per pass over R rows; L2-resident for
// K = 2048, streamed through L2 by all CTAs together for K = 11008).
#pragma once

#include <cuda_fp16.h>

#include "quant.cuh"
#include "wq_common.cuh"

namespace wq {

constexpr int kGptqThreads = 512;  // 16 warps
constexpr int kGptqMaxRows = 16;   // rows per pass: one warp each in the sequential part


struct GptqArgs {
  const uint16_t* W;   // bf16 [N, K]
  const float* U;      // fp32 [K, K], upper triangle read
  int64_t N, K;
  int R;               // rows per pass (<= kGptqMaxRows, fits shared memory)
  uint32_t* qweight;   // [N, K/8]
  uint16_t* scales;    // fp16 [N, K/G]
  uint32_t* zeros;     // [N, ceil(K/G/8)] (asymmetric) or null
};

// shared memory of one CTA: working rows, U's diagonal tile, the block's errors and codes
__host__ __device__ inline size_t gptq_smem_bytes(int R, int64_t K, int G) {
  return size_t(R) * size_t(K) * 4 + size_t(G) * G * 4 + size_t(R) * G * 4 + size_t(R) * G;
}

// RMAX: the largest row count of a pass this instantiation serves (4 for long
// rows, where U streams from DRAM and more loads in flight pay; 16 otherwise).
template <int G, bool ASYM, int RMAX>
__global__ void __launch_bounds__(kGptqThreads, 1) gptq_int4_kernel(const GptqArgs a) {
  constexpr int UCHUNK = RMAX <= 4 ? 32 : 16;  // U loads in flight per thread in the update part
  extern __shared__ __align__(16) float gsm[];
  const int R = a.R;
  const int64_t K = a.K;
  float* w = gsm;                                              // [R][K]
  float* ud = w + size_t(R) * K;                               // [G][G]
  float* errs = ud + G * G;                                    // [R][G] negated errors -e_k
  uint8_t* qb = reinterpret_cast<uint8_t*>(errs + R * G);      // [R][G]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ng = K / G, nzw = (ng + 7) / 8;

  for (int64_t row0 = int64_t(blockIdx.x) * R; row0 < a.N; row0 += int64_t(gridDim.x) * R) {
    const int rows = int(a.N - row0 < R ? a.N - row0 : int64_t(R));
    // working weights: bf16 -> fp32 (8 per 16-byte load; K % 8 == 0)
    for (int64_t u = threadIdx.x; u < int64_t(rows) * (K / 8); u += kGptqThreads) {
      const int64_t r = u / (K / 8), k = (u - r * (K / 8)) * 8;
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(a.W + (row0 + r) * K + k));
      const uint32_t p[4] = {v.x, v.y, v.z, v.w};
      float* d = w + r * K + k;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        d[2 * i] = __uint_as_float(p[i] << 16);
        d[2 * i + 1] = __uint_as_float(p[i] & 0xFFFF0000u);
      }
    }
    uint32_t zacc = 0;  // lane 0 of warp r: zero nibbles of row r's current zero word
    __syncthreads();

    for (int64_t b = 0; b < K; b += G) {
      // ---- 1. U's diagonal tile
      for (int t = threadIdx.x; t < G * G; t += kGptqThreads) ud[t] = __ldg(a.U + (b + t / G) * K + b + t % G);
      __syncthreads();

      // ---- 2. the block, sequentially, one warp per row
      if (warp < rows) {
        constexpr int PL = G / 32;  // columns per lane
        float v[PL], dg[PL];  // this lane's columns and their diagonal entries U[k][k]
#pragma unroll
        for (int i = 0; i < PL; ++i) {
          v[i] = w[int64_t(warp) * K + b + lane + 32 * i];
          dg[i] = ud[(lane + 32 * i) * (G + 1)];
        }
        float mn = v[0], mx = v[0], amax = fabsf(v[0]);
#pragma unroll
        for (int i = 1; i < PL; ++i) {
          mn = fminf(mn, v[i]);
          mx = fmaxf(mx, v[i]);
          amax = fmaxf(amax, fabsf(v[i]));
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) {
          mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, off));
          mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
          amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
        }
        float sc, z;
        uint16_t hbits;
        if (ASYM) {
          hbits = group_scale_f16(__fsub_rn(mx, mn), 15.0f, &sc);
          z = fminf(fmaxf(rintf(__fdiv_rn(-mn, sc)), 0.0f), 15.0f);
        } else {
          hbits = group_scale_f16(amax, 7.0f, &sc);
          z = 8.0f;
        }
#pragma unroll
        for (int i = 0; i < PL; ++i) {
          for (int l2 = 0; l2 < 32; ++l2) {
            const int kk = 32 * i + l2;
            // this step's row of U's tile, read before the step's own stores so
            // that the loads leave the dependency chain
            float urow[PL];
#pragma unroll
            for (int i2 = 0; i2 < PL; ++i2) urow[i2] = ud[kk * G + lane + 32 * i2];
            // every lane quantizes its own column of slot i and divides its error by
            // its own diagonal entry (no divergent branch); the lane holding column kk
            // keeps its code and error, all take its error
            const float q = ASYM ? fminf(fmaxf(__fadd_rn(rintf(__fdiv_rn(v[i], sc)), z), 0.0f), 15.0f)
                                 : __fadd_rn(fminf(fmaxf(rintf(__fdiv_rn(v[i], sc)), -7.0f), 7.0f), 8.0f);
            const float deq = __fmul_rn(__fsub_rn(q, z), sc);  // exact: |q - z| <= 15, sc has 11 bits
            const float e = __shfl_sync(0xFFFFFFFFu, __fdiv_rn(__fsub_rn(v[i], deq), dg[i]), l2);
            if (lane == l2) {
              qb[warp * G + kk] = uint8_t(q);
              errs[warp * G + kk] = -e;
            }
#pragma unroll
            for (int i2 = 0; i2 < PL; ++i2) {
              const int jj = lane + 32 * i2;
              if (jj > kk) v[i2] = __fsub_rn(v[i2], __fmul_rn(e, urow[i2]));
            }
          }
        }
        __syncwarp();
        const int64_t n = row0 + warp;
        if (lane < G / 8) {
          uint32_t word = 0;
#pragma unroll
          for (int t = 0; t < 8; ++t) word |= uint32_t(qb[warp * G + 8 * lane + t]) << (4 * t);
          a.qweight[n * (K / 8) + b / 8 + lane] = word;
        }
        if (lane == 0) {
          const int64_t gi = b / G;
          a.scales[n * ng + gi] = hbits;
          if (ASYM) {
            zacc |= uint32_t(z) << (4 * (gi % 8));
            if (gi % 8 == 7 || gi + 1 == ng) {
              a.zeros[n * nzw + gi / 8] = zacc;
              zacc = 0;
            }
          }
        }
      }
      __syncthreads();

      // ---- 3. the block's errors applied to the later columns, k in order
      for (int64_t j = b + G + threadIdx.x; j < K; j += kGptqThreads) {
        float acc[RMAX];
#pragma unroll
        for (int r = 0; r < RMAX; ++r)
          if (r < rows) acc[r] = w[int64_t(r) * K + j];
        const float* uc = a.U + b * K + j;
        for (int k0 = 0; k0 < G; k0 += UCHUNK) {
          // a chunk of U's column j in flight at once (the loads, not the FMAs,
          // bound this loop when U streams from L2 or DRAM)
          float u[UCHUNK];
#pragma unroll
          for (int q = 0; q < UCHUNK; ++q) u[q] = __ldg(uc + int64_t(k0 + q) * K);
#pragma unroll
          for (int q = 0; q < UCHUNK; q += 4) {  // four k per step: one 16-byte error load per row
#pragma unroll
            for (int r = 0; r < RMAX; ++r)
              if (r < rows) {
                // w - e u as w + (-e) u: negation is exact, the product and the sum
                // each rounded (the intrinsics are never contracted into an FMA)
                const float4 ne = *reinterpret_cast<const float4*>(errs + r * G + k0 + q);
                acc[r] = __fadd_rn(acc[r], __fmul_rn(ne.x, u[q]));
                acc[r] = __fadd_rn(acc[r], __fmul_rn(ne.y, u[q + 1]));
                acc[r] = __fadd_rn(acc[r], __fmul_rn(ne.z, u[q + 2]));
                acc[r] = __fadd_rn(acc[r], __fmul_rn(ne.w, u[q + 3]));
              }
          }
        }
#pragma unroll
        for (int r = 0; r < RMAX; ++r)
          if (r < rows) w[int64_t(r) * K + j] = acc[r];
      }
      __syncthreads();
    }
  }
}

}  // namespace wq
