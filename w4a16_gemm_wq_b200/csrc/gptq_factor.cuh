// gptq_factor.cuh -- GPTQ's second-order information from calibration tokens,
// in fp64 on the GPU ("quantization primer" section 6 "GPTQ": quantize a
// weight, estimate its error with approximate second-order information,
// adjust the rest; the ms-swift page: the information comes from 128-512
// calibration samples).
//
// Computes U (fp32 [K, K], upper triangular, positive diagonal) with
//     U^T U = (H + lambda I)^-1,   H = 2 X^T X,   lambda = damp * mean(diag H)
// over the calibration tokens X (bf16 [T, K]), the factor wq_gptq_int4 reads.
//
// Route (2/3 K^3 flops instead of the 4/3 K^3 of "invert, then factor"): with
// J the index reversal, the damped Hessian in reversed order H' = J H J has a
// lower Cholesky factor L' (H' = L' L'^T), so H = R R^T with the upper R =
// J L' J, H^-1 = R^-T R^-1, and the upper factor of H^-1 with positive
// diagonal is unique: U = R^-1 = J L'^-1 J.  Hence
//   1. H' = 2 Xr^T Xr with Xr = X in reversed column order (fp64, exact
//      products of bf16 values), damped on the diagonal;
//   2. blocked right-looking Cholesky of H' in place (64-wide blocks): factor
//      the diagonal block and invert it in shared memory, panel = panel *
//      inv(L_kk)^T, trailing lower triangle -= panel panel^T;
//   3. Z = L'^-T (upper) by blocked substitution with the stored inverses of
//      the diagonal blocks: Z[:, kb] = Z[:, kb] inv(L_kk)^T, then
//      Z[rows < kb + 64, later columns] -= Z[:, kb] L'[later rows, kb]^T;
//   4. U[i][j] = fp32(Z[K-1-j][K-1-i]) for i <= j, 0 below the diagonal.
// Every product of steps 1-3 runs on one fp64 tensor-core GEMM (mma.sync
// m8n8k4 .f64, "NT": both operands row-major with the reduction index
// contiguous).  Matrices are padded to Kp = a multiple of 64 with an identity
// block after the real indices (exact: the factor and the inverse of
// blockdiag(H', I) are blockdiag(L', I) and blockdiag(L'^-1, I)), so every GEMM
// runs on whole 64 x 64 tiles.
#pragma once

#include "wq_common.cuh"

namespace wq {

constexpr int kFacB = 64;        // block width of the factorisation and GEMM tile side
constexpr int kFacBK = 16;       // reduction slice per pipeline stage
constexpr int kFacStages = 3;
constexpr int kFacThreads = 128;  // 4 warps, 32 x 32 each
constexpr int kFacGemmSmem = kFacStages * 2 * kFacB * kFacBK * 8;  // 48 KB

enum : unsigned { ERR_NOT_POSITIVE_DEFINITE = 1u << 4 };

// fp64 tensor-core product of an 8x4 A fragment and a 4x8 B fragment into an
// 8x8 accumulator.  Fragments (lane l): a = A[l/4][l%4], b = B[k = l%4][n = l/4],
// c0/c1 = C[l/4][2(l%4)], C[l/4][2(l%4)+1].
__device__ __forceinline__ void dmma_8x8x4(double& c0, double& c1, double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
               : "+d"(c0), "+d"(c1)
               : "d"(a), "d"(b));
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Tiles a GEMM launch covers: all of an [mt x nt] grid, or only the lower
// triangle (tile column <= tile row) of a square one.
enum { FAC_TILES_ALL = 0, FAC_TILES_LOWER = 1 };

struct FacGemmArgs {
  const double* A;  // [M, Kd] row-major, leading dimension lda
  const double* B;  // [N, Kd] row-major, leading dimension ldb
  double* C;        // [M, N], leading dimension ldc
  int64_t lda, ldb, ldc;
  int mt, nt;       // tiles of 64 along M and N
  int kd;           // reduction length, a multiple of kFacBK
  double alpha, beta;
};

// C = beta C + alpha A B^T on 64 x 64 tiles.  A tile's operand rows are read
// completely before its outputs are written, so C may alias the rows of A that
// the same tile reads (the panel updates run in place).  beta == 0 reads no C.
template <int TILES>
__global__ void __launch_bounds__(kFacThreads) fac_gemm_nt_kernel(const FacGemmArgs a) {
  extern __shared__ __align__(16) double fsm[];
  // stage s: A slice [kFacBK/4][64][4], then B slice the same; element (r, k) of a
  // slice at ((k / 4) * 64 + r) * 4 + k % 4, so a fragment load is 32 consecutive doubles
  int tm, tn;
  if (TILES == FAC_TILES_LOWER) {
    const int64_t x = blockIdx.x;
    int r = int((sqrt(8.0 * double(x) + 1.0) - 1.0) * 0.5);
    while (int64_t(r + 1) * (r + 2) / 2 <= x) ++r;
    while (int64_t(r) * (r + 1) / 2 > x) --r;
    tm = r;
    tn = int(x - int64_t(r) * (r + 1) / 2);
  } else {
    tm = int(blockIdx.x / a.nt);
    tn = int(blockIdx.x % a.nt);
  }
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wm = warp >> 1, wn = warp & 1;  // this warp's 32 x 32 quarter
  const double* Ab = a.A + int64_t(tm) * kFacB * a.lda;
  const double* Bb = a.B + int64_t(tn) * kFacB * a.ldb;
  const int nslices = a.kd / kFacBK;

  // one slice: 64 rows x 16 doubles of A and of B = 2 x 128 chunks of 16 bytes per
  // operand row block; 128 threads move 4 chunks of each
  const auto load_slice = [&](int slice, int stage) {
    double* As = fsm + stage * 2 * kFacB * kFacBK;
    double* Bs = As + kFacB * kFacBK;
    const int k0 = slice * kFacBK;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int c = tid + i * kFacThreads;  // 0..511
      const int r = c >> 3, kk = (c & 7) * 2;
      const int so = ((kk >> 2) * kFacB + r) * 4 + (kk & 3);
      cp_async16(As + so, Ab + int64_t(r) * a.lda + k0 + kk);
      cp_async16(Bs + so, Bb + int64_t(r) * a.ldb + k0 + kk);
    }
  };

  double acc[4][4][2];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;

#pragma unroll
  for (int s = 0; s < kFacStages - 1; ++s) {
    if (s < nslices) load_slice(s, s);
    cp_async_commit();
  }
  for (int sl = 0; sl < nslices; ++sl) {
    cp_async_wait<kFacStages - 2>();
    __syncthreads();
    // refill the stage consumed one iteration ago
    if (sl + kFacStages - 1 < nslices) load_slice(sl + kFacStages - 1, (sl + kFacStages - 1) % kFacStages);
    cp_async_commit();
    const double* As = fsm + (sl % kFacStages) * 2 * kFacB * kFacBK;
    const double* Bs = As + kFacB * kFacBK;
#pragma unroll
    for (int kq = 0; kq < kFacBK / 4; ++kq) {
      double af[4], bf[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) af[i] = As[(kq * kFacB + wm * 32 + i * 8) * 4 + lane];
#pragma unroll
      for (int j = 0; j < 4; ++j) bf[j] = Bs[(kq * kFacB + wn * 32 + j * 8) * 4 + lane];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) dmma_8x8x4(acc[i][j][0], acc[i][j][1], af[i], bf[j]);
    }
  }
  cp_async_wait<0>();
  __syncthreads();  // every operand read of this tile is done before any output is written

  double* Cb = a.C + int64_t(tm) * kFacB * a.ldc + int64_t(tn) * kFacB;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = wm * 32 + i * 8 + (lane >> 2), c = wn * 32 + j * 8 + (lane & 3) * 2;
      double2* p = reinterpret_cast<double2*>(Cb + int64_t(r) * a.ldc + c);
      double2 v = make_double2(a.alpha * acc[i][j][0], a.alpha * acc[i][j][1]);
      if (a.beta != 0.0) {
        const double2 o = *p;
        v.x = fma(a.beta, o.x, v.x);
        v.y = fma(a.beta, o.y, v.y);
      }
      *p = v;
    }
}

// Xr [Kp, Tp] fp64: Xr[i][t] = X[t][K-1-i] for i < K, t < T, else 0 (the
// reversed channel order, transposed, zero padding; Kp and Tp multiples of 32,
// grid [Tp/32, Kp/32]).  32 x 32 tiles through shared memory so that both
// sides are coalesced.
__global__ void __launch_bounds__(256) fac_xr_kernel(const uint16_t* __restrict__ X, int64_t T, int64_t K,
                                                     int64_t Tp, double* __restrict__ Xr) {
  __shared__ double tile[32][33];
  const int64_t i0 = int64_t(blockIdx.y) * 32, t0 = int64_t(blockIdx.x) * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
  for (int r = ty; r < 32; r += 8) {
    const int64_t t = t0 + r, i = i0 + tx;  // reads along k = K-1-i (consecutive i: descending k)
    double v = 0.0;
    if (t < T && i < K) v = double(bf16_bits_to_f32(X[t * K + (K - 1 - i)]));
    tile[r][tx] = v;
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) Xr[(i0 + r) * Tp + t0 + tx] = tile[tx][r];
}

// Damping, in one CTA: lambda = damp * mean of the K real diagonal entries
// (summed in a fixed order: deterministic), added to them; the padding's
// diagonal becomes 1 (its rows and columns are 0 from the Hessian product).
__global__ void __launch_bounds__(256) fac_damp_kernel(double* H, int64_t K, int64_t Kp, double damp) {
  __shared__ double part[256];
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < K; i += 256) s += H[i * Kp + i];
  part[threadIdx.x] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < 256; ++i) t += part[i];
    part[0] = damp * (t / double(K));
  }
  __syncthreads();
  const double lambda = part[0];
  for (int64_t i = threadIdx.x; i < Kp; i += 256) H[i * Kp + i] = i < K ? H[i * Kp + i] + lambda : 1.0;
}

// One 64 x 64 diagonal block at A[kb][kb] (lower triangle read): Cholesky
// factor L_kk in place (lower; the strict upper part is set to 0) and its
// inverse into Dinv (64 x 64, lower).  A pivot that is not positive (a
// Hessian from non-finite tokens) reports ERR_NOT_POSITIVE_DEFINITE and turns
// into NaN, which then reaches every later entry.
__global__ void __launch_bounds__(256) fac_diag_kernel(double* A, int64_t lda, int64_t kb, double* Dinv) {
  __shared__ double S[kFacB][kFacB + 1];
  __shared__ double col[kFacB];
  const int tid = threadIdx.x;
  double* Ab = A + kb * lda + kb;
  for (int e = tid; e < kFacB * kFacB; e += 256) {
    const int i = e >> 6, c = e & 63;
    S[i][c] = c <= i ? Ab[int64_t(i) * lda + c] : 0.0;
  }
  __syncthreads();
  // column j: every thread derives the pivot itself (no wait on one thread), the
  // scaled column goes to col[], then row i is updated by its 4 threads (columns
  // c = j+1..i with c % 4 == q, independent multiply-adds)
  const int i = tid >> 2, q = tid & 3;
  for (int j = 0; j < kFacB; ++j) {
    const double d = S[j][j];
    const bool ok = d > 0.0 && d < INFINITY;
    const double r = ok ? sqrt(d) : __longlong_as_double(0x7FF8000000000000ll);  // NaN spreads to the rest
    if (!ok && tid == 0) report_error(ERR_NOT_POSITIVE_DEFINITE);
    const double inv = 1.0 / r;
    if (q == 0 && i > j) col[i] = S[i][j] * inv;
    __syncthreads();
    if (i > j) {
      const double li = col[i];
      for (int c = j + 1 + ((q - j - 1) & 3); c <= i; c += 4) S[i][c] = fma(-li, col[c], S[i][c]);
      if (q == 0) S[i][j] = li;
    } else if (i == j && q == 0) {
      S[j][j] = r;
    }
    __syncthreads();
  }
  for (int e = tid; e < kFacB * kFacB; e += 256) {
    const int ii = e >> 6, c = e & 63;
    Ab[int64_t(ii) * lda + c] = S[ii][c];
  }
  // inverse, column by column (columns are independent): 4 lanes per column
  // split each dot product and sum it with shuffles.  Li[c][c] = 1 / L[c][c];
  // Li[i][c] = -(sum_{k = c}^{i-1} L[i][k] Li[k][c]) / L[i][i].  Li is kept in the
  // strict upper part of S as S[c][i] (transposed), which the factor does not use.
  __shared__ double diag_inv[kFacB];
  if (tid < kFacB) diag_inv[tid] = 1.0 / S[tid][tid];
  __syncthreads();
  const int c = i;  // column of this thread's group (4 lanes q per column)
  double* Li = Dinv;
  for (int row = 0; row < kFacB; ++row) {
    double v = 0.0;
    if (row > c) {
      for (int k = c + q; k < row; k += 4) v = fma(S[row][k], (k == c ? diag_inv[c] : S[c][k]), v);
    }
    v += __shfl_xor_sync(0xFFFFFFFFu, v, 1);
    v += __shfl_xor_sync(0xFFFFFFFFu, v, 2);
    if (q == 0 && row > c) S[c][row] = -v * diag_inv[row];
    __syncwarp();
  }
  __syncthreads();
  for (int e = tid; e < kFacB * kFacB; e += 256) {
    const int rr = e >> 6, cc = e & 63;
    Li[e] = rr < cc ? 0.0 : (rr == cc ? diag_inv[rr] : S[cc][rr]);
  }
}

// Z = identity over [Kp, Kp].
__global__ void __launch_bounds__(256) fac_eye_kernel(double* Z, int64_t Kp) {
  const int64_t n = Kp * Kp;
  for (int64_t e = int64_t(blockIdx.x) * 256 + threadIdx.x; e < n; e += int64_t(gridDim.x) * 256)
    Z[e] = (e / Kp == e % Kp) ? 1.0 : 0.0;
}

// U [K, K] fp32: U[i][j] = Z[K-1-j][K-1-i] for i <= j, 0 below the diagonal.
__global__ void __launch_bounds__(256) fac_u_kernel(const double* __restrict__ Z, int64_t K, int64_t Kp,
                                                    float* __restrict__ U) {
  __shared__ float tile[32][33];
  const int64_t i0 = int64_t(blockIdx.y) * 32, j0 = int64_t(blockIdx.x) * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  // tile[jj][ii] = Z[K-1-(j0+jj)][K-1-(i0+ii)], read along ii (consecutive columns of Z)
  for (int r = ty; r < 32; r += 8) {
    const int64_t j = j0 + r, i = i0 + tx;
    float v = 0.f;
    if (i < K && j < K && i <= j) v = float(Z[(K - 1 - j) * Kp + (K - 1 - i)]);
    tile[r][tx] = v;
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    const int64_t i = i0 + r, j = j0 + tx;
    if (i < K && j < K) U[i * K + j] = tile[tx][r];
  }
}

}  // namespace wq
