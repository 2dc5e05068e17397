// gemm_tcgen05.cuh -- prefill GEMM for the quantized Linear at large M on the
// 5th-generation tensor cores (tcgen05, sm_100a).
//
// Y[M, N] = (X * act_inv_s)[M, K] * dequant(Wq)[N, K]^T, bf16 x bf16 -> fp32
// accumulate in tensor memory -> bf16.  This is the fused alternative the
// pages call for ("quantization primer" section 13: read compressed weights,
// dequantize inside the kernel, multiply; "Lance-Quant" section "当前局限":
// a pure dequant-then-matmul module is ~10% slower than bf16).
//
// One CTA computes one BM x BN output tile (BM = 128 rows of X, BN = 128 or
// 256 rows of W) with warp-specialized roles and an mbarrier pipeline of
// STAGES k-blocks (BK = 64):
//   warp 0      TMA producer: X tile [BM x 64] bf16 (128-byte swizzle) and
//               the packed weight tile [BN x 32 bytes] into stage s;
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer
//               (M=128, N=BN, K=16, four per k-block), tcgen05.commit frees
//               the stage and finally signals the epilogue;
//   warps 4..   2 BN dequantizer threads, two per weight row (32 k each):
//               unpack the stage's codes to bf16 (INT4: (q - z) * scale; NVFP4:
//               e2m1 * e4m3 block scale, the fp32 tensor scale is applied in
//               the epilogue) and store them in the canonical K-major
//               128-byte-swizzled layout the MMA reads; then, after the last
//               k-block, the same warps drain the accumulator with
//               tcgen05.ld and write bf16 rows of Y.
// Every wait is bounded (2 s): a stuck pipeline sets the device error word
// and the CTA leaves after releasing its tensor memory.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "wq_common.cuh"

namespace wq {

constexpr int kGemmBM = 128;
constexpr int kGemmBK = 64;

// BMT = 128: one M = 128 MMA per k step; BMT = 256: two (rows 0-127 and
// 128-255 of the X tile) sharing the dequantized W tile, into two tensor-
// memory accumulators side by side (columns [0, BN) and [BN, 2 BN)), which
// halves the dequantization per flop.
template <int BN, int BMT = kGemmBM, bool TMA_B = false>
struct GemmShape {
  static constexpr int STAGES = (BN == 256) ? 3 : 4;
  static constexpr int A_BYTES = BMT * kGemmBK * 2;      // bf16 X tile (16 or 32 KB)
  static constexpr int B_BYTES = BN * kGemmBK * 2;       // dequantized W tile
  static constexpr int P_BYTES = BN * kGemmBK / 2;       // packed 4-bit W tile
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + P_BYTES;
  // dequantizer (then epilogue) threads: two per weight row, each 32 of a k-block's
  // 64 k, so that 8 or 16 warps hide the dequantization's dependency chains; the
  // bf16-B mode only needs the epilogue warps
  static constexpr int DEQ_SPLIT = TMA_B ? 1 : 2;
  static constexpr int DEQ_THREADS = DEQ_SPLIT * BN;
  static constexpr int THREADS = 128 + DEQ_THREADS;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;  // + alignment slack
  static constexpr int NACC = BMT / kGemmBM;             // accumulators
  static constexpr int TMEM_COLS = BN * NACC;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory of one CTA");
  static_assert(TMEM_COLS <= 512, "tensor memory columns");
};

struct GemmArgs {
  CUtensorMap tmA;          // X bf16 [M, K]: dims {K, M}, box {64, 128}, 128B swizzle
  CUtensorMap tmP;          // packed codes u8 [N, K/2]: dims {K/2, N}, box {32, BN}
  const uint16_t* scales;   // INT4 fp16 [N, K/G]
  const uint32_t* zeros;    // INT4 [N, ceil(K/G/8)] or null (symmetric, z = 8)
  const uint8_t* bscale;    // NVFP4 e4m3 [N, K/16]
  const float* gscale;      // NVFP4 fp32 [1]
  const float* inv_s;       // fp32 [K] or null
  uint16_t* Y;              // bf16 [M, N]
  CUtensorMap tmY;          // Y bf16 [M, N], box {32, 32}, 64B swizzle (used iff y_tma)
  CUtensorMap tmPart;       // split-K partials fp32 [tiles * splitk * BMT, BN], box {32, 32}, 128B swizzle
  int y_tma;                // unsplit INT4 / NVFP4 with N % 8 == 0 and Y 16-byte aligned: Y boxes by TMA
  double* sq_partials;      // FMT_BF16_SQ: one partial sum of squares per epilogue warp
  float* part;              // split-K: fp32 partial tiles [tiles][splitk][BMT * BN] (split_reduce_kernel sums them)
  int splitk;               // CTAs per output tile along K (gridDim.z); 1 = no split
  int M, N, K;              // K: reduction length (for FMT_BF16_SQ the length of B's rows)
  int a_kblocks;            // A k-block index wraps modulo this (FMT_BF16_SQ reuses X twice)
  int log2g;
};

// B operand modes of gemm_tcgen05_kernel.
enum { GEMM_INT4 = 0, GEMM_NVFP4 = 1, GEMM_BF16_SQ = 2 };

// ------------------------------------------------------------------ tcgen05 helpers
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulator.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once every previously issued tcgen05.mma of this thread completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Shared-memory matrix descriptor of a K-major tile in the canonical
// 128-byte-swizzle layout: 8-row x 128-byte atoms, atoms 1024 B apart.
__device__ __forceinline__ uint64_t desc_kmajor_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= uint64_t((saddr >> 4) & 0x3FFFu);  // start address
  d |= uint64_t(1) << 16;                 // leading byte offset (unused by swizzled K-major)
  d |= uint64_t(1024 >> 4) << 32;         // stride byte offset: next 8-row atom
  d |= uint64_t(1) << 46;                 // descriptor version of sm_100
  d |= uint64_t(2) << 61;                 // 128-byte swizzle
  return d;
}

// Instruction descriptor: bf16 x bf16 -> fp32, both K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// 32 lanes x 32 columns of fp32 from tensor memory (this warp's lane quarter).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
        "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hsub2(*reinterpret_cast<__nv_bfloat162*>(&a), *reinterpret_cast<__nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&a), *reinterpret_cast<__nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t prmt_b32(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
__device__ __forceinline__ uint32_t lop3_andor(uint32_t a, uint32_t mask, uint32_t bits) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(bits));
  return d;
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

// Byte offset of 16-byte chunk `c` (k = 8c..8c+7) of row `r` in a K-major
// 128B-swizzled tile (rows of 128 bytes, 8-row atoms of 1024 bytes).
__device__ __forceinline__ uint32_t sw128_offset(int r, int c) {
  return uint32_t((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

// INT4: one packed word (codes of k = 8j..8j+7) -> 8 bf16 (q - z) * scale,
// natural k order, as 4 bf16x2 words.
__device__ __forceinline__ uint4 dequant_word_int4(uint32_t w, uint32_t zoff2, uint32_t sc2) {
  // {128 + q_i, 128 + q_{i+4}} for i = 0..3 (bf16 exponent-bias trick), exact
  uint32_t p0 = lop3_andor(w, 0x000F000Fu, 0x43004300u);
  uint32_t p1 = lop3_andor(w >> 4, 0x000F000Fu, 0x43004300u);
  uint32_t p2 = lop3_andor(w >> 8, 0x000F000Fu, 0x43004300u);
  uint32_t p3 = lop3_andor(w >> 12, 0x000F000Fu, 0x43004300u);
  // (128 + q) - (128 + z) = q - z exactly, then * scale (one bf16 rounding)
  p0 = bf16x2_mul(bf16x2_sub(p0, zoff2), sc2);
  p1 = bf16x2_mul(bf16x2_sub(p1, zoff2), sc2);
  p2 = bf16x2_mul(bf16x2_sub(p2, zoff2), sc2);
  p3 = bf16x2_mul(bf16x2_sub(p3, zoff2), sc2);
  // p_i = {w_i, w_{i+4}} -> natural pairs {w0,w1} {w2,w3} {w4,w5} {w6,w7}
  return make_uint4(prmt_b32(p0, p1, 0x5410), prmt_b32(p2, p3, 0x5410), prmt_b32(p0, p1, 0x7632),
                    prmt_b32(p2, p3, 0x7632));
}

// NVFP4: one packed word (codes of k = 8j..8j+7, low nibble = even k) -> 8 bf16
// e2m1 * sb, natural order, with integer and bf16 ALU operations only (no
// conversion instructions): the bf16 bytes of |e2m1| come from two byte
// lookups (prmt over an 8-entry table: magnitude index = the code's low 3
// bits), the bf16 block scale sb2 = {sb, sb} multiplies them (exact: at most
// 6 significant bits, |v| <= 6 * 448), and each code's sign bit is OR-ed into
// its product.
__device__ __forceinline__ uint32_t lop3_or_and(uint32_t a, uint32_t b, uint32_t c) {  // a | (b & c)
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xF8;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint4 dequant_word_nvfp4(uint32_t w, uint32_t sb2) {
  // bf16 of 0, 0.5, 1, 1.5 | 2, 3, 4, 6: low bytes and high bytes, table index = byte index
  constexpr uint32_t kLoA = 0xC0800000u, kLoB = 0xC0804000u, kHiA = 0x3F3F3F00u, kHiB = 0x40404040u;
  const uint32_t s0 = w & 0x7777u, s1 = (w >> 16) & 0x7777u;  // magnitude indices of codes 0-3, 4-7
  const uint32_t l0 = prmt_b32(kLoA, kLoB, s0), h0 = prmt_b32(kHiA, kHiB, s0);
  const uint32_t l1 = prmt_b32(kLoA, kLoB, s1), h1 = prmt_b32(kHiA, kHiB, s1);
  // {code 2i, code 2i+1} as bf16x2 magnitudes, times the block scale
  const uint32_t m0 = bf16x2_mul(prmt_b32(l0, h0, 0x5140), sb2), m1 = bf16x2_mul(prmt_b32(l0, h0, 0x7362), sb2);
  const uint32_t m2 = bf16x2_mul(prmt_b32(l1, h1, 0x5140), sb2), m3 = bf16x2_mul(prmt_b32(l1, h1, 0x7362), sb2);
  // sign of code 2i (bit 8i+3 of w = bit 7 of byte i of w << 4) -> bit 15, of code 2i+1 (bit 7 of byte i of w) -> bit 31
  const uint32_t t = w << 4;
  return make_uint4(lop3_or_and(m0, prmt_b32(t, w, 0x4000), 0x80008000u),
                    lop3_or_and(m1, prmt_b32(t, w, 0x5010), 0x80008000u),
                    lop3_or_and(m2, prmt_b32(t, w, 0x6020), 0x80008000u),
                    lop3_or_and(m3, prmt_b32(t, w, 0x7030), 0x80008000u));
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

template <int FMT, int BN, int BMT = kGemmBM>
__global__ void __launch_bounds__(GemmShape<BN, BMT, FMT == GEMM_BF16_SQ>::THREADS, 1)
    gemm_tcgen05_kernel(const __grid_constant__ GemmArgs a) {
  using S = GemmShape<BN, BMT, FMT == GEMM_BF16_SQ>;
  static_assert(FMT != GEMM_BF16_SQ || BMT == kGemmBM, "the sum-of-squares epilogue uses one accumulator");
  constexpr int STAGES = S::STAGES;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled operand tiles
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
  const uint32_t sbase = smem_u32(smem);
  // stage s: A at s*STAGE, B after A, P after B
  auto a_addr = [&](int s) { return sbase + uint32_t(s * S::STAGE_BYTES); };
  auto b_addr = [&](int s) { return sbase + uint32_t(s * S::STAGE_BYTES + S::A_BYTES); };
  auto p_ptr = [&](int s) { return smem + s * S::STAGE_BYTES + S::A_BYTES + S::B_BYTES; };
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * S::STAGE_BYTES);
  uint64_t* full = bars;                 // TMA landed (A + packed W)
  uint64_t* bready = bars + STAGES;      // dequantized W written
  uint64_t* empty = bars + 2 * STAGES;   // MMAs of the stage finished
  uint64_t* accum = bars + 3 * STAGES;   // accumulator complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * STAGES + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * BMT, n0 = blockIdx.x * BN;
  const int nkb_all = (a.K + kGemmBK - 1) / kGemmBK;
  // split-K: this CTA's k-blocks [kbeg, kbeg + nkb)
  const int splits = a.splitk > 1 ? a.splitk : 1;
  const int kbeg = int((int64_t(nkb_all) * blockIdx.z) / splits);
  const int nkb = int((int64_t(nkb_all) * (blockIdx.z + 1)) / splits) - kbeg;
  constexpr int DEQ_WARP0 = 4;
  constexpr int DEQ_WARPS = S::DEQ_THREADS / 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&bready[s], DEQ_WARPS);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accum, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&a.tmA);
    prefetch_tmap(&a.tmP);
    if (a.y_tma) prefetch_tmap(&a.tmY);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, S::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_acc = *tmem_slot;

  // Let the next kernel in the stream launch; every thread that reads global
  // memory waits for the previous kernel first (griddepcontrol.wait is what makes
  // its writes visible: the weights themselves may have just been quantized).
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      asm volatile("griddepcontrol.wait;" ::: "memory");
      int issued = 0;
      for (int i = 0; i < nkb; ++i) {
        const int kb = kbeg + i, s = i % STAGES, r = i / STAGES;
        if (r > 0 && !mbar_wait(&empty[s], (r - 1) & 1, ERR_TIMEOUT_PIPE, abort_flag)) break;
        if (FMT == GEMM_BF16_SQ) {
          mbar_arrive_expect_tx(&full[s], S::A_BYTES + S::B_BYTES);
          tma_load_2d(smem + s * S::STAGE_BYTES, &a.tmA, &full[s], (kb % a.a_kblocks) * kGemmBK, m0);
          tma_load_2d(smem + s * S::STAGE_BYTES + S::A_BYTES, &a.tmP, &full[s], kb * kGemmBK, n0);
        } else {
          mbar_arrive_expect_tx(&full[s], S::A_BYTES + S::P_BYTES);
          tma_load_2d(smem + s * S::STAGE_BYTES, &a.tmA, &full[s], kb * kGemmBK, m0);
          tma_load_2d(p_ptr(s), &a.tmP, &full[s], kb * (kGemmBK / 2), n0);
        }
        ++issued;
      }
      // On abort, let copies already in flight land before the CTA leaves.
      if (*abort_flag) {
        for (int kb = (issued > STAGES ? issued - STAGES : 0); kb < issued; ++kb)
          mbar_wait(&full[kb % STAGES], (kb / STAGES) & 1, ERR_TIMEOUT_TMA, nullptr);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(kGemmBM, BN);
      bool ok = true;
      for (int i = 0; i < nkb && ok; ++i) {
        const int s = i % STAGES, r = i / STAGES;
        ok = mbar_wait(&full[s], r & 1, ERR_TIMEOUT_TMA, abort_flag) &&
             (FMT == GEMM_BF16_SQ || mbar_wait(&bready[s], r & 1, ERR_TIMEOUT_PIPE, abort_flag));
        if (!ok) break;
        tc_fence_after();
        const uint64_t ad = desc_kmajor_sw128(a_addr(s));
        const uint64_t bd = desc_kmajor_sw128(b_addr(s));
#pragma unroll
        for (int kk = 0; kk < kGemmBK / 16; ++kk) {  // +32 bytes per K=16 step inside the swizzle atom
          umma_bf16(tmem_acc, ad + uint64_t(2 * kk), bd + uint64_t(2 * kk), IDESC, (i | kk) != 0);
          if (S::NACC == 2)  // rows 128-255 of the X tile start 16 KB (16 atoms) further
            umma_bf16(tmem_acc + BN, desc_kmajor_sw128(a_addr(s) + 16384) + uint64_t(2 * kk),
                      bd + uint64_t(2 * kk), IDESC, (i | kk) != 0);
        }
        umma_commit(&empty[s]);
      }
      umma_commit(accum);  // also on abort: completes when issued MMAs are done
    }
  } else if (warp >= DEQ_WARP0) {
    // ---------------------------------------------------------- dequantize, then epilogue
    constexpr int NW = 8 / S::DEQ_SPLIT;         // packed words (8 k each) per thread and k-block
    const int dt = threadIdx.x - DEQ_WARP0 * 32;
    const int t = dt % BN;                       // weight row within the tile
    const int h = dt / BN;                       // which part of the k-block (words NW h .. NW h + NW - 1)
    const int n = min(n0 + t, a.N - 1);          // rows past N dequantize row N-1 (outputs masked)
    const int ng = a.K >> a.log2g;
    const uint32_t zw_stride = (ng + 7) >> 3;
    bool ok = true;
    // Per-row metadata of k-block kb, fetched one k-block ahead so its global
    // (L2) latency overlaps the previous k-block's dequantization.
    auto fetch_meta = [&](int kb, uint32_t& raw_a, uint32_t& raw_b) {
      raw_a = 0;
      raw_b = 0x88888888u;
      if (kb >= kbeg + nkb) return;
      if (FMT == GEMM_INT4) {
        const int g = (kb * kGemmBK) >> a.log2g;
        raw_a = __ldg(a.scales + int64_t(n) * ng + g);
        if (a.log2g == 5 && g + 1 < ng)  // G = 32: the k-block's second group (same zero word: g is even)
          raw_a |= uint32_t(__ldg(a.scales + int64_t(n) * ng + g + 1)) << 16;
        if (a.zeros) raw_b = __ldg(a.zeros + int64_t(n) * zw_stride + (g >> 3));
      } else if (FMT == GEMM_NVFP4) {
        const int nb = a.K >> 4;
        const uint8_t* bs = a.bscale + int64_t(n) * nb + kb * 4;
        const int rem = nb - kb * 4;  // K % 64 == 32 leaves two blocks in the last k-block
        if (rem >= 4 && (reinterpret_cast<uintptr_t>(bs) & 3) == 0) {
          raw_a = __ldg(reinterpret_cast<const uint32_t*>(bs));  // the k-block's 4 scales in one load
        } else {
          raw_a = 0;
          for (int q = 0; q < 4 && q < rem; ++q) raw_a |= uint32_t(__ldg(bs + q)) << (8 * q);
        }
      }
    };
    asm volatile("griddepcontrol.wait;" ::: "memory");
    uint32_t meta_a, meta_b;
    fetch_meta(kbeg, meta_a, meta_b);
    for (int i = 0; i < (FMT == GEMM_BF16_SQ ? 0 : nkb); ++i) {
      const int kb = kbeg + i, s = i % STAGES, r = i / STAGES;
      const uint32_t cur_a = meta_a, cur_b = meta_b;
      fetch_meta(kb + 1, meta_a, meta_b);
      uint32_t sc2[2] = {0, 0}, zoff2[2] = {0, 0};  // INT4: words 0-3 / 4-7 (two groups when G = 32)
      uint32_t sbv[4] = {0, 0, 0, 0};  // NVFP4: the k-block's 4 E4M3 block scales as bf16x2 {sb, sb}
      if (FMT == GEMM_INT4) {
        const int g = (kb * kGemmBK) >> a.log2g;
        if (a.log2g == 5) {  // G = 32: groups g (words 0-3) and g + 1 (words 4-7)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float sc = __half2float(__ushort_as_half(uint16_t(h ? cur_a >> 16 : cur_a)));
            const int z = (cur_b >> (4 * ((g + h) & 7))) & 0xF;
            sc2[h] = pack_bf16x2(sc, sc);
            const uint32_t zb = 0x4300u | uint32_t(z);  // bf16(128 + z)
            zoff2[h] = zb | (zb << 16);
          }
        } else {  // one group covers the k-block
          const float sc = __half2float(__ushort_as_half(uint16_t(cur_a)));
          const int z = (cur_b >> (4 * (g & 7))) & 0xF;
          sc2[0] = sc2[1] = pack_bf16x2(sc, sc);
          const uint32_t zb = 0x4300u | uint32_t(z);
          zoff2[0] = zoff2[1] = zb | (zb << 16);
        }
      } else {
#pragma unroll
        for (int q = 0; q < 4; q += 2) {  // two E4M3 bytes -> f16x2 -> fp32 -> bf16 (all exact), then replicate each
          uint32_t h2;
          asm("{ .reg .b16 t; cvt.u16.u32 t, %1; cvt.rn.f16x2.e4m3x2 %0, t; }"
              : "=r"(h2) : "r"((cur_a >> (8 * q)) & 0x7F7Fu));
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
          sbv[q] = pack_bf16x2(f.x, f.x);
          sbv[q + 1] = pack_bf16x2(f.y, f.y);
        }
      }
      if (!mbar_wait(&full[s], r & 1, ERR_TIMEOUT_TMA, abort_flag)) { ok = false; break; }
      const uint32_t prow = smem_u32(p_ptr(s)) + uint32_t(t * 32 + h * NW * 4);
      uint32_t words[NW];
#pragma unroll
      for (int q = 0; q < NW / 4; ++q) {
        const uint4 qv = ld_shared_v4(prow + 16 * q);
        words[4 * q] = qv.x; words[4 * q + 1] = qv.y; words[4 * q + 2] = qv.z; words[4 * q + 3] = qv.w;
      }
      const uint32_t brow = b_addr(s);
#pragma unroll
      for (int jw = 0; jw < NW; ++jw) {
        const int j = NW * h + jw;  // word of the k-block
        // its scale data, selected without a runtime-indexed array
        const bool hi4 = NW == 8 ? jw >= 4 : h != 0;            // words 4-7: second G = 32 group
        const int blk = NW == 8 ? jw >> 1 : 2 * h + (jw >> 1);  // NVFP4 block of the word
        const uint32_t zz = hi4 ? zoff2[1] : zoff2[0], ss = hi4 ? sc2[1] : sc2[0];
        const uint32_t sbk = blk == 0 ? sbv[0] : blk == 1 ? sbv[1] : blk == 2 ? sbv[2] : sbv[3];
        uint4 v = (FMT == GEMM_INT4) ? dequant_word_int4(words[jw], zz, ss) : dequant_word_nvfp4(words[jw], sbk);
        if (a.inv_s) {
          const int k = kb * kGemmBK + 8 * j;
          if (k < a.K) {
            const float4 i0 = __ldg(reinterpret_cast<const float4*>(a.inv_s + k));
            const float4 i1 = __ldg(reinterpret_cast<const float4*>(a.inv_s + k) + 1);
            v.x = bf16x2_mul(v.x, pack_bf16x2(i0.x, i0.y));
            v.y = bf16x2_mul(v.y, pack_bf16x2(i0.z, i0.w));
            v.z = bf16x2_mul(v.z, pack_bf16x2(i1.x, i1.y));
            v.w = bf16x2_mul(v.w, pack_bf16x2(i1.z, i1.w));
          }
        }
        st_shared_v4(brow + sw128_offset(t, j), v);
      }
      fence_proxy_async_smem();  // generic-proxy stores -> visible to the tensor core
      __syncwarp();
      if (lane == 0) mbar_arrive(&bready[s]);
    }
    // ---------------------------------------------------------- epilogue
    bool go = ok && mbar_wait(accum, 0, ERR_TIMEOUT_MMA, abort_flag);
    go = __all_sync(0xffffffffu, go);  // tcgen05.ld below is warp-collective
    const int quarter = warp & 3;                      // TMEM lanes 32*quarter .. +31
    constexpr int WPQ = DEQ_WARPS / 4;                 // epilogue warps per lane quarter
    const int wi = (warp - DEQ_WARP0) >> 2;            // this warp's index among them
    const bool vec = (a.N % 8) == 0;
    if (a.splitk > 1) {
      // split-K: this CTA's fp32 partial tile leaves by TMA (32 x 32 boxes staged in
      // the freed stage buffers, 128-byte swizzle); split_reduce_kernel, launched
      // next, adds the partials in split order and writes Y (no CTA waits for
      // another; the sum's order does not depend on timing).
      if (go) {
        tc_fence_after();
        const int tile = blockIdx.y * gridDim.x + blockIdx.x;
        const int prow0 = (tile * a.splitk + int(blockIdx.z)) * BMT;  // this partial tile's first row
        int nbox = 0;
        for (int u = wi; u < S::NACC * (BN / 32); u += WPQ) {
          const int acc = u / (BN / 32), c = (u % (BN / 32)) * 32;
          uint32_t v[32];
          tmem_ld32(tmem_acc + (uint32_t(quarter * 32) << 16) + uint32_t(acc * BN + c), v);
          uint8_t* box = smem + (warp - DEQ_WARP0) * 8192 + (nbox & 1) * 4096;
          if (lane == 0) bulk_wait_read<1>();
          __syncwarp();
          const uint32_t rbase = smem_u32(box) + uint32_t(lane * 128);
#pragma unroll
          for (int q = 0; q < 8; ++q)  // 16-byte piece q of the row, at its 128B-swizzled place
            st_shared_v4(rbase + uint32_t((q ^ (lane & 7)) << 4),
                         make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]));
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&a.tmPart, box, c, prow0 + acc * kGemmBM + quarter * 32);
            bulk_commit();
          }
          ++nbox;
        }
        if (lane == 0) bulk_wait_all();  // the partial is stored before the CTA leaves
      }
    } else if (go) {
      tc_fence_after();
      const float gmul = (FMT == GEMM_NVFP4) ? __ldg(a.gscale) : 1.0f;
      double sq = 0.0;
      int nbox = 0;
      // (accumulator, 32-column chunk) units of this quarter, dealt round-robin
      for (int u = wi; u < S::NACC * (BN / 32); u += WPQ) {
        const int acc = u / (BN / 32), c = (u % (BN / 32)) * 32;
        const int row = m0 + acc * kGemmBM + quarter * 32 + lane;
        uint32_t v[32];
        tmem_ld32(tmem_acc + (uint32_t(quarter * 32) << 16) + uint32_t(acc * BN + c), v);
        if (FMT != GEMM_BF16_SQ && a.y_tma) {
          // the unit's 32 x 32 box (row = lane) through shared memory and one TMA store
          // (full lines to L2).  Every k-block's MMAs completed, so the stage buffers
          // are free: each epilogue warp takes two 2 KB boxes of them, alternating; the
          // one used two boxes ago must have been read.
          uint8_t* box = smem + ((warp - DEQ_WARP0) * 2 + (nbox & 1)) * 2048;
          if (lane == 0) bulk_wait_read<1>();
          __syncwarp();
          const uint32_t rbase = smem_u32(box) + uint32_t(lane * 64);
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {  // 16-byte piece qq of the row, at its 64B-swizzled place
            uint4 o;
            o.x = pack_bf16x2(__uint_as_float(v[8 * qq + 0]) * gmul, __uint_as_float(v[8 * qq + 1]) * gmul);
            o.y = pack_bf16x2(__uint_as_float(v[8 * qq + 2]) * gmul, __uint_as_float(v[8 * qq + 3]) * gmul);
            o.z = pack_bf16x2(__uint_as_float(v[8 * qq + 4]) * gmul, __uint_as_float(v[8 * qq + 5]) * gmul);
            o.w = pack_bf16x2(__uint_as_float(v[8 * qq + 6]) * gmul, __uint_as_float(v[8 * qq + 7]) * gmul);
            st_shared_v4(rbase + uint32_t((qq ^ ((lane >> 1) & 3)) << 4), o);
          }
          fence_proxy_async_smem();  // generic-proxy stores -> visible to the TMA
          __syncwarp();
          if (lane == 0) {  // rows or columns past M / N are clipped by the TMA
            tma_store_2d(&a.tmY, box, n0 + c, m0 + acc * kGemmBM + quarter * 32);
            bulk_commit();
          }
          ++nbox;
          continue;
        }
        if (FMT == GEMM_BF16_SQ) {
          float part = 0.f;
          if (row < a.M) {
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              const float x = (n0 + c + q < a.N) ? __uint_as_float(v[q]) : 0.f;
              part = fmaf(x, x, part);
            }
          }
          sq += double(part);
          continue;
        }
        if (row < a.M) {
          uint16_t* yrow = a.Y + int64_t(row) * a.N;
          const int nb = n0 + c;
          if (vec && nb + 32 <= a.N) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4 o;
              o.x = pack_bf16x2(__uint_as_float(v[8 * q + 0]) * gmul, __uint_as_float(v[8 * q + 1]) * gmul);
              o.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]) * gmul, __uint_as_float(v[8 * q + 3]) * gmul);
              o.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]) * gmul, __uint_as_float(v[8 * q + 5]) * gmul);
              o.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]) * gmul, __uint_as_float(v[8 * q + 7]) * gmul);
              *reinterpret_cast<uint4*>(yrow + nb + 8 * q) = o;
            }
          } else {
            for (int q = 0; q < 32; ++q)
              if (nb + q < a.N) yrow[nb + q] = uint16_t(f32_to_bf16_bits(__uint_as_float(v[q]) * gmul));
          }
        }
      }
      if (FMT == GEMM_BF16_SQ) {
        // fixed-order warp reduction; one partial per (tile, epilogue warp)
#pragma unroll
        for (int off = 16; off; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
        if (lane == 0) {
          const int tile = blockIdx.y * gridDim.x + blockIdx.x;
          a.sq_partials[int64_t(tile) * DEQ_WARPS + (warp - DEQ_WARP0)] = sq;
        }
      }
    }
  }
  if (FMT != GEMM_BF16_SQ && a.y_tma && warp >= DEQ_WARP0 && lane == 0) bulk_wait_all();  // Y boxes stored
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_acc, S::TMEM_COLS);
  }
}

// Split-K reduction: Y[m, n] = gmul * sum over the splits, in split order, of the
// fp32 partial tiles part[tile][split][BMT][BN] (tile = (m / BMT) * n_tiles + n / BN).
// Each thread takes 4 consecutive columns of one tile row: every split's float4
// load in flight at once, coalesced across the warp.  A stream-ordered successor
// of the GEMM: it reads the partials only after griddepcontrol.wait.
__global__ void __launch_bounds__(256) split_reduce_kernel(const float* __restrict__ part, int splitk, int bmt,
                                                           int bn, int n_tiles, int64_t quads, int M, int N,
                                                           const float* __restrict__ gscale, uint16_t* __restrict__ Y) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const float gmul = gscale ? __ldg(gscale) : 1.0f;
  const int64_t tile_quads = int64_t(bmt) * bn / 4;
  for (int64_t g = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; g < quads; g += int64_t(gridDim.x) * blockDim.x) {
    const int64_t tile = g / tile_quads;
    const int e = int(g - tile * tile_quads) * 4;  // element within the tile
    const int rt = e / bn, ct = e - rt * bn;
    const int row = int(tile / n_tiles) * bmt + rt, col = int(tile % n_tiles) * bn + ct;
    if (row >= M || col >= N) continue;
    const float4* src = reinterpret_cast<const float4*>(part + tile * splitk * int64_t(bmt) * bn + e);
    const int64_t stride4 = int64_t(bmt) * bn / 4;
    float4 x[8];
#pragma unroll
    for (int sp = 0; sp < 8; ++sp)
      if (sp < splitk) x[sp] = __ldcs(src + sp * stride4);
    float4 t = x[0];
#pragma unroll
    for (int sp = 1; sp < 8; ++sp)
      if (sp < splitk) {
        t.x += x[sp].x; t.y += x[sp].y; t.z += x[sp].z; t.w += x[sp].w;
      }
    uint16_t* yp = Y + int64_t(row) * N + col;
    if ((N & 3) == 0 && (reinterpret_cast<uintptr_t>(Y) & 7) == 0) {
      *reinterpret_cast<uint2*>(yp) = make_uint2(pack_bf16x2(t.x * gmul, t.y * gmul), pack_bf16x2(t.z * gmul, t.w * gmul));
    } else {
      const float tv[4] = {t.x, t.y, t.z, t.w};
      for (int q = 0; q < 4; ++q)
        if (col + q < N) yp[q] = uint16_t(f32_to_bf16_bits(tv[q] * gmul));
    }
  }
}

// Split-K for the AWQ loss GEMM: the sum over one tile's rows ry*16 .. ry*16+15 of
// y^2, y = the splits' partials added in split order, into partials[tile * 8 + ry]
// (gridDim.y = 8 row slices of a 128-row tile).  Each thread takes float4 column
// groups of those rows with every split's load in flight; fixed-order reductions.
__global__ void __launch_bounds__(256) split_sq_reduce_kernel(const float* __restrict__ part, int splitk, int bn,
                                                              int n_tiles, int M, int N, double* __restrict__ partials) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int tile = blockIdx.x, ry = blockIdx.y;
  const int m0 = (tile / n_tiles) * kGemmBM, n0 = (tile % n_tiles) * bn;
  const int64_t tile_elems = int64_t(kGemmBM) * bn;
  const float* base = part + int64_t(tile) * splitk * tile_elems;
  const int quads = 16 * bn / 4;
  double sq = 0.0;
  for (int qd = threadIdx.x; qd < quads; qd += blockDim.x) {
    const int rt = ry * 16 + (qd * 4) / bn, ct = (qd * 4) % bn;
    const float4* src = reinterpret_cast<const float4*>(base + int64_t(rt) * bn + ct);
    float4 x[8];
#pragma unroll
    for (int sp = 0; sp < 8; ++sp)
      if (sp < splitk) x[sp] = __ldcs(src + sp * (tile_elems / 4));
    float4 t = x[0];
#pragma unroll
    for (int sp = 1; sp < 8; ++sp)
      if (sp < splitk) {
        t.x += x[sp].x; t.y += x[sp].y; t.z += x[sp].z; t.w += x[sp].w;
      }
    const int row = m0 + rt, col = n0 + ct;
    float acc = 0.f;
    if (row < M) {
      if (col < N) acc = fmaf(t.x, t.x, acc);
      if (col + 1 < N) acc = fmaf(t.y, t.y, acc);
      if (col + 2 < N) acc = fmaf(t.z, t.z, acc);
      if (col + 3 < N) acc = fmaf(t.w, t.w, acc);
    }
    sq += double(acc);
  }
  __shared__ double red[8];
#pragma unroll
  for (int off = 16; off; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = sq;
  __syncthreads();
  if (threadIdx.x == 0) {
    double tsum = 0.0;
    for (int w = 0; w < int(blockDim.x >> 5); ++w) tsum += red[w];
    partials[int64_t(tile) * 8 + ry] = tsum;
  }
}

}  // namespace wq
