// gemm_fp4.cuh -- NVFP4 W4A4 GEMM on the block-scaled FP4 tensor cores
// (tcgen05.mma kind::mxf4nvf4, one E4M3 scale per 16 elements).
//
// "OmniQuant" section 4.2 (W4A4: weights and activations both 4-bit);
// "Lance-Quant" section "量化应用" (NVFP4 = E2M1 codes + E4M3 scale per 16,
// for Blackwell tensor cores).  The activations were quantized to NVFP4 along
// K just before (same rule as the weight pack, own per-tensor scale g_x):
//   Y[m, n] = g_x g_w sum_b sx[m,b] sw[n,b] sum_{k in b} e2m1(xq[m,k]) e2m1(wq[n,k])
// which is exactly what the block-scaled MMA computes (fp32 accumulation);
// the two per-tensor scales multiply the accumulator in the epilogue.
//
// One CTA = one 128 x BN output tile; k-blocks of 256 elements (128 bytes of
// packed E2M1 per row = one 128-byte swizzle atom), STAGES deep:
//   warp 0      TMA: packed X tile [128 x 128 B] and W tile [BN x 128 B], and
//               (K % 256 == 0) their E4M3 scale tiles [rows x 16 B]
//   warp 1      TMEM allocation (512 columns) and the tcgen05.mma issuer
//               (4 MMAs of K = 64 per k-block)
//   warps 4..11 copy the stage's E4M3 scales into tensor memory with
//               tcgen05.st (warps 4-7: X scales, 8-11: W scales), reading
//               them from the stage in shared memory (or, when K is not a
//               multiple of 256, from global memory one k-block ahead), then
//               run the epilogue (tcgen05.ld, x g_x g_w, bf16 store).
// With K a multiple of 256 the host launches the persistent variant below
// instead.
// Scale-factor placement in tensor memory: the four scales (4 bytes) of row r
// for one K = 64 step form one 32-bit word at column (r / 32) and lane
// (r % 32) of every 32-lane subpartition.
#pragma once

#include "gemm_tcgen05.cuh"

namespace wq {

constexpr int kFp4BK = 256;  // elements per k-block

template <int BN>
struct Fp4Shape {
  static constexpr int STAGES = 4;
  static constexpr int A_BYTES = kGemmBM * kFp4BK / 2;  // 16 KB
  static constexpr int B_BYTES = BN * kFp4BK / 2;       // 32 KB at BN = 256
  static constexpr int SA_BYTES = kGemmBM * 16;         // X scales of the k-block: 16 B per row
  static constexpr int SB_BYTES = BN * 16;              // W scales
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SA_BYTES + SB_BYTES;
  static constexpr int THREADS = 384;
  static constexpr int SFA_COLS = 4 * 4;         // 4 K-steps x 4 row blocks of 32
  static constexpr int SFB_COLS = 4 * (BN / 32);
  static constexpr int SF_STAGE_COLS = SFA_COLS + SFB_COLS;
  static constexpr int TMEM_COLS = 512;
  static_assert(256 + STAGES * SF_STAGE_COLS <= TMEM_COLS, "tensor memory budget");
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 256 + 1024;
  static_assert(STAGE_BYTES % 1024 == 0, "stages keep the 1024-byte alignment of the swizzled tiles");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory of one CTA");
};

struct Fp4Args {
  CUtensorMap tmA;        // X codes u8 [M, K/2], box {128 B, 128}, 128B swizzle
  CUtensorMap tmB;        // W codes u8 [N, K/2], box {128 B, BN}, 128B swizzle
  CUtensorMap tmSA;       // X scales u8 [M, K/16], box {16 B, 128} (used iff sf_tma)
  CUtensorMap tmSB;       // W scales u8 [N, K/16], box {16 B, BN} (used iff sf_tma)
  int sf_tma;             // scale rows 16-byte aligned (K % 256 == 0): scales arrive with the stage
  const uint8_t* sfa;     // X e4m3 [M, K/16]
  const uint8_t* sfb;     // W e4m3 [N, K/16]
  const float* gx;        // fp32 [1]
  const float* gw;        // fp32 [1]
  uint16_t* Y;            // bf16 [M, N]
  CUtensorMap tmY;        // Y bf16 [M, N], box {32, 32}, 64B swizzle (persistent kernel, used iff y_tma)
  int y_tma;              // N % 8 == 0 and Y 16-byte aligned: the epilogue stores Y tiles by TMA
  int M, N, K;            // K % 64 == 0
};

// Instruction descriptor: E2M1 x E2M1 with E4M3 block scales, fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_nvf4(int M, int N) {
  return (1u << 7) | (1u << 10) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);  // scale format 0 = E4M3
}

__device__ __forceinline__ void umma_nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p; }" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

// Four scale bytes (one K = 64 step) of row `row` at k-step `ks`, zero outside.
__device__ __forceinline__ uint32_t sf_word(const uint8_t* __restrict__ sf, int row, int rows, int ks, int ksteps,
                                            int stride) {
  if (row >= rows || ks >= ksteps) return 0u;
  return __ldg(reinterpret_cast<const uint32_t*>(sf + int64_t(row) * stride) + ks);
}

template <int BN>
__global__ void __launch_bounds__(Fp4Shape<BN>::THREADS, 1) gemm_fp4_kernel(const __grid_constant__ Fp4Args a) {
  using S = Fp4Shape<BN>;
  constexpr int STAGES = S::STAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * S::STAGE_BYTES);
  uint64_t* full = bars;
  uint64_t* sfready = bars + STAGES;
  uint64_t* empty = bars + 2 * STAGES;
  uint64_t* accum = bars + 3 * STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * STAGES + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * kGemmBM, n0 = blockIdx.x * BN;
  const int nkb = (a.K + kFp4BK - 1) / kFp4BK;
  const int ksteps = a.K / 64;     // valid K = 64 steps
  const int sf_stride = a.K / 16;  // bytes per row of the scale arrays

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&sfready[s], 8);  // the 8 scale-copy warps
      mbar_init(&empty[s], 1);
    }
    mbar_init(accum, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&a.tmA);
    prefetch_tmap(&a.tmB);
    if (a.sf_tma) {
      prefetch_tmap(&a.tmSA);
      prefetch_tmap(&a.tmSB);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, S::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_acc = tmem;
  auto sfa_col = [&](int s) { return uint32_t(256 + s * S::SF_STAGE_COLS); };
  auto sfb_col = [&](int s) { return uint32_t(256 + s * S::SF_STAGE_COLS + S::SFA_COLS); };

  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == 0) {
    if (lane == 0) {
      asm volatile("griddepcontrol.wait;" ::: "memory");
      int issued = 0;
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % STAGES, r = kb / STAGES;
        if (r > 0 && !mbar_wait(&empty[s], (r - 1) & 1, ERR_TIMEOUT_PIPE, abort_flag)) break;
        uint8_t* st = smem + s * S::STAGE_BYTES;
        mbar_arrive_expect_tx(&full[s], a.sf_tma ? S::STAGE_BYTES : S::A_BYTES + S::B_BYTES);
        tma_load_2d(st, &a.tmA, &full[s], kb * (kFp4BK / 2), m0);
        tma_load_2d(st + S::A_BYTES, &a.tmB, &full[s], kb * (kFp4BK / 2), n0);
        if (a.sf_tma) {  // 16 bytes = the 16 scales of the k-block's 256 elements, per row
          tma_load_2d(st + S::A_BYTES + S::B_BYTES, &a.tmSA, &full[s], kb * 16, m0);
          tma_load_2d(st + S::A_BYTES + S::B_BYTES + S::SA_BYTES, &a.tmSB, &full[s], kb * 16, n0);
        }
        ++issued;
      }
      if (*abort_flag) {
        for (int kb = (issued > STAGES ? issued - STAGES : 0); kb < issued; ++kb)
          mbar_wait(&full[kb % STAGES], (kb / STAGES) & 1, ERR_TIMEOUT_TMA, nullptr);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_nvf4(kGemmBM, BN);
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % STAGES, r = kb / STAGES;
        if (!mbar_wait(&full[s], r & 1, ERR_TIMEOUT_TMA, abort_flag)) break;
        if (!mbar_wait(&sfready[s], r & 1, ERR_TIMEOUT_PIPE, abort_flag)) break;
        tc_fence_after();
        const uint64_t ad = desc_kmajor_sw128(sbase + uint32_t(s * S::STAGE_BYTES));
        const uint64_t bd = desc_kmajor_sw128(sbase + uint32_t(s * S::STAGE_BYTES + S::A_BYTES));
#pragma unroll
        for (int t = 0; t < 4; ++t)  // K = 64 per MMA: +32 bytes inside the swizzle atom
          umma_nvf4(tmem_acc, ad + uint64_t(2 * t), bd + uint64_t(2 * t), IDESC, tmem + sfa_col(s) + 4 * t,
                    tmem + sfb_col(s) + (BN / 32) * t, (kb | t) != 0);
        umma_commit(&empty[s]);
      }
      umma_commit(accum);
    }
  } else if (warp >= 4) {
    asm volatile("griddepcontrol.wait;" ::: "memory");  // the scales may come from the previous kernel
    const int quarter = warp & 3;
    const bool is_b = warp >= 8;
    const uint32_t lane_base = uint32_t(quarter * 32) << 16;
    bool ok = true;
    // Scale words of k-block kb for this lane (16 of them), fetched one
    // k-block ahead so their latency overlaps the previous stage.
    auto fetch_sf = [&](int kb, uint32_t (&v)[16], int part) {
      if (!is_b) {
        if (part > 0) return;  // the X scales of a stage fit one 16-column store
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
          for (int c = 0; c < 4; ++c)
            v[4 * t + c] = kb < nkb ? sf_word(a.sfa, m0 + lane + 32 * c, a.M, 4 * kb + t, ksteps, sf_stride) : 0u;
      } else {
#pragma unroll
        for (int t2 = 0; t2 < 16; ++t2) {
          const int col = 16 * part + t2;  // column within the stage's SFB block
          const int t = col / (BN / 32), c = col % (BN / 32);
          v[t2] = kb < nkb ? sf_word(a.sfb, n0 + lane + 32 * c, a.N, 4 * kb + t, ksteps, sf_stride) : 0u;
        }
      }
    };
    constexpr int PARTS = S::SFB_COLS / 16;  // SFB stores of 16 columns (X scales use one)
    // Scale words of k-block kb from the stage in shared memory: row r's 16
    // bytes are its 4 words (K = 64 steps t); column (rows/32) t + c of lane l
    // takes row 32 c + l (conflict-free 16-byte reads, consecutive rows per lane).
    auto stage_sf = [&](int s, uint32_t (&v)[16], int part) {
      const uint32_t base = sbase + uint32_t(s * S::STAGE_BYTES + S::A_BYTES + S::B_BYTES);
      if (!is_b) {
        if (part > 0) return;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 w = ld_shared_v4(base + uint32_t((32 * c + lane) * 16));
          v[c] = w.x; v[4 + c] = w.y; v[8 + c] = w.z; v[12 + c] = w.w;
        }
      } else {
        constexpr int G = BN / 32;  // row groups of 32
#pragma unroll
        for (int t2 = 0; t2 < 16; t2 += 4) {
          // columns 16 part + t2 .. +3 share k-step t when G >= 4: t = col / G, c = col % G
          const int col = 16 * part + t2, t = col / G, c0 = col % G;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 w = ld_shared_v4(base + uint32_t(S::SA_BYTES + (32 * (c0 + q) + lane) * 16));
            v[t2 + q] = t == 0 ? w.x : t == 1 ? w.y : t == 2 ? w.z : w.w;
          }
        }
      }
    };
    uint32_t nxt[PARTS][16];
    if (!a.sf_tma) {
#pragma unroll
      for (int h = 0; h < PARTS; ++h) fetch_sf(0, nxt[h], h);
    }
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % STAGES, r = kb / STAGES;
      uint32_t cur[PARTS][16];
      if (a.sf_tma) {
        if (!mbar_wait(&full[s], r & 1, ERR_TIMEOUT_TMA, abort_flag)) { ok = false; break; }
#pragma unroll
        for (int h = 0; h < PARTS; ++h) stage_sf(s, cur[h], h);
      } else {
#pragma unroll
        for (int h = 0; h < PARTS; ++h)
#pragma unroll
          for (int i = 0; i < 16; ++i) cur[h][i] = nxt[h][i];
#pragma unroll
        for (int h = 0; h < PARTS; ++h) fetch_sf(kb + 1, nxt[h], h);
      }
      if (r > 0 && !mbar_wait(&empty[s], (r - 1) & 1, ERR_TIMEOUT_PIPE, abort_flag)) { ok = false; break; }
      if (!is_b) {
        tmem_st16(tmem + lane_base + sfa_col(s), cur[0]);
      } else {
#pragma unroll
        for (int h = 0; h < PARTS; ++h) tmem_st16(tmem + lane_base + sfb_col(s) + 16 * h, cur[h]);
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sfready[s]);
    }
    // ---------------------------------------------------------- epilogue
    bool go = ok && mbar_wait(accum, 0, ERR_TIMEOUT_MMA, abort_flag);
    go = __all_sync(0xffffffffu, go);
    if (go) {
      tc_fence_after();
      const int col0 = is_b ? 128 : 0;
      const int row = m0 + quarter * 32 + lane;
      const float gmul = __ldg(a.gx) * __ldg(a.gw);
      const bool vec = (a.N % 8) == 0;
      for (int c = col0; c < min(col0 + 128, BN); c += 32) {
        uint32_t v[32];
        tmem_ld32(tmem_acc + lane_base + uint32_t(c), v);
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
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, S::TMEM_COLS);
  }
}

}  // namespace wq

namespace wq {

// ---------------------------------------------------------------------------
// Persistent variant (scale tiles by TMA, i.e. K % 256 == 0): one CTA per SM
// walks the output tiles t = blockIdx.x, + gridDim.x, ... (N fastest, so
// consecutive tiles of a CTA reuse the X rows in L2).  The TMA / scale /
// MMA pipeline runs on across tiles, and two 128-column accumulators in
// tensor memory alternate, so the epilogue warps drain tile i while the
// MMAs of tile i + 1 proceed:
//   warp 0      TMA producer (codes and scale tiles, STAGES deep)
//   warp 1      TMEM allocation and the MMA issuer
//   warps 4..7  copy each stage's X and W scales into tensor memory (one lane
//               quarter each; every quarter holds the full 128-row block)
//   warps 8..11 epilogue of one lane quarter each (tcgen05.ld, x g_x g_w, bf16)
// Tensor memory: accumulators at columns [0, 256), then STAGES x 32 scale columns.
constexpr int kFp4PBN = 128;

struct Fp4PShape {
  static constexpr int STAGES = 4;
  static constexpr int A_BYTES = kGemmBM * kFp4BK / 2;      // 16 KB
  static constexpr int B_BYTES = kFp4PBN * kFp4BK / 2;      // 16 KB
  static constexpr int SA_BYTES = kGemmBM * 16;
  static constexpr int SB_BYTES = kFp4PBN * 16;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SA_BYTES + SB_BYTES;  // 36 KB
  static constexpr int THREADS = 384;
  static constexpr int SFA_COLS = 16;                       // 4 K-steps x 4 row blocks of 32
  static constexpr int SFB_COLS = 16;                       // 4 K-steps x 4 row blocks of 32
  static constexpr int SF_STAGE_COLS = SFA_COLS + SFB_COLS;
  static constexpr int ACC_COLS = 2 * kFp4PBN;
  static constexpr int TMEM_COLS = 512;
  static_assert(ACC_COLS + STAGES * SF_STAGE_COLS <= TMEM_COLS, "tensor memory budget");
  static constexpr int YBOX_BYTES = 32 * 32 * 2;      // one epilogue warp's 32 x 32 bf16 box of Y
  static constexpr int Y_BYTES = 4 * 2 * YBOX_BYTES;  // two boxes per epilogue warp (store / fill)
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + Y_BYTES + 256 + 1024;
  static_assert(STAGE_BYTES % 1024 == 0, "stages keep the 1024-byte alignment of the swizzled tiles");
};

__global__ void __launch_bounds__(Fp4PShape::THREADS, 1) gemm_fp4_persistent_kernel(const __grid_constant__ Fp4Args a) {
  using S = Fp4PShape;
  constexpr int STAGES = S::STAGES;
  constexpr int BN = kFp4PBN;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
  const uint32_t sbase = smem_u32(smem);
  uint8_t* ybox = smem + STAGES * S::STAGE_BYTES;  // epilogue Y boxes (1024-byte aligned)
  uint64_t* bars = reinterpret_cast<uint64_t*>(ybox + S::Y_BYTES);
  uint64_t* full = bars;                    // TMA landed (codes + scales)
  uint64_t* sfready = bars + STAGES;        // scales in tensor memory
  uint64_t* empty = bars + 2 * STAGES;      // MMAs of the stage finished
  uint64_t* acc_full = bars + 3 * STAGES;   // [2] accumulator complete
  uint64_t* acc_empty = acc_full + 2;       // [2] accumulator drained by the epilogue
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkb = (a.K + kFp4BK - 1) / kFp4BK;
  const int n_tiles = (a.N + BN - 1) / BN, m_tiles = (a.M + kGemmBM - 1) / kGemmBM;
  const int tiles = n_tiles * m_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&sfready[s], 4);  // the 4 scale-copy warps
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);  // the 4 epilogue warps
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&a.tmA);
    prefetch_tmap(&a.tmB);
    prefetch_tmap(&a.tmSA);
    prefetch_tmap(&a.tmSB);
    if (a.y_tma) prefetch_tmap(&a.tmY);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, S::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto sfa_col = [&](int s) { return uint32_t(S::ACC_COLS + s * S::SF_STAGE_COLS); };
  auto sfb_col = [&](int s) { return uint32_t(S::ACC_COLS + s * S::SF_STAGE_COLS + S::SFA_COLS); };

  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      asm volatile("griddepcontrol.wait;" ::: "memory");
      int q = 0;  // global k-block sequence number of this CTA
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        const int m0 = (t / n_tiles) * kGemmBM, n0 = (t % n_tiles) * BN;
        for (int kb = 0; kb < nkb; ++kb, ++q) {
          const int s = q % STAGES, r = q / STAGES;
          if (r > 0 && !mbar_wait(&empty[s], (r - 1) & 1, ERR_TIMEOUT_PIPE, abort_flag)) { ok = false; break; }
          uint8_t* st = smem + s * S::STAGE_BYTES;
          mbar_arrive_expect_tx(&full[s], S::STAGE_BYTES);
          tma_load_2d(st, &a.tmA, &full[s], kb * (kFp4BK / 2), m0);
          tma_load_2d(st + S::A_BYTES, &a.tmB, &full[s], kb * (kFp4BK / 2), n0);
          tma_load_2d(st + S::A_BYTES + S::B_BYTES, &a.tmSA, &full[s], kb * 16, m0);
          tma_load_2d(st + S::A_BYTES + S::B_BYTES + S::SA_BYTES, &a.tmSB, &full[s], kb * 16, n0);
        }
      }
      if (!ok) {  // let copies already issued land before the CTA leaves
        for (int k = (q > STAGES ? q - STAGES : 0); k < q; ++k)
          mbar_wait(&full[k % STAGES], (k / STAGES) & 1, ERR_TIMEOUT_TMA, nullptr);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_nvf4(kGemmBM, BN);
      // stage 0's operand descriptors and scale columns; stage s adds s stages (the
      // descriptor's start address is addr / 16 in its low 14 bits: no carry below 256 KB)
      const uint64_t ad0 = desc_kmajor_sw128(sbase), bd0 = desc_kmajor_sw128(sbase + uint32_t(S::A_BYTES));
      const uint32_t sfa0 = tmem + sfa_col(0), sfb0 = tmem + sfb_col(0);
      int q = 0, i = 0, s = 0;
      uint32_t par = 0;  // phase parity of stage s's barriers
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++i) {
        const int b = i & 1, u = i >> 1;
        if (u > 0 && !mbar_wait(&acc_empty[b], (u - 1) & 1, ERR_TIMEOUT_PIPE, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dacc = tmem + uint32_t(b * BN);
        for (int kb = 0; kb < nkb; ++kb, ++q) {
          if (!mbar_wait(&full[s], par, ERR_TIMEOUT_TMA, abort_flag) ||
              !mbar_wait(&sfready[s], par, ERR_TIMEOUT_PIPE, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = ad0 + uint64_t(s * (S::STAGE_BYTES >> 4));
          const uint64_t bd = bd0 + uint64_t(s * (S::STAGE_BYTES >> 4));
          const uint32_t sfa = sfa0 + uint32_t(s * S::SF_STAGE_COLS), sfb = sfb0 + uint32_t(s * S::SF_STAGE_COLS);
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4)
            umma_nvf4(dacc, ad + uint64_t(2 * k4), bd + uint64_t(2 * k4), IDESC, sfa + 4 * k4, sfb + 4 * k4,
                      (kb | k4) != 0);
          umma_commit(&empty[s]);
          if (++s == STAGES) {
            s = 0;
            par ^= 1u;
          }
        }
        umma_commit(&acc_full[b]);  // also after an abort: completes when the issued MMAs are done
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ---------------------------------------------------------- scales -> tensor memory
    const int quarter = warp & 3;
    const uint32_t lane_base = uint32_t(quarter * 32) << 16;
    int q = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
      for (int kb = 0; kb < nkb; ++kb, ++q) {
        const int s = q % STAGES, r = q / STAGES;
        if (!mbar_wait(&full[s], r & 1, ERR_TIMEOUT_TMA, abort_flag)) { ok = false; break; }
        // row r of a scale tile: its 4 words (K = 64 steps k4); column 4 k4 + c of
        // lane l takes row 32 c + l
        const uint32_t base = sbase + uint32_t(s * S::STAGE_BYTES + S::A_BYTES + S::B_BYTES);
        uint32_t va[16], vb[16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 wa = ld_shared_v4(base + uint32_t((32 * c + lane) * 16));
          const uint4 wb = ld_shared_v4(base + uint32_t(S::SA_BYTES + (32 * c + lane) * 16));
          va[c] = wa.x; va[4 + c] = wa.y; va[8 + c] = wa.z; va[12 + c] = wa.w;
          vb[c] = wb.x; vb[4 + c] = wb.y; vb[8 + c] = wb.z; vb[12 + c] = wb.w;
        }
        if (r > 0 && !mbar_wait(&empty[s], (r - 1) & 1, ERR_TIMEOUT_PIPE, abort_flag)) { ok = false; break; }
        tmem_st16(tmem + lane_base + sfa_col(s), va);
        tmem_st16(tmem + lane_base + sfb_col(s), vb);
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sfready[s]);
      }
    }
  } else if (warp >= 8) {
    // ---------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const uint32_t lane_base = uint32_t(quarter * 32) << 16;
    const float gmul = __ldg(a.gx) * __ldg(a.gw);
    const bool vec = (a.N % 8) == 0;
    int i = 0, nbox = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
      const int b = i & 1, u = i >> 1;
      bool go = mbar_wait(&acc_full[b], u & 1, ERR_TIMEOUT_MMA, abort_flag);
      go = __all_sync(0xffffffffu, go);  // tcgen05.ld is warp-collective
      if (!go) break;
      tc_fence_after();
      const int m0 = (t / n_tiles) * kGemmBM, n0 = (t % n_tiles) * BN;
      const int row = m0 + quarter * 32 + lane;
      for (int c = 0; c < BN; c += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + uint32_t(b * BN + c), v);
        if (a.y_tma) {
          // the warp's 32 x 32 box (row = lane) through shared memory and one TMA
          // store: full 128-byte lines to L2 instead of 16-byte pieces of 32 rows.
          // Box buffers alternate; the one used two boxes ago must have been read.
          uint8_t* box = ybox + (quarter * 2 + (nbox & 1)) * S::YBOX_BYTES;
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
            tma_store_2d(&a.tmY, box, n0 + c, m0 + quarter * 32);
            bulk_commit();
          }
          ++nbox;
          continue;
        }
        if (row < a.M) {
          uint16_t* yrow = a.Y + int64_t(row) * a.N;
          const int nb = n0 + c;
          if (vec && nb + 32 <= a.N) {
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
              uint4 o;
              o.x = pack_bf16x2(__uint_as_float(v[8 * qq + 0]) * gmul, __uint_as_float(v[8 * qq + 1]) * gmul);
              o.y = pack_bf16x2(__uint_as_float(v[8 * qq + 2]) * gmul, __uint_as_float(v[8 * qq + 3]) * gmul);
              o.z = pack_bf16x2(__uint_as_float(v[8 * qq + 4]) * gmul, __uint_as_float(v[8 * qq + 5]) * gmul);
              o.w = pack_bf16x2(__uint_as_float(v[8 * qq + 6]) * gmul, __uint_as_float(v[8 * qq + 7]) * gmul);
              *reinterpret_cast<uint4*>(yrow + nb + 8 * qq) = o;
            }
          } else {
            for (int qq = 0; qq < 32; ++qq)
              if (nb + qq < a.N) yrow[nb + qq] = uint16_t(f32_to_bf16_bits(__uint_as_float(v[qq]) * gmul));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
    }
    if (lane == 0) bulk_wait_all();  // the Y stores are complete before the CTA leaves
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, S::TMEM_COLS);
  }
}

}  // namespace wq
