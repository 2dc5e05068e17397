// gemv_tc.cuh -- decode GEMV (M = 1 or 2 activation rows) on the tensor
// cores, for one quantized Linear or a list of independent ones (INT4 g64,
// INT4 g128 and NVFP4 mixed) in a single launch.
//
// Decode reads every packed weight once per token ("quantization primer"
// section 13: memory-bound decode is where 4-bit weights pay off).  On B200 an
// SM must retire ~46 weights per clock to keep HBM busy, so the kernel is
// built around few instructions per weight and long per-row bursts:
//
// Step: 16 weight rows ("row block") x 128 k.  Lane (g, c) (g = lane / 4,
// c = lane % 4) loads 16 bytes (32 codes) of rows g and g + 8 at
// k = 128 j + 32 c, so every row is read in 64-byte runs and a warp keeps
// kTcDepth steps (3 KB) in flight in registers.
//
// Partition: CTA b owns the row blocks [bounds[b], bounds[b+1]) of the
// launch (items in order, balanced by time on the host); its 16 warps split
// the CTA's steps evenly (stream-K inside the CTA).  A row block inside one
// warp's range is written directly; one split over warps leaves an fp32
// partial per warp in shared memory, and the warp that arrives last (shared
// atomicInc, which wraps back to 0) sums the partials in warp order and writes
// Y.  No warp ever waits.
//
// Math: codes -> f16 mma.sync m16n8k16 A fragments.  A lane's 4 words of a
// row feed 8 mma; the k order inside an mma is free, and the B columns that
// M = 1..2 leaves empty separate partial sums that need different scales:
//   INT4  0x6400 | nibble = 1024 + q (even k) / 1024 + 16 q (odd k; the staged
//         activation is divided by 16): the mma yields sum q x + 1024 P; with
//         per-group activation sums P (staged values) and Q (= sum x),
//         sum (q - z) x = d - 1024 P - z Q, times the fp16 group scale.
//         G = 64: lanes c < 2 hold group 2 j, lanes c >= 2 group 2 j + 1; B
//         column 2 m + (c >= 2) keeps the two groups apart.
//   NVFP4 e2m1x2 -> f16x2 in hardware.  M = 1: lane c's two 16-k blocks go to
//         B columns 2 c and 2 c + 1 (8 columns = the 8 blocks of a step), so
//         the E4M3 block scales multiply fp32 sums after the mma.  M = 2: the
//         block scale multiplies the f16 codes (exact: at most 6 significant
//         bits, at most 6 x 448).  The fp32 tensor scale multiplies Y.
// Activations are staged once per CTA in shared memory as f16 in fragment
// order (bf16 -> f16 is exact in the normal range; x / s is rounded once),
// INT4 with the group sums (of the f16 values the mma sees, so that the 1024 P
// bias cancels exactly); the first weight loads are in flight meanwhile.
// Lanes whose B column must stay empty (INT4 g64, NVFP4 at M = 1) read a
// zeroed row with stride 0 instead of the activations, so the math has no
// selects.  The host precomputes each CTA's first item, kind, step count and
// activation vectors, so a CTA reaches the dependency wait after a few
// parameter reads.  Code loads carry a 256-byte L2 prefetch hint.
// Weights are prefetched into L2 before the programmatic-launch dependency
// wait (L2 is the point of coherence, so this never yields stale data); every
// load that feeds the math is issued after the wait.
#pragma once

#include <cuda_fp16.h>

#include "gemv.cuh"
#include "wq_common.cuh"

namespace wq {

enum TcKind { TC_INT4_G64 = 0, TC_INT4_G128 = 1, TC_NVFP4_COLS = 2, TC_NVFP4_MUL = 3 };

constexpr int kTcMaxItems = 24;
constexpr int kTcMaxX = 8;        // distinct staged activation vectors
constexpr int kTcRows = 16;       // rows per row block
constexpr int kTcStepK = 128;     // k per step
constexpr int kTcWarps = 16;
constexpr int kTcThreads = kTcWarps * 32;
constexpr int kTcDepth = 3;       // steps in flight per warp (3 KB; 48 KB per SM)
constexpr int kTcPrefetchFirst = 4;  // steps per warp brought into L2 before the dependency wait
constexpr int kTcMaxCtas = 148;
constexpr int kTcMaxSmem = 200 * 1024;

struct TcItem {
  const uint8_t* packed;    // codes, [N, K/2] bytes (INT4 words are little-endian nibbles)
  const uint16_t* scales;   // INT4 fp16 [N, K/G]
  const uint32_t* zeros;    // INT4 [N, ceil(K/G/8)] or null (symmetric: codes carry +8)
  const uint8_t* bscale;    // NVFP4 E4M3 [N, K/16]
  const float* gscale;      // NVFP4 fp32 [1]
  uint16_t* Y;              // bf16 [M, N]
  int N, K;
  int xslot;                // staged activation vector
  int kind;                 // TcKind of the weights
  int nrb, steps;           // row blocks, steps per row block (K / 128)
  int rb0;                  // first row block in the launch's row-block sequence
};

struct TcX {
  const uint16_t* X;        // bf16 [M, K]
  const float* inv_s;       // fp32 [K] or null
  int K;
  int g;                    // INT4 group size (INT4 order + group sums), 0 for NVFP4
};

struct TcArgs {
  TcItem items[kTcMaxItems];
  TcX xs[kTcMaxX];
  int bounds[kTcMaxCtas + 1];  // row-block range of each CTA
  uint32_t cta[kTcMaxCtas];    // per CTA: first item | last item << 5 | kind << 10 | steps << 12
  uint8_t xused[kTcMaxCtas];   // per CTA: mask of the activation vectors its items read
  int n_items, n_x;
};
static_assert(sizeof(TcArgs) <= 4096, "kernel parameters must fit the 4 KB limit");

// bytes of one staged activation vector (M rows) and its INT4 group sums
__host__ __device__ inline int tc_x_bytes(int K, int g, int M) { return M * K * 2 + (g ? (K / g) * M * 8 : 0); }

__device__ __forceinline__ uint32_t tc_hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t tc_e2m1x2(uint32_t byte) {
  uint32_t h;
  asm("{ .reg .b8 q; cvt.u8.u32 q, %1; cvt.rn.f16x2.e2m1x2 %0, q; }" : "=r"(h) : "r"(byte));
  return h;
}
// two E4M3 bytes (sign clear) -> f16x2 {lo byte, hi byte}
__device__ __forceinline__ uint32_t tc_e4m3x2(uint32_t two) {
  uint32_t h;
  asm("{ .reg .b16 q; cvt.u16.u32 q, %1; cvt.rn.f16x2.e4m3x2 %0, q; }" : "=r"(h) : "r"(two & 0x7F7Fu));
  return h;
}
__device__ __forceinline__ void tc_mma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                       uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint4 tc_ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ void tc_prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

// What one lane loads per step: 16 code bytes of rows g and g + 8 and their
// scale data (INT4 G64: fp16 scale pair of groups 2j, 2j+1 + zero word;
// G128: fp16 scale + zero word; NVFP4: the two E4M3 bytes of the lane's blocks).
struct TcEntry {
  uint4 lo, hi;
  uint32_t slo, shi, zlo, zhi;
};

// Position of a walk: item, row block, step inside the row block.
struct TcPos {
  int i, rb, j;
};

// Per-row-block load pointers of one lane.
struct TcLoadPtrs {
  const uint8_t* clo;
  const uint8_t* chi;
  const uint8_t* mlo;  // scales (INT4) or block scales (NVFP4) of row g
  const uint8_t* mhi;
  const uint32_t* zlo;
  const uint32_t* zhi;
};

template <int KIND>
__device__ __forceinline__ void tc_load_ptrs(const TcItem& I, int rb, int g, int c, TcLoadPtrs& p) {
  const int nlo = min(rb * kTcRows + g, I.N - 1), nhi = min(rb * kTcRows + g + 8, I.N - 1);
  const int64_t rbytes = I.K >> 1;
  p.clo = I.packed + nlo * rbytes + 16 * c;
  p.chi = I.packed + nhi * rbytes + 16 * c;
  if (KIND == TC_INT4_G64 || KIND == TC_INT4_G128) {
    const int ng = I.K / (KIND == TC_INT4_G64 ? 64 : 128), zw = (ng + 7) >> 3;
    p.mlo = reinterpret_cast<const uint8_t*>(I.scales + int64_t(nlo) * ng);
    p.mhi = reinterpret_cast<const uint8_t*>(I.scales + int64_t(nhi) * ng);
    p.zlo = I.zeros ? I.zeros + int64_t(nlo) * zw : nullptr;
    p.zhi = I.zeros ? I.zeros + int64_t(nhi) * zw : nullptr;
  } else {
    const int nb = I.K >> 4;
    p.mlo = I.bscale + int64_t(nlo) * nb + 2 * c;
    p.mhi = I.bscale + int64_t(nhi) * nb + 2 * c;
    p.zlo = p.zhi = nullptr;
  }
}

template <int KIND>
__device__ __forceinline__ void tc_load_step(const TcLoadPtrs& p, int j, TcEntry& e) {
  e.lo = tc_ld_stream(p.clo + 64 * j);
  e.hi = tc_ld_stream(p.chi + 64 * j);
  if (KIND == TC_INT4_G64) {
    e.slo = __ldg(reinterpret_cast<const uint32_t*>(p.mlo) + j);  // groups 2j, 2j+1
    e.shi = __ldg(reinterpret_cast<const uint32_t*>(p.mhi) + j);
    e.zlo = p.zlo ? __ldg(p.zlo + (j >> 2)) : 0x88888888u;
    e.zhi = p.zhi ? __ldg(p.zhi + (j >> 2)) : 0x88888888u;
  } else if (KIND == TC_INT4_G128) {
    e.slo = __ldg(reinterpret_cast<const uint16_t*>(p.mlo) + j);
    e.shi = __ldg(reinterpret_cast<const uint16_t*>(p.mhi) + j);
    e.zlo = p.zlo ? __ldg(p.zlo + (j >> 3)) : 0x88888888u;
    e.zhi = p.zhi ? __ldg(p.zhi + (j >> 3)) : 0x88888888u;
  } else {
    e.slo = __ldg(reinterpret_cast<const uint16_t*>(p.mlo + 8 * j));  // blocks 8j + 2c, 8j + 2c + 1
    e.shi = __ldg(reinterpret_cast<const uint16_t*>(p.mhi + 8 * j));
  }
}

// (w & 0x000F000F) | 0x64006400 and (w & 0x00F000F0) | 0x64006400 with the
// constants as immediates (no register traffic for them)
__device__ __forceinline__ uint32_t tc_nib_lo(uint32_t w) {
  uint32_t d;
  asm("lop3.b32 %0, %1, 0x000F000F, 0x64006400, 0xEA;" : "=r"(d) : "r"(w));
  return d;
}
__device__ __forceinline__ uint32_t tc_nib_hi(uint32_t w) {
  uint32_t d;
  asm("lop3.b32 %0, %1, 0x00F000F0, 0x64006400, 0xEA;" : "=r"(d) : "r"(w));
  return d;
}

template <int KIND>
__device__ __forceinline__ void tc_unpack(uint32_t w, uint32_t& a0, uint32_t& a2, uint32_t& a0n, uint32_t& a2n) {
  if (KIND == TC_INT4_G64 || KIND == TC_INT4_G128) {
    const uint32_t w8 = w >> 8;
    a0 = tc_nib_lo(w);
    a2 = tc_nib_hi(w);
    a0n = tc_nib_lo(w8);
    a2n = tc_nib_hi(w8);
  } else {
    a0 = tc_e2m1x2(w);
    a2 = tc_e2m1x2(w >> 8);
    a0n = tc_e2m1x2(w >> 16);
    a2n = tc_e2m1x2(w >> 24);
  }
}

// Sum of the whole row block's (row, m) values for the partial / final write:
// lanes with c == 0 end up holding v[0..M-1] of row g and v[M..2M-1] of row g + 8.
template <int M, int KIND>
__device__ __forceinline__ void tc_gather(const float (&acc)[4], int lane, float (&v)[2 * M]) {
  if (KIND == TC_INT4_G64) {  // lane c holds m = c
#pragma unroll
    for (int m = 0; m < M; ++m) {
      v[m] = __shfl_sync(0xFFFFFFFFu, acc[0], (lane & ~3) + m);
      v[M + m] = __shfl_sync(0xFFFFFFFFu, acc[2], (lane & ~3) + m);
    }
  } else if (KIND == TC_NVFP4_COLS) {  // every lane holds its two blocks
    float lo = acc[0], hi = acc[2];
    lo += __shfl_xor_sync(0xFFFFFFFFu, lo, 1);
    hi += __shfl_xor_sync(0xFFFFFFFFu, hi, 1);
    lo += __shfl_xor_sync(0xFFFFFFFFu, lo, 2);
    hi += __shfl_xor_sync(0xFFFFFFFFu, hi, 2);
    v[0] = lo;
    v[M] = hi;
  } else {  // lane c = 0 holds m = 0, 1 in acc[0..1] (row g) and acc[2..3] (row g + 8)
#pragma unroll
    for (int m = 0; m < M; ++m) {
      v[m] = acc[m];
      v[M + m] = acc[2 + m];
    }
  }
}

// Row block done with a split over warps w0..w1 of this CTA (steps [sa, sb)
// of the CTA's sequence; its first Wc = min(8, S) warps share the S steps,
// warp w owning [lo(w), lo(w + 1)), none empty): store this warp's
// partial in shared memory, count the arrival on the first piece's counter,
// and if it is the last one sum the partials in warp order and write Y.
template <int M>
__device__ __noinline__ void tc_flush_split(const float* v, int lane, int warp, int S, int Wc, int sa, int sb,
                                            const TcItem* I, int rb, float gmul, float* spart, unsigned* sctr) {
  const int g = lane >> 2, c = lane & 3;
  const auto lo_of = [&](int w) { return (w * S) / Wc; };
  int w0 = 0, w1 = 0;
  for (int w = 1; w < Wc; ++w) {
    if (lo_of(w) <= sa) w0 = w;
    if (lo_of(w) <= sb - 1) w1 = w;
  }
  const int slot = sa < lo_of(warp) ? 0 : 1;
  float* mine = spart + (warp * 2 + slot) * kTcRows * M;
  if (c == 0) {
#pragma unroll
    for (int m = 0; m < M; ++m) {
      mine[g * M + m] = v[m];
      mine[(g + 8) * M + m] = v[M + m];
    }
  }
  __threadfence_block();
  __syncwarp();
  unsigned old = 0;
  if (lane == 0) old = atomicInc(sctr + w0, unsigned(w1 - w0));
  old = __shfl_sync(0xFFFFFFFFu, old, 0);
  if (old != unsigned(w1 - w0)) return;  // not the last arrival
  __threadfence_block();
  if (lane < kTcRows * M) {
    const int r = lane / M, m = lane % M;
    float s = 0.f;
    for (int w = w0; w <= w1; ++w) {
      const int sl = sa < lo_of(w) ? 0 : 1;
      s += *reinterpret_cast<volatile const float*>(spart + (w * 2 + sl) * kTcRows * M + r * M + m);
    }
    const int n = rb * kTcRows + r;
    if (n < I->N) I->Y[int64_t(m) * I->N + n] = uint16_t(f32_to_bf16_bits(s * gmul));
  }
}

// L2 prefetch of steps [j, j + 4) of the 16 rows of row block rb: lane l takes
// row l % 16 and the 128-byte line of steps j + 2 (l / 16), + 1 (as far as
// the row block has steps).
__device__ __forceinline__ void tc_prefetch_rows(const TcItem& I, int rb, int j, int lane) {
  j += 2 * (lane >> 4);
  if (rb < I.nrb && j < I.steps) {
    const int n = min(rb * kTcRows + (lane & 15), I.N - 1);
    tc_prefetch_l2(I.packed + int64_t(n) * (I.K >> 1) + 64 * j);
  }
}

// Position (item, row block, step) of step t of the CTA's sequence over the
// global row blocks [R0, R1).
__device__ __forceinline__ TcPos tc_pos(const TcArgs& a, int i0, int R0, int R1, int t) {
  TcPos p{i0, 0, 0};
  for (;; ++p.i) {
    const TcItem& I = a.items[p.i];
    const int r0 = max(R0, I.rb0), r1 = min(R1, I.rb0 + I.nrb);
    const int span = (r1 - r0) * I.steps;
    if (t < span || p.i + 1 == a.n_items) {
      const int q = t / I.steps;
      p.rb = r0 - I.rb0 + q;
      p.j = t - q * I.steps;
      return p;
    }
    t -= span;
  }
}

// The work of one CTA whose row blocks all hold weights of kind KIND.
template <int M, int KIND>
__device__ __forceinline__ void gemv_tc_cta(const TcArgs& a, uint8_t* tc_smem, float* spart, unsigned* sctr,
                                            int* xoff, const uint16_t* zrow) {
  static_assert(M == 1 || M == 2, "M is 1 or 2");
  static_assert(KIND != TC_NVFP4_COLS || M == 1, "NVFP4 block columns need all 8 B columns");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int R0 = a.bounds[blockIdx.x], R1 = a.bounds[blockIdx.x + 1];
  const uint32_t info = a.cta[blockIdx.x];
  const int i0 = int(info & 31u), S = int(info >> 12);  // first item, steps of this CTA
  const int Wc = min(kTcWarps, S);  // warps that share the steps (none empty)
  const int lo = warp < Wc ? (warp * S) / Wc : S, hi = warp < Wc ? ((warp + 1) * S) / Wc : S;
  if (threadIdx.x < kTcWarps) sctr[threadIdx.x] = 0;
  if (threadIdx.x < 4) reinterpret_cast<uint4*>(const_cast<uint16_t*>(zrow))[threadIdx.x] = make_uint4(0, 0, 0, 0);

  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // this warp's walk: loads run kTcDepth steps ahead of the math
  TcPos L = tc_pos(a, i0, R0, R1, lo);
  TcPos C = L;
  TcLoadPtrs lp;
  tc_load_ptrs<KIND>(a.items[L.i], L.rb, g, c, lp);
  // warm L2 with the first steps while the previous grid drains (L2 is the
  // point of coherence: this never yields stale data; the loads come after the wait)
  if (lo < hi) {
    const TcItem& I = a.items[L.i];
    int rb = L.rb, j = L.j;
    for (int t = 0; t < min(kTcPrefetchFirst, hi - lo); t += 4) {  // may run into the next row block
      tc_prefetch_rows(I, rb, j, lane);
      if ((j += 4) >= I.steps) {
        j = 0;
        ++rb;
      }
    }
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");

  int lsteps = a.items[L.i].steps;
  const auto load_advance = [&]() {
    if (++L.j == lsteps) {
      L.j = 0;
      if (++L.rb == a.items[L.i].nrb) {
        L.rb = 0;
        ++L.i;
      }
      if (L.i < a.n_items) {
        tc_load_ptrs<KIND>(a.items[L.i], L.rb, g, c, lp);
        lsteps = a.items[L.i].steps;
      }
    }
  };
  TcEntry R[kTcDepth];
#pragma unroll
  for (int u = 0; u < kTcDepth; ++u)
    if (lo + u < hi) {
      tc_load_step<KIND>(lp, L.j, R[u]);
      load_advance();
    }

  // ---- stage this CTA's activation vectors (f16, fragment order, INT4 group sums)
  if (threadIdx.x == 0) {
    const uint32_t used = a.xused[blockIdx.x];
    int off = 0;
    for (int v = 0; v < kTcMaxX; ++v) {
      xoff[v] = -1;
      if (v < a.n_x && ((used >> v) & 1)) {
        xoff[v] = off;
        off += tc_x_bytes(a.xs[v].K, a.xs[v].g, M);
      }
    }
  }
  __syncthreads();
  for (int v = 0; v < a.n_x; ++v) {
    if (xoff[v] < 0) continue;
    const TcX& X = a.xs[v];
    const int n8 = X.K >> 3;  // 8-value chunks per row
    const int cpg = X.g >> 3;  // chunks per group
    uint16_t* xs = reinterpret_cast<uint16_t*>(tc_smem + xoff[v]);
    float2* sums = reinterpret_cast<float2*>(tc_smem + xoff[v] + M * X.K * 2);  // [K/G][M] {P, Q}
    for (int m = 0; m < M; ++m) {
      const uint16_t* src = X.X + int64_t(m) * X.K;
      for (int base = 0; base < n8; base += 2 * kTcThreads) {  // same trip count in every lane (shuffles)
        uint4 raw[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int p = base + threadIdx.x + u * kTcThreads;
          raw[u] = p < n8 ? __ldg(reinterpret_cast<const uint4*>(src) + p) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int p = base + threadIdx.x + u * kTcThreads;
          float f[8];
          const uint32_t wv[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            f[2 * q] = __uint_as_float(wv[q] << 16);
            f[2 * q + 1] = __uint_as_float(wv[q] & 0xFFFF0000u);
          }
          if (X.inv_s && p < n8) {
            const float4 i0v = __ldg(reinterpret_cast<const float4*>(X.inv_s) + 2 * p);
            const float4 i1v = __ldg(reinterpret_cast<const float4*>(X.inv_s) + 2 * p + 1);
            f[0] *= i0v.x; f[1] *= i0v.y; f[2] *= i0v.z; f[3] *= i0v.w;
            f[4] *= i1v.x; f[5] *= i1v.y; f[6] *= i1v.z; f[7] *= i1v.w;
          }
          __half2 hv[4];
          if (X.g) {  // INT4 order {x0, x4}, {x1, x5} / 16, {x2, x6}, {x3, x7} / 16
            hv[0] = __floats2half2_rn(f[0], f[4]);
            hv[1] = __floats2half2_rn(f[1] * 0.0625f, f[5] * 0.0625f);
            hv[2] = __floats2half2_rn(f[2], f[6]);
            hv[3] = __floats2half2_rn(f[3] * 0.0625f, f[7] * 0.0625f);
            const float2 e0 = __half22float2(hv[0]), o0 = __half22float2(hv[1]);
            const float2 e1 = __half22float2(hv[2]), o1 = __half22float2(hv[3]);
            const float se = (e0.x + e0.y) + (e1.x + e1.y), so = (o0.x + o0.y) + (o1.x + o1.y);
            float P = se + so, Q = fmaf(16.f, so, se);
            for (int o = 1; o < cpg; o <<= 1) {  // a group's chunks are aligned consecutive lanes
              P += __shfl_xor_sync(0xFFFFFFFFu, P, o);
              Q += __shfl_xor_sync(0xFFFFFFFFu, Q, o);
            }
            if (p < n8 && (p & (cpg - 1)) == 0) sums[(p / cpg) * M + m] = make_float2(P, Q);
          } else {
            hv[0] = __floats2half2_rn(f[0], f[1]);
            hv[1] = __floats2half2_rn(f[2], f[3]);
            hv[2] = __floats2half2_rn(f[4], f[5]);
            hv[3] = __floats2half2_rn(f[6], f[7]);
          }
          if (p < n8) *reinterpret_cast<uint4*>(xs + m * X.K + 8 * p) = *reinterpret_cast<const uint4*>(hv);
        }
      }
    }
  }
  __syncthreads();
  if (lo >= hi) return;

  // per-item compute state: this lane's B sources for words 0-1 / 2-3 and
  // their stride per step (0 on the zeroed row when the lane's column must stay
  // empty), the INT4 group sums
  const uint16_t* xa = nullptr;
  const uint16_t* xb = nullptr;
  int xsa = 0, xsb = 0;
  const float2* sums = nullptr;
  int csteps = 0;
  float gmul = 1.f;
  const auto compute_enter = [&]() {
    const TcItem& I = a.items[C.i];
    const uint8_t* xbase = tc_smem + xoff[I.xslot];
    csteps = I.steps;
    sums = reinterpret_cast<const float2*>(xbase + M * I.K * 2);
    gmul = (KIND == TC_NVFP4_COLS || KIND == TC_NVFP4_MUL) ? __ldg(I.gscale) : 1.f;
    bool va = true, vb = true;
    int m = 0;
    if (KIND == TC_INT4_G64) {  // column 2m + (c >= 2)
      const int d = g - (c >> 1);
      va = vb = d >= 0 && (d & 1) == 0 && (d >> 1) < M;
      m = va ? d >> 1 : 0;
    } else if (KIND == TC_NVFP4_COLS) {  // column = block 2c + (word >= 2)
      va = g == 2 * c;
      vb = g == 2 * c + 1;
    } else {  // column m; the outputs of the other columns are never read
      m = g < M ? g : 0;
    }
    const uint16_t* xl = reinterpret_cast<const uint16_t*>(xbase) + m * I.K + 32 * c;
    xa = va ? xl : zrow;
    xb = vb ? xl : zrow;
    xsa = va ? kTcStepK : 0;
    xsb = vb ? kTcStepK : 0;
  };
  compute_enter();

  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int base = lo; base < hi; base += kTcDepth) {
#pragma unroll
    for (int u = 0; u < kTcDepth; ++u) {
      const int s = base + u;
      if (s >= hi) break;
      // ---------------------------------------------------------- math of step s
      {
        const TcEntry& e = R[u];
        const uint16_t* xsA = xa + C.j * xsa;
        const uint16_t* xsB = xb + C.j * xsb;
        float d[4] = {0.f, 0.f, 0.f, 0.f}, f[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t sbl = 0, sbh = 0;
        if (KIND == TC_NVFP4_MUL) {
          sbl = tc_e4m3x2(e.slo);
          sbh = tc_e4m3x2(e.shi);
        }
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const uint4 b = *reinterpret_cast<const uint4*>((w < 2 ? xsA : xsB) + 8 * w);
          const uint32_t wl = w == 0 ? e.lo.x : w == 1 ? e.lo.y : w == 2 ? e.lo.z : e.lo.w;
          const uint32_t wh = w == 0 ? e.hi.x : w == 1 ? e.hi.y : w == 2 ? e.hi.z : e.hi.w;
          uint32_t l0, l2, l0n, l2n, h0, h2, h0n, h2n;
          tc_unpack<KIND>(wl, l0, l2, l0n, l2n);
          tc_unpack<KIND>(wh, h0, h2, h0n, h2n);
          if (KIND == TC_NVFP4_MUL) {  // block 2c + (w >= 2): scale byte lo / hi of the pair
            const uint32_t sl = __byte_perm(sbl, 0, w < 2 ? 0x1010 : 0x3232);
            const uint32_t sh = __byte_perm(sbh, 0, w < 2 ? 0x1010 : 0x3232);
            l0 = tc_hmul2(l0, sl); l2 = tc_hmul2(l2, sl); l0n = tc_hmul2(l0n, sl); l2n = tc_hmul2(l2n, sl);
            h0 = tc_hmul2(h0, sh); h2 = tc_hmul2(h2, sh); h0n = tc_hmul2(h0n, sh); h2n = tc_hmul2(h2n, sh);
          }
          float(&t)[4] = (w & 1) ? f : d;
          tc_mma(t, l0, h0, l2, h2, b.x, b.y);
          tc_mma(t, l0n, h0n, l2n, h2n, b.z, b.w);
        }
        if (KIND == TC_INT4_G64) {
          // lane c: m = c; d[0]/d[2] group 2j (rows g / g+8), d[1]/d[3] group 2j + 1
          const int m = c < M ? c : M - 1;
          const float2 pa = sums[(2 * C.j) * M + m], pb = sums[(2 * C.j + 1) * M + m];
          const int sft = (C.j & 3) << 3;
          const float zla = float((e.zlo >> sft) & 0xFu), zlb = float((e.zlo >> (sft + 4)) & 0xFu);
          const float zha = float((e.zhi >> sft) & 0xFu), zhb = float((e.zhi >> (sft + 4)) & 0xFu);
          const float2 sl = __half22float2(*reinterpret_cast<const __half2*>(&e.slo));
          const float2 sh = __half22float2(*reinterpret_cast<const __half2*>(&e.shi));
          acc[0] = fmaf(sl.x, fmaf(-zla, pa.y, fmaf(-1024.f, pa.x, d[0] + f[0])), acc[0]);
          acc[0] = fmaf(sl.y, fmaf(-zlb, pb.y, fmaf(-1024.f, pb.x, d[1] + f[1])), acc[0]);
          acc[2] = fmaf(sh.x, fmaf(-zha, pa.y, fmaf(-1024.f, pa.x, d[2] + f[2])), acc[2]);
          acc[2] = fmaf(sh.y, fmaf(-zhb, pb.y, fmaf(-1024.f, pb.x, d[3] + f[3])), acc[2]);
        } else if (KIND == TC_INT4_G128) {
          const int sft = (C.j & 7) << 2;
          const float zl = float((e.zlo >> sft) & 0xFu), zh = float((e.zhi >> sft) & 0xFu);
          const float sl = __half2float(__ushort_as_half(uint16_t(e.slo)));
          const float sh = __half2float(__ushort_as_half(uint16_t(e.shi)));
#pragma unroll
          for (int m = 0; m < M; ++m) {
            const float2 pq = sums[C.j * M + m];
            acc[m] = fmaf(sl, fmaf(-zl, pq.y, fmaf(-1024.f, pq.x, d[m] + f[m])), acc[m]);
            acc[2 + m] = fmaf(sh, fmaf(-zh, pq.y, fmaf(-1024.f, pq.x, d[2 + m] + f[2 + m])), acc[2 + m]);
          }
        } else if (KIND == TC_NVFP4_COLS) {
          const uint32_t bl = tc_e4m3x2(e.slo), bh = tc_e4m3x2(e.shi);
          const float2 sl = __half22float2(*reinterpret_cast<const __half2*>(&bl));
          const float2 sh = __half22float2(*reinterpret_cast<const __half2*>(&bh));
          acc[0] = fmaf(sl.x, d[0] + f[0], fmaf(sl.y, d[1] + f[1], acc[0]));
          acc[2] = fmaf(sh.x, d[2] + f[2], fmaf(sh.y, d[3] + f[3], acc[2]));
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[q] += d[q] + f[q];
        }
      }
      // ---------------------------------------------------------- refill the slot
      if (s + kTcDepth < hi) {
        tc_load_step<KIND>(lp, L.j, R[u]);
        load_advance();
      }
      // ---------------------------------------------------------- row block end
      if (C.j + 1 == csteps || s + 1 == hi) {
        const TcItem& I = a.items[C.i];
        const int sa = s - C.j, sb = sa + csteps;  // the row block's steps in the CTA sequence
        float v[2 * M];
        tc_gather<M, KIND>(acc, lane, v);
        if (sa >= lo && sb <= hi) {  // whole row block in this warp
          if (c == 0) {
#pragma unroll
            for (int m = 0; m < M; ++m) {
              const int nl = C.rb * kTcRows + g, nh = nl + 8;
              if (nl < I.N) I.Y[int64_t(m) * I.N + nl] = uint16_t(f32_to_bf16_bits(v[m] * gmul));
              if (nh < I.N) I.Y[int64_t(m) * I.N + nh] = uint16_t(f32_to_bf16_bits(v[M + m] * gmul));
            }
          }
        } else {
          tc_flush_split<M>(v, lane, warp, S, Wc, sa, sb, &I, C.rb, gmul, spart, sctr);
        }
        acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
        C.j = 0;
        if (++C.rb == I.nrb) {
          C.rb = 0;
          ++C.i;
          if (s + 1 < hi) compute_enter();
        }
      } else {
        ++C.j;
      }
    }
  }
}

// One launch for a group of any weight kinds: every CTA's row blocks are of
// one kind (the host splits the CTAs over the kinds by bytes), and the CTA
// runs that kind's code.
template <int M>
__global__ void __launch_bounds__(kTcThreads, 1) gemv_tc_kernel(const __grid_constant__ TcArgs a) {
  extern __shared__ __align__(16) uint8_t tc_smem[];
  __shared__ float spart[kTcWarps * 2 * kTcRows * M];  // partials of row blocks split over warps
  __shared__ unsigned sctr[kTcWarps];                   // their arrival counters (by first piece's warp)
  __shared__ int xoff[kTcMaxX];                         // byte offset of each staged vector, -1 if unused
  __shared__ __align__(16) uint16_t zrow[32];           // B source of lanes whose column stays empty
  const int kind = int((a.cta[blockIdx.x] >> 10) & 3u);
  if (kind == TC_INT4_G64) {
    gemv_tc_cta<M, TC_INT4_G64>(a, tc_smem, spart, sctr, xoff, zrow);
  } else if (kind == TC_INT4_G128) {
    gemv_tc_cta<M, TC_INT4_G128>(a, tc_smem, spart, sctr, xoff, zrow);
  } else if constexpr (M == 1) {
    gemv_tc_cta<M, TC_NVFP4_COLS>(a, tc_smem, spart, sctr, xoff, zrow);
  } else {
    gemv_tc_cta<M, TC_NVFP4_MUL>(a, tc_smem, spart, sctr, xoff, zrow);
  }
}

}  // namespace wq
