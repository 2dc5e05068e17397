// wq_api.cu -- host side of libwq: argument validation, launch configuration
// and the extern "C" entry points declared in include/wq.h.  All kernels are
// compiled into this one translation unit for sm_100a.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

#include "wq.h"
#include "awq.cuh"
#include "gemm_fp4.cuh"
#include "gemm_tcgen05.cuh"
#include "gemv.cuh"
#include "gemv_mma.cuh"
#include "gemv_tc.cuh"
#include "gptq.cuh"
#include "gptq_factor.cuh"
#include "quant.cuh"
#include "wq_common.cuh"

namespace {

thread_local char g_last_error[512] = "";

int fail(int status, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
  va_end(ap);
  return status;
}

int cuda_check(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return WQ_OK;
  return fail(WQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define REQUIRE(cond, ...)                         \
  do {                                             \
    if (!(cond)) return fail(WQ_ERR_ARG, __VA_ARGS__); \
  } while (0)

#define REQUIRE_PTR(p)                                                        \
  do {                                                                        \
    if (!(p)) return fail(WQ_ERR_ARG, "%s must not be NULL", #p);             \
    if (!aligned16(p)) return fail(WQ_ERR_ARG, "%s must be 16-byte aligned", #p); \
  } while (0)

#define REQUIRE_OPT_PTR(p)                                                    \
  do {                                                                        \
    if ((p) && !aligned16(p)) return fail(WQ_ERR_ARG, "%s must be 16-byte aligned", #p); \
  } while (0)

int check_shape(int64_t N, int64_t K) {
  REQUIRE(N > 0 && K > 0, "N and K must be positive (got N=%lld K=%lld)", (long long)N, (long long)K);
  REQUIRE(K % 32 == 0, "K must be a multiple of 32 (got %lld)", (long long)K);
  REQUIRE(N <= (int64_t(1) << 30) && K <= (int64_t(1) << 30), "N and K must be below 2^30");
  return WQ_OK;
}

int check_group(int group_size, int64_t K) {
  if (group_size != 32 && group_size != 64 && group_size != 128)
    return fail(WQ_ERR_UNSUPPORTED, "group_size must be 32, 64 or 128 (got %d)", group_size);
  REQUIRE(K % group_size == 0, "K (%lld) must be a multiple of group_size (%d)", (long long)K, group_size);
  return WQ_OK;
}

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

int launched(const char* what) { return cuda_check(cudaGetLastError(), what); }

// The dynamic shared-memory limit of a kernel (cudaFuncSetAttribute) belongs
// to the current device's context, so it is set once per device: bit d of
// *done records device d (devices 64 and up set it on every call).  Racing
// threads may both set it, which is harmless.
template <typename Kern>
int ensure_smem_attr(Kern* kern, int bytes, std::atomic<uint64_t>* done, const char* what) {
  int dev = 0;
  if (int e = cuda_check(cudaGetDevice(&dev), "cudaGetDevice")) return e;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t(1) << dev) : 0;
  if (bit && (done->load(std::memory_order_acquire) & bit)) return WQ_OK;
  if (int e = cuda_check(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes), what))
    return e;
  if (bit) done->fetch_or(bit, std::memory_order_acq_rel);
  return WQ_OK;
}

// ---------------------------------------------------------------- GEMV launch
// Launch shape of the CUDA-core GEMV, measured per weight kind on the decode
// shapes: INT4 at N <= 2048 takes 2 rows per warp (twice the CTAs); INT4 with
// long K (>= 8 k-iterations) targets 4 CTAs per SM through more split-K, the
// rest 2 CTAs per SM.
template <int FMT, int MT, int R>
int launch_gemv_mtr(const wq::GemvArgs& a0, cudaStream_t st, int ctas_per_sm) {
  wq::GemvArgs a = a0;
  const int rows_per_cta = wq::kGemvWarps * R;
  const int gx = (a.N + rows_per_cta - 1) / rows_per_cta;
  const int gz = (a.M + MT - 1) / MT;
  const int iters = (a.K + wq::kGemvKPerIter - 1) / wq::kGemvKPerIter;
  int splits = (ctas_per_sm * 148 + gx * gz - 1) / (gx * gz);
  splits = std::max(1, std::min({splits, wq::kGemvMaxSplits, iters}));
  a.iters_per_split = (iters + splits - 1) / splits;
  splits = (iters + a.iters_per_split - 1) / a.iters_per_split;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(gx, splits, gz);
  cfg.blockDim = dim3(wq::kGemvWarps * 32, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  // Programmatic dependent launch: the kernel streams its weights before it
  // waits (griddepcontrol.wait) for the previous kernel's outputs.
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (splits > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 1;
    attr[na].val.clusterDim.y = splits;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cuda_check(cudaLaunchKernelEx(&cfg, wq::gemv_kernel<FMT, MT, R>, a), "gemv launch");
}

template <int FMT, int MT>
int launch_gemv_mt(const wq::GemvArgs& a, cudaStream_t st) {
  const int iters = (a.K + wq::kGemvKPerIter - 1) / wq::kGemvKPerIter;
  if (FMT == wq::FMT_INT4 && MT == 1) {
    if (a.N <= 2048 && iters < 8) return launch_gemv_mtr<FMT, MT, 2>(a, st, 2);
    return launch_gemv_mtr<FMT, MT, wq::kGemvRows>(a, st, iters >= 8 ? 4 : 2);
  }
  return launch_gemv_mtr<FMT, MT, wq::kGemvRows>(a, st, 2);
}

template <int FMT>
int launch_gemv(const wq::GemvArgs& a, cudaStream_t st) {
  if (a.M == 1) return launch_gemv_mt<FMT, 1>(a, st);
  if (a.M == 2) return launch_gemv_mt<FMT, 2>(a, st);
  return launch_gemv_mt<FMT, 4>(a, st);
}

// ---------------------------------------------------------------- tensor-core GEMV, 3 <= M <= 16
// Serves K % 128 == 0 up to 8 slices of kMmaMaxSliceSteps steps (K <= 24576).
bool gemv_mma_serves(int64_t M, int64_t K) {
  return M >= 3 && M <= 16 && K % wq::kMmaStepK == 0 &&
         K <= int64_t(wq::kMmaMaxSplits) * wq::kMmaMaxSliceSteps * wq::kMmaStepK;
}

template <int FMT, int NT>
int launch_gemv_mma_nt(const wq::GemvMmaArgs& a0, cudaStream_t st) {
  wq::GemvMmaArgs a = a0;
  const int nsteps = a.K / wq::kMmaStepK;
  const int gx = (a.N + wq::kMmaWarps * 16 - 1) / (wq::kMmaWarps * 16);
  // about two CTAs per SM, at most a portable cluster of slices, each slice small
  // enough to stage
  int S = std::max(1, std::min({(2 * 148 + gx - 1) / gx, wq::kMmaMaxSplits, nsteps}));
  S = std::max(S, (nsteps + wq::kMmaMaxSliceSteps - 1) / wq::kMmaMaxSliceSteps);
  a.slice_steps = (nsteps + S - 1) / S;
  S = (nsteps + a.slice_steps - 1) / a.slice_steps;
  const int smem = NT * 8 * (a.slice_steps * wq::kMmaStepK * 2 + 16);
  // the attribute is the kernel's largest staged slice, set once per device
  constexpr int kMaxSmem = NT * 8 * (wq::kMmaMaxSliceSteps * wq::kMmaStepK * 2 + 16);
  static std::atomic<uint64_t> attr_done{0};
  if (int e = ensure_smem_attr(wq::gemv_mma_kernel<FMT, NT>, kMaxSmem, &attr_done, "gemv_mma smem attribute"))
    return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(gx, S, 1);
  cfg.blockDim = dim3(wq::kMmaWarps * 32, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (S > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 1;
    attr[na].val.clusterDim.y = S;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cuda_check(cudaLaunchKernelEx(&cfg, wq::gemv_mma_kernel<FMT, NT>, a), "gemv_mma launch");
}

template <int FMT>
int launch_gemv_mma(const wq::GemvMmaArgs& a, cudaStream_t st) {
  return a.M <= 8 ? launch_gemv_mma_nt<FMT, 1>(a, st) : launch_gemv_mma_nt<FMT, 2>(a, st);
}

int log2i(int v) {
  int r = 0;
  while ((1 << r) < v) ++r;
  return r;
}

// ---------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D row-major tensor [rows, cols] of `elem` bytes, box [box_rows, box_cols].
int make_tmap_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem, uint64_t rows, uint64_t cols,
                 uint32_t box_rows, uint32_t box_cols, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(WQ_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * uint64_t(elem)};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(WQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return WQ_OK;
}

// ---------------------------------------------------------------- GEMM launch
template <int FMT, int BN, int BMT = wq::kGemmBM>
int launch_gemm_prepared(const wq::GemmArgs& a, cudaStream_t st) {
  using S = wq::GemmShape<BN, BMT, FMT == wq::GEMM_BF16_SQ>;
  static std::atomic<uint64_t> attr_done{0};
  if (int e = ensure_smem_attr(wq::gemm_tcgen05_kernel<FMT, BN, BMT>, S::SMEM_BYTES, &attr_done,
                               "gemm smem attribute"))
    return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.N + BN - 1) / BN, (a.M + BMT - 1) / BMT, a.splitk > 1 ? a.splitk : 1);
  cfg.blockDim = dim3(S::THREADS, 1, 1);
  cfg.dynamicSmemBytes = S::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_check(cudaLaunchKernelEx(&cfg, wq::gemm_tcgen05_kernel<FMT, BN, BMT>, a), "gemm launch");
}

template <int FMT, int BN, int BMT = wq::kGemmBM>
int launch_gemm_bn(wq::GemmArgs& a, const uint16_t* X, const void* packed, cudaStream_t st) {
  if (int e = make_tmap_2d(&a.tmA, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, uint64_t(a.M), uint64_t(a.K), BMT,
                           wq::kGemmBK, CU_TENSOR_MAP_SWIZZLE_128B))
    return e;
  if (int e = make_tmap_2d(&a.tmP, packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, uint64_t(a.N), uint64_t(a.K / 2), BN,
                           wq::kGemmBK / 2, CU_TENSOR_MAP_SWIZZLE_NONE))
    return e;
  // unsplit products store Y by TMA when its rows are 16-byte aligned
  a.y_tma = a.splitk <= 1 && (a.N % 8 == 0) && aligned16(a.Y);
  if (a.y_tma) {
    if (int e = make_tmap_2d(&a.tmY, a.Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, uint64_t(a.M), uint64_t(a.N), 32, 32,
                             CU_TENSOR_MAP_SWIZZLE_64B))
      return e;
  }
  return launch_gemm_prepared<FMT, BN, BMT>(a, st);
}

int gemm_bn(int64_t M, int64_t N);

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Plan of a quantized GEMM: the tile (BMT x BN) and how many CTAs share each
// output tile along K (fp32 partial tiles, then the reduction launch), chosen by
// a cost model fitted to measured CTA rates on B200: a CTA spends t_kb per
// 64-deep k-block (set by its dequantization and MMA work: 0.60 us for 128 x 128,
// 0.80 for 256 x 128, 0.85 for 128 x 256 and 256 x 256 with every SM busy)
// plus ~3 us to start and drain; CTAs beyond one wave of 148 queue; a split adds
// the partial tiles' round trip (~10 TB/s while they fit in L2, ~5 TB/s beyond)
// and ~3.5 us for the reduction launch.  Splits stay within one wave and keep at
// least 4 k-blocks per CTA.  Without a workspace (allow_split false) the best
// unsplit plan is taken.
struct GemmPlan {
  int bn, bmt, splitk;
  int64_t tiles;
  size_t part_bytes, ws_bytes;
};
GemmPlan gemm_plan(int64_t M, int64_t N, int64_t K, bool allow_split = true) {
  struct Cfg {
    int bmt, bn;
    double t_kb;
  };
  static const Cfg cfgs[4] = {{256, 256, 0.85}, {256, 128, 0.80}, {128, 256, 0.85}, {128, 128, 0.60}};
  const int64_t nkb = (K + wq::kGemmBK - 1) / wq::kGemmBK;
  const int64_t sms = wq::kTcMaxCtas;
  GemmPlan best = {};
  double best_t = 0.0;
  for (const Cfg& c : cfgs) {
    const int64_t tiles = ((N + c.bn - 1) / c.bn) * ((M + c.bmt - 1) / c.bmt);
    for (int64_t sp = 1; sp <= 8; sp *= 2) {
      if (sp > 1 && (!allow_split || tiles * sp > sms || nkb / sp < 4)) continue;
      const double waves = double((tiles * sp + sms - 1) / sms);
      double t = waves * (double((nkb + sp - 1) / sp) * c.t_kb + 3.0);
      const double part = double(tiles * sp) * c.bmt * c.bn * 4.0;
      // the partials' write and read: ~10 TB/s while they fit in L2 (24 MB), ~5 TB/s past it
      if (sp > 1) t += 2.0 * part / (part <= 24.0 * 1048576.0 ? 10.0e6 : 5.0e6) + 3.5;
      if (best.tiles == 0 || t < best_t) {  // ties keep the earlier (larger-tile, unsplit) plan
        best_t = t;
        best.bmt = c.bmt;
        best.bn = c.bn;
        best.tiles = tiles;
        best.splitk = int(sp);
        best.part_bytes = sp > 1 ? align256(size_t(part)) : 0;
      }
    }
  }
  best.ws_bytes = best.part_bytes;
  return best;
}

// The quantized GEMM with the plan's tile: a 256-row CTA shares each
// dequantized W tile between two accumulators (half the dequantization per
// flop), a 256-wide W tile shares each X tile; the plan splits K when the
// caller's workspace holds the partials, else it takes the best unsplit tile.
template <int FMT>
int launch_gemm(wq::GemmArgs& a, const uint16_t* X, const void* packed, cudaStream_t st, void* ws = nullptr,
                size_t ws_bytes = 0) {
  GemmPlan p = gemm_plan(a.M, a.N, a.K);
  a.splitk = 1;
  if (p.splitk > 1 && !(ws && ws_bytes >= p.ws_bytes && aligned16(ws))) p = gemm_plan(a.M, a.N, a.K, false);
  if (p.splitk > 1) {
    a.splitk = p.splitk;
    a.part = static_cast<float*>(ws);
    // the partial tiles as one fp32 matrix [tiles * splitk * BMT, BN] for the TMA stores
    if (int e = make_tmap_2d(&a.tmPart, a.part, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4,
                             uint64_t(p.tiles) * uint64_t(p.splitk) * uint64_t(p.bmt), uint64_t(p.bn), 32, 32,
                             CU_TENSOR_MAP_SWIZZLE_128B))
      return e;
  }
  int e = WQ_OK;
  if (p.bmt == 256)
    e = p.bn == 256 ? launch_gemm_bn<FMT, 256, 256>(a, X, packed, st) : launch_gemm_bn<FMT, 128, 256>(a, X, packed, st);
  else
    e = p.bn == 256 ? launch_gemm_bn<FMT, 256>(a, X, packed, st) : launch_gemm_bn<FMT, 128>(a, X, packed, st);
  if (e || a.splitk <= 1) return e;
  // the split partials' sum, in split order, as a stream-ordered successor
  const int64_t quads = p.tiles * int64_t(p.bmt) * p.bn / 4;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(std::min<int64_t>((quads + 255) / 256, 148 * 8)), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const int n_tiles = int((a.N + p.bn - 1) / p.bn);
  return cuda_check(cudaLaunchKernelEx(&cfg, wq::split_reduce_kernel, static_cast<const float*>(a.part), a.splitk,
                                       p.bmt, p.bn, n_tiles, quads, a.M, a.N,
                                       FMT == wq::GEMM_NVFP4 ? a.gscale : static_cast<const float*>(nullptr), a.Y),
                    "split reduce launch");
}

int gemm_bn(int64_t M, int64_t N) {
  const int64_t tiles256 = int64_t((N + 255) / 256) * ((M + wq::kGemmBM - 1) / wq::kGemmBM);
  return tiles256 >= 148 ? 256 : 128;
}

// Workspace of awq_search_scale: a (fp64 [K]), s (fp32 [K]), loss partials
// (fp64 [n_alpha, P]) and, with calibration tokens, Delta (bf16 [N, 2K]).
struct AwqLayout {
  size_t off_a, off_s, off_p, off_d, total;
  int64_t P;
  int bn;
  int splitk;          // loss GEMM: CTAs per output tile along K (1 = the fused sum-of-squares epilogue)
  int64_t tiles;       // loss GEMM output tiles
  size_t off_part;     // loss GEMM split partial tiles (fp32 [tiles * splitk * 128, bn])
};

// Without tokens and with at most kAwqProxyMaxAlphas alphas the search runs the
// all-alpha proxy kernel: partial slots for up to 64 stacked matrices (each
// starts a new 4-row block), and the s / 1/s / a table in place of Delta.
bool awq_fused_proxy(bool has_x, int n_alpha) { return !has_x && n_alpha <= wq::kAwqProxyMaxAlphas; }
int64_t awq_proxy_kx(int64_t K) { return (K / 8 + wq::kAwqProxyThreads - 1) / wq::kAwqProxyThreads; }

// The loss GEMM [T, 2K] x [N, 2K]^T (K' = 2K) splits K' when its tiles leave SMs idle:
// the split partial tiles, then kAwqSqRows reduction CTAs per tile that add them in
// split order, square and sum (one partial slot each).
constexpr int kAwqSqRows = 8;
AwqLayout awq_layout(int64_t N, int64_t K, int64_t T, bool has_x, int n_alpha) {
  AwqLayout L = {};
  L.splitk = 1;
  if (has_x) {
    L.bn = gemm_bn(T, N);
    L.tiles = ((N + L.bn - 1) / L.bn) * ((T + wq::kGemmBM - 1) / wq::kGemmBM);
    const int64_t nkb = 2 * K / wq::kGemmBK;
    for (int sp = 8; sp >= 2; sp /= 2)  // the most splits that stay within one wave, >= 8 k-blocks each
      if (L.splitk == 1 && L.tiles * sp <= wq::kTcMaxCtas && nkb / sp >= 8) L.splitk = sp;
    L.P = L.splitk > 1 ? L.tiles * kAwqSqRows : L.tiles * (L.bn / 32);
  } else if (awq_fused_proxy(has_x, n_alpha)) {
    L.bn = 0;
    L.P = awq_proxy_kx(K) * ((N + wq::kAwqProxyRows - 1) / wq::kAwqProxyRows + 63);
  } else {
    L.bn = 0;
    L.P = ((K / 8 + wq::kQuantThreads - 1) / wq::kQuantThreads) * N;
  }
  L.off_a = 0;
  L.off_s = align256(L.off_a + size_t(K) * 8);
  L.off_p = align256(L.off_s + size_t(K) * 4);
  L.off_d = align256(L.off_p + size_t(n_alpha) * size_t(L.P) * 8);
  if (has_x) {
    L.off_part = align256(L.off_d + size_t(N) * size_t(2 * K) * 2);
    L.total = L.off_part + (L.splitk > 1 ? align256(size_t(L.tiles) * L.splitk * wq::kGemmBM * L.bn * 4) : 0);
  } else if (awq_fused_proxy(has_x, n_alpha))
    L.total = align256(L.off_d + size_t(2 * n_alpha + 1) * size_t(K) * 4);
  else
    L.total = L.off_d;
  return L;
}

// Workspace of the W4A4 path: X as NVFP4 (codes [M, K/2], E4M3 scales
// [M, K/16]) and its per-tensor scale g_x.
struct W4A4Layout {
  size_t off_codes, off_sf, off_g, total;
};

// The activation amax pass's per-CTA maxima follow g_x's 256-byte slot.
constexpr int kW4A4AmaxSlot = 64;  // floats past g_x
W4A4Layout w4a4_layout(int64_t M, int64_t K) {
  W4A4Layout L = {};
  L.off_codes = 0;
  L.off_sf = align256(size_t(M) * size_t(K / 2));
  L.off_g = align256(L.off_sf + size_t(M) * size_t(K / 16));
  L.total = L.off_g + 256 + align256(size_t(4 * 148 * 8));
  return L;
}

// Persistent FP4 GEMM (scale tiles by TMA): one CTA per SM over 128 x 128 tiles.
int launch_fp4_persistent(wq::Fp4Args& a, const uint8_t* wcodes, cudaStream_t st) {
  using S = wq::Fp4PShape;
  if (int e = make_tmap_2d(&a.tmB, wcodes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, uint64_t(a.N), uint64_t(a.K / 2),
                           wq::kFp4PBN, wq::kFp4BK / 2, CU_TENSOR_MAP_SWIZZLE_128B))
    return e;
  if (int e = make_tmap_2d(&a.tmSB, a.sfb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, uint64_t(a.N), uint64_t(a.K / 16),
                           wq::kFp4PBN, 16, CU_TENSOR_MAP_SWIZZLE_NONE))
    return e;
  // the epilogue stores Y by TMA when its rows are 16-byte aligned
  a.y_tma = (a.N % 8 == 0) && aligned16(a.Y);
  if (a.y_tma) {
    if (int e = make_tmap_2d(&a.tmY, a.Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, uint64_t(a.M), uint64_t(a.N), 32, 32,
                             CU_TENSOR_MAP_SWIZZLE_64B))
      return e;
  }
  static std::atomic<uint64_t> attr_done{0};
  if (int e = ensure_smem_attr(wq::gemm_fp4_persistent_kernel, S::SMEM_BYTES, &attr_done,
                               "fp4 persistent smem attribute"))
    return e;
  const int64_t tiles = ((a.N + wq::kFp4PBN - 1) / wq::kFp4PBN) * int64_t((a.M + wq::kGemmBM - 1) / wq::kGemmBM);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(std::min<int64_t>(tiles, 148)), 1, 1);
  cfg.blockDim = dim3(S::THREADS, 1, 1);
  cfg.dynamicSmemBytes = S::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_check(cudaLaunchKernelEx(&cfg, wq::gemm_fp4_persistent_kernel, a), "fp4 persistent gemm launch");
}

template <int BN>
int launch_fp4_bn(wq::Fp4Args& a, const uint8_t* xcodes, const uint8_t* wcodes, cudaStream_t st) {
  using S = wq::Fp4Shape<BN>;
  if (int e = make_tmap_2d(&a.tmA, xcodes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, uint64_t(a.M), uint64_t(a.K / 2),
                           wq::kGemmBM, wq::kFp4BK / 2, CU_TENSOR_MAP_SWIZZLE_128B))
    return e;
  if (int e = make_tmap_2d(&a.tmB, wcodes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, uint64_t(a.N), uint64_t(a.K / 2), BN,
                           wq::kFp4BK / 2, CU_TENSOR_MAP_SWIZZLE_128B))
    return e;
  // scale tiles ride with the stage when their rows are 16-byte aligned
  a.sf_tma = (a.K % wq::kFp4BK == 0) && aligned16(a.sfa) && aligned16(a.sfb);
  if (a.sf_tma) {
    if (int e = make_tmap_2d(&a.tmSA, a.sfa, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, uint64_t(a.M), uint64_t(a.K / 16),
                             wq::kGemmBM, 16, CU_TENSOR_MAP_SWIZZLE_NONE))
      return e;
    if (int e = make_tmap_2d(&a.tmSB, a.sfb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, uint64_t(a.N), uint64_t(a.K / 16), BN,
                             16, CU_TENSOR_MAP_SWIZZLE_NONE))
      return e;
  }
  if (a.sf_tma) return launch_fp4_persistent(a, wcodes, st);
  static std::atomic<uint64_t> attr_done{0};
  if (int e = ensure_smem_attr(wq::gemm_fp4_kernel<BN>, S::SMEM_BYTES, &attr_done,
                               "fp4 gemm smem attribute"))
    return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.N + BN - 1) / BN, (a.M + wq::kGemmBM - 1) / wq::kGemmBM, 1);
  cfg.blockDim = dim3(S::THREADS, 1, 1);
  cfg.dynamicSmemBytes = S::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_check(cudaLaunchKernelEx(&cfg, wq::gemm_fp4_kernel<BN>, a), "fp4 gemm launch");
}

// NVFP4 quantization of a bf16 [R, C] tensor (optionally times s per column)
// into codes / scales / g: the stream-ordered passes of wq_quantize_nvfp4
// (zeroing, an atomic amax pass, pack, and a one-thread pass that turns the
// amax in *g into g).  With block_max scratch (kNvfp4AmaxBlocks floats the caller
// does not otherwise use) the amax pass leaves one maximum per CTA there and the
// pack pass reduces them and writes g itself: two launches fewer.
constexpr int kNvfp4AmaxBlocks = 148 * 8;
int nvfp4_quantize_launch(const uint16_t* A, int64_t R, int64_t C, const float* s, uint8_t* codes, uint8_t* bscale,
                          float* g, cudaStream_t st, float* block_max = nullptr) {
  const int64_t words = R * C / 8;
  const int amax_blocks = int(std::max<int64_t>(1, std::min<int64_t>((words + 255) / 256, kNvfp4AmaxBlocks)));
  if (!block_max)
    if (int e = cuda_check(cudaMemsetAsync(g, 0, sizeof(float), st), "memset")) return e;
  wq::nvfp4_amax_kernel<<<amax_blocks, 256, 0, st>>>(A, s, R, C, g, block_max);
  if (int e = launched("nvfp4_amax launch")) return e;
  const int64_t nblk = R * C / 16;
  const int pack_blocks = int(std::max<int64_t>(1, std::min<int64_t>((nblk + 255) / 256, 148 * 16)));
  wq::nvfp4_pack_kernel<<<pack_blocks, 256, 0, st>>>(A, s, R, C, g, codes, bscale, block_max ? g : nullptr,
                                                      block_max, amax_blocks);
  if (int e = launched("nvfp4_pack launch")) return e;
  if (block_max) return WQ_OK;
  wq::nvfp4_finalize_kernel<<<1, 1, 0, st>>>(g);
  return launched("nvfp4_finalize launch");
}

// ---------------------------------------------------------------- tensor-core decode GEMV
// One entry of a gemv_tc launch (the single-item calls and wq_linear_group
// both build these).
struct TcCall {
  int fmt;  // wq::FMT_INT4 / wq::FMT_NVFP4
  int64_t N, K;
  const uint16_t* X;
  const float* inv_s;
  const void* packed;
  const uint16_t* scales;
  const uint32_t* zeros;
  int group_size;
  const uint8_t* bscale;
  const float* gscale;
  uint16_t* Y;
};

// Kernel variant of a call (-1: gemv_tc does not serve it).  Needs M <= 2,
// K a multiple of 128 (whole steps), 16-byte aligned codes / X / 1/s and
// 4-byte aligned scale data.
int tc_kind(const TcCall& c, int64_t M) {
  if (M < 1 || M > 2 || c.K % wq::kTcStepK != 0 || c.K > (int64_t(1) << 20)) return -1;
  if (!aligned16(c.packed) || !aligned16(c.X) || (c.inv_s && !aligned16(c.inv_s))) return -1;
  const auto a4 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 3) == 0; };
  if (c.fmt == wq::FMT_INT4) {
    if (!a4(c.scales) || (c.zeros && !a4(c.zeros))) return -1;
    if (c.group_size != 64 && c.group_size != 128) return -1;  // G = 32: the CUDA-core GEMV serves it
    return c.group_size == 64 ? wq::TC_INT4_G64 : wq::TC_INT4_G128;
  }
  if (!a4(c.bscale)) return -1;
  return M == 1 ? wq::TC_NVFP4_COLS : wq::TC_NVFP4_MUL;
}

// Builds one launch over calls (each with its kind; all kinds in one launch):
// items ordered by kind with their row-block offsets, distinct activation
// vectors, the CTAs split over the kinds by bytes and, within a kind, into
// byte-balanced contiguous row-block ranges, and the staged activation bytes
// the busiest CTA needs.  Returns false when the calls do not fit one launch.
bool build_tc_args(const TcCall* calls, const int* kinds, int count, int64_t M, wq::TcArgs* g, int* nctas,
                   size_t* smem) {
  if (count < 1 || count > wq::kTcMaxItems) return false;
  memset(g, 0, sizeof(*g));
  g->n_items = count;
  int rb = 0;
  std::vector<double> cost;
  double kcost[4] = {0, 0, 0, 0};
  int krb[4] = {0, 0, 0, 0};
  int n = 0;
  for (int kind = 0; kind < 4; ++kind) {
    for (int i = 0; i < count; ++i) {
      if (kinds[i] != kind) continue;
      const TcCall& c = calls[i];
      wq::TcItem& d = g->items[n++];
      d.packed = static_cast<const uint8_t*>(c.packed);
      d.scales = c.scales;
      d.zeros = c.zeros;
      d.bscale = c.bscale;
      d.gscale = c.gscale;
      d.Y = c.Y;
      d.N = int(c.N);
      d.K = int(c.K);
      d.kind = kind;
      d.nrb = int((c.N + wq::kTcRows - 1) / wq::kTcRows);
      d.steps = int(c.K / wq::kTcStepK);
      d.rb0 = rb;
      const int xg = c.fmt == wq::FMT_INT4 ? c.group_size : 0;
      int slot = -1;
      for (int v = 0; v < g->n_x; ++v)
        if (g->xs[v].X == c.X && g->xs[v].K == d.K && g->xs[v].inv_s == c.inv_s && g->xs[v].g == xg) slot = v;
      if (slot < 0) {
        if (g->n_x == wq::kTcMaxX) return false;
        slot = g->n_x++;
        g->xs[slot] = wq::TcX{c.X, c.inv_s, d.K, xg};
      }
      d.xslot = slot;
      // time of a row block: its steps (one 1 KB code tile each, at the kind's
      // measured cost per step relative to INT4 g128) plus an allowance for its end
      static const double kStepCost[4] = {1.04, 1.0, 0.975, 1.0};
      const double per = double(d.steps) * 1024.0 * kStepCost[kind] + 1024.0;
      for (int r = 0; r < d.nrb; ++r) cost.push_back(per);
      kcost[kind] += per * d.nrb;
      krb[kind] += d.nrb;
      rb += d.nrb;
      if (rb >= (1 << 28)) return false;
    }
  }
  if (n != count) return false;
  // CTAs per kind in proportion to bytes (at least one, at most one per row block)
  double total = 0;
  int kinds_used = 0;
  for (int k = 0; k < 4; ++k) {
    total += kcost[k];
    kinds_used += krb[k] > 0;
  }
  int kctas[4] = {0, 0, 0, 0};
  int B = 0;
  for (int k = 0; k < 4; ++k) {
    if (!krb[k]) continue;
    kctas[k] = std::min(krb[k], std::max(1, int(wq::kTcMaxCtas * kcost[k] / total)));
    B += kctas[k];
  }
  while (B > wq::kTcMaxCtas) {  // rounding overflow: take from the largest
    int kk = 0;
    for (int k = 1; k < 4; ++k)
      if (kctas[k] > kctas[kk]) kk = k;
    --kctas[kk];
    --B;
  }
  // contiguous byte-balanced ranges inside each kind's row blocks
  int b = 0, r0 = 0;
  g->bounds[0] = 0;
  for (int k = 0; k < 4; ++k) {
    if (!krb[k]) continue;
    const int r1 = r0 + krb[k], Bk = kctas[k];
    double accum = 0;
    int made = 0;
    for (int r = r0; r < r1 && made < Bk - 1; ++r) {
      accum += cost[size_t(r)];
      const int left = r1 - 1 - r, ctas_left = Bk - 1 - made;
      if (accum >= kcost[k] * (made + 1) / Bk || left == ctas_left) {
        g->bounds[++b] = r + 1;
        ++made;
      }
    }
    while (made < Bk - 1) {  // cannot happen with Bk <= row blocks; kept for safety
      g->bounds[++b] = r1;
      ++made;
    }
    g->bounds[++b] = r1;
    r0 = r1;
  }
  // drop empty ranges (bounds must be strictly increasing)
  int B2 = 0;
  for (int i = 0; i < b; ++i)
    if (g->bounds[i + 1] > g->bounds[i]) g->bounds[++B2] = g->bounds[i + 1];
  B = B2;
  // per CTA: first / last item, kind, steps, activation vectors; the staged
  // activations of the busiest CTA
  const auto item_of = [&](int r) {
    int i = 0;
    while (i + 1 < count && g->items[i + 1].rb0 <= r) ++i;
    return i;
  };
  size_t xmax = 0;
  for (int cb = 0; cb < B; ++cb) {
    const int R0 = g->bounds[cb], R1 = g->bounds[cb + 1];
    const int i0 = item_of(R0), i1 = item_of(R1 - 1);
    uint32_t used = 0;
    int64_t steps = 0;
    for (int i = i0; i <= i1; ++i) {
      const wq::TcItem& I = g->items[i];
      used |= 1u << I.xslot;
      steps += int64_t(std::min(R1, I.rb0 + I.nrb) - std::max(R0, I.rb0)) * I.steps;
    }
    if (steps >= (int64_t(1) << 20) || g->items[i0].kind != g->items[i1].kind) return false;
    g->cta[cb] = uint32_t(i0) | uint32_t(i1) << 5 | uint32_t(g->items[i0].kind) << 10 | uint32_t(steps) << 12;
    g->xused[cb] = uint8_t(used);
    size_t x = 0;
    for (int v = 0; v < g->n_x; ++v)
      if ((used >> v) & 1) x += size_t(wq::tc_x_bytes(g->xs[v].K, g->xs[v].g, int(M)));
    xmax = std::max(xmax, x);
  }
  *smem = xmax;
  if (*smem > size_t(wq::kTcMaxSmem)) return false;
  *nctas = B;
  (void)kinds_used;
  return true;
}

template <int M>
int launch_tc_m(const wq::TcArgs& g, int nctas, size_t smem, cudaStream_t st) {
  static std::atomic<uint64_t> attr_done{0};
  if (int e = ensure_smem_attr(wq::gemv_tc_kernel<M>, wq::kTcMaxSmem, &attr_done,
                               "gemv_tc smem attribute"))
    return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nctas, 1, 1);
  cfg.blockDim = dim3(wq::kTcThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_check(cudaLaunchKernelEx(&cfg, wq::gemv_tc_kernel<M>, g), "gemv_tc launch");
}

// Runs calls (each with its kind, -1 = not served) through the tensor-core
// decode GEMV: one launch for up to kTcMaxItems of them, all kinds together;
// done[i] tells which calls it took.
int run_tc(const TcCall* calls, const int* kinds, int count, int64_t M, cudaStream_t st, char* done) {
  static thread_local wq::TcArgs g;  // ~3 KB: keep it off the stack
  for (int i = 0; i < count; ++i) done[i] = 0;
  for (int start = 0; start < count;) {
    TcCall sub[wq::kTcMaxItems];
    int sk[wq::kTcMaxItems], idx[wq::kTcMaxItems];
    int n = 0, i = start;
    for (; i < count && n < wq::kTcMaxItems; ++i)
      if (kinds[i] >= 0) {
        idx[n] = i;
        sk[n] = kinds[i];
        sub[n++] = calls[i];
      }
    start = i;
    if (n == 0) break;
    int nctas = 0;
    size_t smem = 0;
    if (!build_tc_args(sub, sk, n, M, &g, &nctas, &smem)) continue;
    if (int e = (M == 1 ? launch_tc_m<1>(g, nctas, smem, st) : launch_tc_m<2>(g, nctas, smem, st))) return e;
    for (int j = 0; j < n; ++j) done[idx[j]] = 1;
  }
  return WQ_OK;
}

// ---------------------------------------------------------------- GPTQ factor
// Workspace of wq_gptq_hessian_factor: the fp64 Hessian / Cholesky factor
// [Kp, Kp], Z [Kp, Kp], the inverses of the 64 x 64 diagonal blocks, and the
// reversed, transposed tokens Xr [Kp, Tp] (inside Z's bytes when they fit:
// Z is first written after the Hessian product).
struct FacLayout {
  int64_t Kp, Tp;
  size_t off_a, off_z, off_dinv, off_xr, total;
};

FacLayout fac_layout(int64_t K, int64_t T) {
  FacLayout L = {};
  L.Kp = (K + wq::kFacB - 1) / wq::kFacB * wq::kFacB;
  L.Tp = (T + 31) / 32 * 32;
  const size_t mat = size_t(L.Kp) * size_t(L.Kp) * 8;
  L.off_a = 0;
  L.off_z = align256(mat);
  L.off_dinv = align256(L.off_z + mat);
  L.total = align256(L.off_dinv + size_t(L.Kp) * wq::kFacB * 8);
  if (L.Tp <= L.Kp) {
    L.off_xr = L.off_z;
  } else {
    L.off_xr = L.total;
    L.total = align256(L.total + size_t(L.Kp) * size_t(L.Tp) * 8);
  }
  return L;
}

constexpr int kMaxDevicesFac = 64;
// A second stream per device for the factor's inverse, created on first use
// (the library's only other per-device state besides the error word and the
// no-allocation scratch).
std::mutex g_fac_mu;
cudaStream_t g_fac_stream[kMaxDevicesFac] = {};

int fac_aux_stream(cudaStream_t* out) {
  int dev = 0;
  if (int e = cuda_check(cudaGetDevice(&dev), "cudaGetDevice")) return e;
  if (dev < 0 || dev >= kMaxDevicesFac) return fail(WQ_ERR_CUDA, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_fac_mu);
  if (!g_fac_stream[dev]) {
    if (int e = cuda_check(cudaStreamCreateWithFlags(&g_fac_stream[dev], cudaStreamNonBlocking), "stream create"))
      return e;
  }
  *out = g_fac_stream[dev];
  return WQ_OK;
}

int fac_gemm(const wq::FacGemmArgs& a, bool lower, cudaStream_t st) {
  static std::atomic<uint64_t> done_all{0}, done_lower{0};
  const int64_t tiles = lower ? int64_t(a.mt) * (a.mt + 1) / 2 : int64_t(a.mt) * a.nt;
  if (tiles <= 0) return WQ_OK;
  if (lower) {
    if (int e = ensure_smem_attr(wq::fac_gemm_nt_kernel<wq::FAC_TILES_LOWER>, wq::kFacGemmSmem, &done_lower,
                                 "factor gemm smem attribute"))
      return e;
    wq::fac_gemm_nt_kernel<wq::FAC_TILES_LOWER><<<unsigned(tiles), wq::kFacThreads, wq::kFacGemmSmem, st>>>(a);
  } else {
    if (int e = ensure_smem_attr(wq::fac_gemm_nt_kernel<wq::FAC_TILES_ALL>, wq::kFacGemmSmem, &done_all,
                                 "factor gemm smem attribute"))
      return e;
    wq::fac_gemm_nt_kernel<wq::FAC_TILES_ALL><<<unsigned(tiles), wq::kFacThreads, wq::kFacGemmSmem, st>>>(a);
  }
  return launched("factor gemm launch");
}

wq::FacGemmArgs fac_args(const double* A, int64_t lda, const double* B, int64_t ldb, double* C, int64_t ldc,
                         int64_t m, int64_t n, int64_t kd, double alpha, double beta) {
  wq::FacGemmArgs a;
  a.A = A; a.B = B; a.C = C;
  a.lda = lda; a.ldb = ldb; a.ldc = ldc;
  a.mt = int(m / wq::kFacB); a.nt = int(n / wq::kFacB); a.kd = int(kd);
  a.alpha = alpha; a.beta = beta;
  return a;
}

// Decode GEMV up to this many activation rows, tensor-core GEMM above.
constexpr int64_t kGemvMaxM = 16;

// ---------------------------------------------------------------- fixed scratch
// Scratch memory of wq_linear_nvfp4_w4a4_noalloc, owned by the library: the
// NVFP4 pack of X (codes | E4M3 scales | g_x, laid out as w4a4_layout) lives
// in this array instead of a caller-provided workspace.  Every GPU that loads
// the library holds these bytes until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB per GPU
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current GPU.  In host code the
// array's name only stands for the symbol, so the address is looked up once
// per device (cudaGetSymbolAddress, with that device current) and cached.
int noalloc_scratch(void** out) {
  int dev = 0;
  if (int e = cuda_check(cudaGetDevice(&dev), "cudaGetDevice")) return e;
  if (dev < 0 || dev >= kMaxDevices) return fail(WQ_ERR_CUDA, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (int e = cuda_check(cudaGetSymbolAddress(&p, g_noalloc_scratch), "cudaGetSymbolAddress")) return e;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return WQ_OK;
}

}  // namespace

extern "C" {

const char* wq_status_string(int status) {
  switch (status) {
    case WQ_OK: return "WQ_OK";
    case WQ_ERR_ARG: return "WQ_ERR_ARG (invalid argument)";
    case WQ_ERR_CUDA: return "WQ_ERR_CUDA (CUDA runtime failure)";
    case WQ_ERR_UNSUPPORTED: return "WQ_ERR_UNSUPPORTED (unsupported parameters)";
    case WQ_ERR_TIMEOUT: return "WQ_ERR_TIMEOUT (device-side wait gave up)";
    default: return "unknown wq status";
  }
}

const char* wq_last_error(void) { return g_last_error; }

int wq_int4_sizes(int64_t N, int64_t K, int group_size, size_t* qweight_bytes, size_t* scales_bytes,
                  size_t* zeros_bytes) {
  if (int e = check_shape(N, K)) return e;
  if (int e = check_group(group_size, K)) return e;
  const int64_t ng = K / group_size;
  if (qweight_bytes) *qweight_bytes = size_t(N) * size_t(K / 8) * 4;
  if (scales_bytes) *scales_bytes = size_t(N) * size_t(ng) * 2;
  if (zeros_bytes) *zeros_bytes = size_t(N) * size_t((ng + 7) / 8) * 4;
  return WQ_OK;
}

int wq_nvfp4_sizes(int64_t N, int64_t K, size_t* codes_bytes, size_t* bscale_bytes) {
  if (int e = check_shape(N, K)) return e;
  if (codes_bytes) *codes_bytes = size_t(N) * size_t(K / 2);
  if (bscale_bytes) *bscale_bytes = size_t(N) * size_t(K / 16);
  return WQ_OK;
}

int wq_linear_workspace_size(int64_t M, int64_t N, int64_t K, int format, int act_fp4, size_t* bytes) {
  REQUIRE(bytes, "bytes must not be NULL");
  REQUIRE(M > 0, "M must be positive");
  if (int e = check_shape(N, K)) return e;
  REQUIRE(format == WQ_FMT_INT4 || format == WQ_FMT_NVFP4, "unknown format %d", format);
  REQUIRE(act_fp4 == 0 || act_fp4 == 1, "act_fp4 must be 0 or 1");
  REQUIRE(!act_fp4 || format == WQ_FMT_NVFP4, "act_fp4 needs the NVFP4 format");
  if (act_fp4) {
    *bytes = w4a4_layout(M, K).total;
  } else {
    *bytes = M > kGemvMaxM ? gemm_plan(M, N, K).ws_bytes : 0;
  }
  return WQ_OK;
}

int awq_search_workspace_size(int64_t N, int64_t K, int64_t T, int n_alpha, int group_size, size_t* bytes) {
  REQUIRE(bytes, "bytes must not be NULL");
  if (int e = check_shape(N, K)) return e;
  if (int e = check_group(group_size, K)) return e;
  REQUIRE(T >= 0, "T must not be negative");
  REQUIRE(n_alpha > 0 && n_alpha <= 1024, "n_alpha must be in 1..1024");
  *bytes = awq_layout(N, K, T, T > 0, n_alpha).total;
  return WQ_OK;
}

int wq_quantize_int4(const uint16_t* W, int64_t N, int64_t K, int bits, int group_size, int zero_point,
                     const float* scale_s, uint32_t* qweight, uint16_t* scales, uint32_t* zeros, void* stream) {
  if (bits != 4) return fail(WQ_ERR_UNSUPPORTED, "bits must be 4 (got %d)", bits);
  if (int e = check_shape(N, K)) return e;
  if (int e = check_group(group_size, K)) return e;
  REQUIRE(zero_point == 0 || zero_point == 1, "zero_point must be 0 or 1");
  REQUIRE_PTR(W);
  REQUIRE_PTR(qweight);
  REQUIRE_PTR(scales);
  REQUIRE_OPT_PTR(scale_s);
  if (zero_point) {
    REQUIRE_PTR(zeros);
  } else {
    REQUIRE(!zeros, "zeros must be NULL for a symmetric (zero_point=0) pack");
  }
  const dim3 grid(unsigned((K / 8 + wq::kQuantThreads - 1) / wq::kQuantThreads), unsigned(N));
  cudaStream_t st = as_stream(stream);
  if (group_size == 32) {
    if (zero_point)
      wq::quantize_int4_kernel<32, true><<<grid, wq::kQuantThreads, 0, st>>>(W, scale_s, N, K, qweight, scales, zeros);
    else
      wq::quantize_int4_kernel<32, false><<<grid, wq::kQuantThreads, 0, st>>>(W, scale_s, N, K, qweight, scales, zeros);
  } else if (group_size == 64) {
    if (zero_point)
      wq::quantize_int4_kernel<64, true><<<grid, wq::kQuantThreads, 0, st>>>(W, scale_s, N, K, qweight, scales, zeros);
    else
      wq::quantize_int4_kernel<64, false><<<grid, wq::kQuantThreads, 0, st>>>(W, scale_s, N, K, qweight, scales, zeros);
  } else {
    if (zero_point)
      wq::quantize_int4_kernel<128, true><<<grid, wq::kQuantThreads, 0, st>>>(W, scale_s, N, K, qweight, scales, zeros);
    else
      wq::quantize_int4_kernel<128, false><<<grid, wq::kQuantThreads, 0, st>>>(W, scale_s, N, K, qweight, scales, zeros);
  }
  return launched("quantize_int4 launch");
}

int wq_gptq_int4(const uint16_t* W, int64_t N, int64_t K, const float* U, int group_size, int zero_point,
                 uint32_t* qweight, uint16_t* scales, uint32_t* zeros, void* stream) {
  if (int e = check_shape(N, K)) return e;
  if (int e = check_group(group_size, K)) return e;
  REQUIRE(zero_point == 0 || zero_point == 1, "zero_point must be 0 or 1");
  REQUIRE_PTR(W);
  REQUIRE(aligned16(W), "W must be 16-byte aligned");
  REQUIRE_PTR(U);
  REQUIRE_PTR(qweight);
  REQUIRE_PTR(scales);
  if (zero_point) {
    REQUIRE_PTR(zeros);
  } else {
    REQUIRE(!zeros, "zeros must be NULL for a symmetric (zero_point=0) pack");
  }
  int dev = 0, optin = 0, sms = 0;
  if (int e = cuda_check(cudaGetDevice(&dev), "cudaGetDevice")) return e;
  if (int e = cuda_check(cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev), "smem attr"))
    return e;
  if (int e = cuda_check(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev), "SM count")) return e;
  const int G = group_size;
  const int64_t fit = (int64_t(optin) - int64_t(G) * G * 4) / (K * 4 + int64_t(G) * 5);
  const int R = int(std::min<int64_t>({int64_t(wq::kGptqMaxRows), N, fit}));
  if (R < 1) return fail(WQ_ERR_UNSUPPORTED, "K = %lld is too long for one row in shared memory", (long long)K);
  wq::GptqArgs a = {W, U, N, K, R, qweight, scales, zeros};
  const size_t smem = wq::gptq_smem_bytes(R, K, G);
  const unsigned grid = unsigned(std::min<int64_t>((N + R - 1) / R, sms));
  cudaStream_t st = as_stream(stream);
  const auto go = [&](auto kern) -> int {
    if (int e = cuda_check(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)),
                           "gptq smem attribute"))
      return e;
    kern<<<grid, wq::kGptqThreads, smem, st>>>(a);
    return launched("gptq_int4 launch");
  };
  if (R <= 4) {
    if (G == 32) return zero_point ? go(wq::gptq_int4_kernel<32, true, 4>) : go(wq::gptq_int4_kernel<32, false, 4>);
    if (G == 64) return zero_point ? go(wq::gptq_int4_kernel<64, true, 4>) : go(wq::gptq_int4_kernel<64, false, 4>);
    return zero_point ? go(wq::gptq_int4_kernel<128, true, 4>) : go(wq::gptq_int4_kernel<128, false, 4>);
  }
  if (G == 32) return zero_point ? go(wq::gptq_int4_kernel<32, true, 16>) : go(wq::gptq_int4_kernel<32, false, 16>);
  if (G == 64) return zero_point ? go(wq::gptq_int4_kernel<64, true, 16>) : go(wq::gptq_int4_kernel<64, false, 16>);
  return zero_point ? go(wq::gptq_int4_kernel<128, true, 16>) : go(wq::gptq_int4_kernel<128, false, 16>);
}

int wq_gptq_factor_workspace_size(int64_t K, int64_t T, size_t* bytes) {
  REQUIRE(bytes, "bytes must not be NULL");
  if (int e = check_shape(1, K)) return e;
  REQUIRE(K <= 65536, "K must be at most 65536 (got %lld)", (long long)K);
  REQUIRE(T > 0 && T <= (int64_t(1) << 24), "T must be in 1..2^24 (got %lld)", (long long)T);
  *bytes = fac_layout(K, T).total;
  return WQ_OK;
}

int wq_gptq_hessian_factor(const uint16_t* X, int64_t T, int64_t K, double damp, float* U, void* ws,
                           size_t ws_bytes, void* stream) {
  if (int e = check_shape(1, K)) return e;
  REQUIRE(K <= 65536, "K must be at most 65536 (got %lld)", (long long)K);
  REQUIRE(T > 0, "empty calibration set: T=%lld tokens", (long long)T);
  REQUIRE(T <= (int64_t(1) << 24), "T must be at most 2^24");
  REQUIRE(damp >= 0.0 && damp < 1e30, "damp must be finite and non-negative");
  REQUIRE_PTR(X);
  REQUIRE_PTR(U);
  const FacLayout L = fac_layout(K, T);
  REQUIRE(ws && ws_bytes >= L.total, "workspace too small: need %zu bytes (wq_gptq_factor_workspace_size)",
          L.total);
  REQUIRE_PTR(ws);
  cudaStream_t st = as_stream(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  double* A = reinterpret_cast<double*>(wsb + L.off_a);
  double* Z = reinterpret_cast<double*>(wsb + L.off_z);
  double* Dinv = reinterpret_cast<double*>(wsb + L.off_dinv);
  double* Xr = reinterpret_cast<double*>(wsb + L.off_xr);
  const int64_t Kp = L.Kp, Tp = L.Tp, B = wq::kFacB;

  // 1. H' = 2 Xr Xr^T (lower tiles), damped
  wq::fac_xr_kernel<<<dim3(unsigned(Tp / 32), unsigned(Kp / 32)), 256, 0, st>>>(X, T, K, Tp, Xr);
  if (int e = launched("factor tokens launch")) return e;
  if (int e = fac_gemm(fac_args(Xr, Tp, Xr, Tp, A, Kp, Kp, Kp, Tp, 2.0, 0.0), true, st)) return e;
  wq::fac_damp_kernel<<<1, 256, 0, st>>>(A, K, Kp, damp);
  if (int e = launched("factor damping launch")) return e;
  // 2 and 3 run on two streams: the inverse of a 256-wide super-panel (Z's columns of
  // it) needs only that super-panel's factor (its diagonal-block inverses and its L
  // panel, final once its 64-wide steps are done), so it overlaps the rest of the
  // factorisation.  The inverse's stream joins the caller's before U is written,
  // also when a launch fails, so no work outlives the call's use of the workspace.
  cudaStream_t zs = nullptr;
  if (int e = fac_aux_stream(&zs)) return e;
  cudaEvent_t fork = nullptr, join = nullptr;
  if (int e = cuda_check(cudaEventCreateWithFlags(&fork, cudaEventDisableTiming), "event create")) return e;
  if (int e = cuda_check(cudaEventCreateWithFlags(&join, cudaEventDisableTiming), "event create")) {
    cudaEventDestroy(fork);
    return e;
  }
  const auto to_z = [&]() -> int {  // the inverse's stream waits for the work enqueued so far
    if (int e = cuda_check(cudaEventRecord(fork, st), "event record")) return e;
    return cuda_check(cudaStreamWaitEvent(zs, fork, 0), "stream wait");
  };
  const int64_t SB = 4 * B;
  const auto factor_and_invert = [&]() -> int {
    // Z's bytes also hold Xr, read by the Hessian product: Z is initialised after it
    if (int e = to_z()) return e;
    wq::fac_eye_kernel<<<unsigned(std::min<int64_t>((Kp * Kp + 255) / 256, 148 * 16)), 256, 0, zs>>>(Z, Kp);
    if (int e = launched("factor identity launch")) return e;
    for (int64_t KB = 0; KB < Kp; KB += SB) {
      const int64_t E = std::min(KB + SB, Kp);
      // 2. Cholesky of the super-panel: 64-wide steps, each updating only the
      // super-panel's later columns
      for (int64_t kb = KB; kb < E; kb += B) {
        const int64_t e = kb + B, rest = Kp - e;
        double* Di = Dinv + (kb / B) * B * B;
        wq::fac_diag_kernel<<<1, 256, 0, st>>>(A, Kp, kb, Di);
        if (int er = launched("factor diagonal block launch")) return er;
        if (rest == 0) break;
        double* P = A + e * Kp + kb;  // panel [rest, B]
        if (int er = fac_gemm(fac_args(P, Kp, Di, B, P, Kp, rest, B, B, 1.0, 0.0), false, st)) return er;
        if (e < E) {
          if (int er = fac_gemm(fac_args(P, Kp, P, Kp, A + e * Kp + e, Kp, rest, E - e, B, -1.0, 1.0), false, st))
            return er;
        }
      }
      // 3. this super-panel's part of Z = L'^-T, on the inverse's stream
      if (int e = to_z()) return e;
      for (int64_t kb = KB; kb < E; kb += B) {
        const int64_t e = kb + B;
        const double* Di = Dinv + (kb / B) * B * B;
        if (int er = fac_gemm(fac_args(Z + kb, Kp, Di, B, Z + kb, Kp, e, B, B, 1.0, 0.0), false, zs)) return er;
        if (e < E) {
          if (int er = fac_gemm(fac_args(Z + kb, Kp, A + e * Kp + kb, Kp, Z + e, Kp, e, E - e, B, -1.0, 1.0), false,
                                zs))
            return er;
        }
      }
      if (E < Kp) {
        // rows [e, E) of the super-panel's columns of Z are still 0 (Z is upper
        // triangular), so the update may span rows 0..E with the reduction over all its columns
        if (int er = fac_gemm(fac_args(Z + KB, Kp, A + E * Kp + KB, Kp, Z + E, Kp, E, Kp - E, E - KB, -1.0, 1.0),
                              false, zs))
          return er;
        // the rest of the trailing matrix: one update with a reduction depth of 256
        // (a quarter of the trailing-matrix traffic of an update per 64-wide step)
        const double* Q = A + E * Kp + KB;  // [Kp - E, E - KB]
        if (int er = fac_gemm(fac_args(Q, Kp, Q, Kp, A + E * Kp + E, Kp, Kp - E, Kp - E, E - KB, -1.0, 1.0), true, st))
          return er;
      }
    }
    return WQ_OK;
  };
  const int err = factor_and_invert();
  // join (always): the caller's stream waits for everything enqueued on the inverse's stream
  int jerr = cuda_check(cudaEventRecord(join, zs), "event record");
  if (!jerr) jerr = cuda_check(cudaStreamWaitEvent(st, join, 0), "stream wait");
  cudaEventDestroy(fork);
  cudaEventDestroy(join);
  if (err) return err;
  if (jerr) return jerr;
  // 4. U from Z, reversed and transposed, fp32
  const unsigned kt = unsigned((K + 31) / 32);
  wq::fac_u_kernel<<<dim3(kt, kt), 256, 0, st>>>(Z, K, Kp, U);
  return launched("factor output launch");
}

int wq_quantize_nvfp4(const uint16_t* W, int64_t N, int64_t K, const float* scale_s, uint8_t* codes,
                      uint8_t* bscale, float* global_scale, void* stream) {
  if (int e = check_shape(N, K)) return e;
  REQUIRE_PTR(W);
  REQUIRE_PTR(codes);
  REQUIRE_PTR(bscale);
  REQUIRE_PTR(global_scale);
  REQUIRE_OPT_PTR(scale_s);
  // global_scale first accumulates amax, then the pack pass reads it, then it
  // is replaced by g: three stream-ordered steps, no scratch memory.
  return nvfp4_quantize_launch(W, N, K, scale_s, codes, bscale, global_scale, as_stream(stream));
}

// The grid search over the rows of one or more weight matrices that share one
// s (their Delta rows stacked in one buffer, one loss over all of them).
static int awq_search_pieces(const uint16_t* const* Ws, const int64_t* Ns, int n_mats, int64_t K, const uint16_t* X,
                             int64_t T, const float* act_mean, const float* alphas, int n_alpha, int group_size,
                             float* s_out, float* loss_out, int* best_idx, void* ws, size_t ws_bytes, void* stream) {
  REQUIRE(Ws && Ns && n_mats > 0 && n_mats <= 64, "need 1..64 weight matrices");
  int64_t N = 0;
  for (int p = 0; p < n_mats; ++p) {
    if (int e = check_shape(Ns[p], K)) return e;
    REQUIRE(Ws[p], "weight matrix %d is NULL", p);
    REQUIRE(aligned16(Ws[p]), "weight matrix %d must be 16-byte aligned", p);
    N += Ns[p];
  }
  if (int e = check_shape(N, K)) return e;
  if (int e = check_group(group_size, K)) return e;
  if (X) {
    REQUIRE_PTR(X);
    REQUIRE(T > 0, "empty calibration set: X given with T=%lld tokens", (long long)T);
  } else {
    REQUIRE(act_mean, "either X (calibration tokens) or act_mean is required");
    REQUIRE_PTR(act_mean);
  }
  REQUIRE(n_alpha > 0 && n_alpha <= 1024, "n_alpha must be in 1..1024");
  REQUIRE_PTR(alphas);
  REQUIRE_PTR(s_out);
  REQUIRE_PTR(loss_out);
  REQUIRE_PTR(best_idx);
  const AwqLayout L = awq_layout(N, K, X ? T : 0, X != nullptr, n_alpha);
  REQUIRE(ws && ws_bytes >= L.total, "workspace too small: need %zu bytes (awq_search_workspace_size)", L.total);
  REQUIRE_PTR(ws);
  cudaStream_t st = as_stream(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  double* a = reinterpret_cast<double*>(wsb + L.off_a);
  float* s = reinterpret_cast<float*>(wsb + L.off_s);
  double* partials = reinterpret_cast<double*>(wsb + L.off_p);
  uint16_t* D = X ? reinterpret_cast<uint16_t*>(wsb + L.off_d) : nullptr;

  wq::awq_act_mean_kernel<<<unsigned((K + 255) / 256), 256, 0, st>>>(X, T, K, act_mean, a);
  if (int e = launched("awq_act_mean launch")) return e;
  if (awq_fused_proxy(X != nullptr, n_alpha)) {
    // one pass over each matrix for all alphas; unused partial slots stay 0
    float* tab = reinterpret_cast<float*>(wsb + L.off_d);
    wq::awq_proxy_table_kernel<<<dim3(unsigned((K + 255) / 256), unsigned(n_alpha + 1)), 256, 0, st>>>(
        a, alphas, n_alpha, K, tab);
    if (int e = launched("awq_proxy_table launch")) return e;
    if (int e = cuda_check(cudaMemsetAsync(partials, 0, size_t(n_alpha) * size_t(L.P) * 8, st), "memset")) return e;
    const int64_t kx = awq_proxy_kx(K);
    int64_t p0 = 0;
    for (int p = 0; p < n_mats; ++p) {
      const int64_t ry = (Ns[p] + wq::kAwqProxyRows - 1) / wq::kAwqProxyRows;
      const dim3 grid{unsigned(kx), unsigned(ry), 1u};
      if (group_size == 32)
        wq::awq_proxy_kernel<32><<<grid, wq::kAwqProxyThreads, 0, st>>>(Ws[p], Ns[p], K, tab, n_alpha, partials,
                                                                        L.P, p0);
      else if (group_size == 64)
        wq::awq_proxy_kernel<64><<<grid, wq::kAwqProxyThreads, 0, st>>>(Ws[p], Ns[p], K, tab, n_alpha, partials,
                                                                        L.P, p0);
      else
        wq::awq_proxy_kernel<128><<<grid, wq::kAwqProxyThreads, 0, st>>>(Ws[p], Ns[p], K, tab, n_alpha, partials,
                                                                         L.P, p0);
      if (int e = launched("awq_proxy launch")) return e;
      p0 += kx * ry;
    }
    wq::awq_finalize_kernel<<<1, 256, 0, st>>>(partials, L.P, n_alpha, a, alphas, K, loss_out, best_idx, s_out);
    return launched("awq_finalize launch");
  }
  wq::GemmArgs g = {};
  if (X) {
    g.M = int(T); g.N = int(N); g.K = int(2 * K); g.a_kblocks = int(K / wq::kGemmBK);
    if (int e = make_tmap_2d(&g.tmA, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, uint64_t(T), uint64_t(K), wq::kGemmBM,
                             wq::kGemmBK, CU_TENSOR_MAP_SWIZZLE_128B))
      return e;
    if (int e = make_tmap_2d(&g.tmP, D, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, uint64_t(N), uint64_t(2 * K), L.bn,
                             wq::kGemmBK, CU_TENSOR_MAP_SWIZZLE_128B))
      return e;
    if (L.splitk > 1) {  // partial tiles by TMA, then the sum-of-squares reduction
      g.splitk = L.splitk;
      g.part = reinterpret_cast<float*>(wsb + L.off_part);
      if (int e = make_tmap_2d(&g.tmPart, g.part, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4,
                               uint64_t(L.tiles) * uint64_t(L.splitk) * wq::kGemmBM, uint64_t(L.bn), 32, 32,
                               CU_TENSOR_MAP_SWIZZLE_128B))
        return e;
    }
  }
  const unsigned gx = unsigned((K / 8 + wq::kQuantThreads - 1) / wq::kQuantThreads);
  for (int i = 0; i < n_alpha; ++i) {
    wq::awq_scale_kernel<<<unsigned((K + 255) / 256), 256, 0, st>>>(a, alphas + i, K, s);
    if (int e = launched("awq_scale launch")) return e;
    double* part_i = partials + int64_t(i) * L.P;
    int64_t row = 0;  // first stacked row of matrix p
    for (int p = 0; p < n_mats; ++p) {
      const dim3 dgrid(gx, unsigned(Ns[p]));
      uint16_t* Dp = D ? D + row * 2 * K : nullptr;
      double* pp = D ? part_i : part_i + row * gx;  // proxy partials: one per (row, CTA column)
      if (group_size == 32)
        wq::awq_delta_kernel<32><<<dgrid, wq::kQuantThreads, 0, st>>>(Ws[p], s, Ns[p], K, Dp, a, pp);
      else if (group_size == 64)
        wq::awq_delta_kernel<64><<<dgrid, wq::kQuantThreads, 0, st>>>(Ws[p], s, Ns[p], K, Dp, a, pp);
      else
        wq::awq_delta_kernel<128><<<dgrid, wq::kQuantThreads, 0, st>>>(Ws[p], s, Ns[p], K, Dp, a, pp);
      if (int e = launched("awq_delta launch")) return e;
      row += Ns[p];
    }
    if (X) {
      g.sq_partials = part_i;
      const int e = (L.bn == 256) ? launch_gemm_prepared<wq::GEMM_BF16_SQ, 256>(g, st)
                                  : launch_gemm_prepared<wq::GEMM_BF16_SQ, 128>(g, st);
      if (e) return e;
      if (L.splitk > 1) {
        const int n_tiles = int((N + L.bn - 1) / L.bn);
        wq::split_sq_reduce_kernel<<<dim3(unsigned(L.tiles), kAwqSqRows), 256, 0, st>>>(
            g.part, L.splitk, L.bn, n_tiles, int(T), int(N), part_i);
        if (int e2 = launched("awq loss reduce launch")) return e2;
      }
    }
  }
  wq::awq_finalize_kernel<<<1, 256, 0, st>>>(partials, L.P, n_alpha, a, alphas, K, loss_out, best_idx, s_out);
  return launched("awq_finalize launch");
}

int awq_search_scale(const uint16_t* W, int64_t N, int64_t K, const uint16_t* X, int64_t T, const float* act_mean,
                     const float* alphas, int n_alpha, int group_size, float* s_out, float* loss_out, int* best_idx,
                     void* ws, size_t ws_bytes, void* stream) {
  REQUIRE_PTR(W);
  return awq_search_pieces(&W, &N, 1, K, X, T, act_mean, alphas, n_alpha, group_size, s_out, loss_out, best_idx, ws,
                           ws_bytes, stream);
}

int awq_search_scale_shared(const uint16_t* const* Ws, const int64_t* Ns, int n_mats, int64_t K, const uint16_t* X,
                            int64_t T, const float* act_mean, const float* alphas, int n_alpha, int group_size,
                            float* s_out, float* loss_out, int* best_idx, void* ws, size_t ws_bytes, void* stream) {
  return awq_search_pieces(Ws, Ns, n_mats, K, X, T, act_mean, alphas, n_alpha, group_size, s_out, loss_out, best_idx,
                           ws, ws_bytes, stream);
}

namespace {
int check_layer_items(const wq_layer_item* items, int count, int n_alpha, int group_size, size_t* ws_need) {
  REQUIRE(items, "items must not be NULL");
  REQUIRE(count > 0, "count must be positive");
  if (int e = check_group(group_size, 128)) return e;
  REQUIRE(n_alpha > 0 && n_alpha <= 1024, "n_alpha must be in 1..1024");
  size_t need = 0;
  for (int i = 0; i < count; ++i) {
    const wq_layer_item& it = items[i];
    if (int e = check_shape(it.N, it.K)) return e;
    if (int e = check_group(group_size, it.K)) return e;
    REQUIRE(it.W && aligned16(it.W), "item %d: W must be a 16-byte aligned device pointer", i);
    if (it.act_mean) {
      REQUIRE(aligned16(it.act_mean), "item %d: act_mean must be 16-byte aligned", i);
      REQUIRE(it.s_out && aligned16(it.s_out), "item %d: s_out (16-byte aligned) is required with act_mean", i);
      REQUIRE(it.loss_out && aligned16(it.loss_out), "item %d: loss_out (16-byte aligned) is required", i);
      REQUIRE(it.best_idx && aligned16(it.best_idx), "item %d: best_idx (16-byte aligned) is required", i);
      need = std::max(need, awq_layout(it.N, it.K, 0, false, n_alpha).total);
    }
    if (it.qweight) {
      REQUIRE(aligned16(it.qweight) && it.scales && aligned16(it.scales) && it.zeros && aligned16(it.zeros),
              "item %d: qweight, scales and zeros must be 16-byte aligned device pointers", i);
    }
    if (it.codes) {
      REQUIRE(aligned16(it.codes) && it.bscale && aligned16(it.bscale) && it.global_scale &&
                  aligned16(it.global_scale),
              "item %d: codes, bscale and global_scale must be 16-byte aligned device pointers", i);
    }
  }
  *ws_need = need;
  return WQ_OK;
}
}  // namespace

int wq_quantize_layers_workspace_size(const wq_layer_item* items, int count, int n_alpha, int group_size,
                                      size_t* bytes) {
  REQUIRE(bytes, "bytes must not be NULL");
  return check_layer_items(items, count, n_alpha, group_size, bytes);
}

int wq_quantize_layers(const wq_layer_item* items, int count, const float* alphas, int n_alpha, int group_size,
                       void* ws, size_t ws_bytes, void* stream) {
  size_t need = 0;
  if (int e = check_layer_items(items, count, n_alpha, group_size, &need)) return e;
  if (need) {
    REQUIRE_PTR(alphas);
    REQUIRE(ws && ws_bytes >= need, "workspace too small: need %zu bytes (wq_quantize_layers_workspace_size)",
            need);
    REQUIRE_PTR(ws);
  }
  for (int i = 0; i < count; ++i) {
    const wq_layer_item& it = items[i];
    if (it.act_mean) {
      if (int e = awq_search_pieces(&it.W, &it.N, 1, it.K, nullptr, 0, it.act_mean, alphas, n_alpha, group_size,
                                    it.s_out, it.loss_out, it.best_idx, ws, ws_bytes, stream))
        return e;
    }
    if (it.qweight) {
      if (int e = wq_quantize_int4(it.W, it.N, it.K, 4, group_size, 1, it.act_mean ? it.s_out : nullptr, it.qweight,
                                   it.scales, it.zeros, stream))
        return e;
    }
    if (it.codes) {
      if (int e = wq_quantize_nvfp4(it.W, it.N, it.K, nullptr, it.codes, it.bscale, it.global_scale, stream))
        return e;
    }
  }
  return WQ_OK;
}

int wq_linear_int4(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* qweight,
                   const uint16_t* scales, const uint32_t* zeros, int group_size, int zero_point,
                   const float* act_inv_s, uint16_t* Y, void* ws, size_t ws_bytes, void* stream) {
  REQUIRE(M > 0 && M <= (int64_t(1) << 30), "M must be positive");
  if (int e = check_shape(N, K)) return e;
  if (int e = check_group(group_size, K)) return e;
  REQUIRE(zero_point == 0 || zero_point == 1, "zero_point must be 0 or 1");
  REQUIRE_PTR(X);
  REQUIRE_PTR(qweight);
  REQUIRE_PTR(scales);
  REQUIRE_PTR(Y);
  REQUIRE_OPT_PTR(act_inv_s);
  if (zero_point) {
    REQUIRE_PTR(zeros);
  } else {
    REQUIRE(!zeros, "zeros must be NULL for a symmetric (zero_point=0) pack");
  }
  if (M > kGemvMaxM) {
    wq::GemmArgs g = {};
    g.scales = scales; g.zeros = zeros; g.inv_s = act_inv_s; g.Y = Y;
    g.M = int(M); g.N = int(N); g.K = int(K); g.log2g = log2i(group_size);
    return launch_gemm<wq::FMT_INT4>(g, X, qweight, as_stream(stream), ws, ws_bytes);
  }
  if (gemv_mma_serves(M, K)) {
    wq::GemvMmaArgs m = {};
    m.X = X; m.inv_s = act_inv_s; m.packed = reinterpret_cast<const uint8_t*>(qweight); m.scales = scales;
    m.zeros = zeros; m.Y = Y; m.M = int(M); m.N = int(N); m.K = int(K); m.log2g = log2i(group_size);
    return launch_gemv_mma<wq::FMT_INT4>(m, as_stream(stream));
  }
  wq::GemvArgs a = {};
  a.X = X; a.inv_s = act_inv_s; a.wq = qweight; a.scales = scales; a.zeros = zeros;
  a.Y = Y; a.M = int(M); a.N = int(N); a.K = int(K); a.log2g = log2i(group_size);
  return launch_gemv<wq::FMT_INT4>(a, as_stream(stream));
}

int wq_linear_nvfp4(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint8_t* codes,
                    const uint8_t* bscale, const float* global_scale, int act_fp4, const float* act_inv_s,
                    uint16_t* Y, void* ws, size_t ws_bytes, void* stream) {
  REQUIRE(M > 0 && M <= (int64_t(1) << 30), "M must be positive");
  if (int e = check_shape(N, K)) return e;
  REQUIRE(act_fp4 == 0 || act_fp4 == 1, "act_fp4 must be 0 or 1");
  REQUIRE_PTR(X);
  REQUIRE_PTR(codes);
  REQUIRE_PTR(bscale);
  REQUIRE_PTR(global_scale);
  REQUIRE_PTR(Y);
  REQUIRE_OPT_PTR(act_inv_s);
  if (act_fp4) {
    REQUIRE(K % 64 == 0, "W4A4 needs K %% 64 == 0 (got %lld)", (long long)K);
    const W4A4Layout L = w4a4_layout(M, K);
    REQUIRE(ws && ws_bytes >= L.total, "workspace too small: need %zu bytes (wq_linear_workspace_size)", L.total);
    REQUIRE_PTR(ws);
    cudaStream_t st = as_stream(stream);
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    uint8_t* xcodes = wsb + L.off_codes;
    uint8_t* xsf = wsb + L.off_sf;
    float* gx = reinterpret_cast<float*>(wsb + L.off_g);
    if (int e = nvfp4_quantize_launch(X, M, K, act_inv_s, xcodes, xsf, gx, st, gx + kW4A4AmaxSlot)) return e;
    wq::Fp4Args f = {};
    f.sfa = xsf; f.sfb = bscale; f.gx = gx; f.gw = global_scale; f.Y = Y;
    f.M = int(M); f.N = int(N); f.K = int(K);
    return gemm_bn(M, N) == 256 ? launch_fp4_bn<256>(f, xcodes, codes, st) : launch_fp4_bn<128>(f, xcodes, codes, st);
  }
  if (M > kGemvMaxM) {
    wq::GemmArgs g = {};
    g.bscale = bscale; g.gscale = global_scale; g.inv_s = act_inv_s; g.Y = Y;
    g.M = int(M); g.N = int(N); g.K = int(K);
    return launch_gemm<wq::FMT_NVFP4>(g, X, codes, as_stream(stream), ws, ws_bytes);
  }
  if (gemv_mma_serves(M, K)) {
    wq::GemvMmaArgs m = {};
    m.X = X; m.inv_s = act_inv_s; m.packed = codes; m.bscale = bscale; m.gscale = global_scale;
    m.Y = Y; m.M = int(M); m.N = int(N); m.K = int(K);
    return launch_gemv_mma<wq::FMT_NVFP4>(m, as_stream(stream));
  }
  wq::GemvArgs a = {};
  a.X = X; a.inv_s = act_inv_s; a.wq = codes; a.bscale = bscale; a.gscale = global_scale;
  a.Y = Y; a.M = int(M); a.N = int(N); a.K = int(K);
  return launch_gemv<wq::FMT_NVFP4>(a, as_stream(stream));
}

namespace {
TcCall tc_call_of(const wq_linear_item& it) {
  const bool int4 = it.format == WQ_FMT_INT4;
  return TcCall{int4 ? wq::FMT_INT4 : wq::FMT_NVFP4, it.N, it.K, it.X, it.act_inv_s, it.packed,
                int4 ? it.scales : nullptr, int4 && it.zero_point ? it.zeros : nullptr, int4 ? it.group_size : 0,
                int4 ? nullptr : it.bscale, int4 ? nullptr : it.global_scale, it.Y};
}

int check_items(const wq_linear_item* items, int count, int64_t M) {
  REQUIRE(items, "items must not be NULL");
  REQUIRE(count > 0, "count must be positive");
  REQUIRE(M > 0 && M <= 16, "wq_linear_group serves decode sizes: 1 <= M <= 16 (got %lld)", (long long)M);
  for (int i = 0; i < count; ++i) {
    const wq_linear_item& it = items[i];
    REQUIRE(it.format == WQ_FMT_INT4 || it.format == WQ_FMT_NVFP4, "item %d: unknown format %d", i, it.format);
    if (int e = check_shape(it.N, it.K)) return e;
    REQUIRE_PTR(it.X);
    REQUIRE_PTR(it.packed);
    REQUIRE_PTR(it.Y);
    REQUIRE_OPT_PTR(it.act_inv_s);
    if (it.format == WQ_FMT_INT4) {
      if (int e = check_group(it.group_size, it.K)) return e;
      REQUIRE(it.zero_point == 0 || it.zero_point == 1, "item %d: zero_point must be 0 or 1", i);
      REQUIRE_PTR(it.scales);
      if (it.zero_point) REQUIRE_PTR(it.zeros);
    } else {
      REQUIRE_PTR(it.bscale);
      REQUIRE_PTR(it.global_scale);
    }
  }
  return WQ_OK;
}
}  // namespace

int wq_linear_group(const wq_linear_item* items, int count, int64_t M, void* stream) {
  if (int e = check_items(items, count, M)) return e;
  cudaStream_t st = as_stream(stream);
  // items the tensor-core decode GEMV serves run first (one launch per kernel
  // variant); the rest, and any that do not fit a launch, one by one
  std::vector<char> done(static_cast<size_t>(count), 0);
  if (M <= 2) {
    std::vector<TcCall> calls(static_cast<size_t>(count));
    std::vector<int> kinds(static_cast<size_t>(count));
    for (int i = 0; i < count; ++i) {
      calls[size_t(i)] = tc_call_of(items[i]);
      kinds[size_t(i)] = tc_kind(calls[size_t(i)], M);
    }
    if (int e = run_tc(calls.data(), kinds.data(), count, M, st, done.data())) return e;
  }
  for (int i = 0; i < count; ++i) {
    if (done[size_t(i)]) continue;
    const wq_linear_item& it = items[i];
    const int e = it.format == WQ_FMT_INT4
                      ? wq_linear_int4(it.X, M, it.N, it.K, static_cast<const uint32_t*>(it.packed), it.scales,
                                       it.zero_point ? it.zeros : nullptr, it.group_size, it.zero_point, it.act_inv_s,
                                       it.Y, nullptr, 0, stream)
                      : wq_linear_nvfp4(it.X, M, it.N, it.K, static_cast<const uint8_t*>(it.packed), it.bscale,
                                        it.global_scale, 0, it.act_inv_s, it.Y, nullptr, 0, stream);
    if (e) return e;
  }
  return WQ_OK;
}

int wq_linear_nvfp4_w4a4_noalloc(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint8_t* codes,
                                  const uint8_t* bscale, const float* global_scale, const float* act_inv_s,
                                  uint16_t* Y, void* stream) {
  REQUIRE(M > 0 && M <= (int64_t(1) << 30), "M must be positive");
  if (int e = check_shape(N, K)) return e;
  REQUIRE(K % 64 == 0, "W4A4 needs K %% 64 == 0 (got %lld)", (long long)K);
  REQUIRE_PTR(X);
  REQUIRE_PTR(codes);
  REQUIRE_PTR(bscale);
  REQUIRE_PTR(global_scale);
  REQUIRE_PTR(Y);
  REQUIRE_OPT_PTR(act_inv_s);
  const W4A4Layout L = w4a4_layout(M, K);
  REQUIRE(L.total <= kNoAllocScratchBytes,
          "M x K = %lld x %lld needs %zu bytes of scratch, more than the fixed %zu bytes of this entry point; "
          "use wq_linear_nvfp4 with a workspace",
          (long long)M, (long long)K, L.total, kNoAllocScratchBytes);
  void* scratch = nullptr;
  if (int e = noalloc_scratch(&scratch)) return e;
  cudaStream_t st = as_stream(stream);
  uint8_t* wsb = static_cast<uint8_t*>(scratch);
  uint8_t* xcodes = wsb + L.off_codes;
  uint8_t* xsf = wsb + L.off_sf;
  float* gx = reinterpret_cast<float*>(wsb + L.off_g);
  // the amax pass's per-CTA maxima go after g_x's slot; the pack pass reduces them and writes g_x
  if (int e = nvfp4_quantize_launch(X, M, K, act_inv_s, xcodes, xsf, gx, st, gx + kW4A4AmaxSlot)) return e;
  wq::Fp4Args f = {};
  f.sfa = xsf; f.sfb = bscale; f.gx = gx; f.gw = global_scale; f.Y = Y;
  f.M = int(M); f.N = int(N); f.K = int(K);
  return gemm_bn(M, N) == 256 ? launch_fp4_bn<256>(f, xcodes, codes, st) : launch_fp4_bn<128>(f, xcodes, codes, st);
}

int wq_selftest_timeout(int* waited_ok, void* stream) {
  REQUIRE_PTR(waited_ok);
  wq::selftest_timeout_kernel<<<1, 32, 0, as_stream(stream)>>>(waited_ok);
  return launched("selftest_timeout launch");
}

int wq_device_error(void* stream) {
  cudaStream_t st = as_stream(stream);
  if (int e = cuda_check(cudaStreamSynchronize(st), "stream synchronize")) return e;
  unsigned word = 0;
  if (int e = cuda_check(cudaMemcpyFromSymbol(&word, wq::g_error_word, sizeof word), "read error word")) return e;
  if (!word) return WQ_OK;
  const unsigned zero = 0;
  if (int e = cuda_check(cudaMemcpyToSymbol(wq::g_error_word, &zero, sizeof zero), "clear error word")) return e;
  if (word == wq::ERR_NOT_POSITIVE_DEFINITE)
    return fail(WQ_ERR_ARG, "GPTQ Hessian factor: the damped Hessian is not positive definite "
                            "(non-finite calibration tokens?); U holds NaN");
  return fail(WQ_ERR_TIMEOUT, "device error word 0x%x (1=TMA wait, 2=MMA wait, 4=pipeline wait, 8=bounds, "
                              "16=Hessian not positive definite)", word);
}

}  // extern "C"
