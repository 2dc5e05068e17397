/*
 * wq.h -- C ABI of libwq, a B200 (sm_100a) library for group-wise 4-bit
 * weight-only quantization of transformer Linear layers and for the
 * quantized Linear Y = X * dequant(Wq)^T with bf16 activations.
 *
 * Method (page titles and sections):
 *  - "Lance-Quant" (zingnex.cn), section "量化应用": AWQ-style grid search of
 *    an activation-aware per-input-channel scale, group-wise INT4 packing,
 *    and the NVFP4 pack (E2M1 codes with one FP8-E4M3 scale per 16
 *    elements) for Blackwell tensor cores; section "当前局限": the quantized
 *    Linear should run as a fused dequant GEMM, not a dequant-then-matmul.
 *  - "quantization primer" (xingyuwang.me), section 2: asymmetric
 *    q = round(x/s) + z, x_hat = (q - z) s with clipping; section 3:
 *    per-group scales; section 4: W4A16 (4-bit weights, 16-bit
 *    activations); section 6: GPTQ (quantize, estimate the error with
 *    second-order information, adjust the remaining weights); section 12:
 *    FP8 E4M3 bit layout; section 13: a fused kernel reads compressed
 *    weights and dequantizes inside the matmul.
 *  - the ms-swift article (maplevalley.com.cn): GPTQ from 128-512
 *    calibration samples with group size 128 and no activation reordering.
 *  - "OmniQuant" tutorial (cyqw.cn), section 2.1: scale and zero point;
 *    section 2.2.2: the equivalence Y = (X s)(W / s); section 4.2: W4A4.
 *
 * Conventions for every entry point:
 *  - Matrices are row-major.  W and Wq are [N, K] (N = out_features, row n
 *    holds the K input-channel weights of output n); X is [M, K]; Y [M, N].
 *  - bf16 and fp16 values travel as their 16-bit patterns (uint16_t).
 *  - All data pointers are DEVICE pointers owned by the caller; the library
 *    allocates no memory and keeps no state except one device error word
 *    per loaded GPU (see wq_device_error), the fixed scratch array of
 *    wq_linear_nvfp4_w4a4_noalloc, and one internal CUDA stream per GPU that
 *    wq_gptq_hessian_factor creates on first use (its work is joined back to
 *    the caller's stream before the call's last launch).
 *  - `stream` is a cudaStream_t (0 = legacy default stream).  Every call is
 *    asynchronous on that stream; validation happens on the host before any
 *    launch, so an error return means nothing was launched.
 *  - Data pointers must be 16-byte aligned; K must be a multiple of 32.
 *  - Status codes mirror the exit codes 0 / 1 / 2 of the "llm-quantize"
 *    guide (blog.yoooo.fun): 0 ok, 1 argument validation failed, 2 runtime
 *    (CUDA) failure; 3 = valid but unsupported parameters; 4 = a kernel's
 *    bounded wait ran out (reported by wq_device_error).
 *
 * Packed INT4 format (the pages fix no layout; this library's choice):
 *    qweight uint32 [N, K/8]   nibble j (bits 4j..4j+3) of word k/8 = code of k%8 == j
 *    scales  fp16   [N, K/G]   one scale per group of G consecutive k
 *    zeros   uint32 [N, ceil(K/G/8)]  nibble g%8 of word g/8 = zero point of
 *                              group g; unused high nibbles of the last word are 0
 *    asymmetric (zero_point=1): w_hat = (q - z) * scale
 *    symmetric  (zero_point=0): w_hat = (q - 8) * scale, no zeros buffer
 * Packed NVFP4 format:
 *    codes   uint8 [N, K/2]    low nibble = element 2j, high nibble = 2j+1,
 *                              E2M1 (1 sign, 2 exponent, 1 mantissa)
 *    bscale  uint8 [N, K/16]   FP8 E4M3 block scale, one per 16 consecutive k
 *    global_scale float [1]    per-tensor fp32 scale g
 *    w_hat = e2m1(code) * e4m3(bscale) * g
 */
#ifndef WQ_H_
#define WQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  WQ_OK = 0,
  WQ_ERR_ARG = 1,         /* null/misaligned pointer, bad size, too-small workspace */
  WQ_ERR_CUDA = 2,        /* a CUDA launch or runtime call failed */
  WQ_ERR_UNSUPPORTED = 3, /* bits != 4, group_size not in {32, 64, 128}, ... */
  WQ_ERR_TIMEOUT = 4      /* a device-side bounded wait gave up (see wq_device_error) */
} wq_status;

/* Linear formats for wq_linear_workspace_size. */
enum { WQ_FMT_INT4 = 0, WQ_FMT_NVFP4 = 1 };

/* Human-readable name of a status code (static string, never NULL). */
const char* wq_status_string(int status);

/* Message of the last error this thread saw inside the library ("" if none). */
const char* wq_last_error(void);

/* ---------------------------------------------------------------- sizes
 * Host-only; no device work.  Byte counts of the packed buffers above. */
int wq_int4_sizes(int64_t N, int64_t K, int group_size, size_t* qweight_bytes,
                  size_t* scales_bytes, size_t* zeros_bytes);
int wq_nvfp4_sizes(int64_t N, int64_t K, size_t* codes_bytes, size_t* bscale_bytes);

/* Scratch bytes wq_linear_int4 / wq_linear_nvfp4 use for an [M, K] x [N, K]
 * problem (format WQ_FMT_*, act_fp4 as in wq_linear_nvfp4).  W4A4 requires a
 * workspace of this size.  W4A16 never requires one: a non-zero size means a
 * prefill GEMM with few output tiles (under half the SMs) that, given a
 * workspace of at least this size, splits K over several CTAs per tile (fp32
 * partial tiles, then a reduction launch that sums them in split order, so the
 * result does not depend on timing); with ws = NULL or a smaller one it runs
 * unsplit. */
int wq_linear_workspace_size(int64_t M, int64_t N, int64_t K, int format, int act_fp4,
                             size_t* bytes);

/* Scratch bytes awq_search_scale needs. */
int awq_search_workspace_size(int64_t N, int64_t K, int64_t T, int n_alpha, int group_size,
                              size_t* bytes);

/* ---------------------------------------------------------------- stage 1: quantize + pack
 * wq_quantize_int4 -- group-wise INT4 quantization ("quantization primer"
 * sections 2-3; "Lance-Quant" section "量化应用": pack by group).
 *   W        bf16 [N, K]
 *   bits     must be 4
 *   group_size 32, 64 or 128 (K % group_size == 0)
 *   zero_point 1 = asymmetric with per-group zero point, 0 = symmetric
 *   scale_s  fp32 [K] AWQ per-input-channel scale, or NULL; when given the
 *            library quantizes w' = W[n,k] * scale_s[k] (fp32 multiply)
 *   qweight, scales, zeros: outputs in the packed INT4 format above; zeros
 *            must be NULL when zero_point == 0 and non-NULL otherwise.
 * Per group (all fp32, IEEE round-to-nearest-even, rint ties to even):
 *   asymmetric: scale = fp16(clamp((max - min) / 15, 1e-5, 65504)),
 *               z = clamp(rint(-min / scale), 0, 15),
 *               q = clamp(rint(w' / scale) + z, 0, 15)
 *   symmetric:  scale = fp16(clamp(max|w'| / 7, 1e-5, 65504)),
 *               q = clamp(rint(w' / scale), -7, 7) + 8
 * Results are bit-for-bit deterministic. */
int wq_quantize_int4(const uint16_t* W, int64_t N, int64_t K, int bits, int group_size,
                     int zero_point, const float* scale_s, uint32_t* qweight, uint16_t* scales,
                     uint32_t* zeros, void* stream);

/* wq_quantize_nvfp4 -- NVFP4 pack ("Lance-Quant" section "量化应用": E2M1 +
 * FP8-E4M3 per 16 elements; "quantization primer" section 12: E4M3 layout).
 *   W        bf16 [N, K] (K % 16 == 0; K % 32 == 0 as everywhere)
 *   scale_s  fp32 [K] or NULL, as for INT4
 *   codes, bscale, global_scale: outputs in the packed NVFP4 format above.
 * g = amax|w'| / (6 * 448) (1 if all zero); per block of 16 along k:
 * bscale = E4M3 round-to-nearest-even satfinite of (amax_block / 6) / g;
 * code = nearest E2M1 of w' / (e4m3(bscale) * g), ties to the even code,
 * saturating at 6, sign bit = sign of the quotient; all-zero codes when the
 * block scale is 0.  Bit-for-bit deterministic. */
int wq_quantize_nvfp4(const uint16_t* W, int64_t N, int64_t K, const float* scale_s,
                      uint8_t* codes, uint8_t* bscale, float* global_scale, void* stream);

/* wq_gptq_int4 -- GPTQ INT4 quantize-and-pack with second-order error
 * feedback ("quantization primer" section 6 "GPTQ": quantize a weight,
 * estimate its error with second-order information, adjust the weights not
 * yet quantized, continue; ms-swift page: Hessian from calibration samples,
 * group size 128, no activation reordering).
 *   W        bf16 [N, K], 16-byte aligned
 *   U        fp32 [K, K] row-major, device: the upper Cholesky factor of the
 *            damped inverse Hessian, U^T U = (2 X^T X + lambda I)^-1 over the
 *            caller's calibration tokens X (only the upper triangle is read),
 *            as wq_gptq_hessian_factor computes it
 *   group_size, zero_point, qweight, scales, zeros: as wq_quantize_int4, and
 *            the same packed format (so every linear entry point takes it)
 * Per row, columns k = 0..K-1 in order: at a group's first column its scale
 * and zero point follow wq_quantize_int4's rule applied to the group's
 * weights as they stand; q_k as wq_quantize_int4;
 * e_k = (w_k - (q_k - z) * scale) / U[k][k]; then w_j = w_j - e_k * U[k][j]
 * for all j > k.  All in fp32, each operation rounded on its own (no fused
 * multiply-add), every w_j adjusted in increasing k: the codes are bit-for-bit
 * deterministic.  Returns
 * WQ_ERR_UNSUPPORTED if one row of K fp32 weights plus a G x G tile of U does
 * not fit the GPU's shared memory (K up to ~40000). */
int wq_gptq_int4(const uint16_t* W, int64_t N, int64_t K, const float* U, int group_size,
                 int zero_point, uint32_t* qweight, uint16_t* scales, uint32_t* zeros,
                 void* stream);

/* wq_gptq_hessian_factor -- GPTQ's second-order information from
 * calibration tokens ("quantization primer" section 6 "GPTQ": the error of
 * each quantized weight is estimated with approximate second-order
 * information; the ms-swift page: it comes from 128-512 calibration samples):
 * the factor U that wq_gptq_int4 takes,
 *     U^T U = (H + lambda I)^-1,  H = 2 X^T X,  lambda = damp * mean(diag H),
 * U upper triangular with a positive diagonal (unique), fp32 [K, K]
 * row-major with zeros below the diagonal.  Computed in fp64 on the GPU:
 * the Hessian of the bf16 tokens, the damping, a blocked Cholesky
 * factorisation of the Hessian in reversed channel order and a blocked
 * triangular inverse (the reversed order turns the inverse's upper factor
 * into the inverse of an ordinary lower factor), rounded to fp32 once.
 *   X        bf16 [T, K] calibration tokens (T > 0: an empty calibration set
 *            is an error), 16-byte aligned
 *   damp     relative damping (0.01 is the customary value), finite, >= 0
 *   U        fp32 [K, K] output, 16-byte aligned
 *   ws, ws_bytes  scratch of wq_gptq_factor_workspace_size bytes (about
 *            16 K^2 bytes: 1.9 GB at K = 11008)
 * K up to 65536.  A Hessian that is not positive definite (non-finite
 * tokens, or damp = 0 with fewer independent tokens than channels) makes U
 * NaN and is reported by the next wq_device_error as WQ_ERR_ARG.  The
 * inverse runs on an internal stream that overlaps the factorisation and
 * joins `stream` before U is written; calls on one GPU share that stream. */
int wq_gptq_factor_workspace_size(int64_t K, int64_t T, size_t* bytes);
int wq_gptq_hessian_factor(const uint16_t* X, int64_t T, int64_t K, double damp, float* U,
                           void* ws, size_t ws_bytes, void* stream);

/* awq_search_scale -- AWQ grid search of the per-input-channel scale
 * ("Lance-Quant" section "量化应用": grid-search AWQ scale equalization;
 * "quantization primer" section 7: scale salient channels by activation
 * magnitude).  For each alpha_i:
 *   a_k = max(mean_t |X[t,k]|, 1e-4)   (or max(act_mean[k], 1e-4) if X == NULL)
 *   s_k = fp32(a_k ^ alpha_i)
 *   Delta = W - dequant(Q_int4(W s)) / s     (asymmetric INT4, group_size)
 *   loss_i = || X Delta^T ||_F^2            (X given, T tokens)
 *   loss_i = sum_{n,k} (a_k Delta[n,k])^2    (X == NULL: diagonal proxy from
 *                                             mean |activation| only)
 *   best = first index of the minimum loss; s_out = s of best.
 *   W bf16 [N, K]; X bf16 [T, K] or NULL (T > 0 required when X given: an
 *   empty calibration set is an error); act_mean fp32 [K] used iff X == NULL;
 *   alphas fp32 [n_alpha] device array; s_out fp32 [K]; loss_out fp32
 *   [n_alpha]; best_idx int32 [1]; ws/ws_bytes from awq_search_workspace_size.
 * The chosen s then goes to wq_quantize_int4 / wq_quantize_nvfp4 and its
 * reciprocal to the linear entry points as act_inv_s. */
int awq_search_scale(const uint16_t* W, int64_t N, int64_t K, const uint16_t* X, int64_t T,
                     const float* act_mean, const float* alphas, int n_alpha, int group_size,
                     float* s_out, float* loss_out, int* best_idx, void* ws, size_t ws_bytes,
                     void* stream);

/* awq_search_scale_shared -- the same grid search for several weight
 * matrices that consume one input and therefore share one s ("Lance-Quant"
 * section "量化应用：网格搜索与分组策略": the AWQ scale of a norm and the
 * linear layers consuming it is folded into that RMSNorm, so q/k/v share one
 * s and gate/up share one; section "v2改进" notes o/down cannot).  The loss
 * of alpha_i is the loss of the stacked matrix [W_0; W_1; ...] (N = sum of
 * Ns rows): the sum of the matrices' losses under the one s.
 *   Ws       host array of n_mats (1..64) device pointers, bf16 [Ns[p], K],
 *            16-byte aligned
 *   Ns       host array of the row counts
 *   ws_bytes from awq_search_workspace_size(sum of Ns, K, T, n_alpha, G)
 * Every other argument and the errors are those of awq_search_scale; the
 * chosen s then quantizes each matrix (wq_quantize_int4 with scale_s = s), or
 * the stacked matrix once, whose pack is the stack of the matrices' packs
 * (rows are quantized independently), for one fused linear over N rows. */
int awq_search_scale_shared(const uint16_t* const* Ws, const int64_t* Ns, int n_mats, int64_t K,
                            const uint16_t* X, int64_t T, const float* act_mean, const float* alphas,
                            int n_alpha, int group_size, float* s_out, float* loss_out, int* best_idx,
                            void* ws, size_t ws_bytes, void* stream);

/* One weight matrix of wq_quantize_layers. */
typedef struct {
  const uint16_t* W;        /* bf16 [N, K], 16-byte aligned */
  int64_t N, K;
  const float* act_mean;    /* fp32 [K] mean |activation| per input channel (the
                               calibration statistic), or NULL: no search, the INT4
                               pack uses no scale (the plain min-max rule) */
  float* s_out;             /* fp32 [K] chosen AWQ scale; required with act_mean */
  float* loss_out;          /* fp32 [n_alpha] diagonal-proxy losses; required with act_mean */
  int* best_idx;            /* int32 [1] index of the chosen alpha; required with act_mean */
  uint32_t* qweight;        /* INT4 pack (asymmetric, group_size) of W * s, or NULL to skip */
  uint16_t* scales;
  uint32_t* zeros;
  uint8_t* codes;           /* NVFP4 pack of W, or NULL to skip */
  uint8_t* bscale;
  float* global_scale;
} wq_layer_item;

/* wq_quantize_layers -- quantize and pack a list of Linear weights in one
 * call, as a whole model's target layers are ("Lance-Quant", section
 * "校准阶段": 504 target Linear layers with saved per-channel mean
 * |activation|, min-max fallback for layers without statistics; section
 * "量化应用": AWQ grid search then group-wise INT4 packing, and the NVFP4 pack).
 * For each item, in order, on `stream`:
 *   1. with act_mean: awq_search_scale with X = NULL (the diagonal-proxy loss
 *      from the mean |activation| alone) over `alphas` at group_size;
 *   2. with qweight: wq_quantize_int4 (asymmetric, group_size) of W with the
 *      chosen s (no scale without act_mean);
 *   3. with codes: wq_quantize_nvfp4 of W (no scale).
 * Each result equals the single entry point's.  Every item is validated
 * before anything is launched.  ws / ws_bytes: at least
 * wq_quantize_layers_workspace_size bytes (reused item after item). */
int wq_quantize_layers_workspace_size(const wq_layer_item* items, int count, int n_alpha,
                                      int group_size, size_t* bytes);
int wq_quantize_layers(const wq_layer_item* items, int count, const float* alphas, int n_alpha,
                       int group_size, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- stage 2: quantized Linear
 * wq_linear_int4 -- Y = (X * act_inv_s) * dequant(Wq)^T, bf16 in, fp32
 * accumulate, bf16 out ("quantization primer" sections 4 and 13).
 *   X        bf16 [M, K]
 *   qweight/scales/zeros/group_size/zero_point: an INT4 pack from
 *            wq_quantize_int4 (zeros NULL for symmetric packs)
 *   act_inv_s fp32 [K] or NULL: multiplies column k of X (the 1/s of an AWQ
 *            scale that could not be folded into a preceding norm)
 *   Y        bf16 [M, N]
 *   ws, ws_bytes: optional scratch (NULL allowed): with at least
 *            wq_linear_workspace_size bytes, a prefill GEMM with few output
 *            tiles splits K over several CTAs per tile
 * M <= 16 runs the split-K CUDA-core decode GEMV (one launch, lowest
 * latency for a single projection); larger M runs the tensor-core GEMM.
 * wq_linear_group runs decode projections on the tensor-core decode GEMV. */
int wq_linear_int4(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* qweight,
                   const uint16_t* scales, const uint32_t* zeros, int group_size, int zero_point,
                   const float* act_inv_s, uint16_t* Y, void* ws, size_t ws_bytes, void* stream);

/* wq_linear_nvfp4 -- Y = (X * act_inv_s) * dequant(Wq)^T for an NVFP4 pack.
 *   act_fp4 = 0: W4A16, activations stay bf16.
 *   act_fp4 = 1: W4A4 ("OmniQuant" section 4.2): X is first quantized to
 *            NVFP4 along K with its own per-tensor scale (the
 *            wq_quantize_nvfp4 rule applied to X), and the product runs on
 *            the block-scaled FP4 tensor cores; needs workspace.
 *   other arguments as for wq_linear_int4. */
int wq_linear_nvfp4(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint8_t* codes,
                    const uint8_t* bscale, const float* global_scale, int act_fp4,
                    const float* act_inv_s, uint16_t* Y, void* ws, size_t ws_bytes, void* stream);

/* One quantized Linear of a group (W4A16; see wq_linear_int4 / wq_linear_nvfp4
 * for the meaning of each field).  `format` is WQ_FMT_INT4 or WQ_FMT_NVFP4;
 * fields of the other format are ignored. */
typedef struct {
  int format;
  int64_t N, K;
  const uint16_t* X;          /* bf16 [M, K] */
  const float* act_inv_s;     /* fp32 [K] or NULL */
  const void* packed;         /* INT4 qweight (uint32 [N, K/8]) or NVFP4 codes (uint8 [N, K/2]) */
  const uint16_t* scales;     /* INT4 fp16 [N, K/G] */
  const uint32_t* zeros;      /* INT4 packed zero points, NULL for a symmetric pack */
  int group_size;             /* INT4: 32, 64 or 128 (32 runs the CUDA-core GEMV) */
  int zero_point;             /* INT4: 1 asymmetric, 0 symmetric */
  const uint8_t* bscale;      /* NVFP4 E4M3 [N, K/16] */
  const float* global_scale;  /* NVFP4 fp32 [1] */
  uint16_t* Y;                /* bf16 [M, N] */
} wq_linear_item;

/* wq_linear_group -- the decode-time (M <= 16) quantized Linears of a group
 * of independent projections at once, e.g. the projections of one
 * transformer block that read the same normalised activations ("quantization
 * primer" section 13: decode is memory-bound, so the weights must stream at
 * HBM speed; one launch pays the launch and ramp cost once for the whole
 * group).  Each item's Y is what its single entry point computes.  At M <= 2
 * the items the tensor-core decode GEMV serves (K % 128 == 0, INT4 group 64
 * or 128 or NVFP4, 16-byte aligned X / packed / act_inv_s, 4-byte aligned
 * scale data) run as one launch for all their weight kinds together, up to 24
 * items and 8 distinct activation vectors; the other items (M > 2, group 32,
 * other K) run one by one after them.  Items must not alias each other's
 * outputs.  Needs no workspace.
 * Returns the first failing item's status. */
int wq_linear_group(const wq_linear_item* items, int count, int64_t M, void* stream);

/* wq_linear_nvfp4_w4a4_noalloc -- the W4A4 product of wq_linear_nvfp4
 * (act_fp4 = 1) for callers that cannot allocate device memory when they
 * call, and so cannot hand over a workspace: for example a runtime that
 * plans every device buffer up front and forbids allocation afterwards, or
 * code running where no device allocator is reachable.  The pages have no
 * counterpart of this entry point; it exists only for such callers.
 *   Arguments as for wq_linear_nvfp4 with act_fp4 = 1, minus the workspace.
 *   The NVFP4 pack of X is kept in a scratch array inside the library
 *   (8 MiB per GPU that loads the library, held until the process exits).
 *   The pack needs M*K/2 + M*K/16 bytes plus alignment; larger problems are
 *   rejected with WQ_ERR_ARG (use wq_linear_nvfp4 with a workspace then).
 *   The call allocates nothing.  Its first call on a GPU looks up the
 *   scratch array's device address there; make that first call before any
 *   CUDA graph capture.  All calls on a GPU share the one array: calls whose
 *   execution overlaps on the GPU (different streams without ordering) race
 *   on it and give undefined results. */
int wq_linear_nvfp4_w4a4_noalloc(const uint16_t* X, int64_t M, int64_t N, int64_t K,
                                 const uint8_t* codes, const uint8_t* bscale,
                                 const float* global_scale, const float* act_inv_s, uint16_t* Y,
                                 void* stream);

/* wq_selftest_timeout -- exercises the failure path of the bounded waits on
 * the GPU without a fault: launches one kernel whose single thread waits on
 * an mbarrier that nothing arrives on.  After the 2 s limit the wait gives
 * up, records a timeout in the device error word, stores 0 into
 * *waited_ok (device int; 1 would mean the wait completed) and the kernel
 * returns.  A following wq_device_error reports WQ_ERR_TIMEOUT and clears the
 * word.  The pages have no counterpart: it is a test hook of this library. */
int wq_selftest_timeout(int* waited_ok, void* stream);

/* Synchronizes `stream`, then reads and clears the device error word of the
 * current GPU.  WQ_OK if no kernel reported a problem since the last call,
 * WQ_ERR_TIMEOUT if a bounded wait inside a kernel gave up (the kernel then
 * exited early and its outputs are undefined), WQ_ERR_ARG if
 * wq_gptq_hessian_factor met a Hessian that is not positive definite,
 * WQ_ERR_CUDA if the stream itself failed. */
int wq_device_error(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* WQ_H_ */
