"""B200-native group-wise 4-bit weight-only quantization (INT4 / NVFP4) and the
quantized Linear Y = X * dequant(Wq)^T.

This module is a thin ctypes binding over ``libwq.so`` (C ABI in
``include/wq.h``).  It only checks tensor properties and marshals pointers
and the current CUDA stream; every step of the computation runs in the
library's CUDA kernels.  There is no CPU fallback: if the library cannot be
loaded every call raises.

Functions carry the C names:
    wq_quantize_int4, wq_gptq_hessian_factor, wq_gptq_int4, wq_quantize_nvfp4, awq_search_scale,
    awq_search_scale_shared, wq_quantize_layers, wq_linear_int4, wq_linear_nvfp4, wq_linear_group,
    wq_device_error
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libwq.so")

WQ_OK, WQ_ERR_ARG, WQ_ERR_CUDA, WQ_ERR_UNSUPPORTED, WQ_ERR_TIMEOUT = range(5)
WQ_FMT_INT4, WQ_FMT_NVFP4 = 0, 1

# (name, restype, argtypes) of every symbol declared in include/wq.h
_P, _I64, _I, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
_PSZ = ctypes.POINTER(ctypes.c_size_t)
SIGNATURES = {
    "wq_status_string": (ctypes.c_char_p, [_I]),
    "wq_last_error": (ctypes.c_char_p, []),
    "wq_int4_sizes": (_I, [_I64, _I64, _I, _PSZ, _PSZ, _PSZ]),
    "wq_nvfp4_sizes": (_I, [_I64, _I64, _PSZ, _PSZ]),
    "wq_linear_workspace_size": (_I, [_I64, _I64, _I64, _I, _I, _PSZ]),
    "awq_search_workspace_size": (_I, [_I64, _I64, _I64, _I, _I, _PSZ]),
    "wq_quantize_int4": (_I, [_P, _I64, _I64, _I, _I, _I, _P, _P, _P, _P, _P]),
    "wq_gptq_int4": (_I, [_P, _I64, _I64, _P, _I, _I, _P, _P, _P, _P]),
    "wq_gptq_factor_workspace_size": (_I, [_I64, _I64, _PSZ]),
    "wq_gptq_hessian_factor": (_I, [_P, _I64, _I64, ctypes.c_double, _P, _P, _SZ, _P]),
    "wq_quantize_nvfp4": (_I, [_P, _I64, _I64, _P, _P, _P, _P, _P]),
    "awq_search_scale": (_I, [_P, _I64, _I64, _P, _I64, _P, _P, _I, _I, _P, _P, _P, _P, _SZ, _P]),
    "awq_search_scale_shared": (_I, [_P, _P, _I, _I64, _P, _I64, _P, _P, _I, _I, _P, _P, _P, _P, _SZ, _P]),
    "wq_linear_int4": (_I, [_P, _I64, _I64, _I64, _P, _P, _P, _I, _I, _P, _P, _P, _SZ, _P]),
    "wq_linear_nvfp4": (_I, [_P, _I64, _I64, _I64, _P, _P, _P, _I, _P, _P, _P, _SZ, _P]),
    "wq_linear_nvfp4_w4a4_noalloc": (_I, [_P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P]),
    "wq_linear_group": (_I, [_P, _I, _I64, _P]),
    "wq_quantize_layers_workspace_size": (_I, [_P, _I, _I, _I, _PSZ]),
    "wq_quantize_layers": (_I, [_P, _I, _P, _I, _I, _P, _SZ, _P]),
    "wq_selftest_timeout": (_I, [_P, _P]),
    "wq_device_error": (_I, [_P]),
}

_lib = None


class WQError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        self.status = status
        super().__init__(f"{where}: status {status} ({msg})")


def load(path: str | None = None) -> ctypes.CDLL:
    """Load libwq.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"{p} is missing: build it with `python -m w4a16_gemm_wq_b200.build`")
    lib = ctypes.CDLL(p)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status: int, where: str):
    if status != WQ_OK:
        msg = load().wq_last_error().decode(errors="replace")
        raise WQError(status, where, msg)


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dev(t: torch.Tensor, name: str, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _opt_f32(t, name, K):
    if t is None:
        return None
    return _dev(t, name, torch.float32, (K,))


# ---------------------------------------------------------------- packed formats
@dataclasses.dataclass
class PackedInt4:
    qweight: torch.Tensor  # int32 view of uint32 [N, K/8]
    scales: torch.Tensor   # fp16 [N, K/G]
    zeros: torch.Tensor | None  # int32 view of uint32 [N, ceil(K/G/8)]
    N: int
    K: int
    group_size: int
    zero_point: int

    def nbytes(self) -> int:
        z = 0 if self.zeros is None else self.zeros.numel() * 4
        return self.qweight.numel() * 4 + self.scales.numel() * 2 + z


@dataclasses.dataclass
class PackedNVFP4:
    codes: torch.Tensor        # uint8 [N, K/2]
    bscale: torch.Tensor       # uint8 [N, K/16] (E4M3 bits)
    global_scale: torch.Tensor  # fp32 [1]
    N: int
    K: int

    def nbytes(self) -> int:
        return self.codes.numel() + self.bscale.numel() + 4


def int4_sizes(N: int, K: int, group_size: int):
    q, s, z = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(load().wq_int4_sizes(N, K, group_size, ctypes.byref(q), ctypes.byref(s), ctypes.byref(z)), "wq_int4_sizes")
    return q.value, s.value, z.value


def nvfp4_sizes(N: int, K: int):
    c, b = ctypes.c_size_t(), ctypes.c_size_t()
    _check(load().wq_nvfp4_sizes(N, K, ctypes.byref(c), ctypes.byref(b)), "wq_nvfp4_sizes")
    return c.value, b.value


def linear_workspace_size(M: int, N: int, K: int, fmt: int, act_fp4: int = 0) -> int:
    b = ctypes.c_size_t()
    _check(load().wq_linear_workspace_size(M, N, K, fmt, act_fp4, ctypes.byref(b)), "wq_linear_workspace_size")
    return b.value


def _workspace(nbytes: int, device) -> torch.Tensor | None:
    if nbytes == 0:
        return None
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


# ---------------------------------------------------------------- stage 1
def wq_quantize_int4(W: torch.Tensor, group_size: int = 64, zero_point: int = 1, scale_s=None,
                     bits: int = 4) -> PackedInt4:
    if isinstance(W, (PackedInt4, PackedNVFP4)):
        raise ValueError("the layer is already quantized")  # "llm-quantize": refuse re-quantizing
    _dev(W, "W", torch.bfloat16)
    N, K = W.shape
    lib = load()
    ng = K // group_size if group_size and K % group_size == 0 else 1
    qweight = torch.empty((N, max(K // 8, 1)), dtype=torch.int32, device=W.device)
    scales = torch.empty((N, ng), dtype=torch.float16, device=W.device)
    zeros = torch.empty((N, (ng + 7) // 8), dtype=torch.int32, device=W.device) if zero_point else None
    s = _opt_f32(scale_s, "scale_s", K)
    _check(lib.wq_quantize_int4(_ptr(W), N, K, bits, group_size, zero_point, _ptr(s), _ptr(qweight),
                                _ptr(scales), _ptr(zeros), _stream()), "wq_quantize_int4")
    return PackedInt4(qweight, scales, zeros, N, K, group_size, zero_point)


def wq_gptq_int4(W: torch.Tensor, U: torch.Tensor, group_size: int = 128, zero_point: int = 1) -> PackedInt4:
    """GPTQ INT4 pack of W with the inverse-Hessian factor U (fp32 [K, K] upper
    Cholesky factor of the damped inverse Hessian; see wq_gptq_hessian_factor).
    Same packed format as wq_quantize_int4."""
    if isinstance(W, (PackedInt4, PackedNVFP4)):
        raise ValueError("the layer is already quantized")
    _dev(W, "W", torch.bfloat16)
    N, K = W.shape
    _dev(U, "U", torch.float32)
    if tuple(U.shape) != (K, K):
        raise ValueError(f"U must be [{K}, {K}]")
    lib = load()
    ng = K // group_size if group_size and K % group_size == 0 else 1
    qweight = torch.empty((N, max(K // 8, 1)), dtype=torch.int32, device=W.device)
    scales = torch.empty((N, ng), dtype=torch.float16, device=W.device)
    zeros = torch.empty((N, (ng + 7) // 8), dtype=torch.int32, device=W.device) if zero_point else None
    _check(lib.wq_gptq_int4(_ptr(W), N, K, _ptr(U), group_size, zero_point, _ptr(qweight), _ptr(scales),
                            _ptr(zeros), _stream()), "wq_gptq_int4")
    return PackedInt4(qweight, scales, zeros, N, K, group_size, zero_point)


def gptq_factor_workspace_size(K: int, T: int) -> int:
    b = ctypes.c_size_t()
    _check(load().wq_gptq_factor_workspace_size(K, T, ctypes.byref(b)), "wq_gptq_factor_workspace_size")
    return b.value


def wq_gptq_hessian_factor(X: torch.Tensor, damp: float = 0.01, out: torch.Tensor | None = None,
                           ws: torch.Tensor | None = None) -> torch.Tensor:
    """U (fp32 [K, K], upper) with U^T U = (2 X^T X + lambda I)^-1 for calibration
    tokens X (bf16 [T, K]), lambda = damp * mean(diag 2 X^T X): the factor
    wq_gptq_int4 takes, computed by the library in fp64."""
    _dev(X, "X", torch.bfloat16)
    if X.dim() != 2:
        raise ValueError("X must be [T, K]")
    T, K = X.shape
    U = out if out is not None else torch.empty((K, K), dtype=torch.float32, device=X.device)
    _dev(U, "out", torch.float32, (K, K))
    need = gptq_factor_workspace_size(K, T)
    if ws is None or ws.numel() < need:
        ws = _workspace(need, X.device)
    _check(load().wq_gptq_hessian_factor(_ptr(X), T, K, float(damp), _ptr(U), _ptr(ws), ws.numel(), _stream()),
           "wq_gptq_hessian_factor")
    return U


def wq_quantize_nvfp4(W: torch.Tensor, scale_s=None) -> PackedNVFP4:
    if isinstance(W, (PackedInt4, PackedNVFP4)):
        raise ValueError("the layer is already quantized")
    _dev(W, "W", torch.bfloat16)
    N, K = W.shape
    lib = load()
    codes = torch.empty((N, max(K // 2, 1)), dtype=torch.uint8, device=W.device)
    bscale = torch.empty((N, max(K // 16, 1)), dtype=torch.uint8, device=W.device)
    g = torch.empty((1,), dtype=torch.float32, device=W.device)
    s = _opt_f32(scale_s, "scale_s", K)
    _check(lib.wq_quantize_nvfp4(_ptr(W), N, K, _ptr(s), _ptr(codes), _ptr(bscale), _ptr(g), _stream()),
           "wq_quantize_nvfp4")
    return PackedNVFP4(codes, bscale, g, N, K)


def awq_search_scale(W: torch.Tensor, alphas: torch.Tensor, group_size: int = 64, X: torch.Tensor | None = None,
                     act_mean: torch.Tensor | None = None):
    """Returns (s fp32 [K], losses fp32 [n_alpha], best int32 [1]) as device tensors."""
    _dev(W, "W", torch.bfloat16)
    N, K = W.shape
    T = 0
    if X is not None:
        _dev(X, "X", torch.bfloat16)
        if X.dim() != 2 or X.shape[1] != K:
            raise ValueError("X must be [T, K]")
        T = X.shape[0]
    am = _opt_f32(act_mean, "act_mean", K)
    _dev(alphas, "alphas", torch.float32)
    lib = load()
    n_alpha = alphas.numel()
    b = ctypes.c_size_t()
    _check(lib.awq_search_workspace_size(N, K, T, n_alpha, group_size, ctypes.byref(b)), "awq_search_workspace_size")
    ws = _workspace(b.value, W.device)
    s = torch.empty(K, dtype=torch.float32, device=W.device)
    losses = torch.empty(n_alpha, dtype=torch.float32, device=W.device)
    best = torch.empty(1, dtype=torch.int32, device=W.device)
    _check(lib.awq_search_scale(_ptr(W), N, K, _ptr(X), T, _ptr(am), _ptr(alphas), n_alpha, group_size, _ptr(s),
                                _ptr(losses), _ptr(best), _ptr(ws), b.value, _stream()), "awq_search_scale")
    return s, losses, best


def awq_search_scale_shared(Ws: list, alphas: torch.Tensor, group_size: int = 64, X: torch.Tensor | None = None,
                            act_mean: torch.Tensor | None = None):
    """One AWQ scale for several weights that consume the same input (q/k/v,
    gate/up): the loss is taken over their stacked rows.  Returns (s fp32 [K],
    losses fp32 [n_alpha], best int32 [1]) as device tensors."""
    if not Ws:
        raise ValueError("need at least one weight matrix")
    for i, W in enumerate(Ws):
        _dev(W, f"Ws[{i}]", torch.bfloat16)
    K = Ws[0].shape[1]
    if any(W.dim() != 2 or W.shape[1] != K for W in Ws):
        raise ValueError("every weight must be [N_i, K] with the same K")
    T = 0
    if X is not None:
        _dev(X, "X", torch.bfloat16)
        if X.dim() != 2 or X.shape[1] != K:
            raise ValueError("X must be [T, K]")
        T = X.shape[0]
    am = _opt_f32(act_mean, "act_mean", K)
    _dev(alphas, "alphas", torch.float32)
    lib = load()
    n_alpha = alphas.numel()
    Ntot = sum(int(W.shape[0]) for W in Ws)
    b = ctypes.c_size_t()
    _check(lib.awq_search_workspace_size(Ntot, K, T, n_alpha, group_size, ctypes.byref(b)),
           "awq_search_workspace_size")
    ws = _workspace(b.value, Ws[0].device)
    ptrs = (ctypes.c_void_p * len(Ws))(*[W.data_ptr() for W in Ws])
    ns = (ctypes.c_int64 * len(Ws))(*[int(W.shape[0]) for W in Ws])
    s = torch.empty(K, dtype=torch.float32, device=Ws[0].device)
    losses = torch.empty(n_alpha, dtype=torch.float32, device=Ws[0].device)
    best = torch.empty(1, dtype=torch.int32, device=Ws[0].device)
    _check(lib.awq_search_scale_shared(ctypes.cast(ptrs, ctypes.c_void_p), ctypes.cast(ns, ctypes.c_void_p),
                                       len(Ws), K, _ptr(X), T, _ptr(am), _ptr(alphas), n_alpha, group_size,
                                       _ptr(s), _ptr(losses), _ptr(best), _ptr(ws), b.value, _stream()),
           "awq_search_scale_shared")
    return s, losses, best


class LayerItem(ctypes.Structure):
    """Mirror of wq_layer_item (include/wq.h)."""

    _fields_ = [("W", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64), ("act_mean", ctypes.c_void_p),
                ("s_out", ctypes.c_void_p), ("loss_out", ctypes.c_void_p), ("best_idx", ctypes.c_void_p),
                ("qweight", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("zeros", ctypes.c_void_p),
                ("codes", ctypes.c_void_p), ("bscale", ctypes.c_void_p), ("global_scale", ctypes.c_void_p)]


@dataclasses.dataclass
class QuantizedLayer:
    """Outputs of one wq_quantize_layers item (None where not requested)."""
    int4: PackedInt4 | None
    nvfp4: PackedNVFP4 | None
    s: torch.Tensor | None       # fp32 [K] chosen AWQ scale
    losses: torch.Tensor | None  # fp32 [n_alpha]
    best: torch.Tensor | None    # int32 [1]


def make_layer_items(Ws: list, act_means: list, n_alpha: int, group_size: int = 64, int4: bool = True,
                     nvfp4: bool = True):
    """(ctypes array of wq_layer_item, [QuantizedLayer]) for the weights Ws with their
    act_mean vectors (fp32 [K] or None): the outputs are allocated here and filled by
    every wq_quantize_layers call made with the array."""
    if len(Ws) != len(act_means) or not Ws:
        raise ValueError("need one act_mean (or None) per weight matrix")
    arr = (LayerItem * len(Ws))()
    outs = []
    for i, (W, am) in enumerate(zip(Ws, act_means)):
        if isinstance(W, (PackedInt4, PackedNVFP4)):
            raise ValueError("the layer is already quantized")
        _dev(W, f"Ws[{i}]", torch.bfloat16)
        N, K = W.shape
        dev = W.device
        it = arr[i]
        it.W, it.N, it.K = W.data_ptr(), N, K
        s = losses = best = None
        if am is not None:
            _dev(am, f"act_means[{i}]", torch.float32, (K,))
            s = torch.empty(K, dtype=torch.float32, device=dev)
            losses = torch.empty(max(n_alpha, 4), dtype=torch.float32, device=dev)[:n_alpha]
            best = torch.empty(4, dtype=torch.int32, device=dev)[:1]
            it.act_mean, it.s_out = am.data_ptr(), s.data_ptr()
            it.loss_out, it.best_idx = losses.data_ptr(), best.data_ptr()
        p4 = pn = None
        if int4:
            ng = K // group_size if K % group_size == 0 else 1
            p4 = PackedInt4(torch.empty((N, K // 8), dtype=torch.int32, device=dev),
                            torch.empty((N, ng), dtype=torch.float16, device=dev),
                            torch.empty((N, (ng + 7) // 8), dtype=torch.int32, device=dev), N, K, group_size, 1)
            it.qweight, it.scales, it.zeros = p4.qweight.data_ptr(), p4.scales.data_ptr(), p4.zeros.data_ptr()
        if nvfp4:
            pn = PackedNVFP4(torch.empty((N, K // 2), dtype=torch.uint8, device=dev),
                             torch.empty((N, K // 16), dtype=torch.uint8, device=dev),
                             torch.empty(4, dtype=torch.float32, device=dev)[:1], N, K)
            it.codes, it.bscale, it.global_scale = pn.codes.data_ptr(), pn.bscale.data_ptr(), pn.global_scale.data_ptr()
        outs.append(QuantizedLayer(p4, pn, s, losses, best))
    return arr, outs


def quantize_layers_workspace_size(items, n_alpha: int, group_size: int) -> int:
    b = ctypes.c_size_t()
    _check(load().wq_quantize_layers_workspace_size(ctypes.cast(items, ctypes.c_void_p), len(items), n_alpha,
                                                    group_size, ctypes.byref(b)), "wq_quantize_layers_workspace_size")
    return b.value


def wq_quantize_layers(Ws: list, act_means: list, alphas: torch.Tensor, group_size: int = 64, int4: bool = True,
                       nvfp4: bool = True, ws: torch.Tensor | None = None, prepared=None) -> list:
    """Quantize and pack many Linear weights in one library call: per matrix the AWQ
    diagonal-proxy search when its act_mean (fp32 [K] or None) is given, the INT4
    pack with the chosen s, and the NVFP4 pack.  Returns a QuantizedLayer per matrix.
    `prepared` = make_layer_items(...) reuses its item array and outputs."""
    _dev(alphas, "alphas", torch.float32)
    n_alpha = alphas.numel()
    arr, outs = prepared if prepared is not None else make_layer_items(Ws, act_means, n_alpha, group_size, int4,
                                                                       nvfp4)
    need = quantize_layers_workspace_size(arr, n_alpha, group_size)
    if ws is None or ws.numel() < need:
        ws = _workspace(need, alphas.device)
    _check(load().wq_quantize_layers(ctypes.cast(arr, ctypes.c_void_p), len(arr), _ptr(alphas), n_alpha, group_size,
                                     _ptr(ws), 0 if ws is None else ws.numel(), _stream()), "wq_quantize_layers")
    return outs


# ---------------------------------------------------------------- stage 2
def wq_linear_int4(X: torch.Tensor, p: PackedInt4, act_inv_s=None, out: torch.Tensor | None = None,
                   ws: torch.Tensor | None = None) -> torch.Tensor:
    _dev(X, "X", torch.bfloat16)
    M, K = X.shape
    if K != p.K:
        raise ValueError(f"X has K={K}, the pack K={p.K}")
    Y = out if out is not None else torch.empty((M, p.N), dtype=torch.bfloat16, device=X.device)
    _dev(Y, "out", torch.bfloat16, (M, p.N))
    lib = load()
    need = linear_workspace_size(M, p.N, K, WQ_FMT_INT4)
    if ws is None:
        ws = _workspace(need, X.device)
    s = _opt_f32(act_inv_s, "act_inv_s", K)
    _check(lib.wq_linear_int4(_ptr(X), M, p.N, K, _ptr(p.qweight), _ptr(p.scales), _ptr(p.zeros), p.group_size,
                              p.zero_point, _ptr(s), _ptr(Y), _ptr(ws), 0 if ws is None else ws.numel(), _stream()),
           "wq_linear_int4")
    return Y


def wq_linear_nvfp4(X: torch.Tensor, p: PackedNVFP4, act_fp4: int = 0, act_inv_s=None,
                    out: torch.Tensor | None = None, ws: torch.Tensor | None = None) -> torch.Tensor:
    _dev(X, "X", torch.bfloat16)
    M, K = X.shape
    if K != p.K:
        raise ValueError(f"X has K={K}, the pack K={p.K}")
    Y = out if out is not None else torch.empty((M, p.N), dtype=torch.bfloat16, device=X.device)
    _dev(Y, "out", torch.bfloat16, (M, p.N))
    lib = load()
    need = linear_workspace_size(M, p.N, K, WQ_FMT_NVFP4, act_fp4)
    if ws is None:
        ws = _workspace(need, X.device)
    s = _opt_f32(act_inv_s, "act_inv_s", K)
    _check(lib.wq_linear_nvfp4(_ptr(X), M, p.N, K, _ptr(p.codes), _ptr(p.bscale), _ptr(p.global_scale), act_fp4,
                               _ptr(s), _ptr(Y), _ptr(ws), 0 if ws is None else ws.numel(), _stream()),
           "wq_linear_nvfp4")
    return Y


def wq_linear_nvfp4_w4a4_noalloc(X: torch.Tensor, p: PackedNVFP4, act_inv_s=None,
                                 out: torch.Tensor | None = None) -> torch.Tensor:
    """W4A4 product without a workspace: the library's fixed scratch holds the
    NVFP4 pack of X (for callers that cannot allocate at call time)."""
    _dev(X, "X", torch.bfloat16)
    M, K = X.shape
    if K != p.K:
        raise ValueError(f"X has K={K}, the pack K={p.K}")
    Y = out if out is not None else torch.empty((M, p.N), dtype=torch.bfloat16, device=X.device)
    _dev(Y, "out", torch.bfloat16, (M, p.N))
    s = _opt_f32(act_inv_s, "act_inv_s", K)
    _check(load().wq_linear_nvfp4_w4a4_noalloc(_ptr(X), M, p.N, K, _ptr(p.codes), _ptr(p.bscale),
                                               _ptr(p.global_scale), _ptr(s), _ptr(Y), _stream()),
           "wq_linear_nvfp4_w4a4_noalloc")
    return Y


class LinearItem(ctypes.Structure):
    """Mirror of wq_linear_item (include/wq.h)."""

    _fields_ = [("format", ctypes.c_int), ("N", ctypes.c_int64), ("K", ctypes.c_int64), ("X", ctypes.c_void_p),
                ("act_inv_s", ctypes.c_void_p), ("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("zeros", ctypes.c_void_p), ("group_size", ctypes.c_int), ("zero_point", ctypes.c_int),
                ("bscale", ctypes.c_void_p), ("global_scale", ctypes.c_void_p), ("Y", ctypes.c_void_p)]


def make_group(calls):
    """(ctypes array of wq_linear_item, M) for [(X, pack, out[, act_inv_s]), ...].
    Keeps no tensor alive: the caller holds the tensors for as long as the array is used."""
    arr = (LinearItem * len(calls))()
    M = None
    for i, c in enumerate(calls):
        X, p, Y = c[0], c[1], c[2]
        inv_s = c[3] if len(c) > 3 else None
        _dev(X, "X", torch.bfloat16)
        if M is None:
            M = X.shape[0]
        if X.shape != (M, p.K):
            raise ValueError(f"item {i}: X must be [{M}, {p.K}]")
        _dev(Y, "out", torch.bfloat16, (M, p.N))
        s = _opt_f32(inv_s, "act_inv_s", p.K)
        it = arr[i]
        it.N, it.K, it.X, it.Y = p.N, p.K, X.data_ptr(), Y.data_ptr()
        it.act_inv_s = None if s is None else s.data_ptr()
        if isinstance(p, PackedInt4):
            it.format, it.packed, it.scales = WQ_FMT_INT4, p.qweight.data_ptr(), p.scales.data_ptr()
            it.zeros = None if p.zeros is None else p.zeros.data_ptr()
            it.group_size, it.zero_point = p.group_size, p.zero_point
        else:
            it.format, it.packed = WQ_FMT_NVFP4, p.codes.data_ptr()
            it.bscale, it.global_scale = p.bscale.data_ptr(), p.global_scale.data_ptr()
    return arr, M


def wq_linear_group(calls, group=None):
    """Run the W4A16 decode Linears [(X, pack, out[, act_inv_s]), ...] of independent
    projections as one group (one tensor-core GEMV launch per kernel variant for the
    items it serves)."""
    arr, M = group if group is not None else make_group(calls)
    _check(load().wq_linear_group(ctypes.cast(arr, ctypes.c_void_p), len(arr), M, _stream()), "wq_linear_group")


def wq_selftest_timeout() -> int:
    """Launch the self-test whose bounded device wait runs out (about 2 s); returns the
    kernel's waited_ok flag (0: the wait gave up as designed). Read the outcome with
    wq_device_error(), which then raises WQError with WQ_ERR_TIMEOUT."""
    flag = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    _check(load().wq_selftest_timeout(_ptr(flag), _stream()), "wq_selftest_timeout")
    torch.cuda.synchronize()
    return int(flag.item())


def wq_device_error() -> int:
    """Synchronize the current stream and read/clear the device error word (raises on error)."""
    st = load().wq_device_error(_stream())
    _check(st, "wq_device_error")
    return st
