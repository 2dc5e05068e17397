"""CPU oracle for the 4-bit weight-only quantization path (test infrastructure).

Only the test-suite, the package smoke check and the benchmark's CPU-baseline
leg may import this package.  The product path (the CUDA library and its
binding) never does, and this package never imports the product.

The arithmetic lives in ``oracle.c`` (plain C, fp64 for real values, fp32 for
quantization decisions); this module compiles it on first use with gcc and
wraps it with ctypes + numpy.  Inputs are numpy arrays (bf16 passed as their
uint16 bit patterns) or torch CPU tensors.

Parity pins: every function here is checked in ``tests/test_oracle_pins.py``
against closed forms, invariants, library routines or brute force.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-shared", "-fPIC"]


def build(force: bool = False) -> str:
    """Compile liboracle.so next to oracle.c (gcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _L():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        lib.oracle_bf16_to_f64.restype = ctypes.c_double
        lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_f16_to_f64.restype = ctypes.c_double
        lib.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_f32_to_f16_rne_sat.restype = ctypes.c_uint16
        lib.oracle_f32_to_f16_rne_sat.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_encode_sat.restype = ctypes.c_uint8
        lib.oracle_e4m3_encode_sat.argtypes = [ctypes.c_float]
        lib.oracle_e2m1_decode.restype = ctypes.c_double
        lib.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e2m1_encode.restype = ctypes.c_uint8
        lib.oracle_e2m1_encode.argtypes = [ctypes.c_float]
        lib.oracle_quantize_int4.restype = I
        lib.oracle_quantize_int4.argtypes = [P, I64, I64, I, I, I, P, P, P, P]
        lib.oracle_dequant_int4.restype = None
        lib.oracle_dequant_int4.argtypes = [P, P, P, I64, I64, I, I, P, I64, P]
        lib.oracle_quantize_nvfp4.restype = I
        lib.oracle_quantize_nvfp4.argtypes = [P, I64, I64, P, P, P, P]
        lib.oracle_dequant_nvfp4.restype = None
        lib.oracle_dequant_nvfp4.argtypes = [P, P, ctypes.c_float, I64, I64, P, I64, P]
        lib.oracle_activations_f64.restype = None
        lib.oracle_activations_f64.argtypes = [P, I64, I64, P, P]
        lib.oracle_matmul_abT.restype = None
        lib.oracle_matmul_abT.argtypes = [P, I64, I64, P, I64, P]
        lib.oracle_awq_delta.restype = I
        lib.oracle_awq_delta.argtypes = [P, I64, I64, P, I, P]
        lib.oracle_awq_search.restype = I
        lib.oracle_awq_search.argtypes = [P, I64, I64, P, I64, P, P, I, I, P, P, P]
        lib.oracle_gptq_int4.restype = I
        lib.oracle_gptq_int4.argtypes = [P, I64, I64, P, I, I, P, P, P, P]
        lib.oracle_num_threads.restype = I
        lib.oracle_num_threads.argtypes = []
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def as_bits16(t) -> np.ndarray:
    """bf16/fp16 torch tensor (or uint16 array) -> contiguous uint16 numpy array of bit patterns."""
    if isinstance(t, np.ndarray):
        assert t.dtype == np.uint16
        return np.ascontiguousarray(t)
    import torch

    return np.ascontiguousarray(t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def _f32(a):
    if a is None:
        return None
    if not isinstance(a, np.ndarray):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.float32)


def num_threads() -> int:
    return _L().oracle_num_threads()


# ---------------------------------------------------------------- scalar codecs
def bf16_to_f64(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).ravel()
    return np.array([_L().oracle_bf16_to_f64(int(v)) for v in b])


def f16_to_f64(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).ravel()
    return np.array([_L().oracle_f16_to_f64(int(v)) for v in b])


def f32_to_f16(x) -> np.ndarray:
    x = np.asarray(x, dtype=np.float32).ravel()
    return np.array([_L().oracle_f32_to_f16_rne_sat(float(v)) for v in x], dtype=np.uint16)


def e4m3_decode(b) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint8).ravel()
    return np.array([_L().oracle_e4m3_decode(int(v)) for v in b])


def e4m3_encode(x) -> np.ndarray:
    x = np.asarray(x, dtype=np.float32).ravel()
    return np.array([_L().oracle_e4m3_encode_sat(float(v)) for v in x], dtype=np.uint8)


def e2m1_decode(c) -> np.ndarray:
    c = np.asarray(c, dtype=np.uint8).ravel()
    return np.array([_L().oracle_e2m1_decode(int(v)) for v in c])


def e2m1_encode(x) -> np.ndarray:
    x = np.asarray(x, dtype=np.float32).ravel()
    return np.array([_L().oracle_e2m1_encode(float(v)) for v in x], dtype=np.uint8)


# ---------------------------------------------------------------- INT4
def quantize_int4(W, group_size: int, zero_point: int = 1, s=None, bits: int = 4) -> dict:
    w = as_bits16(W)
    N, K = w.shape
    ng = K // group_size
    qweight = np.zeros((N, K // 8), dtype=np.uint32)
    scales = np.zeros((N, ng), dtype=np.uint16)
    zeros = np.zeros((N, (ng + 7) // 8), dtype=np.uint32) if zero_point else None
    s32 = _f32(s)
    rc = _L().oracle_quantize_int4(_ptr(w), N, K, bits, group_size, zero_point, _ptr(s32),
                                   _ptr(qweight), _ptr(scales), _ptr(zeros))
    if rc != 0:
        raise ValueError("oracle_quantize_int4: invalid arguments")
    return dict(qweight=qweight, scales=scales, zeros=zeros, N=N, K=K, group_size=group_size,
                zero_point=zero_point)


def dequant_int4(p: dict, rows=None) -> np.ndarray:
    N, K = p["N"], p["K"]
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nr = N if r is None else len(r)
    out = np.empty((nr, K), dtype=np.float64)
    _L().oracle_dequant_int4(_ptr(np.ascontiguousarray(p["qweight"], dtype=np.uint32)),
                             _ptr(np.ascontiguousarray(p["scales"], dtype=np.uint16)),
                             _ptr(None if p["zeros"] is None else np.ascontiguousarray(p["zeros"], dtype=np.uint32)),
                             N, K, p["group_size"], p["zero_point"], _ptr(r), nr, _ptr(out))
    return out


# ---------------------------------------------------------------- NVFP4
def quantize_nvfp4(A, s=None) -> dict:
    a = as_bits16(A)
    R, C = a.shape
    codes = np.zeros((R, C // 2), dtype=np.uint8)
    bscale = np.zeros((R, C // 16), dtype=np.uint8)
    g = ctypes.c_float(0.0)
    rc = _L().oracle_quantize_nvfp4(_ptr(a), R, C, _ptr(_f32(s)), _ptr(codes), _ptr(bscale),
                                    ctypes.cast(ctypes.pointer(g), ctypes.c_void_p))
    if rc != 0:
        raise ValueError("oracle_quantize_nvfp4: invalid arguments")
    return dict(codes=codes, bscale=bscale, g=np.float32(g.value), N=R, K=C)


def dequant_nvfp4(p: dict, rows=None) -> np.ndarray:
    R, C = p["N"], p["K"]
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nr = R if r is None else len(r)
    out = np.empty((nr, C), dtype=np.float64)
    _L().oracle_dequant_nvfp4(_ptr(np.ascontiguousarray(p["codes"], dtype=np.uint8)),
                              _ptr(np.ascontiguousarray(p["bscale"], dtype=np.uint8)),
                              float(p["g"]), R, C, _ptr(r), nr, _ptr(out))
    return out


# ---------------------------------------------------------------- linear
def activations_f64(X, inv_s=None) -> np.ndarray:
    x = as_bits16(X)
    M, K = x.shape
    out = np.empty((M, K), dtype=np.float64)
    _L().oracle_activations_f64(_ptr(x), M, K, _ptr(_f32(inv_s)), _ptr(out))
    return out


def matmul_abT(A: np.ndarray, B: np.ndarray) -> np.ndarray:
    A = np.ascontiguousarray(A, dtype=np.float64)
    B = np.ascontiguousarray(B, dtype=np.float64)
    M, K = A.shape
    N, K2 = B.shape
    assert K == K2
    Y = np.empty((M, N), dtype=np.float64)
    _L().oracle_matmul_abT(_ptr(A), M, K, _ptr(B), N, _ptr(Y))
    return Y


def linear(X, W_hat: np.ndarray, inv_s=None) -> np.ndarray:
    """Y = (X * inv_s) W_hat^T in fp64; W_hat from dequant_int4 / dequant_nvfp4."""
    return matmul_abT(activations_f64(X, inv_s), W_hat)


# ---------------------------------------------------------------- AWQ
def awq_delta(W, s, group_size: int) -> np.ndarray:
    """Delta = W - dequant(Q(W s)) / s in fp64 [N, K]."""
    w = as_bits16(W)
    N, K = w.shape
    out = np.empty((N, K), dtype=np.float64)
    rc = _L().oracle_awq_delta(_ptr(w), N, K, _ptr(_f32(s)), group_size, _ptr(out))
    if rc != 0:
        raise ValueError("oracle_awq_delta: invalid arguments")
    return out


def awq_mean_abs(X) -> np.ndarray:
    """a_k = max(mean_t |X[t,k]|, 1e-4) in fp64 (the AWQ activation statistic)."""
    x = activations_f64(X)
    return np.maximum(np.abs(x).mean(axis=0), 1e-4)


def awq_search(W, group_size: int, alphas, X=None, act_mean=None):
    """Returns (s fp32 [K], losses fp64 [n_alpha], best index)."""
    w = as_bits16(W)
    N, K = w.shape
    x = None if X is None else as_bits16(X)
    T = 0 if x is None else x.shape[0]
    al = np.ascontiguousarray(alphas, dtype=np.float32)
    s = np.zeros(K, dtype=np.float32)
    losses = np.zeros(len(al), dtype=np.float64)
    best = ctypes.c_int(-1)
    rc = _L().oracle_awq_search(_ptr(w), N, K, _ptr(x), T, _ptr(_f32(act_mean)), _ptr(al), len(al),
                                group_size, _ptr(s), _ptr(losses),
                                ctypes.cast(ctypes.pointer(best), ctypes.c_void_p))
    if rc != 0:
        raise ValueError("oracle_awq_search: invalid arguments")
    return s, losses, best.value


def gptq_hessian_factor(X, damp: float = 0.01) -> np.ndarray:
    """U (fp32 [K, K], upper triangular) with U^T U = (H + lambda I)^-1, where
    H = 2 X^T X over the calibration tokens X [T, K] and lambda = damp times the
    mean of diag(H) ("quantization primer" section 6 and the ms-swift page: the
    second-order information of GPTQ comes from 128-512 calibration samples;
    the damping is a reading, the pages are silent).  fp64 throughout, numpy's
    inverse and Cholesky factorisation as library steps, rounded to fp32 once."""
    x = activations_f64(X)
    H = 2.0 * (x.T @ x)
    K = H.shape[0]
    H[np.diag_indices(K)] += damp * np.mean(np.diag(H))
    Hinv = np.linalg.inv(H)
    Hinv = 0.5 * (Hinv + Hinv.T)
    return np.ascontiguousarray(np.linalg.cholesky(Hinv).T.astype(np.float32))


def gptq_int4(W, U, group_size: int, zero_point: int = 1, want_err: bool = False) -> dict:
    """GPTQ INT4 pack of W [N, K] with the inverse-Hessian factor U (fp32 [K, K]):
    columns in order, group scale/zero from the weights as they stand at the
    group's first column, error e_k = (w_k - deq(q_k)) / U[k][k], later columns
    w_j = w_j - e_k U[k][j], fp32 with every operation rounded on its own.
    Returns the pack (and e [N, K] fp32)."""
    w = as_bits16(W)
    N, K = w.shape
    u = np.ascontiguousarray(U, dtype=np.float32)
    if u.shape != (K, K):
        raise ValueError("U must be [K, K]")
    ng = K // group_size
    out = {"qweight": np.zeros((N, K // 8), dtype=np.uint32),
           "scales": np.zeros((N, ng), dtype=np.uint16),
           "zeros": np.zeros((N, (ng + 7) // 8), dtype=np.uint32) if zero_point else None}
    err = np.zeros((N, K), dtype=np.float32) if want_err else None
    rc = _L().oracle_gptq_int4(_ptr(w), N, K, _ptr(u), group_size, zero_point, _ptr(out["qweight"]),
                               _ptr(out["scales"]), _ptr(out["zeros"]), _ptr(err))
    if rc != 0:
        raise ValueError("oracle_gptq_int4: invalid arguments")
    out.update(N=N, K=K, group_size=group_size, zero_point=zero_point)
    if want_err:
        out["err"] = err
    return out
