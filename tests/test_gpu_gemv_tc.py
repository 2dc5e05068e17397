"""Tensor-core decode GEMV (M <= 2, row blocks balanced over the SMs, split over
the warps of a CTA): parity against the oracle on shapes chosen to exercise
every way a 16-row block can be split over warps (whole in one warp, split over
several, a CTA with fewer steps than warps, ragged N), and repeatability (the
split sums are taken in a fixed order)."""
import numpy as np
import pytest
import torch

import w4a16_gemm_wq_b200 as wq
from w4a16_gemm_wq_b200 import synth
from tests._parity import assert_linear_close
from tests.test_gpu_gemv import _ref_int4, _ref_nvfp4

pytestmark = pytest.mark.gpu

FORMATS = ["int4_g64", "int4_g128", "int4_sym", "nvfp4"]
# (K, N): long K / few rows (every row block split across CTAs), one step per
# row block, more warps than steps, ragged N, the block shapes
SHAPES = [(11008, 40), (128, 4000), (256, 17), (2048, 2048), (1024, 2304), (11008, 2048)]


def _pack(lib, W, fmt):
    if fmt == "nvfp4":
        return lib.wq_quantize_nvfp4(W.cuda())
    if fmt == "int4_sym":
        return lib.wq_quantize_int4(W.cuda(), 128, 0)
    return lib.wq_quantize_int4(W.cuda(), int(fmt.split("_g")[1]), 1)


def _run(lib, X, p, inv_s=None):
    # a one-item group: the tensor-core decode GEMV (single calls take the CUDA-core kernel)
    Y = torch.empty((X.shape[0], p.N), dtype=torch.bfloat16, device="cuda")
    lib.wq_linear_group([(X, p, Y) if inv_s is None else (X, p, Y, inv_s)])
    return Y


def _ref(p, X, inv_s=None):
    return _ref_nvfp4(p, X, inv_s) if isinstance(p, wq.PackedNVFP4) else _ref_int4(p, X, inv_s)


@pytest.mark.parametrize("K,N", SHAPES)
@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("M", [1, 2])
def test_stream_k_parity(lib, K, N, fmt, M):
    W = synth.weight(N, K, seed=K * 7 + N)
    X = synth.activations(M, K, seed=K + N + M)
    p = _pack(lib, W, fmt)
    inv_s = (1.0 / synth.act_mean_lognormal(K, seed=K).sqrt()) if N % 2 else None
    Y = _run(lib, X.cuda(), p, None if inv_s is None else inv_s.cuda())
    ref = _ref(p, X, None if inv_s is None else inv_s.numpy())
    assert_linear_close(Y, ref, what=f"{fmt} M={M} {K}x{N}")


@pytest.mark.parametrize("fmt", FORMATS)
def test_repeatable(lib, fmt):
    # the split row blocks are summed in warp order: the same bits every call
    M, K, N = 1, 11008, 72
    W = synth.weight(N, K, seed=3)
    X = synth.activations(M, K, seed=4).cuda()
    p = _pack(lib, W, fmt)
    first = _run(lib, X, p).clone()
    for _ in range(3):
        again = _run(lib, X, p)
        assert torch.equal(first.view(torch.int16), again.view(torch.int16)), "split sums must not depend on timing"


def test_alternating_m(lib):
    # M = 2 and M = 1 launches back to back on one stream
    K, N = 11008, 96
    p = _pack(lib, synth.weight(N, K, seed=11), "int4_g128")
    for M in (2, 1, 2, 1):
        X = synth.activations(M, K, seed=20 + M)
        assert_linear_close(_run(lib, X.cuda(), p), _ref(p, X), what=f"alternating M={M}")
