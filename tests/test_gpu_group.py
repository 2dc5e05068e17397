"""Grouped decode GEMV (one persistent launch for a list of independent
projections): every item's output equals the oracle's, and equals what the
single-item entry point computes within the linear tolerance."""
import numpy as np
import pytest
import torch

import w4a16_gemm_wq_b200 as wq
from w4a16_gemm_wq_b200 import synth
from tests._parity import assert_linear_close
from tests.test_gpu_gemv import _ref_int4, _ref_nvfp4

pytestmark = pytest.mark.gpu


def _pack(lib, W, fmt):
    if fmt == "nvfp4":
        return lib.wq_quantize_nvfp4(W.cuda())
    if fmt == "int4_sym":
        return lib.wq_quantize_int4(W.cuda(), 128, 0)
    return lib.wq_quantize_int4(W.cuda(), int(fmt.split("_g")[1]), 1)


def _ref(p, X, inv_s=None):
    return _ref_nvfp4(p, X, inv_s) if isinstance(p, wq.PackedNVFP4) else _ref_int4(p, X, inv_s)


def _single(lib, X, p, inv_s=None):
    if isinstance(p, wq.PackedNVFP4):
        return lib.wq_linear_nvfp4(X, p, act_inv_s=inv_s)
    return lib.wq_linear_int4(X, p, act_inv_s=inv_s)


@pytest.mark.parametrize("M", [1, 2])
def test_decode_sweep_group(lib, M):
    # the 4 block shapes x {INT4 g128, INT4 g64, NVFP4}: 12 items, one launch
    items, refs = [], []
    Xs = {K: synth.activations(M, K, seed=K + M).cuda() for K, _ in synth.DECODE_SHAPES}
    for si, (K, N) in enumerate(synth.DECODE_SHAPES):
        W = synth.weight(N, K, seed=synth.layer_seed(2, si))
        for fmt in ("int4_g128", "int4_g64", "nvfp4"):
            p = _pack(lib, W, fmt)
            Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
            items.append((Xs[K], p, Y))
    lib.wq_linear_group(items)
    torch.cuda.synchronize()
    for X, p, Y in items:
        assert_linear_close(Y, _ref(p, X.cpu()), what=f"group {type(p).__name__} {p.K}x{p.N} M={M}")
        single = _single(lib, X, p)
        assert_linear_close(Y, single.double().cpu().numpy(), what="group vs single entry point")
    assert lib.wq_device_error() == 0


def test_ragged_shapes_scales_and_symmetric(lib):
    M = 1
    shapes = [(96, 40, "nvfp4"), (1088, 200, "int4_g64"), (2048, 17, "int4_sym"), (11008, 33, "nvfp4"),
              (512, 16, "int4_g128"), (3072, 1, "int4_g64"), (2048, 96, "int4_g32")]
    items = []
    for i, (K, N, fmt) in enumerate(shapes):
        W = synth.weight(N, K, seed=100 + i)
        X = synth.activations(M, K, seed=200 + i).cuda()
        inv_s = (1.0 / synth.act_mean_lognormal(K, seed=i).sqrt()).cuda() if i % 2 else None
        p = _pack(lib, W, fmt)
        items.append((X, p, torch.empty((M, N), dtype=torch.bfloat16, device="cuda"), inv_s))
    lib.wq_linear_group(items)
    torch.cuda.synchronize()
    for X, p, Y, inv_s in items:
        ref = _ref(p, X.cpu(), None if inv_s is None else inv_s.cpu().numpy())
        assert_linear_close(Y, ref, what=f"ragged {type(p).__name__} {p.K}x{p.N}")


def test_groups_outside_the_single_launch_limits_fall_back(lib):
    # 25 items (> 24: the 25th runs alone) and M = 3 (> 2: item by item) give identical results
    K, N = 1024, 64
    W = synth.weight(N, K, seed=7)
    p = _pack(lib, W, "int4_g64")
    for M, count in ((1, 25), (3, 2)):
        X = synth.activations(M, K, seed=M).cuda()
        items = [(X, p, torch.empty((M, N), dtype=torch.bfloat16, device="cuda")) for _ in range(count)]
        lib.wq_linear_group(items)
        torch.cuda.synchronize()
        ref = _ref(p, X.cpu())
        for _, _, Y in items:
            assert_linear_close(Y, ref, what=f"fallback M={M} count={count}")
