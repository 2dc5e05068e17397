"""The no-allocation W4A4 entry point.

Some callers cannot allocate device memory at the moment they call the
library -- a runtime that plans every device buffer up front, or code
running where no allocator is reachable -- so they cannot pass a workspace.
wq_linear_nvfp4_w4a4_noalloc keeps the activation pack in a fixed scratch
array inside the library instead.  This file checks it through the C ABI,
twice in a row (the array keeps the previous call's bytes): its output must
be bit-identical to the workspace-taking entry point (wq_linear_nvfp4 with
act_fp4 = 1 runs the same kernels on the same bytes), and both must match the
oracle's fp64 product of the NVFP4-quantized activations and weights.  It
also checks that problems larger than the array are refused.  It is named so
that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import w4a16_gemm_wq_b200 as wq
from w4a16_gemm_wq_b200 import synth
from tests._parity import assert_linear_close, bits

pytestmark = pytest.mark.gpu


def _noalloc(lib, X, p, Y, inv_s=None):
    P = ctypes.c_void_p
    rc = lib.wq_linear_nvfp4_w4a4_noalloc(P(X.data_ptr()), X.shape[0], p.N, p.K, P(p.codes.data_ptr()),
                                          P(p.bscale.data_ptr()), P(p.global_scale.data_ptr()),
                                          None if inv_s is None else P(inv_s.data_ptr()), P(Y.data_ptr()),
                                          P(torch.cuda.current_stream().cuda_stream))
    return rc


def _oracle_w4a4(X, inv_s, p):
    xq = oracle.quantize_nvfp4(X.cpu(), s=None if inv_s is None else inv_s.cpu().numpy())
    wh = oracle.dequant_nvfp4(dict(codes=p.codes.cpu().numpy(), bscale=p.bscale.cpu().numpy(),
                                   g=p.global_scale.cpu().numpy()[0], N=p.N, K=p.K))
    return oracle.matmul_abT(oracle.dequant_nvfp4(xq), wh)


def test_noalloc_matches_workspace_entry_point_twice():
    lib = wq.load()
    cases = [(200, 2048, 384, 11), (64, 1024, 256, 12)]  # second call differs in shape and values
    for M, K, N, seed in cases:
        W = synth.weight(N, K, seed=seed).cuda()
        X = synth.activations(M, K, seed=seed + 1).cuda()
        inv_s = (1.0 / synth.act_mean_lognormal(K, seed=seed).sqrt()).cuda()
        p = wq.wq_quantize_nvfp4(W)
        ref = wq.wq_linear_nvfp4(X, p, act_fp4=1, act_inv_s=inv_s)
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _noalloc(lib, X, p, Y, inv_s) == wq.WQ_OK, lib.wq_last_error().decode()
        torch.cuda.synchronize()
        np.testing.assert_array_equal(bits(Y), bits(ref), err_msg=f"noalloc M={M} K={K} N={N}")
        assert_linear_close(Y, _oracle_w4a4(X, inv_s, p), what=f"noalloc vs oracle M={M} K={K} N={N}")
    assert wq.wq_device_error() == 0


def test_noalloc_rejects_problems_beyond_its_scratch():
    lib = wq.load()
    M, K, N = 8192, 2048, 128  # pack of X needs ~9.4 MB > 8 MiB
    p = wq.wq_quantize_nvfp4(synth.weight(N, K, seed=3).cuda())
    X = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    assert _noalloc(lib, X, p, Y) == wq.WQ_ERR_ARG
    assert "scratch" in lib.wq_last_error().decode()
