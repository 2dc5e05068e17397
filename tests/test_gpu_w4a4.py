"""NVFP4 W4A4 parity (block-scaled FP4 tensor cores): the activation pack in
the workspace is bit-exact against the oracle's NVFP4 rule applied to X, and
Y matches the oracle's fp64 product of both dequantized operands."""
import numpy as np
import pytest
import torch

import oracle
import w4a16_gemm_wq_b200 as wq
from w4a16_gemm_wq_b200 import synth
from tests._parity import assert_linear_close

pytestmark = pytest.mark.gpu


def _wref(p):
    return oracle.dequant_nvfp4(dict(codes=p.codes.cpu().numpy(), bscale=p.bscale.cpu().numpy(),
                                     g=p.global_scale.cpu().numpy()[0], N=p.N, K=p.K))


def _run(lib, X, p, inv_s=None):
    M, K = X.shape
    nb = wq.linear_workspace_size(M, p.N, K, wq.WQ_FMT_NVFP4, 1)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    Y = lib.wq_linear_nvfp4(X.cuda(), p, act_fp4=1, act_inv_s=None if inv_s is None else torch.tensor(inv_s).cuda(),
                            ws=ws)
    torch.cuda.synchronize()
    # workspace layout: codes [M, K/2] | e4m3 scales [M, K/16] | g_x (each 256-byte aligned)
    a256 = lambda v: (v + 255) // 256 * 256
    w = ws.cpu().numpy()
    off_sf = a256(M * K // 2)
    off_g = a256(off_sf + M * K // 16)
    xq = dict(codes=w[:M * K // 2].reshape(M, K // 2), bscale=w[off_sf:off_sf + M * K // 16].reshape(M, K // 16),
              g=w[off_g:off_g + 4].view(np.float32)[0], N=M, K=K)
    return Y, xq


@pytest.mark.parametrize("M", [1, 17, 128, 200])
@pytest.mark.parametrize("K,N", [(64, 40), (320, 256), (2048, 384), (2048, 203)])
def test_w4a4_small(lib, M, K, N):
    # N = 203 (N % 8 != 0) stores Y row by row instead of by TMA boxes
    W = synth.weight(N, K, seed=K + N)
    X = synth.activations(M, K, seed=M + K, channels=synth.outlier_channels(K, 0.01, 1))
    p = lib.wq_quantize_nvfp4(W.cuda())
    Y, xq = _run(lib, X, p)
    ref = oracle.quantize_nvfp4(X)
    np.testing.assert_array_equal(xq["codes"], ref["codes"])
    np.testing.assert_array_equal(xq["bscale"], ref["bscale"])
    assert np.float32(xq["g"]) == ref["g"]
    yref = oracle.matmul_abT(oracle.dequant_nvfp4(ref), _wref(p))
    assert_linear_close(Y, yref, what=f"w4a4 M={M} {K}x{N}")


def test_w4a4_with_awq_inv_scale(lib):
    M, K, N = 96, 1024, 512
    W = synth.weight(N, K, seed=3)
    X = synth.activations(M, K, seed=4)
    inv_s = (1.0 / synth.act_mean_lognormal(K, seed=5).numpy() ** 0.5).astype(np.float32)
    p = lib.wq_quantize_nvfp4(W.cuda())
    Y, xq = _run(lib, X, p, inv_s)
    ref = oracle.quantize_nvfp4(X, s=inv_s)
    np.testing.assert_array_equal(xq["codes"], ref["codes"])
    np.testing.assert_array_equal(xq["bscale"], ref["bscale"])
    assert_linear_close(Y, oracle.matmul_abT(oracle.dequant_nvfp4(ref), _wref(p)), what="w4a4 inv_s")


@pytest.mark.parametrize("name,K,N", list(synth.PROJECTIONS)
                         + [p for p in synth.FUSED_PROJECTIONS if p[0] in ("qkv_proj", "gate_up_proj")])
@pytest.mark.parametrize("M", [512, 2048, 8192])
def test_config4_w4a4_sampled(lib, name, K, N, M):
    # every Linear of the block (both layouts) at every prefill size the benchmark times:
    # the activation pack bit-exact in full, Y on sampled rows
    W = synth.weight(N, K, seed=synth.layer_seed(4, K + N), device="cuda")
    X = synth.activations(M, K, seed=synth.layer_seed(4, M), device="cuda")
    p = lib.wq_quantize_nvfp4(W)
    Y, xq = _run(lib, X, p)
    ref = oracle.quantize_nvfp4(X.cpu())
    np.testing.assert_array_equal(xq["codes"], ref["codes"])
    np.testing.assert_array_equal(xq["bscale"], ref["bscale"])
    rows = np.array(sorted(set(range(0, M, M // 16)) | {127, 128, M - 1}))
    xr = oracle.dequant_nvfp4(ref, rows=rows)
    assert_linear_close(Y[rows], oracle.matmul_abT(xr, _wref(p)), what=f"w4a4 {name} M={M}")


def test_w4a4_rejects_bad_args(lib):
    p = lib.wq_quantize_nvfp4(synth.weight(64, 96, seed=1).cuda())
    with pytest.raises(wq.WQError):  # K % 64 != 0
        lib.wq_linear_nvfp4(synth.activations(4, 96, seed=1).cuda(), p, act_fp4=1)
    p = lib.wq_quantize_nvfp4(synth.weight(64, 128, seed=1).cuda())
    with pytest.raises(wq.WQError):  # workspace too small
        lib.wq_linear_nvfp4(synth.activations(4, 128, seed=1).cuda(), p, act_fp4=1,
                            ws=torch.zeros(16, dtype=torch.uint8, device="cuda"))
