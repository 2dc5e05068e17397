"""Decode-GEMV parity (M <= 16): the CUDA split-K GEMV against the oracle's
fp64 product of the same dequantized weights."""
import numpy as np
import pytest
import torch

import oracle
from w4a16_gemm_wq_b200 import synth
from tests._parity import assert_linear_close

pytestmark = pytest.mark.gpu


def _ref_int4(p, X, inv_s=None):
    ref = oracle.dequant_int4(dict(qweight=p.qweight.cpu().numpy().view(np.uint32),
                                   scales=p.scales.cpu().view(torch.int16).numpy().view(np.uint16),
                                   zeros=None if p.zeros is None else p.zeros.cpu().numpy().view(np.uint32),
                                   N=p.N, K=p.K, group_size=p.group_size, zero_point=p.zero_point))
    return oracle.linear(X, ref, inv_s)


def _ref_nvfp4(p, X, inv_s=None):
    ref = oracle.dequant_nvfp4(dict(codes=p.codes.cpu().numpy(), bscale=p.bscale.cpu().numpy(),
                                    g=p.global_scale.cpu().numpy()[0], N=p.N, K=p.K))
    return oracle.linear(X, ref, inv_s)


def test_config1_awq_m1_m16(lib):
    d = synth.config1(seed=0)
    xc = d["X_calib"].double().numpy()
    s = np.power(np.maximum(np.abs(xc).mean(0), 1e-4), 0.5).astype(np.float32)
    inv_s = (1.0 / s).astype(np.float32)
    p = lib.wq_quantize_int4(d["W"].cuda(), 64, 1, torch.tensor(s).cuda())
    for X in (d["X1"], d["X16"]):
        Y = lib.wq_linear_int4(X.cuda(), p, act_inv_s=torch.tensor(inv_s).cuda())
        assert_linear_close(Y, _ref_int4(p, X, inv_s), what=f"cfg1 M={X.shape[0]}")
    # the AWQ transform keeps the product close to the bf16 layer itself
    Yq = lib.wq_linear_int4(d["X16"].cuda(), p, act_inv_s=torch.tensor(inv_s).cuda()).double().cpu().numpy()
    Yf = d["X16"].double().numpy() @ d["W"].double().numpy().T
    assert np.max(np.abs(Yq - Yf)) / np.max(np.abs(Yf)) < 0.05


@pytest.mark.parametrize("K,N", synth.DECODE_SHAPES)
@pytest.mark.parametrize("fmt", ["int4_g128", "int4_g64", "int4_g32", "nvfp4"])
def test_config2_decode_m1(lib, K, N, fmt):
    W = synth.weight(N, K, seed=synth.layer_seed(2, K + N))
    X = synth.activations(1, K, seed=synth.layer_seed(2, K))
    if fmt == "nvfp4":
        p = lib.wq_quantize_nvfp4(W.cuda())
        Y = lib.wq_linear_nvfp4(X.cuda(), p)
        ref = _ref_nvfp4(p, X)
    else:
        p = lib.wq_quantize_int4(W.cuda(), int(fmt[-3:].lstrip("g")), 1)
        Y = lib.wq_linear_int4(X.cuda(), p)
        ref = _ref_int4(p, X)
    assert_linear_close(Y, ref, what=f"{fmt} {K}x{N}")


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 13, 16])
def test_m_sweep_and_symmetric(lib, M):
    K, N = 2048, 200  # ragged N
    W = synth.weight(N, K, seed=40 + M)
    X = synth.activations(M, K, seed=40 + M)
    p = lib.wq_quantize_int4(W.cuda(), 128, 0)
    assert_linear_close(lib.wq_linear_int4(X.cuda(), p), _ref_int4(p, X), what=f"sym M={M}")
    p = lib.wq_quantize_nvfp4(W.cuda())
    assert_linear_close(lib.wq_linear_nvfp4(X.cuda(), p), _ref_nvfp4(p, X), what=f"nvfp4 M={M}")


@pytest.mark.parametrize("K,N", [(96, 8), (11008, 37), (3072, 1), (1024, 4096)])
def test_ragged_shapes_split_k(lib, K, N):
    W = synth.weight(N, K, seed=K + N)
    X = synth.activations(3, K, seed=K)
    inv_s = synth.act_mean_lognormal(K, seed=K).numpy().astype(np.float32)
    p = lib.wq_quantize_nvfp4(W.cuda())
    Y = lib.wq_linear_nvfp4(X.cuda(), p, act_inv_s=torch.tensor(inv_s).cuda())
    assert_linear_close(Y, _ref_nvfp4(p, X, inv_s), what=f"nvfp4 {K}x{N}")
    if K % 64 == 0:
        p = lib.wq_quantize_int4(W.cuda(), 64, 1)
        Y = lib.wq_linear_int4(X.cuda(), p, act_inv_s=torch.tensor(inv_s).cuda())
        assert_linear_close(Y, _ref_int4(p, X, inv_s), what=f"int4 {K}x{N}")


def test_no_device_error_reported(lib):
    assert lib.wq_device_error() == 0


@pytest.mark.parametrize("M", [3, 8, 9, 16])
@pytest.mark.parametrize("K,N", [(128, 24), (2048, 2048), (2048, 300), (11008, 2048), (24576, 40)])
@pytest.mark.parametrize("fmt", ["int4_g32", "int4_g64", "int4_g128_sym", "nvfp4"])
def test_tensor_core_gemv_m3_to_16(lib, M, K, N, fmt):
    # 3 <= M <= 16 with K % 128 == 0: the weights are read once and multiplied on
    # the tensor cores (one or two n8 tiles of activation rows), split-K slices
    # reduced through the cluster; ragged N, the projections' K, the longest K the
    # split serves, and an act_inv_s on half the cases
    W = synth.weight(N, K, seed=K + N + M, device="cuda")
    X = synth.activations(M, K, seed=M + K, device="cuda")
    inv_s = synth.act_mean_lognormal(K, seed=K).numpy().astype(np.float32) if (M + K) % 2 else None
    s = None if inv_s is None else torch.tensor(inv_s).cuda()
    if fmt == "nvfp4":
        p = lib.wq_quantize_nvfp4(W)
        Y = lib.wq_linear_nvfp4(X, p, act_inv_s=s)
        ref = _ref_nvfp4(p, X.cpu(), inv_s)
    else:
        G = {"int4_g32": 32, "int4_g64": 64}.get(fmt, 128)
        p = lib.wq_quantize_int4(W, G, 0 if fmt.endswith("sym") else 1)
        Y = lib.wq_linear_int4(X, p, act_inv_s=s)
        ref = _ref_int4(p, X.cpu(), inv_s)
    assert_linear_close(Y, ref, what=f"{fmt} M={M} {K}x{N}")
