"""Prefill GEMM parity (M > 16, tcgen05 tensor cores): outputs against the
oracle's fp64 product of the same dequantized weights, on all rows for small
problems and on sampled rows (every tile row band plus the ragged tail) at
the full transformer-block shapes."""
import numpy as np
import pytest
import torch

import oracle
from w4a16_gemm_wq_b200 import synth
from tests._parity import assert_linear_close
from tests.test_gpu_gemv import _ref_int4, _ref_nvfp4

pytestmark = pytest.mark.gpu


def _deq(p):
    if hasattr(p, "qweight"):
        return oracle.dequant_int4(dict(qweight=p.qweight.cpu().numpy().view(np.uint32),
                                        scales=p.scales.cpu().view(torch.int16).numpy().view(np.uint16),
                                        zeros=None if p.zeros is None else p.zeros.cpu().numpy().view(np.uint32),
                                        N=p.N, K=p.K, group_size=p.group_size, zero_point=p.zero_point))
    return oracle.dequant_nvfp4(dict(codes=p.codes.cpu().numpy(), bscale=p.bscale.cpu().numpy(),
                                     g=p.global_scale.cpu().numpy()[0], N=p.N, K=p.K))


@pytest.mark.parametrize("M", [17, 64, 128, 129, 200, 512])
@pytest.mark.parametrize("fmt", ["int4_g64", "int4_g128", "int4_g32", "int4_sym", "nvfp4"])
def test_small_gemm_all_rows(lib, M, fmt):
    K, N = 512, 384  # 3 N-tiles of 128, ragged M tiles
    W = synth.weight(N, K, seed=M)
    X = synth.activations(M, K, seed=M + 1)
    if fmt == "nvfp4":
        p = lib.wq_quantize_nvfp4(W.cuda())
        Y = lib.wq_linear_nvfp4(X.cuda(), p)
        ref = _ref_nvfp4(p, X)
    else:
        G = {"int4_g128": 128, "int4_g32": 32}.get(fmt, 64)
        p = lib.wq_quantize_int4(W.cuda(), G, 0 if fmt == "int4_sym" else 1)
        Y = lib.wq_linear_int4(X.cuda(), p)
        ref = _ref_int4(p, X)
    assert_linear_close(Y, ref, what=f"{fmt} M={M}")


@pytest.mark.parametrize("K,N", [(96, 40), (1056, 200), (2048, 520), (2048, 203)])
def test_ragged_k_and_n(lib, K, N):
    # N % 8 != 0 (203) stores Y row by row instead of by TMA boxes
    M = 160
    W = synth.weight(N, K, seed=K)
    X = synth.activations(M, K, seed=N)
    inv_s = synth.act_mean_lognormal(K, seed=K).numpy().astype(np.float32)
    p = lib.wq_quantize_nvfp4(W.cuda())
    Y = lib.wq_linear_nvfp4(X.cuda(), p, act_inv_s=torch.tensor(inv_s).cuda())
    assert_linear_close(Y, _ref_nvfp4(p, X, inv_s), what=f"nvfp4 {K}x{N}")
    if K % 64 == 0:
        p = lib.wq_quantize_int4(W.cuda(), 64, 1)
        Y = lib.wq_linear_int4(X.cuda(), p, act_inv_s=torch.tensor(inv_s).cuda())
        assert_linear_close(Y, _ref_int4(p, X, inv_s), what=f"int4 {K}x{N}")


@pytest.mark.parametrize("K", [96, 1056])
@pytest.mark.parametrize("zp", [1, 0])
def test_int4_g32_odd_group_count(lib, K, zp):
    # G = 32 with an odd number of groups (K % 64 == 32): the dequantizer's last
    # 64-wide k-block holds one real group, its upper half lies past K
    M, N = 160, 200
    W = synth.weight(N, K, seed=K + zp)
    X = synth.activations(M, K, seed=K + 1)
    inv_s = synth.act_mean_lognormal(K, seed=K).numpy().astype(np.float32)
    p = lib.wq_quantize_int4(W.cuda(), 32, zp)
    Y = lib.wq_linear_int4(X.cuda(), p, act_inv_s=torch.tensor(inv_s).cuda())
    assert_linear_close(Y, _ref_int4(p, X, inv_s), what=f"int4 g32 zp={zp} K={K}")


def _sampled_rows(M, n=24):
    rows = set(range(0, M, max(1, M // n)))
    rows.update({0, 127, 128, M - 1})
    return np.array(sorted(r for r in rows if r < M))


# the 7 projections, and the stacked q/k/v and gate/up Linears of the fused block layout
_BLOCK_SHAPES = list(synth.PROJECTIONS) + [p for p in synth.FUSED_PROJECTIONS if p[0] in ("qkv_proj", "gate_up_proj")]


@pytest.mark.parametrize("name,K,N", _BLOCK_SHAPES)
@pytest.mark.parametrize("M", [512, 2048, 8192])
@pytest.mark.parametrize("fmt", ["int4_g64", "nvfp4"])
def test_config4_block_projection_sampled(lib, name, K, N, M, fmt):
    # every Linear of the block (both layouts) at every prefill size the benchmark times,
    # in the benchmark's launch configuration (no workspace), on sampled rows (every row
    # band of the tiles plus the ragged tail)
    W = synth.weight(N, K, seed=synth.layer_seed(4, K + N), device="cuda")
    X = synth.activations(M, K, seed=synth.layer_seed(4, M), device="cuda")
    if fmt == "nvfp4":
        p = lib.wq_quantize_nvfp4(W)
        Y = lib.wq_linear_nvfp4(X, p)
    else:
        p = lib.wq_quantize_int4(W, 64, 1)
        Y = lib.wq_linear_int4(X, p)
    rows = _sampled_rows(M)
    ref = oracle.linear(X[rows].cpu(), _deq(p))
    assert lib.wq_device_error() == 0
    assert_linear_close(Y[rows], ref, what=f"{fmt} {name} M={M}")


@pytest.mark.parametrize("M,N", [(2300, 4200), (2300, 4100), (2300, 2100)])
@pytest.mark.parametrize("fmt", ["int4_g64", "int4_g128", "int4_sym", "nvfp4"])
def test_two_accumulator_tiles_ragged(lib, M, N, fmt):
    # enough tiles for 256-row CTAs (two tensor-memory accumulators sharing each
    # dequantized W tile): W tiles of 256 (4200, 4100: vector and scalar stores)
    # and of 128 (2100); M = 2300 leaves a ragged last row band
    K = 1024
    W = synth.weight(N, K, seed=M + N, device="cuda")
    X = synth.activations(M, K, seed=N, device="cuda")
    inv_s = (1.0 / synth.act_mean_lognormal(K, seed=5).sqrt()).cuda() if fmt == "int4_g128" else None
    if fmt == "nvfp4":
        p = lib.wq_quantize_nvfp4(W)
        Y = lib.wq_linear_nvfp4(X, p)
    else:
        p = lib.wq_quantize_int4(W, 128 if fmt == "int4_g128" else 64, 0 if fmt == "int4_sym" else 1)
        Y = lib.wq_linear_int4(X, p, act_inv_s=inv_s)
    # the second accumulator of the first tile, a full band around 2048 and the tail
    rows = np.array(sorted(set(range(120, 264, 3)) | set(range(2040, 2300, 7)) | {M - 1}))
    ref = oracle.linear(X[rows].cpu(), _deq(p), None if inv_s is None else inv_s.cpu().numpy())
    assert_linear_close(Y[rows], ref, what=f"{fmt} M={M} N={N}")


@pytest.mark.parametrize("fmt", ["int4", "nvfp4"])
@pytest.mark.parametrize("M,N,K", [(512, 256, 11008), (2048, 256, 4096), (512, 2048, 11008), (300, 200, 3072),
                                   (512, 203, 11008)])
def test_split_k_few_tiles(lib, fmt, M, N, K):
    # few output tiles: K split over several CTAs per tile through the workspace
    # (fp32 partial tiles by TMA, then the reduction launch sums them in split
    # order): sampled rows against the oracle, bit-identical on a second run with the
    # same (garbage-filled) workspace, and close to the unsplit run; N = 203 takes the
    # reduction's element-wise Y stores
    W = synth.weight(N, K, seed=M + N + K, device="cuda")
    X = synth.activations(M, K, seed=K, device="cuda")
    p = lib.wq_quantize_int4(W, 64, 1) if fmt == "int4" else lib.wq_quantize_nvfp4(W)
    call = lib.wq_linear_int4 if fmt == "int4" else lib.wq_linear_nvfp4
    fmt_id = lib.WQ_FMT_INT4 if fmt == "int4" else lib.WQ_FMT_NVFP4
    need = lib.linear_workspace_size(M, N, K, fmt_id)
    assert need > 0, "these shapes take the split"
    ws = torch.full((need,), 0xAB, dtype=torch.uint8, device="cuda")
    y1 = call(X, p, ws=ws).clone()
    y2 = call(X, p, ws=ws).clone()
    y0 = call(X, p, ws=torch.empty(16, dtype=torch.uint8, device="cuda"))  # too small: unsplit
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16)), "split sums must not depend on timing"
    rows = _sampled_rows(M)
    ref = oracle.linear(X[rows].cpu(), _deq(p))
    assert_linear_close(y1[rows], ref, what=f"split-K {fmt} {M}x{N}x{K}")
    assert_linear_close(y0[rows], ref, what=f"unsplit {fmt} {M}x{N}x{K}")
    assert lib.wq_device_error() == 0
