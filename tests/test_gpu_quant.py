"""Stage-1 parity: packed INT4 / NVFP4 bytes from the CUDA kernels equal the
oracle's bit for bit (same fp32 decisions, round-half-to-even)."""
import numpy as np
import pytest
import torch

import oracle
from w4a16_gemm_wq_b200 import synth
from tests._parity import bits

pytestmark = pytest.mark.gpu


def _check_int4(lib, W, G, zp=1, s=None):
    Wd = W.cuda()
    sd = None if s is None else torch.as_tensor(s, dtype=torch.float32).cuda()
    p = lib.wq_quantize_int4(Wd, G, zp, sd)
    torch.cuda.synchronize()
    ref = oracle.quantize_int4(W, G, zero_point=zp, s=s)
    np.testing.assert_array_equal(bits(p.qweight), ref["qweight"])
    np.testing.assert_array_equal(bits(p.scales), ref["scales"])
    if zp:
        np.testing.assert_array_equal(bits(p.zeros), ref["zeros"])
    else:
        assert p.zeros is None
    return p


def _check_nvfp4(lib, W, s=None):
    sd = None if s is None else torch.as_tensor(s, dtype=torch.float32).cuda()
    p = lib.wq_quantize_nvfp4(W.cuda(), sd)
    torch.cuda.synchronize()
    ref = oracle.quantize_nvfp4(W, s=s)
    np.testing.assert_array_equal(bits(p.codes), ref["codes"])
    np.testing.assert_array_equal(bits(p.bscale), ref["bscale"])
    assert bits(p.global_scale)[0] == np.float32(ref["g"]).view(np.uint32)
    return p


def test_config1_awq_int4_g64(lib):
    d = synth.config1(seed=0)
    xc = d["X_calib"].double().numpy()
    s = np.power(np.maximum(np.abs(xc).mean(0), 1e-4), 0.5).astype(np.float32)
    _check_int4(lib, d["W"], 64, 1, s)
    _check_int4(lib, d["W"], 64, 1, None)


@pytest.mark.parametrize("K,N", synth.DECODE_SHAPES)
@pytest.mark.parametrize("G", [128, 64, 32])
def test_config2_int4_shapes(lib, K, N, G):
    W = synth.weight(N, K, seed=synth.layer_seed(2, K + N))
    _check_int4(lib, W, G)


@pytest.mark.parametrize("K,N", synth.DECODE_SHAPES)
def test_config2_nvfp4_shapes(lib, K, N):
    W = synth.weight(N, K, seed=synth.layer_seed(2, K + N))
    _check_nvfp4(lib, W)


def test_symmetric_int4_and_awq_scaled_nvfp4(lib):
    W = synth.weight(96, 1024, seed=5)
    _check_int4(lib, W, 128, zp=0)
    _check_int4(lib, W, 64, zp=0)
    s = synth.act_mean_lognormal(1024, seed=5).numpy() ** 0.5
    _check_nvfp4(lib, W, s=s.astype(np.float32))


def test_int4_exact_ties_and_degenerate_groups(lib):
    G, K = 64, 256
    rows = []
    # group range [0, 15/16] -> scale 1/16 exactly, zero 0; values on half steps tie
    ties = np.arange(G, dtype=np.float32) % 31 / 32.0
    ties[0], ties[1] = 0.0, 15 / 16
    rows.append(np.tile(ties, K // G))
    rows.append(np.full(K, 0.3, dtype=np.float32))       # degenerate: max == min
    rows.append(np.zeros(K, dtype=np.float32))           # all zero
    neg = -np.tile(ties, K // G)
    rows.append(neg)                                     # zero point 15 side
    W = torch.tensor(np.stack(rows)).to(torch.bfloat16)
    _check_int4(lib, W, G)
    _check_int4(lib, W, G, zp=0)


def test_nvfp4_exact_ties_zero_blocks_and_spikes(lib):
    # g = 10.5 / 2688 = 2^-8; block 0 scale 448 -> step 1.75, block 1 scale 1 -> step 2^-8
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0])
    b0 = np.concatenate([mids * 1.75, -mids * 1.75])
    b0[7] = 10.5 / 1.75 * 1.75 if False else 10.5
    b1 = np.concatenate([mids, -mids]) * 2.0 ** -8
    b2 = np.zeros(16)
    b3 = np.zeros(16)
    b3[3] = -1e-3  # tiny spike: tiny block scale
    row = np.concatenate([b0, b1, b2, b3]).astype(np.float32)
    W = torch.tensor(np.stack([row, -row, np.zeros_like(row)])).to(torch.bfloat16)
    _check_nvfp4(lib, W)
    _check_nvfp4(lib, torch.zeros(4, 64, dtype=torch.bfloat16))


def test_ragged_row_counts_and_long_k(lib):
    # N not a multiple of anything, K = 11008 with g128 -> 86 groups (zero word padding)
    W = synth.weight(37, 11008, seed=7)
    _check_int4(lib, W, 128)
    _check_int4(lib, W, 64)
    _check_nvfp4(lib, W)
    W = synth.weight(3, 32 * 3, seed=8)  # K = 96: only with G... K % 64 != 0 -> nvfp4 only
    _check_nvfp4(lib, W)


def test_nvfp4_tiny_tensor_without_finite_reciprocal(lib):
    # a tensor with amax ~2e-36: g and many block denominators e4m3(sb) * g fall
    # below 2^-128, where 1 / denominator overflows fp32; the codes must still be
    # those of the IEEE quotients w / denominator
    W = synth.weight(8, 256, seed=9).float()
    mag = (10.0 ** -np.repeat(np.arange(16) % 4, 16)).astype(np.float32)
    Wt = (W * torch.tensor(mag)[None, :] * 3e-35).to(torch.bfloat16)
    ref = oracle.quantize_nvfp4(Wt)
    denom = oracle.e4m3_decode(ref["bscale"]).astype(np.float32) * np.float32(ref["g"])
    assert np.any((denom > 0) & (denom < np.float32(2.0 ** -128)))
    _check_nvfp4(lib, Wt)
