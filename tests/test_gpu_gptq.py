"""GPTQ INT4 ("quantization primer" section 6): the pack bit-exact against the
oracle's column-by-column definition fed the same inverse-Hessian factor U,
at small sizes spanning several groups and passes of rows, ragged row counts,
both group sizes, symmetric packs, and sampled rows at the 7-projection sizes;
the packs run through the linear entry points like any INT4 pack."""
import numpy as np
import pytest
import torch

import oracle
import w4a16_gemm_wq_b200 as wq
from w4a16_gemm_wq_b200 import synth
from tests._parity import bits, assert_linear_close

pytestmark = pytest.mark.gpu


def _factor(K, seed, T=256):
    X = synth.activations_student_t(T, K, seed=seed)
    return X, oracle.gptq_hessian_factor(X)


def _check(p, ref, rows=None):
    for name in ("qweight", "scales", "zeros"):
        got = getattr(p, name)
        if ref[name] is None:
            assert got is None
            continue
        g = bits(got)
        np.testing.assert_array_equal(g if rows is None else g[rows], ref[name], err_msg=name)


@pytest.mark.parametrize("G", [32, 64, 128])
@pytest.mark.parametrize("zp", [1, 0])
@pytest.mark.parametrize("N,K", [(37, 256), (16, 1024), (100, 512)])
def test_gptq_bit_exact(lib, G, zp, N, K):
    W = synth.weight(N, K, seed=N + K, outlier_frac=0.02)
    X, U = _factor(K, seed=K)
    p = lib.wq_gptq_int4(W.cuda(), torch.tensor(U).cuda(), G, zp)
    torch.cuda.synchronize()
    _check(p, oracle.gptq_int4(W, U, G, zp))


def _synthetic_factor(K, seed):
    # an upper-triangular factor with a positive diagonal and small couplings (the
    # definition holds for any such U; a real factor at K = 11008 costs minutes of fp64)
    rng = np.random.default_rng(seed)
    U = np.triu(rng.standard_normal((K, K), dtype=np.float32) * np.float32(0.01), 1)
    U[np.diag_indices(K)] = (1.0 + rng.random(K)).astype(np.float32)
    return U


@pytest.mark.parametrize("K,N", [(2048, 2048), (11008, 64)])
def test_gptq_full_size_sampled_rows(lib, K, N):
    # the projections' K (2048: 16 rows per pass; 11008: 3 rows per pass at G = 128),
    # rows from the first, a middle and the last pass checked against the oracle
    W = synth.weight(N, K, seed=K + 1, outlier_frac=0.005)
    U = _factor(K, seed=K + 1, T=512)[1] if K <= 2048 else _synthetic_factor(K, K + 1)
    p = lib.wq_gptq_int4(W.cuda(), torch.tensor(U).cuda(), 128, 1)
    torch.cuda.synchronize()
    rows = np.array(sorted({0, 1, N // 2, N - 2, N - 1}))
    _check(p, oracle.gptq_int4(W[torch.tensor(rows)], U, 128, 1), rows)


def test_gptq_pack_runs_through_the_linears(lib):
    # a GPTQ pack is a plain INT4 pack: decode GEMV and prefill GEMM against the oracle
    K, N = 1024, 384
    W = synth.weight(N, K, seed=7, outlier_frac=0.01)
    X, U = _factor(K, seed=7)
    p = lib.wq_gptq_int4(W.cuda(), torch.tensor(U).cuda(), 64, 1)
    ref = oracle.gptq_int4(W, U, 64, 1)
    What = oracle.dequant_int4(ref)
    for M in (1, 600):
        Xa = synth.activations(M, K, seed=M)
        Y = lib.wq_linear_int4(Xa.cuda(), p)
        assert_linear_close(Y, oracle.linear(Xa, What), what=f"gptq pack M={M}")


@pytest.mark.parametrize("T,K", [(128, 256), (100, 288), (37, 1056), (512, 2048), (512, 11008)])
def test_gptq_hessian_factor_matches_oracle(lib, T, K):
    # the library's fp64 factor (Hessian, damping, reversed-order Cholesky, triangular
    # inverse) against the oracle's (numpy fp64 inverse, then Cholesky), both rounded to
    # fp32 once: K not a multiple of the 64-wide blocks (288, 1056), T not a multiple of
    # 32, fewer tokens than channels (the damping keeps H positive definite), and the
    # projections' K
    X = synth.activations_student_t(T, K, seed=T + K)
    U = lib.wq_gptq_hessian_factor(X.cuda()).cpu().numpy()
    assert lib.wq_device_error() == 0
    ref = oracle.gptq_hessian_factor(X)
    assert np.all(np.tril(U, -1) == 0) and np.all(np.diag(U) > 0)
    np.testing.assert_allclose(U, ref, rtol=1e-5, atol=1e-6 * np.abs(ref).max())


def test_gptq_pack_with_library_factor(lib):
    # the whole GPTQ path on the GPU (factor, then pack) against the oracle's pack with
    # the same factor
    K, N, T = 2048, 256, 512
    W = synth.weight(N, K, seed=21, outlier_frac=0.005)
    X = synth.activations_student_t(T, K, seed=22)
    Ud = lib.wq_gptq_hessian_factor(X.cuda())
    p = lib.wq_gptq_int4(W.cuda(), Ud, 128, 1)
    torch.cuda.synchronize()
    _check(p, oracle.gptq_int4(W, Ud.cpu().numpy(), 128, 1))


def test_gptq_hessian_factor_rejects_empty_calibration(lib):
    X = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(wq.WQError):
        lib.wq_gptq_hessian_factor(X)


def test_gptq_hessian_factor_reports_non_finite_tokens(lib):
    X = synth.activations(64, 256, seed=5)
    X[3, 17] = float("inf")
    U = lib.wq_gptq_hessian_factor(X.cuda())
    with pytest.raises(wq.WQError) as e:
        lib.wq_device_error()
    assert e.value.status == wq.WQ_ERR_ARG
    assert torch.isnan(U).any()
    assert lib.wq_device_error() == 0  # the word was cleared


def test_gptq_rejects_bad_factor_shape(lib):
    W = synth.weight(8, 256, seed=1).cuda()
    with pytest.raises(ValueError):
        lib.wq_gptq_int4(W, torch.eye(128, device="cuda"), 64, 1)
