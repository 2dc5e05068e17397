"""AWQ grid-search parity: losses, chosen alpha and scale against the oracle,
and the packed weights of the chosen scale bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from w4a16_gemm_wq_b200 import synth
from tests._parity import bits

pytestmark = pytest.mark.gpu

ALPHAS = np.array(synth.ALPHA_GRID, dtype=np.float32)
LOSS_RTOL = 1e-3  # Delta carried as bf16 hi+lo (~16 bits), fp32 MMA accumulation


def _run(lib, W, G, X=None, act_mean=None, alphas=ALPHAS):
    s, losses, best = lib.awq_search_scale(W.cuda(), torch.tensor(alphas).cuda(), G,
                                           X=None if X is None else X.cuda(),
                                           act_mean=None if act_mean is None else torch.tensor(act_mean).cuda())
    torch.cuda.synchronize()
    return s.cpu().numpy(), losses.cpu().numpy().astype(np.float64), int(best.cpu()[0])


def _check_choice(losses_ref, best_gpu, best_ref):
    # equal, or a near-tie: the oracle's loss at the GPU's choice is within the loss tolerance of its minimum
    assert best_gpu == best_ref or losses_ref[best_gpu] <= losses_ref[best_ref] * (1 + LOSS_RTOL), \
        (best_gpu, best_ref, losses_ref[best_gpu], losses_ref[best_ref])


def _ulps(a, b):
    return np.max(np.abs(a.view(np.int32).astype(np.int64) - b.view(np.int32).astype(np.int64)))


@pytest.mark.parametrize("G", [32, 64, 128])
@pytest.mark.parametrize("N,K,T", [(48, 256, 64), (200, 1024, 130), (256, 512, 512)])
def test_search_with_tokens_small(lib, G, N, K, T):
    W = synth.weight(N, K, seed=N + K, outlier_frac=0.02)
    X = synth.activations_student_t(T, K, seed=T)
    s, losses, best = _run(lib, W, G, X=X)
    s_ref, losses_ref, best_ref = oracle.awq_search(W, G, ALPHAS, X=X)
    np.testing.assert_allclose(losses, losses_ref, rtol=LOSS_RTOL)
    assert best == int(np.argmin(losses))
    _check_choice(losses_ref, best, best_ref)
    a = oracle.awq_mean_abs(X)
    s_at_best = np.power(a, float(ALPHAS[best])).astype(np.float32)
    assert _ulps(s, s_at_best) <= 4
    # the pack with the GPU's s is bit-exact against the oracle's quantizer fed the same s
    p = lib.wq_quantize_int4(W.cuda(), G, 1, torch.tensor(s).cuda())
    torch.cuda.synchronize()
    ref = oracle.quantize_int4(W, G, s=s)
    np.testing.assert_array_equal(bits(p.qweight), ref["qweight"])
    np.testing.assert_array_equal(bits(p.scales), ref["scales"])
    np.testing.assert_array_equal(bits(p.zeros), ref["zeros"])


def test_search_diagonal_proxy(lib):
    N, K, G = 96, 2048, 64
    W = synth.weight(N, K, seed=5)
    am = synth.act_mean_lognormal(K, seed=5).numpy()
    s, losses, best = _run(lib, W, G, act_mean=am)
    s_ref, losses_ref, best_ref = oracle.awq_search(W, G, ALPHAS, act_mean=am)
    np.testing.assert_allclose(losses, losses_ref, rtol=1e-5)
    _check_choice(losses_ref, best, best_ref)
    assert _ulps(s, s_ref) <= 4 if best == best_ref else True


def test_alpha_zero_is_plain_rtn(lib):
    N, K, G, T = 64, 512, 64, 32
    W = synth.weight(N, K, seed=6)
    X = synth.activations_student_t(T, K, seed=6)
    s, losses, best = _run(lib, W, G, X=X, alphas=np.array([0.0], dtype=np.float32))
    assert best == 0 and np.all(s == 1.0)
    delta = W.double().numpy() - oracle.dequant_int4(oracle.quantize_int4(W, G))
    y = X.double().numpy() @ delta.T
    np.testing.assert_allclose(losses[0], np.sum(y * y), rtol=LOSS_RTOL)


def test_config1_awq_alpha(lib):
    d = synth.config1(seed=0)
    s, losses, best = _run(lib, d["W"], 64, X=d["X_calib"])
    s_ref, losses_ref, best_ref = oracle.awq_search(d["W"], 64, ALPHAS, X=d["X_calib"])
    np.testing.assert_allclose(losses, losses_ref, rtol=LOSS_RTOL)
    _check_choice(losses_ref, best, best_ref)


@pytest.mark.parametrize("name,K,N", synth.PROJECTIONS)
def test_config3_full_shapes_two_alphas(lib, name, K, N):
    # full size (T = 512 calibration tokens): the GPU searches all 20 alphas; the
    # oracle's literal loss ||X Delta^T||^2 (Delta from the oracle, product in
    # fp64) is evaluated at alpha = 0 and at the GPU's choice.
    T = 512
    W = synth.weight(N, K, seed=synth.layer_seed(3, K + N))
    X = synth.activations_student_t(T, K, seed=synth.layer_seed(3, K))
    s, losses, best = _run(lib, W, 64, X=X)
    assert np.all(np.isfinite(losses)) and np.all(losses > 0)
    assert best == int(np.argmin(losses))
    a = oracle.awq_mean_abs(X)
    x = X.double().numpy()
    for i in sorted({0, best}):
        si = np.power(a, float(ALPHAS[i])).astype(np.float32)
        d = oracle.awq_delta(W, si, 64)
        y = x @ d.T
        ref = float(np.sum(y * y))
        assert abs(losses[i] - ref) <= LOSS_RTOL * ref, (i, losses[i], ref)
    assert _ulps(s, np.power(a, float(ALPHAS[best])).astype(np.float32)) <= 4


@pytest.mark.slow
@pytest.mark.parametrize("name,K,N", [p for p in synth.PROJECTIONS if p[0] in ("q_proj", "down_proj")])
def test_config3_full_size_search_against_oracle(lib, name, K, N):
    # the whole config-3 search at full size (T = 512 Student-t tokens, 20 alphas, G = 64)
    # on the oracle too (fp64 literal losses ||X Delta^T||^2): all 20 losses, the choice
    # (equal or a near tie), s, and the pack with the chosen s bit-exact.  Minutes of
    # fp64 on the host for down_proj.
    T = 512
    W = synth.weight(N, K, seed=synth.layer_seed(3, K + N))
    X = synth.activations_student_t(T, K, seed=synth.layer_seed(3, K))
    s, losses, best = _run(lib, W, 64, X=X)
    s_ref, losses_ref, best_ref = oracle.awq_search(W, 64, ALPHAS, X=X)
    np.testing.assert_allclose(losses, losses_ref, rtol=LOSS_RTOL)
    _check_choice(losses_ref, best, best_ref)
    a = oracle.awq_mean_abs(X)
    assert _ulps(s, np.power(a, float(ALPHAS[best])).astype(np.float32)) <= 4
    p = lib.wq_quantize_int4(W.cuda(), 64, 1, torch.tensor(s).cuda())
    torch.cuda.synchronize()
    ref = oracle.quantize_int4(W, 64, s=s)
    for key in ("qweight", "scales", "zeros"):
        np.testing.assert_array_equal(bits(getattr(p, key)), ref[key])


@pytest.mark.parametrize("G", [64, 128])
@pytest.mark.parametrize("proxy", [False, True])
def test_shared_scale_qkv_like(lib, G, proxy):
    # one s for three matrices that consume one input (q/k/v-like row counts, one of
    # them ragged): losses, choice and s against the oracle's search over the stacked
    # rows; each matrix's pack with that s bit-exact; the stacked pack is the stack of packs
    K, T = 512, 96
    Ns = (80, 24, 17)
    Ws = [synth.weight(n, K, seed=50 + i, outlier_frac=0.02) for i, n in enumerate(Ns)]
    X = None if proxy else synth.activations_student_t(T, K, seed=50)
    am = synth.act_mean_lognormal(K, seed=50).numpy() if proxy else None
    s, losses, best = lib.awq_search_scale_shared(
        [W.cuda() for W in Ws], torch.tensor(ALPHAS).cuda(), G, X=None if X is None else X.cuda(),
        act_mean=None if am is None else torch.tensor(am).cuda())
    torch.cuda.synchronize()
    s, losses, best = s.cpu().numpy(), losses.cpu().numpy().astype(np.float64), int(best.cpu()[0])
    s_ref, losses_ref, best_ref = oracle.awq_search(torch.cat(Ws), G, ALPHAS, X=X, act_mean=am)
    np.testing.assert_allclose(losses, losses_ref, rtol=LOSS_RTOL)
    assert best == int(np.argmin(losses))
    _check_choice(losses_ref, best, best_ref)
    a = oracle.awq_mean_abs(X) if X is not None else np.maximum(am.astype(np.float64), 1e-4)
    assert _ulps(s, np.power(a, float(ALPHAS[best])).astype(np.float32)) <= 4
    st = torch.tensor(s).cuda()
    stacked = lib.wq_quantize_int4(torch.cat(Ws).cuda(), G, 1, st)
    packs = [lib.wq_quantize_int4(W.cuda(), G, 1, st) for W in Ws]
    torch.cuda.synchronize()
    for W, p in zip(Ws, packs):
        ref = oracle.quantize_int4(W, G, s=s)
        np.testing.assert_array_equal(bits(p.qweight), ref["qweight"])
        np.testing.assert_array_equal(bits(p.scales), ref["scales"])
        np.testing.assert_array_equal(bits(p.zeros), ref["zeros"])
    for name in ("qweight", "scales", "zeros"):
        np.testing.assert_array_equal(bits(getattr(stacked, name)),
                                      np.concatenate([bits(getattr(p, name)) for p in packs]))


def test_shared_scale_rejects_mismatched_k(lib):
    Ws = [synth.weight(16, 256, seed=1).cuda(), synth.weight(16, 512, seed=2).cuda()]
    with pytest.raises(ValueError):
        lib.awq_search_scale_shared(Ws, torch.tensor(ALPHAS).cuda(), 64, act_mean=torch.ones(256).cuda())
