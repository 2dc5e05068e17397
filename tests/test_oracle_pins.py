"""Pins of the CPU oracle to facts other than itself (no GPU needed).

Each test checks one oracle function against a closed form, a library
routine (numpy / torch conversions), a value worked by hand from the pages
(tests/golden), an invariant, or brute force on tiny inputs.  They are chosen
so that a plausible slip in the oracle (a dropped term, a wrong sign or
index, a transposed operand, a wrong tie rule) fails at least one of them.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from w4a16_gemm_wq_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    rows = []
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def _bf16(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


# ---------------------------------------------------------------- scalar codecs
def test_bf16_decode_matches_torch():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 1 << 16, size=4000, dtype=np.uint16)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF]  # finite only
    ref = torch.tensor(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(oracle.bf16_to_f64(bits), ref)


def test_f16_decode_matches_numpy_all_patterns():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    finite = ((bits >> 10) & 0x1F) != 0x1F
    ref = bits.view(np.float16).astype(np.float64)
    np.testing.assert_array_equal(oracle.f16_to_f64(bits[finite]), ref[finite])


def test_f32_to_f16_rne_matches_numpy():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(3000).astype(np.float32) * np.float32(0.05),
        (rng.random(1000) * 65000).astype(np.float32),
        (rng.random(1000) * 1e-4).astype(np.float32),  # subnormal fp16 range
        # exact ties between fp16 neighbours (1 + (2j+1) * 2^-11)
        (np.float32(1.0) + (2 * np.arange(50, dtype=np.float32) + 1) * np.float32(2.0 ** -11)),
        np.array([0.0, -0.0, 1e-5, 65504.0, -65504.0, 6.1035156e-05, 5.9604645e-08], dtype=np.float32),
    ])
    ref = x.astype(np.float16).view(np.uint16)
    np.testing.assert_array_equal(oracle.f32_to_f16(x), ref)
    # saturation (pages silent; reading: saturate to the largest finite half)
    assert oracle.f32_to_f16([1e6])[0] == 0x7BFF
    assert oracle.f32_to_f16([-70000.0])[0] == 0xFBFF


def test_e4m3_golden_codes():
    for code, val in _golden("e4m3_codes.txt"):
        got = oracle.e4m3_decode([int(code, 16)])[0]
        if val == "nan":
            assert np.isnan(got)
        else:
            assert got == float(val) and np.signbit(got) == np.signbit(float(val)), code


def test_e4m3_decode_matches_torch_float8():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.tensor(codes).view(torch.float8_e4m3fn).double().numpy()
    got = oracle.e4m3_decode(codes)
    nan = np.isnan(ref)
    np.testing.assert_array_equal(np.isnan(got), nan)
    np.testing.assert_array_equal(got[~nan], ref[~nan])


def test_e4m3_encode_matches_torch_rne_and_saturates():
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.random(3000) * 448, rng.random(1000) * 0.02, rng.random(200) * 2 ** -8]).astype(np.float32)
    # exact midpoints between neighbouring codes (ties -> even code)
    mids = []
    for c in range(0, 0x7E):
        a, b = oracle.e4m3_decode([c, c + 1])
        mids.append((a + b) / 2)
    x = np.concatenate([x, np.array(mids, dtype=np.float32)])
    ref = torch.tensor(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(oracle.e4m3_encode(x), ref)
    assert list(oracle.e4m3_encode([448.0, 460.0, 470.0, 1e9])) == [0x7E] * 4


def test_e2m1_golden_table_and_ties():
    for code, val in _golden("e2m1_codes.txt"):
        got = oracle.e2m1_decode([int(code)])[0]
        assert got == float(val) and np.signbit(got) == np.signbit(float(val))
    # ties go to the even code; saturation at 6; sign copied from the input
    cases = [(0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6), (7.0, 7),
             (100.0, 7), (0.2, 0), (0.3, 1), (-0.1, 8), (-0.0, 8), (0.0, 0), (-5.5, 15), (-2.6, 13)]
    got = oracle.e2m1_encode([c[0] for c in cases])
    assert [int(v) for v in got] == [c[1] for c in cases]


def test_e2m1_encode_is_nearest():
    x = np.linspace(-8, 8, 4001, dtype=np.float32)
    codes = oracle.e2m1_encode(x)
    vals = oracle.e2m1_decode(codes)
    table = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    best = np.min(np.abs(np.abs(x)[:, None] - table[None, :]), axis=1)
    np.testing.assert_allclose(np.abs(np.abs(x) - np.abs(vals)), best, rtol=0, atol=0)


# ---------------------------------------------------------------- INT4
def _unpack_nibbles(words, count):
    words = np.asarray(words, dtype=np.uint32)
    shifts = np.arange(8, dtype=np.uint32) * 4
    nib = (words[..., None] >> shifts) & 0xF
    return nib.reshape(*words.shape[:-1], -1)[..., :count]


def test_int4_golden_range_example():
    rows = _golden("int4_range_example.txt")
    vals = [float(r[0]) for r in rows]
    G = 64
    group = np.zeros(G, dtype=np.float32)
    group[: len(vals)] = vals
    W = _bf16(group[None, :])
    p = oracle.quantize_int4(W, G)
    assert p["scales"][0, 0] == 0x3377
    assert p["zeros"][0, 0] & 0xF == 6
    codes = _unpack_nibbles(p["qweight"][0], G)
    deq = oracle.dequant_int4(p)[0]
    for i, r in enumerate(rows):
        assert codes[i] == int(r[1]), r
        assert deq[i] == float(r[2]), r


def test_int4_symmetric_example():
    # "quantization primer" section 2: symmetric range [-1, 1], zero maps to integer zero.
    G = 64
    g = np.zeros(G, dtype=np.float32)
    g[:3] = [1.0, -1.0, 0.0]
    p = oracle.quantize_int4(_bf16(g[None]), G, zero_point=0)
    sc = oracle.f16_to_f64([p["scales"][0, 0]])[0]
    assert sc == float(np.float16(np.float32(1.0) / np.float32(7.0)))
    codes = _unpack_nibbles(p["qweight"][0], G)
    assert list(codes[:3]) == [15, 1, 8]
    deq = oracle.dequant_int4(p)[0]
    assert deq[0] == 7 * sc and deq[1] == -7 * sc and deq[2] == 0.0


@pytest.mark.parametrize("G", [32, 64, 128])
def test_int4_round_trip_bound_and_brute_force(G):
    N, K = 48, 512
    W = synth.weight(N, K, seed=11)
    p = oracle.quantize_int4(W, G)
    w = W.float().numpy().astype(np.float64)
    sc = oracle.f16_to_f64(p["scales"].ravel()).reshape(N, K // G)
    z = _unpack_nibbles(p["zeros"], K // G).astype(np.float64)
    q = _unpack_nibbles(p["qweight"], K).astype(np.float64)
    scf = np.repeat(sc, G, axis=1)
    zf = np.repeat(z, G, axis=1)
    deq = oracle.dequant_int4(p)
    np.testing.assert_array_equal(deq, (q - zf) * scf)
    lo, hi = (0 - zf) * scf, (15 - zf) * scf
    inside = (w >= lo) & (w <= hi)
    assert inside.mean() > 0.95  # only group extremes can fall just outside
    err = np.abs(w - deq)
    assert np.all(err[inside] <= scf[inside] / 2 * (1 + 2 ** -20))
    # brute force: the stored code minimises |w - (c - z) sc| over all 16 codes
    cand = (np.arange(16)[None, None, :] - zf[..., None]) * scf[..., None]
    d = np.abs(w[..., None] - cand)
    best = d.min(axis=-1)
    np.testing.assert_allclose(np.abs(w - deq), best, rtol=1e-6, atol=0)
    # the group's min lies within half a step of the bottom code; the max within half a
    # step of the top code plus the fp16 rounding of the scale over 15 steps (2^-11 each)
    wg = w.reshape(N, K // G, G)
    assert np.all(wg.min(-1) >= (0 - z) * sc - sc / 2 - 1e-12)
    assert np.all(wg.max(-1) <= (15 - z) * sc + sc / 2 + 15 * 2 ** -11 * sc + 1e-12)
    # the scale is the min-max range over 15 levels, to fp16 precision
    rng_ = (wg.max(-1) - wg.min(-1)) / 15
    np.testing.assert_allclose(sc, np.maximum(rng_, 1e-5), rtol=2 ** -10)


def test_int4_groups_are_independent_and_row_major():
    N, K, G = 8, 512, 64
    W = synth.weight(N, K, seed=12)
    full = oracle.quantize_int4(W, G)
    deq = oracle.dequant_int4(full)
    for g in range(K // G):
        part = oracle.quantize_int4(W[:, g * G:(g + 1) * G].contiguous(), G)
        np.testing.assert_array_equal(oracle.dequant_int4(part), deq[:, g * G:(g + 1) * G])
        np.testing.assert_array_equal(part["scales"][:, 0], full["scales"][:, g])
    for n in range(N):
        row = oracle.quantize_int4(W[n:n + 1].contiguous(), G)
        np.testing.assert_array_equal(row["qweight"][0], full["qweight"][n])
    # row subset dequant
    np.testing.assert_array_equal(oracle.dequant_int4(full, rows=[5, 2]), deq[[5, 2]])


def test_int4_pack_layout_lsb_first_and_zero_padding():
    N, K, G = 4, 11008, 128  # 86 groups -> 11 zero words, last one padded
    W = synth.weight(N, K, seed=13)
    p = oracle.quantize_int4(W, G)
    assert p["zeros"].shape == (N, 11)
    assert np.all(p["zeros"][:, -1] >> (4 * (86 % 8)) == 0)
    # repack codes recovered from the dequantized values by independent numpy code
    deq = oracle.dequant_int4(p)
    sc = np.repeat(oracle.f16_to_f64(p["scales"].ravel()).reshape(N, -1), G, axis=1)
    z = np.repeat(_unpack_nibbles(p["zeros"], K // G), G, axis=1)
    q = np.rint(deq / sc).astype(np.int64) + z
    words = np.zeros((N, K // 8), dtype=np.uint64)
    for j in range(8):
        words |= (q[:, j::8].astype(np.uint64) << np.uint64(4 * j))
    np.testing.assert_array_equal(words.astype(np.uint32), p["qweight"])


def test_int4_degenerate_group_and_scale_floor():
    G = 64
    g = np.full((2, G), 0.25, dtype=np.float32)
    g[1] = 0.0
    p = oracle.quantize_int4(_bf16(g), G)
    sc = oracle.f16_to_f64(p["scales"].ravel())
    assert np.all(sc == float(np.float16(1e-5)))
    deq = oracle.dequant_int4(p)
    assert np.all(deq[1] == 0.0)  # all-zero group is exact


def test_int4_awq_scale_path():
    N, K, G = 16, 256, 64
    W = synth.weight(N, K, seed=14)
    base = oracle.quantize_int4(W, G)
    ones = oracle.quantize_int4(W, G, s=np.ones(K, dtype=np.float32))
    for key in ("qweight", "scales", "zeros"):
        np.testing.assert_array_equal(base[key], ones[key])
    # a power-of-two s scales w' exactly: codes unchanged, scales x4
    four = oracle.quantize_int4(W, G, s=np.full(K, 4.0, dtype=np.float32))
    np.testing.assert_array_equal(four["qweight"], base["qweight"])
    np.testing.assert_array_equal(four["zeros"], base["zeros"])
    np.testing.assert_array_equal(oracle.f16_to_f64(four["scales"].ravel()),
                                  4 * oracle.f16_to_f64(base["scales"].ravel()))
    # s differing per column scales column k of w' only: check against w*s quantized
    rng = np.random.default_rng(3)
    s = (2.0 ** rng.integers(-2, 3, size=K)).astype(np.float32)
    ps = oracle.quantize_int4(W, G, s=s)
    ws = (W.float() * torch.tensor(s)).to(torch.bfloat16)  # exact: powers of two
    pw = oracle.quantize_int4(ws, G)
    for key in ("qweight", "scales", "zeros"):
        np.testing.assert_array_equal(ps[key], pw[key])


# ---------------------------------------------------------------- NVFP4
def test_nvfp4_block_structure_and_error_bound():
    N, K = 32, 512
    W = synth.weight(N, K, seed=21)
    p = oracle.quantize_nvfp4(W)
    w = W.float().numpy().astype(np.float64)
    amax = np.abs(w).max()
    assert p["g"] == np.float32(np.float32(amax) / np.float32(2688.0))
    sb = oracle.e4m3_decode(p["bscale"].ravel()).reshape(N, K // 16)
    # the block holding the tensor maximum gets the largest E4M3 scale (448)
    assert p["bscale"].max() == 0x7E
    deq = oracle.dequant_nvfp4(p)
    step = np.repeat(sb, 16, axis=1) * float(p["g"])
    # each element is the nearest E2M1 multiple of its block step (ties aside)
    table = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    v = np.abs(w) / step
    best = np.min(np.abs(v[..., None] - table), axis=-1) * step
    np.testing.assert_allclose(np.abs(np.abs(w) - np.abs(deq)), best, rtol=1e-6, atol=1e-30)
    # the block maximum lands near the top code: |w|max / step within E4M3 rounding of 6
    bm = np.abs(w).reshape(N, K // 16, 16).max(-1)
    ratio = bm / (sb * float(p["g"]))
    assert np.all((ratio > 6 / (1 + 2 ** -3)) & (ratio < 6 * (1 + 2 ** -3)))


def test_nvfp4_pack_low_nibble_even_and_scale_invariance():
    N, K = 8, 256
    W = synth.weight(N, K, seed=22)
    p = oracle.quantize_nvfp4(W)
    deq = oracle.dequant_nvfp4(p)
    sb = np.repeat(oracle.e4m3_decode(p["bscale"].ravel()).reshape(N, -1), 16, axis=1)
    vals = deq / (sb * float(p["g"]))
    table = {0.0: 0, 0.5: 1, 1.0: 2, 1.5: 3, 2.0: 4, 3.0: 5, 4.0: 6, 6.0: 7}
    codes = np.vectorize(lambda v: table[abs(v)] | (8 if v < 0 else 0))(vals)
    wneg = W.float().numpy() < 0
    codes = np.where((vals == 0) & wneg, 8, codes)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    np.testing.assert_array_equal(packed, p["codes"])
    # scaling the whole tensor by a power of two only scales g
    p2 = oracle.quantize_nvfp4((W.float() * 8).to(torch.bfloat16))
    np.testing.assert_array_equal(p2["codes"], p["codes"])
    np.testing.assert_array_equal(p2["bscale"], p["bscale"])
    assert p2["g"] == p["g"] * 8


def test_nvfp4_zero_tensor_and_single_spike():
    z = oracle.quantize_nvfp4(torch.zeros(2, 32, dtype=torch.bfloat16))
    assert z["g"] == 1.0 and not z["codes"].any() and not z["bscale"].any()
    a = torch.zeros(1, 32)
    a[0, 5] = -3.0
    p = oracle.quantize_nvfp4(a.to(torch.bfloat16))
    assert p["bscale"][0, 0] == 0x7E and p["bscale"][0, 1] == 0
    assert (p["codes"][0, 2] >> 4) == 0xF  # element 5: high nibble of byte 2, code -6
    # exact up to the fp32 rounding of g = 3 / 2688
    np.testing.assert_allclose(oracle.dequant_nvfp4(p)[0], a[0].double().numpy(), rtol=2 ** -23, atol=0)


# ---------------------------------------------------------------- linear
def test_matmul_matches_numpy_and_transpose_order():
    rng = np.random.default_rng(4)
    A = rng.standard_normal((5, 33))
    B = rng.standard_normal((7, 33))
    np.testing.assert_allclose(oracle.matmul_abT(A, B), A @ B.T, rtol=1e-13, atol=1e-13)


def test_activations_and_equivalence_transform():
    # "OmniQuant" section 2.2.2: Y = (X diag(s)) (diag(1/s) W)^T is exact before quantization.
    rng = np.random.default_rng(5)
    M, K, N = 4, 64, 12
    X = _bf16(rng.standard_normal((M, K)))
    W = rng.standard_normal((N, K))
    s = rng.uniform(0.25, 4.0, size=K).astype(np.float32)
    xf = oracle.activations_f64(X)
    np.testing.assert_array_equal(xf, X.double().numpy())
    y_plain = oracle.linear(X, W)
    y_eq = oracle.linear(X, W * s.astype(np.float64)[None, :], inv_s=(1.0 / s.astype(np.float64)))
    # exact in real arithmetic; here only 1/s is rounded (to fp32, the kernels' type)
    np.testing.assert_allclose(y_eq, y_plain, rtol=0, atol=1e-6 * np.abs(y_plain).max())


# ---------------------------------------------------------------- AWQ
ALPHAS = np.array([i / 20 for i in range(20)], dtype=np.float32)


def test_awq_alpha0_is_plain_rtn():
    # alpha = 0 gives s = 1: the "simple min-max" fallback of Lance-Quant
    N, K, G, T = 8, 128, 64, 16
    W = synth.weight(N, K, seed=31)
    X = synth.activations_student_t(T, K, seed=31)
    s, losses, best = oracle.awq_search(W, G, ALPHAS[:1], X=X)
    assert best == 0 and np.all(s == 1.0)
    p = oracle.quantize_int4(W, G)
    delta = W.double().numpy() - oracle.dequant_int4(p)
    y = X.double().numpy() @ delta.T
    np.testing.assert_allclose(losses[0], np.sum(y * y), rtol=1e-12)


def test_awq_brute_force_direct_form():
    # L(alpha) = || X W^T - (X/s) Q(W s)^T ||^2 evaluated literally in numpy fp64
    T, N, K, G = 4, 8, 64, 64
    W = synth.weight(N, K, seed=32, outlier_frac=0.05)
    X = synth.activations_student_t(T, K, seed=32)
    s_best, losses, best = oracle.awq_search(W, G, ALPHAS, X=X)
    x = X.double().numpy()
    w = W.double().numpy()
    a = np.maximum(np.abs(x).mean(0), 1e-4)
    direct = []
    for al in ALPHAS:
        s = np.power(a, float(al)).astype(np.float32)
        q = oracle.dequant_int4(oracle.quantize_int4(W, G, s=s))
        r = x @ w.T - (x / s.astype(np.float64)) @ q.T
        direct.append(np.sum(r * r))
    direct = np.array(direct)
    np.testing.assert_allclose(losses, direct, rtol=1e-9)
    assert best == int(np.argmin(direct))
    np.testing.assert_array_equal(s_best, np.power(a, float(ALPHAS[best])).astype(np.float32))


def test_awq_diagonal_proxy_matches_full_loss_for_diagonal_calibration():
    # With X = diag(c) (T = K tokens), mean_t |X_tk| = c_k / K and
    # ||X Delta^T||^2 = sum_nk c_k^2 Delta_nk^2 = K^2 * sum_nk (a_k Delta_nk)^2.
    K, N, G = 64, 8, 64
    rng = np.random.default_rng(6)
    c = (2.0 ** rng.integers(-1, 4, size=K)).astype(np.float32)
    X = _bf16(np.diag(c))
    a = (c / K).astype(np.float32)
    W = synth.weight(N, K, seed=33, outlier_frac=0.05)
    _, full, bf = oracle.awq_search(W, G, ALPHAS, X=X)
    _, proxy, bp = oracle.awq_search(W, G, ALPHAS, act_mean=a)
    np.testing.assert_allclose(full, K * K * proxy, rtol=1e-9)
    assert bf == bp


def test_awq_helps_on_outlier_channels():
    # the search finds a non-trivial alpha that beats plain RTN when a few
    # activation channels dominate (the premise of AWQ, "quantization primer" section 7)
    T, N, K, G = 64, 32, 256, 64
    d = synth.config1(seed=0)
    W = synth.weight(N, K, seed=34, outlier_frac=0.01)
    ch = synth.outlier_channels(K, 0.05, 34)
    X = synth.activations(T, K, seed=34, channels=ch, mult=30.0)
    s, losses, best = oracle.awq_search(W, G, ALPHAS, X=X)
    assert best > 0 and losses[best] < losses[0]
    assert d["W"].shape == (512, 512)


def test_awq_shared_scale_is_the_search_over_stacked_rows():
    # Matrices that consume one normalised input (q/k/v, gate/up) share one s, since
    # the scale is folded into that RMSNorm ("Lance-Quant", section 量化应用): the loss
    # of the stack [W_0; W_1; W_2] under s is the sum of the matrices' losses under the
    # same s, for the token loss and for the diagonal proxy alike.
    T, K, G = 32, 256, 64
    Ws = [synth.weight(n, K, seed=40 + i, outlier_frac=0.02) for i, n in enumerate((32, 8, 8))]
    X = synth.activations_student_t(T, K, seed=40)
    a = synth.act_mean_lognormal(K, seed=40).numpy()
    for kw in ({"X": X}, {"act_mean": a}):
        parts = np.sum([oracle.awq_search(W, G, ALPHAS, **kw)[1] for W in Ws], axis=0)
        s, shared, best = oracle.awq_search(torch.cat(Ws), G, ALPHAS, **kw)
        np.testing.assert_allclose(shared, parts, rtol=1e-12)
        assert best == int(np.argmin(parts))


# ---------------------------------------------------------------- GPTQ
def _spd_factor(K, seed, corr=0.9):
    # calibration tokens with strongly correlated channels (so that the second-order
    # adjustment matters), and the inverse-Hessian factor from them
    rng = np.random.default_rng(seed)
    base = rng.standard_normal((256, K // 4))
    x = np.repeat(base, 4, axis=1) * corr + rng.standard_normal((256, K)) * (1 - corr)
    X = _bf16(x.astype(np.float32))
    return X, oracle.gptq_hessian_factor(X)


@pytest.mark.parametrize("zp", [1, 0])
def test_gptq_identity_factor_is_plain_rtn(zp):
    # U = I: no second-order coupling, nothing to adjust -> the plain min-max quantizer
    # ("quantization primer" section 6 reduces to sections 2-3), and e = w - deq(q)
    N, K, G = 16, 256, 64
    W = synth.weight(N, K, seed=60, outlier_frac=0.02)
    g = oracle.gptq_int4(W, np.eye(K, dtype=np.float32), G, zp, want_err=True)
    r = oracle.quantize_int4(W, G, zp)
    for key in ("qweight", "scales", "zeros"):
        if r[key] is not None:
            np.testing.assert_array_equal(g[key], r[key])
    np.testing.assert_array_equal(g["err"], (W.float().numpy() - oracle.dequant_int4(r)).astype(np.float32))


@pytest.mark.parametrize("zp", [1, 0])
def test_gptq_diagonal_factor_divides_by_the_diagonal(zp):
    # U diagonal: the columns do not couple, so no weight is adjusted and the codes are
    # the plain quantizer's, while each error is the IEEE fp32 quotient
    # (w_k - deq(q_k)) / U[k][k] ("quantization primer" section 6: the error is scaled by
    # the second-order information).  Diagonal values that are not powers of two make a
    # reciprocal-then-multiply evaluation differ from the quotient on many elements, so
    # that reading would fail here.
    N, K, G = 16, 256, 64
    W = synth.weight(N, K, seed=63, outlier_frac=0.02)
    d = np.array([3.0, 7.0, 0.3, 1.7, 5.9, 0.11, 2.6, 9.3], dtype=np.float32)[np.arange(K) % 8]
    g = oracle.gptq_int4(W, np.diag(d).astype(np.float32), G, zp, want_err=True)
    r = oracle.quantize_int4(W, G, zp)
    for key in ("qweight", "scales", "zeros"):
        if r[key] is not None:
            np.testing.assert_array_equal(g[key], r[key])
    diff = W.float().numpy() - oracle.dequant_int4(r).astype(np.float32)  # fp32 - fp32, IEEE
    quotient = diff / d[None, :]
    np.testing.assert_array_equal(g["err"], quotient)
    assert np.any(diff * (np.float32(1.0) / d)[None, :] != quotient)


@pytest.mark.parametrize("G", [64, 128])
def test_gptq_error_identity(G):
    # The adjustments accumulate so that w - deq(q) = e U for every row (U upper
    # triangular): column j carries e_k U[k][j] from every k < j plus its own
    # e_j U[j][j].  A dropped, mis-signed or transposed term breaks it.
    N, K = 12, 256
    W = synth.weight(N, K, seed=61, outlier_frac=0.02)
    _, U = _spd_factor(K, 61)
    g = oracle.gptq_int4(W, U, G, want_err=True)
    lhs = W.double().numpy() - oracle.dequant_int4(g)
    rhs = g["err"].astype(np.float64) @ np.triu(U).astype(np.float64)
    np.testing.assert_allclose(lhs, rhs, rtol=0, atol=2e-5 * np.abs(W.double().numpy()).max())


def test_gptq_factor_and_loss():
    # U^T U is the damped inverse Hessian; GPTQ's output error under H, |X (W - Q)^T|^2,
    # beats plain rounding on correlated calibration data (the point of the method)
    N, K, G = 24, 256, 64
    W = synth.weight(N, K, seed=62, outlier_frac=0.02)
    X, U = _spd_factor(K, 62)
    x = X.double().numpy()
    H = 2 * x.T @ x
    H[np.diag_indices(K)] += 0.01 * np.mean(np.diag(H))
    np.testing.assert_allclose(U.astype(np.float64).T @ U.astype(np.float64), np.linalg.inv(H),
                               rtol=0, atol=1e-6 * np.abs(np.linalg.inv(H)).max())
    assert np.all(np.tril(U, -1) == 0)
    w = W.double().numpy()
    loss = lambda q: float(np.sum((x @ (w - oracle.dequant_int4(q)).T) ** 2))
    assert loss(oracle.gptq_int4(W, U, G)) < 0.8 * loss(oracle.quantize_int4(W, G))
