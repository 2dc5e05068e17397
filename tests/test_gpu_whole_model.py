"""Whole-model quantize + pack ("Lance-Quant", sections "校准阶段" and "量化应用":
504 target Linear layers -- 36 layers x 7 projections and their `_moe_gen`
siblings -- each with its saved mean |activation| per input channel, AWQ grid
search, group-wise INT4 pack and NVFP4 pack).

All 504 seeded matrices go through one wq_quantize_layers call, in the launch
configuration the benchmark times.  The packed byte totals must equal the byte
formula of the packed formats, and a sample of matrices covering every shape,
both siblings and the first and last layer is redone by the oracle: diagonal-
proxy losses within the AWQ loss tolerance, the chosen alpha equal (or a near
tie), s within 4 ulp of fp32(a^alpha), and both packs bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from w4a16_gemm_wq_b200 import synth
from tests._parity import bits

pytestmark = pytest.mark.gpu

ALPHAS = np.array(synth.ALPHA_GRID, dtype=np.float32)
LOSS_RTOL = 1e-3


def _packed_bytes_formula(layers):
    # INT4 g64: N*K/2 codes + N*(K/64) fp16 scales + N*ceil(K/64/8) uint32 zero words;
    # NVFP4: N*K/2 codes + N*K/16 E4M3 scales + one fp32 tensor scale
    i4 = sum(N * K // 2 + N * (K // 64) * 2 + N * (-(-(K // 64) // 8)) * 4 for _, _, K, N, _ in layers)
    nv = sum(N * K // 2 + N * K // 16 + 4 for _, _, K, N, _ in layers)
    return i4, nv


def test_whole_model_504_linears(lib):
    layers = synth.whole_model_layers()
    assert len(layers) == 504
    dev = torch.device("cuda")
    Ws = [synth.weight(N, K, seed=sd, device=dev) for _, _, K, N, sd in layers]
    ams = [synth.act_mean_lognormal(K, seed=sd, device=dev) for _, _, K, _, sd in layers]
    alphas = torch.tensor(ALPHAS, device=dev)
    outs = lib.wq_quantize_layers(Ws, ams, alphas, 64)
    torch.cuda.synchronize()
    assert lib.wq_device_error() == 0

    i4 = sum(o.int4.nbytes() for o in outs)
    nv = sum(o.nvfp4.nbytes() for o in outs)
    assert (i4, nv) == _packed_bytes_formula(layers)
    assert i4 == 2_991_587_328 and nv == 3_121_350_624  # 2.9916 GB and 3.1214 GB

    names = [(l, n) for l, n, _, _, _ in layers]
    sample = [names.index(x) for x in ((0, "q_proj"), (0, "k_proj_moe_gen"), (17, "v_proj"), (17, "o_proj_moe_gen"),
                                       (35, "gate_proj"), (35, "up_proj_moe_gen"), (35, "down_proj"))]
    for i in sample:
        l, name, K, N, _ = layers[i]
        W, am, o = Ws[i].cpu(), ams[i].cpu().numpy(), outs[i]
        s_ref, losses_ref, best_ref = oracle.awq_search(W, 64, ALPHAS, act_mean=am)
        losses = o.losses.cpu().numpy().astype(np.float64)
        best = int(o.best.cpu()[0])
        np.testing.assert_allclose(losses, losses_ref, rtol=LOSS_RTOL, err_msg=f"{l} {name}")
        assert best == best_ref or losses_ref[best] <= losses_ref[best_ref] * (1 + LOSS_RTOL), (l, name)
        s = o.s.cpu().numpy()
        s_at_best = np.power(np.maximum(am.astype(np.float64), 1e-4), float(ALPHAS[best])).astype(np.float32)
        assert np.max(np.abs(s.view(np.int32).astype(np.int64) - s_at_best.view(np.int32).astype(np.int64))) <= 4
        ref4 = oracle.quantize_int4(W, 64, s=s)
        for key in ("qweight", "scales", "zeros"):
            np.testing.assert_array_equal(bits(getattr(o.int4, key)), ref4[key], err_msg=f"{l} {name} {key}")
        refn = oracle.quantize_nvfp4(W)
        np.testing.assert_array_equal(bits(o.nvfp4.codes), refn["codes"], err_msg=f"{l} {name} codes")
        np.testing.assert_array_equal(bits(o.nvfp4.bscale), refn["bscale"], err_msg=f"{l} {name} bscale")
        assert bits(o.nvfp4.global_scale)[0] == np.float32(refn["g"]).view(np.uint32)


def test_layers_without_statistics_fall_back_to_min_max(lib):
    # a layer whose calibration statistics are missing ("Lance-Quant" 校准阶段: such
    # `_moe_gen` layers fall back to simple min-max) is packed without a scale
    W = synth.weight(300, 1024, seed=77, device="cuda")
    am = synth.act_mean_lognormal(1024, seed=77, device="cuda")
    alphas = torch.tensor(ALPHAS, device="cuda")
    with_stats, without = lib.wq_quantize_layers([W, W], [am, None], alphas, 64, nvfp4=False)
    torch.cuda.synchronize()
    assert without.s is None and with_stats.s is not None
    ref = oracle.quantize_int4(W.cpu(), 64)
    np.testing.assert_array_equal(bits(without.int4.qweight), ref["qweight"])
    np.testing.assert_array_equal(bits(without.int4.scales), ref["scales"])
    ref_s = oracle.quantize_int4(W.cpu(), 64, s=with_stats.s.cpu().numpy())
    np.testing.assert_array_equal(bits(with_stats.int4.qweight), ref_s["qweight"])


def test_layers_validate_every_item_before_launching(lib):
    W = synth.weight(64, 256, seed=1, device="cuda")
    bad = synth.weight(64, 100 * 8, seed=1, device="cuda")  # K = 800: not a multiple of group 64
    alphas = torch.tensor(ALPHAS, device="cuda")
    with pytest.raises(lib.WQError):
        lib.wq_quantize_layers([W, bad], [None, None], alphas, 64)
