"""The C-ABI library: builds for sm_100a, loads, exports every declared symbol,
and validates arguments on the host (no GPU needed for any of this)."""
import ctypes
import os
import re

import pytest

import w4a16_gemm_wq_b200 as wq
from w4a16_gemm_wq_b200 import build

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "wq.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(\w+)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return wq.load()


def test_header_declares_the_five_entry_points():
    names = declared_functions()
    for n in ("wq_quantize_int4", "wq_quantize_nvfp4", "awq_search_scale", "wq_linear_int4", "wq_linear_nvfp4"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(names) == set(wq.SIGNATURES), "binding signatures out of sync with include/wq.h"
    for n in names:
        assert hasattr(lib, n), n


def test_size_queries(lib):
    assert wq.int4_sizes(2048, 11008, 128) == (2048 * 11008 // 2, 2048 * 86 * 2, 2048 * 11 * 4)
    assert wq.int4_sizes(512, 512, 64) == (512 * 256, 512 * 8 * 2, 512 * 1 * 4)
    assert wq.nvfp4_sizes(2048, 2048) == (2048 * 1024, 2048 * 128)
    with pytest.raises(wq.WQError) as e:
        wq.int4_sizes(16, 100, 64)  # K not a multiple of 32
    assert e.value.status == wq.WQ_ERR_ARG
    assert wq.int4_sizes(16, 512, 32) == (16 * 256, 16 * 16 * 2, 16 * 2 * 4)
    with pytest.raises(wq.WQError) as e:
        wq.int4_sizes(16, 512, 256)
    assert e.value.status == wq.WQ_ERR_UNSUPPORTED


def _st(lib, rc):
    return rc, lib.wq_last_error().decode()


def test_host_validation_rejects_before_any_launch(lib):
    P = ctypes.c_void_p
    good = P(1 << 20)  # 16-byte aligned, never dereferenced: validation fails first
    bad = P((1 << 20) + 8)
    # bits != 4 -> unsupported
    assert lib.wq_quantize_int4(good, 16, 64, 8, 64, 1, None, good, good, good, None) == wq.WQ_ERR_UNSUPPORTED
    # null input, misaligned output, zeros with a symmetric pack
    assert lib.wq_quantize_int4(None, 16, 64, 4, 64, 1, None, good, good, good, None) == wq.WQ_ERR_ARG
    assert lib.wq_quantize_int4(good, 16, 64, 4, 64, 1, None, bad, good, good, None) == wq.WQ_ERR_ARG
    assert lib.wq_quantize_int4(good, 16, 64, 4, 64, 0, None, good, good, good, None) == wq.WQ_ERR_ARG
    assert "zeros" in lib.wq_last_error().decode()
    # K % group_size
    assert lib.wq_quantize_int4(good, 16, 96, 4, 64, 1, None, good, good, good, None) == wq.WQ_ERR_ARG
    # empty calibration set is an error ("llm-quantize": reject empty calibration)
    assert lib.awq_search_scale(good, 16, 64, good, 0, None, good, 20, 64, good, good, good, None, 0, None) \
        in (wq.WQ_ERR_ARG,)
    # M <= 0, act_fp4 out of range
    assert lib.wq_linear_int4(good, 0, 16, 64, good, good, good, 64, 1, None, good, None, 0, None) == wq.WQ_ERR_ARG
    assert lib.wq_linear_nvfp4(good, 1, 16, 64, good, good, good, 2, None, good, None, 0, None) == wq.WQ_ERR_ARG
    assert lib.wq_status_string(4).decode().startswith("WQ_ERR_TIMEOUT")


def test_binding_refuses_requantizing():
    p = wq.PackedInt4(None, None, None, 1, 32, 64, 1)
    with pytest.raises(ValueError):
        wq.wq_quantize_int4(p)


def test_gptq_and_shared_awq_validate_on_the_host(lib):
    P = ctypes.c_void_p
    good = P(1 << 20)
    bad = P((1 << 20) + 8)
    # GPTQ: unsupported group, null W, misaligned W, zeros without / with a zero point
    assert lib.wq_gptq_int4(good, 16, 256, good, 256, 1, good, good, good, None) == wq.WQ_ERR_UNSUPPORTED
    assert lib.wq_gptq_int4(None, 16, 256, good, 64, 1, good, good, good, None) == wq.WQ_ERR_ARG
    assert lib.wq_gptq_int4(bad, 16, 256, good, 64, 1, good, good, good, None) == wq.WQ_ERR_ARG
    assert lib.wq_gptq_int4(good, 16, 256, good, 64, 1, good, good, None, None) == wq.WQ_ERR_ARG
    assert lib.wq_gptq_int4(good, 16, 256, good, 64, 0, good, good, good, None) == wq.WQ_ERR_ARG
    assert lib.wq_gptq_int4(good, 16, 256, None, 64, 1, good, good, good, None) == wq.WQ_ERR_ARG
    # shared-s AWQ: no matrices, a null or misaligned one, an empty calibration set
    ptrs = (ctypes.c_void_p * 2)(1 << 20, 1 << 21)
    ns = (ctypes.c_int64 * 2)(16, 8)
    args = (256, good, 4, None, good, 20, 64, good, good, good, good, 1 << 30, None)
    assert lib.awq_search_scale_shared(ctypes.cast(ptrs, P), ctypes.cast(ns, P), 0, *args) == wq.WQ_ERR_ARG
    nulls = (ctypes.c_void_p * 2)(1 << 20, None)
    assert lib.awq_search_scale_shared(ctypes.cast(nulls, P), ctypes.cast(ns, P), 2, *args) == wq.WQ_ERR_ARG
    odd = (ctypes.c_void_p * 2)(1 << 20, (1 << 21) + 8)
    assert lib.awq_search_scale_shared(ctypes.cast(odd, P), ctypes.cast(ns, P), 2, *args) == wq.WQ_ERR_ARG
    empty = (256, good, 0, None, good, 20, 64, good, good, good, good, 1 << 30, None)
    assert lib.awq_search_scale_shared(ctypes.cast(ptrs, P), ctypes.cast(ns, P), 2, *empty) == wq.WQ_ERR_ARG


def test_split_k_plan_is_host_logic():
    # the prefill GEMM's plan (tile and split count from a cost model of CTA rates) is
    # host logic: K splits only where the tiles leave SMs idle and K is long enough; the
    # workspace query is the partial tiles' size (whole fp32 tiles, one wave of CTAs at
    # most) and 0 when nothing splits
    split = [(512, 256, 11008), (512, 2048, 11008), (2048, 256, 4096), (512, 256, 2048), (512, 2048, 2048),
             (2048, 2048, 11008), (512, 2560, 2048)]
    # (the last three: q/k/v and gate/up stacked along N, whose tiles fill the SMs)
    unsplit = [(8192, 11008, 2048), (2048, 2048, 2048), (16, 256, 11008), (512, 11008, 2048),
               (2048, 2560, 2048), (2048, 22016, 2048), (8192, 2560, 2048)]
    for M, N, K in split:
        for fmt in (wq.WQ_FMT_INT4, wq.WQ_FMT_NVFP4):
            ws = wq.linear_workspace_size(M, N, K, fmt)
            assert ws > 0, (M, N, K)
            assert ws % (128 * 128 * 4) == 0 and ws <= 148 * 256 * 256 * 4, (M, N, K, ws)
    for M, N, K in unsplit:
        assert wq.linear_workspace_size(M, N, K, wq.WQ_FMT_INT4) == 0, (M, N, K)
    # the plan depends on the shape only: the same query twice, and INT4 / NVFP4 alike
    assert wq.linear_workspace_size(512, 2048, 11008, wq.WQ_FMT_INT4) == \
        wq.linear_workspace_size(512, 2048, 11008, wq.WQ_FMT_NVFP4)