"""Failure detection on the GPU without a fault: a bounded mbarrier wait that
nothing completes gives up after its limit, the kernel returns, the device
error word reports WQ_ERR_TIMEOUT, and the context stays usable."""
import pytest
import torch

import w4a16_gemm_wq_b200 as wq
from w4a16_gemm_wq_b200 import synth
from tests._parity import assert_linear_close
from tests.test_gpu_gemv import _ref_int4

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_is_reported(lib):
    assert lib.wq_device_error() == 0  # nothing pending from earlier tests
    assert lib.wq_selftest_timeout() == 0, "the wait must give up, not complete"
    with pytest.raises(wq.WQError) as e:
        lib.wq_device_error()
    assert e.value.status == wq.WQ_ERR_TIMEOUT
    assert lib.wq_device_error() == 0  # the word was cleared
    # the context is still usable: a linear call afterwards is correct
    K, N = 1024, 64
    p = lib.wq_quantize_int4(synth.weight(N, K, seed=3).cuda(), 64, 1)
    X = synth.activations(1, K, seed=4)
    assert_linear_close(lib.wq_linear_int4(X.cuda(), p), _ref_int4(p, X), what="after timeout")
