"""The bounded-wait failure path on the GPU, without a fault: a self-test kernel built from the
GEMM kernels' wait helpers waits on a barrier that nothing arrives on, gives up after a short
limit, records FP8Q_ERR_TIMEOUT in the device error word, stops its other warps through the abort
flag and releases TMEM.  The host reads the status, and the next kernels run correctly on the same
context."""
import time

import numpy as np
import pytest

import oracle
import fp8_blockwise_w8a8_b200 as fq
from fp8_blockwise_w8a8_b200 import inputs

from helpers import dev_bf16, dev_f32, dev_u8, host_bf16_f64, assert_within_gemm_tolerance, promoted_steps

pytestmark = pytest.mark.gpu


def test_timeout_is_reported_and_the_context_stays_usable():
    assert fq.check_device_error() == 0
    t0 = time.perf_counter()
    fq.selftest_timeout(2_000_000)                       # 2 ms
    assert fq.check_device_error() == fq.FP8Q_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    assert fq.check_device_error() == 0                  # the word was cleared by the read
    # the same context quantizes and multiplies correctly afterwards
    d = inputs.tiny_linear()
    aq, sa = oracle.quant_token_1x128(d["A"])
    wq, sw = oracle.quant_weight_block(d["W"], 0)
    q, s = fq.quant_weight_block(dev_bf16(d["W"]), "f32")
    assert np.array_equal(q.cpu().numpy(), wq) and np.array_equal(s.cpu().numpy(), sw)
    out = fq.gemm_w8a8_block(dev_u8(aq), dev_f32(sa), dev_u8(wq), dev_f32(sw), 0)
    assert fq.check_device_error() == 0
    ref, absref = oracle.gemm_w8a8_block(aq, sa, wq, sw, 0)
    assert_within_gemm_tolerance(host_bf16_f64(out), ref, absref, "after timeout",
                                 steps=promoted_steps(aq.shape[1]))


def test_repeated_timeouts():
    for _ in range(3):
        fq.selftest_timeout(500_000)
        assert fq.check_device_error() == fq.FP8Q_ERR_TIMEOUT
