"""Pins of the oracle's SiLU-and-mul front end (reading R8): the fp32 exponential (Cody-Waite
reduction + degree-7 Taylor polynomial) against float64 math.exp, SiLU's sign and limits, the bf16
product against a float64 evaluation, and the fused quant against the pinned 1x128 quant of the
product."""
import math

import numpy as np

import oracle
from fp8_blockwise_w8a8_b200 import inputs


def _ulp32(v):
    return np.spacing(np.float32(abs(v)))


def test_exp_f32_within_two_ulp_of_float64():
    xs = np.concatenate([np.linspace(-87.0, 88.5, 20001), np.linspace(-1.0, 1.0, 2001),
                         [0.0, -0.0, 0.5 * math.log(2), -0.5 * math.log(2)]]).astype(np.float32)
    for x in xs:
        e = oracle.exp_f32(float(x))
        t = math.exp(float(x))
        assert abs(e - t) <= 2 * _ulp32(t), (x, e, t)


def test_exp_f32_special_values_and_subnormal_range():
    assert oracle.exp_f32(0.0) == 1.0
    assert oracle.exp_f32(89.0) == math.inf
    assert oracle.exp_f32(-105.0) == 0.0
    for x in np.linspace(-103.0, -87.5, 501).astype(np.float32):
        e = oracle.exp_f32(float(x))
        assert abs(e - math.exp(float(x))) <= 2.0 ** -149   # subnormal: within one step


def test_silu_sign_limits_and_accuracy():
    assert oracle.silu_f32(0.0) == 0.0
    assert math.copysign(1.0, oracle.silu_f32(-0.0)) == -1.0
    assert oracle.silu_f32(100.0) == 100.0
    s = oracle.silu_f32(-100.0)
    assert s == 0.0 or abs(s) < 1e-40
    assert math.copysign(1.0, oracle.silu_f32(-200.0)) == -1.0     # e^200 = inf: g / inf = -0
    for g in np.linspace(-20.0, 20.0, 4001).astype(np.float32):
        t = float(g) / (1.0 + math.exp(-float(g)))
        assert abs(oracle.silu_f32(float(g)) - t) <= 3 * _ulp32(t) + 1e-45, g


def test_silu_mul_bf16_within_one_bf16_ulp_of_float64():
    h = inputs.randn_bf16((16, 512), 2.0, 21, 0)
    y = oracle.silu_mul_bf16(h)
    hf = (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    g, u = hf[:, :256], hf[:, 256:]
    t = g / (1.0 + np.exp(-g)) * u
    yf = (y.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.all(np.abs(yf - t) <= oracle.bf16_ulp(t))


def test_silu_mul_quant_equals_token_quant_of_the_product():
    h = inputs.randn_bf16((33, 1536), 1.0, 22, 0)
    q, sa = oracle.silu_mul_quant(h, lds=36)
    q2, sa2 = oracle.quant_token_1x128(oracle.silu_mul_bf16(h), lds=36)
    assert np.array_equal(q, q2)
    assert np.array_equal(sa, sa2)
