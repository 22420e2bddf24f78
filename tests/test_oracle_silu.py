"""Pins of the oracle's SiLU-and-mul front end (reading R8): the fp32 exponential (Cody-Waite
reduction + degree-7 Taylor polynomial) against float64 math.exp, SiLU's sign and limits, the bf16
product against a float64 evaluation, and the fused quant against the pinned 1x128 quant of the
product."""
import math
from fractions import Fraction

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


# ln 2 to 40 decimal places (far beyond the 2^-60 needed below)
LN2 = Fraction("0.6931471805599453094172321214581765680755")


def _rn32(q: Fraction) -> np.float32:
    """Round a positive rational to the nearest fp32 (ties to even), exactly."""
    lo = np.float32(float(q))
    while Fraction(float(lo)) > q:
        lo = np.nextafter(lo, np.float32(0))
    while Fraction(float(np.nextafter(lo, np.float32(np.inf)))) <= q:
        lo = np.nextafter(lo, np.float32(np.inf))
    hi = np.nextafter(lo, np.float32(np.inf))
    dlo, dhi = q - Fraction(float(lo)), Fraction(float(hi)) - q
    if dlo < dhi or (dlo == dhi and (lo.view(np.uint32) & 1) == 0):
        return lo
    return hi


def _significant_bits(v: np.float32) -> int:
    m = int(v.view(np.uint32) & 0x7FFFFF) | 0x800000
    return 24 - ((m & -m).bit_length() - 1)


def test_exp_f32_constants_from_their_definitions():
    """Cody-Waite: c1 + c2 splits ln 2 with k c1 exact for |k| <= 150 (8 bits) and c2 the fp32
    rounding of ln 2 - c1; the Taylor coefficients are 1/n! rounded to fp32; 1/ln 2 likewise."""
    c = oracle.exp_constants()
    assert c[0] == _rn32(1 / LN2)
    c1, c2 = c[1], c[2]
    assert _significant_bits(c1) + 8 <= 24            # k c1 exact for |k| < 256
    assert abs(LN2 - Fraction(float(c1))) < Fraction(1, 2 ** 16)
    assert c2 == _rn32(LN2 - Fraction(float(c1)))
    for i, n in enumerate(range(7, -1, -1)):
        assert c[3 + i] == _rn32(Fraction(1, math.factorial(n))), n


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
