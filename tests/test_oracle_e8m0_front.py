"""Pins of the oracle's E8M0 activation scales for the 1x128 front ends (its reading R12): the plain
token quant, RMSNorm + quant, SiLU-and-mul + quant and residual add + RMSNorm + quant, each with
the group scale 2^e, e the smallest integer with 2^e >= fp32(amax / 448) (clamped to
[-127, 127]; 1 for an all-zero group), stored as its fp32 value.

Sources: "DeepSeek V4 performance: FP8 WO_A output projection (vLLM PR 54894 analysis)", section
1 (E8M0: an unsigned exponent with bias 127, lossless only for exact powers of two) and section 3
(group-128 activation quant feeding a GEMM that takes MX scales on both operands); "SGLang ...
(PR 21403 analysis)", section 1 (RMSNorm fused with the FP8 quant).

Every scale is checked against its definition (a power of two, at least fp32(amax/448), its half
below it), every code against numpy's fp32 quotient encoded by ml_dtypes' E4M3 cast, and each
fused front end against the pinned token quant of its bf16 intermediate.  Planted mistakes (the
OCP-MX floor exponent, rounding the exponent to nearest) are rejected.
"""
import ml_dtypes
import numpy as np
import pytest

import oracle
from fp8_blockwise_w8a8_b200 import inputs

E8M0 = oracle.SCALE_E8M0


def _scale_ok(amax32, s32):
    """s is the least power of two >= r = fp32(amax / 448) (1 where amax == 0)."""
    with np.errstate(under="ignore"):
        r = (amax32.astype(np.float32) / np.float32(448.0)).astype(np.float32)
    mant, _ = np.frexp(s32.astype(np.float64))
    pow2 = mant == 0.5
    least = (s32.astype(np.float64) >= r) & (s32.astype(np.float64) / 2 < r)
    zero = (amax32 == 0) & (s32 == 1.0)
    clamped = (s32 == np.float32(2.0 ** -127)) & (r <= 2.0 ** -127)
    return (pow2 & (least | clamped)) | zero


def _codes(y32, s32):
    with np.errstate(under="ignore"):
        t = (y32.astype(np.float32) / s32.astype(np.float32)).astype(np.float32)
    return np.clip(t, -448, 448).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)


def _check(y_bits, q, sa):
    y = inputs.bf16_bits_to_f32(y_bits)
    M, K = y.shape
    g = y.reshape(M, K // 128, 128)
    s = sa[:, :M].T
    amax = np.abs(g).max(axis=2)
    assert _scale_ok(amax, s).all()
    assert np.array_equal(q.reshape(g.shape), _codes(g, s[:, :, None]))
    # the largest code of a non-zero group lies in [224, 448] (unless the exponent was clamped
    # at -127: a group maximum below 448 * 2^-128)
    dec = oracle.e4m3_decode_all()
    vmax = np.abs(dec[q.reshape(g.shape)]).max(axis=2)
    nz = (amax > 0) & (s > np.float32(2.0 ** -127))
    assert np.all((vmax[nz] >= 224) & (vmax[nz] <= 448))


def test_token_quant_e8m0_every_element():
    for a in (inputs.tiny_linear()["A"], inputs.decode_linear(N=128)["A"],
              inputs.randn_bf16((64, 2048), 1e-30, 7, 0), inputs.randn_bf16((8, 512), 1e30, 7, 1)):
        q, sa = oracle.quant_token_1x128(a, fmt=E8M0)
        _check(a, q, sa)


def test_token_quant_e8m0_every_bf16_quotient():
    """Groups holding every bf16 magnitude up to the maximum, for maxima whose amax/448 lands on
    each side of a power of two (and exactly on one)."""
    for amax_bits in (0x3F80, 0x43E0, 0x43DF, 0x43E1, 0x0080):   # 1, 448, just below/above, tiny
        vals = np.arange(0, amax_bits + 1, dtype=np.uint16)
        vals = np.concatenate([vals, vals | np.uint16(0x8000)])
        n = -(-vals.size // 127)
        vals = np.concatenate([vals, np.zeros(n * 127 - vals.size, np.uint16)])
        rows = np.empty((n, 128), np.uint16)
        rows[:, 0] = amax_bits
        rows[:, 1:] = vals.reshape(n, 127)
        q, sa = oracle.quant_token_1x128(rows, fmt=E8M0)
        _check(rows, q, sa)


def test_zero_groups_take_scale_one():
    x = np.zeros((3, 256), np.uint16)
    x[1, 128:] = inputs.randn_bf16((1, 128), 1.0, 3, 0)
    q, sa = oracle.quant_token_1x128(x, fmt=E8M0)
    assert sa[0, 0] == 1.0 and sa[0, 1] == 1.0 and sa[1, 1] != 1.0 and not q[0].any()


def test_planted_exponent_rules_are_rejected():
    """The OCP-MX rule 2^(floor(log2 amax) - 8) and a rounded exponent both break the pin."""
    a = inputs.decode_linear(N=128)["A"]
    x = inputs.bf16_bits_to_f32(a).reshape(a.shape[0], -1, 128)
    amax = np.abs(x).max(axis=2)
    floor_rule = np.ldexp(np.float32(1), (np.floor(np.log2(amax)) - 8).astype(np.int32))
    assert not _scale_ok(amax, floor_rule.astype(np.float32)).all()
    round_rule = np.ldexp(np.float32(1), np.rint(np.log2(amax / 448.0)).astype(np.int32))
    assert not _scale_ok(amax, round_rule.astype(np.float32)).all()


def test_rmsnorm_quant_e8m0_is_the_token_quant_of_the_normalised_rows():
    d = inputs.prefill_linear(M=96, N=128, with_weight=False)
    q, sa = oracle.rmsnorm_quant_token(d["X"], d["gamma"], d["eps"], fmt=E8M0)
    y = oracle.rmsnorm_bf16(d["X"], d["gamma"], d["eps"])
    q2, sa2 = oracle.quant_token_1x128(y, fmt=E8M0)
    assert np.array_equal(q, q2) and np.array_equal(sa, sa2)
    _check(y, q, sa)


def test_silu_mul_quant_e8m0_is_the_token_quant_of_the_product():
    h = inputs.randn_bf16((33, 1536), 1.0, 22, 0)
    q, sa = oracle.silu_mul_quant(h, lds=36, fmt=E8M0)
    y = oracle.silu_mul_bf16(h)
    q2, sa2 = oracle.quant_token_1x128(y, lds=36, fmt=E8M0)
    assert np.array_equal(q, q2) and np.array_equal(sa, sa2)
    _check(y, q, sa)


def test_add_rmsnorm_quant_e8m0_is_the_rmsnorm_quant_of_the_sum():
    x = inputs.randn_bf16((40, 1024), 1.0, 23, 0)
    res = inputs.randn_bf16((40, 1024), 1.0, 23, 1)
    gamma = inputs.to_bf16_bits(np.linspace(0.5, 1.5, 1024).astype(np.float32))
    h, q, sa = oracle.add_rmsnorm_quant(x, res, gamma, 1e-6, fmt=E8M0)
    q2, sa2 = oracle.rmsnorm_quant_token(h, gamma, 1e-6, fmt=E8M0)
    assert np.array_equal(q, q2) and np.array_equal(sa, sa2)
    with pytest.raises(ValueError):
        oracle.add_rmsnorm_quant(x, res, gamma, 1e-6, per_token=True, fmt=E8M0)


def test_inverse_rope_e8m0_without_rotary_dims_is_the_token_quant():
    x = inputs.randn_bf16((50, 1024), 1.0, 24, 0)
    cos = np.ones((1, 1), np.float32)
    q, sa = oracle.inverse_rope_quant(x.reshape(50, 1, 1024), np.zeros(50, np.int64), cos, cos, 0,
                                      fmt=E8M0)
    q2, sa2 = oracle.quant_token_1x128(x, fmt=E8M0)
    assert np.array_equal(q, q2) and np.array_equal(sa, sa2)
