"""Bit-level pins of the oracle's element rule q = RNEsat(RN_fp32(x / s)) and of its scale rule
s = RN_fp32(amax / 448) (1 for an all-zero group).

Sources: "FP8-RL: A Practical and Stable Low-Precision Stack for LLM RL", abstract (i) (blockwise
FP8 W8A8, weights requantized every step); "DeepSeek V4 performance: FP8 WO_A output projection
(vLLM PR 54894 analysis)", sections 1-3 (E4M3 codes with a scale per 128x128 weight block and per
1x128 activation group); the OCP FP8 E4M3 format (max 448, round to nearest even).  The
division and its rounding are the readings the oracle states (its R1): one IEEE fp32 division
x / s, then round-to-nearest-even to E4M3 with saturation at 448.

Every code is checked, not sampled, against a computation that shares nothing with the oracle:

* the quotient t is numpy's IEEE single-precision division, and t is verified to be the correctly
  rounded x / s by the definition of rounding, evaluated exactly in fp64: |x - t s| <= s ulp(t) / 2,
  with an exact tie only at an even t (t s has at most 48 significant bits, and x - t s is exact
  by Sterbenz's lemma);
* the code is ml_dtypes' float8_e4m3fn cast of t clamped to +-448 (pinned against the oracle's
  codec and torch's cast in test_oracle_codec), so the chain never touches the oracle's encoder.

A reciprocal-multiply variant x * RN(1 / s), a plausible slip in either implementation, is
planted on the CPU as a negative control: these checks must reject it.
"""
import ml_dtypes
import numpy as np
import pytest

import oracle
from fp8_blockwise_w8a8_b200 import inputs


def _quotient_is_correctly_rounded(x32, s32, t32):
    """True where t32 is RN_fp32(x32 / s32), checked by the definition of correct rounding."""
    x = x32.astype(np.float64)
    s = np.broadcast_to(np.asarray(s32, np.float32), x32.shape).astype(np.float64)
    t = t32.astype(np.float64)
    ulp = np.spacing(np.abs(t32).astype(np.float32)).astype(np.float64)
    diff = np.abs(x - t * s)            # exact: see the module docstring
    half = s * ulp / 2                  # exact: s times a power of two
    even = (t32.view(np.uint32) & 1) == 0
    return (diff < half) | ((diff == half) & even)


def _independent_codes(x32, s32):
    """Codes of x / s computed without the oracle: numpy fp32 division, then ml_dtypes' E4M3 cast
    (round to nearest even) of the quotient clamped to +-448."""
    with np.errstate(under="ignore"):
        t = (x32.astype(np.float32) / np.asarray(s32, np.float32)).astype(np.float32)
    assert _quotient_is_correctly_rounded(x32, s32, t).all()
    return np.clip(t, -448.0, 448.0).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)


def _reciprocal_variant_codes(x32, s32):
    """The planted mistake: x * RN(1 / s) instead of x / s."""
    inv = (np.float32(1.0) / np.asarray(s32, np.float32)).astype(np.float32)
    with np.errstate(under="ignore"):
        t = (x32.astype(np.float32) * inv).astype(np.float32)
    return np.clip(t, -448.0, 448.0).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)


def _scale_rule(amax32):
    with np.errstate(under="ignore"):
        s = (amax32.astype(np.float32) / np.float32(448.0)).astype(np.float32)
    return np.where(amax32 == 0, np.float32(1.0), s).astype(np.float32)


def _token_groups(x_bits):
    """bf16 [M, K] -> fp32 values [M, K/128, 128] and their group maxima [M, K/128]."""
    x = inputs.bf16_bits_to_f32(x_bits)
    M, K = x.shape
    g = x.reshape(M, K // 128, 128)
    return g, np.abs(g).max(axis=2)


def _check_token_quant(x_bits, q, sa):
    g, amax = _token_groups(x_bits)
    M, KB, _ = g.shape
    s_oracle = sa[:, :M].T                          # sa is [K/128, lds], K-block-major
    assert np.array_equal(s_oracle.view(np.uint32), _scale_rule(amax).view(np.uint32))
    want = _independent_codes(g, s_oracle[:, :, None])
    got = q.reshape(M, KB, 128)
    return int(np.count_nonzero(got != want)), g, s_oracle


def _check_weight_quant(w_bits, q, sw):
    x = inputs.bf16_bits_to_f32(w_bits)
    N, K = x.shape
    b = x.reshape(N // 128, 128, K // 128, 128)
    amax = np.abs(b).max(axis=(1, 3))
    assert np.array_equal(sw.view(np.uint32), _scale_rule(amax).view(np.uint32))
    want = _independent_codes(b, sw[:, None, :, None])
    return int(np.count_nonzero(q.reshape(b.shape) != want)), b, sw[:, None, :, None]


# --- crafted groups: every bf16 value below a chosen maximum ------------------------------------

def _all_bf16_up_to(amax_bits: int, lo_bits: int = 0) -> np.ndarray:
    """Every bf16 pattern with a magnitude between those of lo_bits and amax_bits, both signs."""
    pos = np.arange(lo_bits, amax_bits + 1, dtype=np.uint16)
    return np.concatenate([pos, pos | np.uint16(0x8000)])


def _crafted_rows(amax_bits: int, lo_bits: int = 0) -> np.ndarray:
    """1x128 groups that each hold the maximum once and then 127 values from the full list of
    bf16 values of magnitude <= amax (down to lo_bits): every quotient x / s the scale can
    produce."""
    vals = _all_bf16_up_to(amax_bits, lo_bits)
    n = -(-vals.size // 127)
    vals = np.concatenate([vals, np.zeros(n * 127 - vals.size, np.uint16)])
    rows = np.empty((n, 128), np.uint16)
    rows[:, 0] = amax_bits
    rows[:, 1:] = vals.reshape(n, 127)
    return rows


# bf16 maxima: significand 128 (1.0; 128 = 7*18 + 2: amax/448 inexact), 168 = 7*24 (exact
# quotient, E4M3 ties reachable), 255 (inexact), a huge, a tiny normal and a subnormal maximum
# (scale below 2^-60), and 0x3F2B (significand 171 = 7*24 + 3).
CRAFTED_MAXIMA = [0x3F80, 0x3FA8, 0x3FFF, 0x7F7F, 0x0D80, 0x0042, 0x3F2B]


@pytest.mark.parametrize("amax_bits", CRAFTED_MAXIMA)
def test_token_quant_every_quotient_of_a_scale(amax_bits):
    rows = _crafted_rows(amax_bits)
    q, sa = oracle.quant_token_1x128(rows)
    bad, _, _ = _check_token_quant(rows, q, sa)
    assert bad == 0


def test_every_significand_of_the_maximum_and_the_negative_control_fails():
    """For each of the 128 bf16 significands of the maximum (amax in [1, 2)), every bf16 value
    in [2^-10, amax]: this reaches quotients within 2^-22 (relative) of E4M3 rounding
    midpoints, and the reciprocal-multiply variant is rejected on them."""
    vals = oracle.e4m3_decode_all()
    pos = np.sort(vals[np.isfinite(vals) & (vals >= 0)])
    mids = (pos[1:] + pos[:-1]) / 2
    planted = near_total = 0
    for amax_bits in range(0x3F80, 0x4000):
        rows = _crafted_rows(amax_bits, 0x3A80)
        q, sa = oracle.quant_token_1x128(rows)
        _, g, s = _check_token_quant(rows, q, sa)
        t = np.abs(g.astype(np.float64) / s[:, :, None].astype(np.float64))
        j = np.clip(np.searchsorted(mids, t), 1, mids.size - 1)
        near = np.minimum(np.abs(t - mids[j]), np.abs(t - mids[j - 1])) <= t * 2.0 ** -22
        near_total += int(near.sum())
        bad, _, _ = _check_token_quant(rows, q, sa)
        assert bad == 0, hex(amax_bits)
        wrong = _reciprocal_variant_codes(g, s[:, :, None])
        planted += int(np.count_nonzero(wrong != q.reshape(g.shape)))
    assert near_total > 100
    assert planted > 0


def test_token_quant_workload_inputs_every_element():
    for a in (inputs.tiny_linear()["A"], inputs.decode_linear(N=128)["A"]):
        q, sa = oracle.quant_token_1x128(a, lds=(a.shape[0] + 3) // 4 * 4)
        bad, _, _ = _check_token_quant(a, q, sa)
        assert bad == 0


def test_weight_quant_4096_square_every_element_and_negative_control():
    """All 16.8 M codes of a 4096 x 4096 N(0, 0.02) weight; the reciprocal-multiply variant
    changes thousands of them and must be caught."""
    w = inputs.randn_bf16((4096, 4096), 0.02, 42, 0)
    q, sw = oracle.quant_weight_block(w, oracle.SCALE_F32)
    bad, b, s = _check_weight_quant(w, q, sw)
    assert bad == 0
    wrong = _reciprocal_variant_codes(b, s)
    assert np.count_nonzero(wrong != q.reshape(b.shape)) > 1000


def test_weight_quant_e8m0_every_element():
    """Power-of-two scales: x / 2^e is exact, so the codes are the E4M3 rounding of x 2^-e."""
    w = inputs.randn_bf16((1024, 2048), 0.02, 42, 1)
    q, sw = oracle.quant_weight_block(w, oracle.SCALE_E8M0)
    x = inputs.bf16_bits_to_f32(w).reshape(8, 128, 16, 128)
    s = np.ldexp(np.float32(1.0), sw.astype(np.int32) - 127).astype(np.float32)[:, None, :, None]
    assert np.array_equal(q.reshape(x.shape), _independent_codes(x, s))


def test_weight_quant_crafted_blocks():
    """128x128 blocks built from the crafted groups (the weight path shares the element rule)."""
    rows = _crafted_rows(0x3FFF)
    n = rows.shape[0] // 128 * 128
    w = np.ascontiguousarray(rows[:n].reshape(n // 128, 128, 128).transpose(1, 0, 2)
                             .reshape(128, n))
    q, sw = oracle.quant_weight_block(w, oracle.SCALE_F32)
    bad, _, _ = _check_weight_quant(w, q, sw)
    assert bad == 0


def test_rowwise_quant_every_element():
    """The per-token / per-channel rule (one scale per full row) uses the same element rule."""
    x = inputs.randn_bf16((64, 4096), 1.0, 42, 2)
    x[3] = 0
    q, s = oracle.quant_rowwise(x)
    xf = inputs.bf16_bits_to_f32(x)
    assert np.array_equal(s.view(np.uint32), _scale_rule(np.abs(xf).max(axis=1)).view(np.uint32))
    assert np.array_equal(q, _independent_codes(xf, s[:, None]))


def test_fused_front_ends_inherit_the_rule():
    """RMSNorm + quant, SiLU-and-mul + quant and residual add + RMSNorm + quant each quantize a
    bf16 intermediate; every one of their codes is the rule applied to that intermediate."""
    x = inputs.randn_bf16((48, 2048), 1.0, 42, 3)
    gamma = inputs.to_bf16_bits(np.linspace(0.5, 1.5, 2048).astype(np.float32))
    q, sa = oracle.rmsnorm_quant_token(x, gamma, 1e-6, lds=48)
    assert _check_token_quant(oracle.rmsnorm_bf16(x, gamma, 1e-6), q, sa)[0] == 0
    h = inputs.randn_bf16((40, 1536), 1.0, 42, 4)
    q, sa = oracle.silu_mul_quant(h, lds=40)
    assert _check_token_quant(oracle.silu_mul_bf16(h), q, sa)[0] == 0
