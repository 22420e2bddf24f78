"""Pins of the oracle's inverse-RoPE + group-128 quant front end (reading R9) against what the
mathematics fixes: the inverse rotation is multiplication of each pair, read as a complex number,
by e^(-i theta) (checked in float64 complex arithmetic, within the fp32 error bound before the
bf16 rounding); position 0 is the identity; theta = pi/2 is an exact swap with a sign; forward
then inverse RoPE gives back the input; the pass-through dims are untouched; and the fused quant
equals the pinned 1x128 token quant of the rotated bf16 values (fp32 scales) or the E8M0 power of
two of reading R2 with codes from the pinned encoder."""
import math

import numpy as np
import pytest

import oracle
from fp8_blockwise_w8a8_b200 import inputs


def _f(bits):
    return inputs.bf16_bits_to_f32(bits).astype(np.float64)


def _pairs(R, interleaved):
    i = np.arange(R // 2)
    return (2 * i, 2 * i + 1) if interleaved else (i, i + R // 2)


def _bf16_candidates(v):
    """The bf16 values an fp32 evaluation of v within its error bound may round to."""
    lo = inputs.to_bf16_bits(v[0]).astype(np.int64)
    hi = inputs.to_bf16_bits(v[1]).astype(np.int64)
    return lo, hi


@pytest.mark.parametrize("interleaved", [True, False])
def test_inverse_rope_is_complex_multiplication_by_conjugate(interleaved):
    T, H, D, R = 24, 3, 192, 64
    d = inputs.wo_a(tokens=T, heads=H, head_dim=D, rope_dim=R, max_pos=4096, with_weight=False)
    y = oracle.inverse_rope_bf16(d["o"], d["positions"], d["cos"], d["sin"], R, interleaved)
    x = _f(d["o"])                                                # [T, H, D]
    a, b = _pairs(R, interleaved)
    z = x[:, :, D - R + a] + 1j * x[:, :, D - R + b]
    c = d["cos"][d["positions"]].astype(np.float64)[:, None, :]
    s = d["sin"][d["positions"]].astype(np.float64)[:, None, :]
    w = z * (c - 1j * s)                                          # e^(-i theta) from the caches
    # fp32 evaluation: two rounded products and a rounded sum, relative error <= 2 * 2^-24 of
    # |x_a c| + |x_b s| (and alike for the second).
    mag_a = np.abs(x[:, :, D - R + a] * c) + np.abs(x[:, :, D - R + b] * s)
    mag_b = np.abs(x[:, :, D - R + b] * c) + np.abs(x[:, :, D - R + a] * s)
    yr = y.reshape(T, H, D)
    for part, exact, mag, idx in ((0, w.real, mag_a, a), (1, w.imag, mag_b, b)):
        err = 2.0 ** -23 * mag
        got = yr[:, :, D - R + idx].astype(np.int64)
        lo, hi = _bf16_candidates((exact - err, exact + err))
        near = inputs.to_bf16_bits(exact).astype(np.int64)
        ok = (got == near) | (got == lo) | (got == hi)
        assert ok.all(), (part, np.argwhere(~ok)[:3])
        # away from a bf16 rounding boundary the result is bf16 of the exact value
        assert np.mean(got == near) > 0.99
    assert np.array_equal(yr[:, :, :D - R], d["o"][:, :, :D - R])   # pass-through dims


def test_position_zero_is_identity_and_quarter_turn_is_a_signed_swap():
    T, H, D, R = 4, 2, 128, 32
    o = inputs.randn_bf16((T, H, D), 1.0, 31, 0)
    cos = np.ones((2, R // 2), np.float32)
    sin = np.zeros((2, R // 2), np.float32)
    cos[1] = 0.0
    sin[1] = 1.0                                                  # theta = pi/2 exactly
    y0 = oracle.inverse_rope_bf16(o, np.zeros(T, np.int64), cos, sin, R)
    assert np.array_equal(y0.reshape(T, H, D), o)
    y1 = oracle.inverse_rope_bf16(o, np.ones(T, np.int64), cos, sin, R).reshape(T, H, D)
    x, yf = _f(o), _f(y1)
    a, b = _pairs(R, True)
    # multiplying (x_a + i x_b) by e^(-i pi/2) = -i gives x_b - i x_a
    assert np.array_equal(yf[:, :, D - R + a], x[:, :, D - R + b])
    assert np.array_equal(yf[:, :, D - R + b], -x[:, :, D - R + a])


def test_forward_then_inverse_rope_recovers_the_input():
    T, H, D, R = 16, 2, 256, 64
    d = inputs.wo_a(tokens=T, heads=H, head_dim=D, rope_dim=R, max_pos=8192, with_weight=False)
    x = _f(d["o"])
    a, b = _pairs(R, True)
    c = d["cos"][d["positions"]].astype(np.float64)[:, None, :]
    s = d["sin"][d["positions"]].astype(np.float64)[:, None, :]
    fwd = x.copy()
    fwd[:, :, D - R + a] = x[:, :, D - R + a] * c - x[:, :, D - R + b] * s
    fwd[:, :, D - R + b] = x[:, :, D - R + a] * s + x[:, :, D - R + b] * c
    y = _f(oracle.inverse_rope_bf16(inputs.to_bf16_bits(fwd.astype(np.float32)),
                                    d["positions"], d["cos"], d["sin"], R)).reshape(T, H, D)
    # two bf16 roundings of values of size |x| (the forward pass and the inverse): a few ulp of
    # the pair's magnitude
    mag = np.sqrt(x[:, :, D - R + a] ** 2 + x[:, :, D - R + b] ** 2)
    tol = 3 * 2.0 ** -8 * mag + 1e-30
    assert np.all(np.abs(y[:, :, D - R + a] - x[:, :, D - R + a]) <= tol)
    assert np.all(np.abs(y[:, :, D - R + b] - x[:, :, D - R + b]) <= tol)


@pytest.mark.parametrize("interleaved", [True, False])
def test_fused_fp32_scale_quant_equals_token_quant_of_rotated_values(interleaved):
    T, H, D, R = 37, 4, 192, 64                                   # H*D = 768 = 6 blocks; heads
    d = inputs.wo_a(tokens=T, heads=H, head_dim=D, rope_dim=R,     # straddle block edges
                    max_pos=1024, with_weight=False)
    q, sa = oracle.inverse_rope_quant(d["o"], d["positions"], d["cos"], d["sin"], R,
                                      interleaved, fmt=0, lds=40)
    y = oracle.inverse_rope_bf16(d["o"], d["positions"], d["cos"], d["sin"], R, interleaved)
    q2, sa2 = oracle.quant_token_1x128(y, lds=40)
    assert np.array_equal(q, q2)
    assert np.array_equal(sa[:, :T], sa2[:, :T])
    assert np.all(sa[:, T:] == 0)


def test_fused_e8m0_quant_uses_the_power_of_two_scale():
    T, H, D, R = 9, 2, 128, 64
    d = inputs.wo_a(tokens=T, heads=H, head_dim=D, rope_dim=R, max_pos=512, with_weight=False)
    o = d["o"].copy()
    o[3] = 0                                                      # an all-zero token: scale 1
    q, sa = oracle.inverse_rope_quant(o, d["positions"], d["cos"], d["sin"], R, fmt=1)
    y = _f(oracle.inverse_rope_bf16(o, d["positions"], d["cos"], d["sin"], R)).reshape(T, -1)
    for t in range(T):
        for kb in range(H * D // 128):
            g = y[t, kb * 128:(kb + 1) * 128]
            amax = np.float32(np.abs(g).max())
            s = float(sa[kb, t])
            if amax == 0:
                assert s == 1.0
            else:
                r = float(np.float32(amax) / np.float32(448.0))
                m, e = math.frexp(s)
                assert m == 0.5 and s >= r and s / 2 < r, (t, kb, s, r)
            codes = oracle.e4m3_encode((g / s).astype(np.float32))
            assert np.array_equal(q[t, kb * 128:(kb + 1) * 128], codes)


def test_no_rotary_dims_reduces_to_token_quant():
    o = inputs.randn_bf16((5, 2, 256), 1.0, 32, 0)
    cos = np.ones((1, 1), np.float32)
    sin = np.zeros((1, 1), np.float32)
    q, sa = oracle.inverse_rope_quant(o, np.zeros(5, np.int64), cos, sin, 0)
    q2, sa2 = oracle.quant_token_1x128(o.reshape(5, 512))
    assert np.array_equal(q, q2) and np.array_equal(sa, sa2)


@pytest.mark.parametrize("fmt", [oracle.SCALE_F32, oracle.SCALE_E8M0])
def test_block_diag_gemm_equals_dense_gemm_with_block_diagonal_weight(fmt):
    """The per-group GEMM is the plain GEMM with the groups' weights on the block diagonal of
    one [G N_g, G K_g] matrix (zero codes elsewhere add exact zeros)."""
    G, M, N_g, K_g = 3, 20, 256, 256
    a = inputs.bf16_bits_to_f32(inputs.randn_bf16((M, G * K_g), 40.0, 41, 0))
    aq = oracle.e4m3_encode(a).reshape(M, G * K_g)
    sa = np.abs(inputs.bf16_bits_to_f32(inputs.randn_bf16((G * K_g // 128, M), 0.01, 41, 1)))
    sa += np.float32(1e-4)
    w = inputs.randn_bf16((G, N_g, K_g), 0.02, 41, 2)
    wq = np.empty((G, N_g, K_g), np.uint8)
    sw = []
    for g in range(G):
        wq[g], s = oracle.quant_weight_block(w[g], fmt)
        sw.append(s)
    sw = np.stack(sw)
    ref, absref = oracle.gemm_w8a8_block_diag(aq, sa, wq, sw, fmt)
    wfull = np.zeros((G * N_g, G * K_g), np.uint8)
    swfull = np.full((G * N_g // 128, G * K_g // 128), 1.0 if fmt == oracle.SCALE_F32 else 127,
                     np.float32 if fmt == oracle.SCALE_F32 else np.uint8)
    for g in range(G):
        wfull[g * N_g:(g + 1) * N_g, g * K_g:(g + 1) * K_g] = wq[g]
        swfull[g * N_g // 128:(g + 1) * N_g // 128, g * K_g // 128:(g + 1) * K_g // 128] = sw[g]
    ref2, absref2 = oracle.gemm_w8a8_block(aq, sa, wfull, swfull, fmt)
    assert np.array_equal(ref, ref2) and np.array_equal(absref, absref2)
    assert np.abs(ref).max() > 0
