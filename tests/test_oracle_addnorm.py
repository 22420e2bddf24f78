"""Pins of the oracle's residual add + RMSNorm + quant (reading R11) against what the mathematics
fixes.  The add h = bf16(fp32(x) + fp32(res)) rounds twice, but rounding to fp32 (24 bits) before
bf16 (8 bits) is innocuous for a sum (Figueroa: p' >= 2p + 2), so h must equal ONE round-to-nearest-
even of the exact sum to bf16 -- computed here from float64 (exact for the exponent spreads used)
by frexp and rint, a path that shares nothing with the oracle's bit-level conversion.  Zero and
opposite residuals, a closed form through the whole chain (a constant row normalises to +-1 and
every code is +-448), and the composition with the already pinned front ends complete it."""
import numpy as np
import pytest

import oracle
from fp8_blockwise_w8a8_b200 import inputs


def _bf16_of_f64(v):
    """Round-to-nearest-even of float64 values to bf16 (normal range), via frexp and rint."""
    m, e = np.frexp(v)                       # v = m 2^e, 0.5 <= |m| < 1
    r = np.rint(m * 256.0) * np.exp2(e - 8.0)  # 8 significant bits, ties to even
    return inputs.to_bf16_bits(r.astype(np.float32))   # exact: r has 8 bits, fp32 normal range


def _wide(shape, seed, tid, lo=-40, hi=40):
    rng = inputs.rng_for(seed, tid)
    v = rng.standard_normal(shape).astype(np.float32)
    v *= np.exp2(rng.integers(lo, hi, shape)).astype(np.float32)
    return inputs.to_bf16_bits(v)


def test_add_is_one_rounding_of_the_exact_sum():
    M, K = 48, 1024
    x = _wide((M, K), 51, 0)
    r = _wide((M, K), 51, 1)
    # near-cancellations and near-ties: res = -x (1 + small) and res = x * 2^-9 (1 + 2^-7 k)
    r[:4] = inputs.to_bf16_bits(-inputs.bf16_bits_to_f32(x[:4]) * np.float32(1 + 2 ** -7))
    r[4:8] = inputs.to_bf16_bits(inputs.bf16_bits_to_f32(x[4:8]) * np.float32(2 ** -9 * 1.5))
    g = inputs.randn_bf16((K,), 0.3, 51, 2)
    h, _, _ = oracle.add_rmsnorm_quant(x, r, g)
    exact = (inputs.bf16_bits_to_f32(x).astype(np.float64)
             + inputs.bf16_bits_to_f32(r).astype(np.float64))
    want = _bf16_of_f64(exact)
    nz = exact != 0
    assert np.array_equal(h[nz], want[nz])
    assert np.all(h[~nz] == 0)                    # exact cancellation gives +0


def test_zero_and_opposite_residuals():
    M, K = 6, 256
    x = inputs.randn_bf16((M, K), 1.0, 52, 0)
    g = inputs.randn_bf16((K,), 0.3, 52, 1)
    h, _, _ = oracle.add_rmsnorm_quant(x, np.zeros_like(x), g)
    assert np.array_equal(h, x)
    neg = x ^ np.uint16(0x8000)
    h, q, sa = oracle.add_rmsnorm_quant(x, neg, g)
    assert np.all(h == 0)                         # x + (-x) = +0 in round-to-nearest
    # all-zero blocks: scale 1 and zero codes, signed as 0 * r * gamma is (reading R3)
    assert np.all(sa == 1.0)
    want = np.where(inputs.bf16_bits_to_f32(g) < 0, 0x80, 0x00).astype(np.uint8)
    assert np.array_equal(q, np.broadcast_to(want, q.shape))


@pytest.mark.parametrize("per_token", [False, True])
def test_constant_row_closed_form(per_token):
    """x + res = c on every element, gamma = 1: RMSNorm gives bf16(c / sqrt(c^2 + eps)) = +-1 for
    |c| >> sqrt(eps), every block's amax is 1, s = 1/448, and every code is +-448."""
    M, K = 4, 512
    c = np.array([3.0, -0.5, 40.0, -7.0], np.float32)
    x = inputs.to_bf16_bits(np.repeat(c[:, None] / 2, K, axis=1))
    r = x.copy()
    g = inputs.to_bf16_bits(np.ones(K, np.float32))
    h, q, sa = oracle.add_rmsnorm_quant(x, r, g, 1e-6, per_token)
    assert np.array_equal(inputs.bf16_bits_to_f32(h), np.repeat(c[:, None], K, axis=1))
    want = np.where(c < 0, 0xFE, 0x7E).astype(np.uint8)
    assert np.array_equal(q, np.repeat(want[:, None], K, axis=1))
    assert np.all(sa[..., :M] == np.float32(1.0) / np.float32(448.0))


@pytest.mark.parametrize("per_token", [False, True])
def test_fused_equals_add_then_the_pinned_front_end(per_token):
    M, K = 37, 768
    x = inputs.randn_bf16((M, K), 1.0, 53, 0)
    r = inputs.randn_bf16((M, K), 2.0, 53, 1)
    g = inputs.randn_bf16((K,), 0.3, 53, 2)
    x0, r0 = x.copy(), r.copy()
    h, q, sa = oracle.add_rmsnorm_quant(x, r, g, 1e-6, per_token, lds=40)
    assert np.array_equal(x, x0) and np.array_equal(r, r0)      # inputs untouched
    if per_token:
        q2, sa2 = oracle.quant_rowwise(h, g, 1e-6)
        assert np.array_equal(sa, sa2)
    else:
        q2, sa2 = oracle.rmsnorm_quant_token(h, g, 1e-6, lds=40)
        assert np.array_equal(sa, sa2)
    assert np.array_equal(q, q2)
