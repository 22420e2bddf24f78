"""Pins of the oracle's per-token / per-channel ("PTPC") path: row-wise quantization (one scale per
row of K, optionally after RMSNorm) and the per-channel GEMM reference ("SGLang ... (PR 21403
analysis)" sections 1-3: group_size 0 = per token, CHANNEL weight scales, GEMM on (codes, x_scale)
with weight_scale).  Each check compares against something other than the function itself."""
import numpy as np
import pytest

import oracle
from fp8_blockwise_w8a8_b200 import inputs


def _dec(codes):
    return oracle.e4m3_decode_all()[codes]


def test_rowwise_equals_1x128_token_quant_when_k_is_128():
    x = inputs.randn_bf16((37, 128), 1.0, 11, 0)
    q, s = oracle.quant_rowwise(x)
    q1, sa = oracle.quant_token_1x128(x, lds=40)
    assert np.array_equal(q, q1)
    assert np.array_equal(s, sa[0, :37])


def test_rowwise_rmsnorm_equals_token_rmsnorm_when_k_is_128():
    x = inputs.randn_bf16((21, 128), 1.0, 12, 0)
    g = inputs.randn_bf16((128,), 0.3, 12, 1)
    q, s = oracle.quant_rowwise(x, g, 1e-6)
    q1, sa = oracle.rmsnorm_quant_token(x, g, 1e-6, lds=24)
    assert np.array_equal(q, q1)
    assert np.array_equal(s, sa[0, :21])


def test_fused_rowwise_equals_rmsnorm_then_rowwise():
    x = inputs.randn_bf16((9, 1024), 1.0, 13, 0)
    g = inputs.randn_bf16((1024,), 0.5, 13, 1)
    q, s = oracle.quant_rowwise(x, g, 1e-5)
    y = oracle.rmsnorm_bf16(x, g, 1e-5)
    q2, s2 = oracle.quant_rowwise(y)
    assert np.array_equal(q, q2) and np.array_equal(s, s2)


def test_rowwise_scale_invariants_and_error_bound():
    x = inputs.randn_bf16((16, 768), 1.0, 14, 0)
    x[3] = 0                                   # an all-zero row
    x[5, 100] = 0x4700                         # a large value in one row (bf16 32768.0)
    q, s = oracle.quant_rowwise(x)
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    amax = np.abs(xf).max(axis=1)
    expect = np.where(amax == 0, np.float32(1.0), amax / np.float32(448.0)).astype(np.float32)
    assert np.array_equal(s, expect)           # numpy's float32 division is IEEE round-to-nearest
    assert s[3] == 1.0 and not q[3].any()
    for m in range(16):
        if m == 3:
            continue
        assert ((q[m] & 0x7F) == 0x7E).any()   # the row maximum maps to +-448
        y = xf[m] / s[m]
        d = _dec(q[m])
        # half the E4M3 spacing at |y| (normal: 2^(e-3); subnormal: 2^-9), doubled for safety
        e = np.floor(np.log2(np.maximum(np.abs(y), 2.0 ** -6)))
        assert np.all(np.abs(y - d) <= 2.0 ** (e - 3))


def test_rowwise_gemm_brute_force():
    M, N, K = 5, 128, 256
    rng = np.random.default_rng(15)
    aq = rng.integers(0, 256, (M, K), dtype=np.uint8)
    wq = rng.integers(0, 256, (N, K), dtype=np.uint8)
    aq[(aq & 0x7F) == 0x7F] = 0                # no NaN codes
    wq[(wq & 0x7F) == 0x7F] = 0
    sa = rng.uniform(0.01, 2.0, M).astype(np.float32)
    sw = rng.uniform(0.01, 2.0, N).astype(np.float32)
    ref, absref = oracle.gemm_w8a8_rowwise(aq, sa, wq, sw)
    A, W = _dec(aq), _dec(wq)
    expect = sa.astype(np.float64)[:, None] * sw.astype(np.float64)[None, :] * (A @ W.T)
    assert np.allclose(ref, expect, rtol=1e-12, atol=1e-300)
    sa64, sw64 = np.abs(sa.astype(np.float64)), np.abs(sw.astype(np.float64))
    assert np.allclose(absref, sa64[:, None] * sw64[None, :] * (np.abs(A) @ np.abs(W).T), rtol=1e-12)


def test_rowwise_gemm_equals_blockwise_gemm_with_constant_scales():
    """With sa constant along K and sw constant over each 128-column block, the per-channel and
    the block-scaled definitions describe the same product."""
    M, N, K = 9, 256, 384
    x = inputs.randn_bf16((M, K), 1.0, 16, 0)
    w = inputs.randn_bf16((N, K), 0.02, 16, 1)
    aq, sa = oracle.quant_rowwise(x)
    wq, _ = oracle.quant_rowwise(w)
    swb = np.array([0.5, 2.0], np.float32)                     # one scale per 128 columns
    sw = np.repeat(swb, 128)
    ref, absref = oracle.gemm_w8a8_rowwise(aq, sa, wq, sw)
    sa_blk = np.tile(sa, (K // 128, 1))                        # sa[kb, m] = sa[m]
    sw_blk = np.tile(swb[:, None], (1, K // 128)).astype(np.float32)
    ref2, absref2 = oracle.gemm_w8a8_block(aq, sa_blk, wq, sw_blk, oracle.SCALE_F32)
    assert np.allclose(ref, ref2, rtol=1e-12, atol=1e-30)
    assert np.allclose(absref, absref2, rtol=1e-12)
