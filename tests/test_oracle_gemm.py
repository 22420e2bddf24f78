"""Pins of the oracle's block-scaled W8A8 GEMM reference and its grouped (MoE) form.

Sources: "FP8-RL: A Practical and Stable Low-Precision Stack for LLM RL", abstract (i) (W8A8
linear layers, dense and MoE); "SGLang AMD GPU optimisation ... (SGLang PR 21403 analysis)"
section 3 (the GEMM consumes a pre-quantized (codes, scale) pair, bf16 out); "DeepSeek V4
performance: FP8 WO_A output projection (vLLM PR 54894 analysis)" section 3 (batched per-group
FP8 GEMM with per-group [out/128, in/128] weight scales).
"""
from fractions import Fraction

import numpy as np
import torch

import oracle
from fp8_blockwise_w8a8_b200 import inputs


def _quantized_pair(M, N, K, seed, sw_fmt=oracle.SCALE_F32):
    a = inputs.randn_bf16((M, K), 1.0, seed, 0)
    w = inputs.randn_bf16((N, K), 0.02, seed, 1)
    aq, sa = oracle.quant_token_1x128(a)
    wq, sw = oracle.quant_weight_block(w, sw_fmt)
    return aq, sa, wq, sw


def _dequant(aq, sa, wq, sw, sw_fmt):
    dec = oracle.e4m3_decode_all()
    A = dec[aq] * np.repeat(sa.T.astype(np.float64), 128, axis=1)
    swv = sw.astype(np.float64) if sw_fmt == oracle.SCALE_F32 else \
        np.vectorize(oracle.e8m0_decode)(sw)
    W = dec[wq] * np.repeat(np.repeat(swv, 128, axis=0), 128, axis=1)
    return A, W


def test_matches_torch_matmul_fp64():
    for fmt in (oracle.SCALE_F32, oracle.SCALE_E8M0):
        aq, sa, wq, sw = _quantized_pair(37, 256, 512, 8, fmt)
        ref, absref = oracle.gemm_w8a8_block(aq, sa, wq, sw, fmt)
        A, W = _dequant(aq, sa, wq, sw, fmt)
        t = (torch.from_numpy(A) @ torch.from_numpy(W).T).numpy()
        assert np.all(np.abs(ref - t) <= 1e-12 * absref + 1e-300)
        tabs = (torch.from_numpy(np.abs(A)) @ torch.from_numpy(np.abs(W)).T).numpy()
        assert np.allclose(absref, tabs, rtol=1e-12, atol=0)


def test_exact_rational_brute_force():
    aq, sa, wq, sw = _quantized_pair(2, 128, 256, 9)
    ref, absref = oracle.gemm_w8a8_block(aq, sa, wq, sw)
    dec = oracle.e4m3_decode_all()
    for m in range(2):
        for n in range(0, 128, 9):
            exact = Fraction(0)
            for kb in range(2):
                sc = Fraction(float(sa[kb, m])) * Fraction(float(sw[n // 128, kb]))
                p = sum(Fraction(dec[aq[m, k]]) * Fraction(dec[wq[n, k]])
                        for k in range(kb * 128, kb * 128 + 128))
                exact += sc * p
            assert abs(Fraction(ref[m, n]) - exact) <= Fraction(absref[m, n]) * Fraction(1, 2 ** 50)


def test_identity_blocks_pin_operand_and_scale_indexing():
    """W made of identity 128x128 blocks on the block diagonal (codes 1.0) with a distinct scale
    per block: out[m, n] = sa[m, nb] * sw[nb, nb] * dec(a[m, n]).  A transposed operand, a
    swapped scale index or a wrong scale grid fails this."""
    M, K = 19, 384
    N = K
    a = inputs.randn_bf16((M, K), 1.0, 12, 0)
    aq, sa = oracle.quant_token_1x128(a)
    wq = np.zeros((N, K), np.uint8)
    for i in range(N):
        wq[i, i] = 0x38                     # 1.0
    sw = (np.arange(9, dtype=np.float32).reshape(3, 3) + 1) * np.float32(0.25)
    ref, _ = oracle.gemm_w8a8_block(aq, sa, wq, sw)
    dec = oracle.e4m3_decode_all()
    for m in range(M):
        for n in range(N):
            nb = n // 128
            want = float(sa[nb, m]) * float(sw[nb, nb]) * dec[aq[m, n]]
            assert ref[m, n] == want


def test_single_nonzero_k_block():
    """Only K-block 1 of A is nonzero: the result uses sa[m, 1] and sw[nb, 1] only."""
    aq, sa, wq, sw = _quantized_pair(8, 256, 384, 13)
    aq = aq.copy()
    aq[:, :128] = 0
    aq[:, 256:] = 0
    sw = sw.copy()
    sw[:, 0] = 1e9                        # would blow up if K-block 0 leaked in
    sw[:, 2] = 1e9
    ref, _ = oracle.gemm_w8a8_block(aq, sa, wq, sw)
    dec = oracle.e4m3_decode_all()
    P = dec[aq[:, 128:256]] @ dec[wq[:, 128:256]].T
    want = P * sa[1][:, None].astype(np.float64) * \
        np.repeat(sw[:, 1].astype(np.float64), 128)[None, :]
    assert np.allclose(ref, want, rtol=1e-15, atol=0)


def test_row_subset_equals_full():
    aq, sa, wq, sw = _quantized_pair(50, 128, 256, 14)
    full, fa = oracle.gemm_w8a8_block(aq, sa, wq, sw)
    rows = [49, 0, 17]
    part, pa = oracle.gemm_w8a8_block(aq, sa, wq, sw, rows=rows)
    assert np.array_equal(part, full[rows]) and np.array_equal(pa, fa[rows])


def test_grouped_equals_dense_per_expert():
    E, N, K = 4, 256, 256
    off = np.array([0, 5, 5, 133, 140], np.int32)      # expert 1 empty, expert 2 spans a tile
    M = int(off[-1])
    a = inputs.randn_bf16((M, K), 1.0, 15, 0)
    aq, sa = oracle.quant_token_1x128(a)
    wqs, sws = [], []
    for e in range(E):
        wq, sw = oracle.quant_weight_block(inputs.randn_bf16((N, K), 0.02, 15, 1 + e))
        wqs.append(wq)
        sws.append(sw)
    wq3, sw3 = np.stack(wqs), np.stack(sws)
    ref, absref = oracle.grouped_gemm_w8a8_block(aq, sa, wq3, sw3, off)
    for e in range(E):
        lo, hi = off[e], off[e + 1]
        if hi == lo:
            continue
        d, da = oracle.gemm_w8a8_block(aq, sa, wqs[e], sws[e], rows=np.arange(lo, hi))
        assert np.array_equal(ref[lo:hi], d) and np.array_equal(absref[lo:hi], da)


def test_tolerance_helper():
    ref = np.array([0.0, 1.0, -3.0, 2.0 ** -130])
    absref = np.array([0.0, 2.0, 3.0, 0.0])
    tol = oracle.gemm_tolerance(ref, absref)
    assert tol[0] == 2.0 ** -133
    assert tol[1] == 8e-3 * 2 + 2.0 ** -7
    assert tol[2] == 8e-3 * 3 + 2.0 ** -6
    assert tol[3] == 2.0 ** -133


# --- the tight fp32 bound the GPU tests apply, and its negative control ---------------------------

def _bf16_round(x):
    return inputs.bf16_bits_to_f32(inputs.to_bf16_bits(np.asarray(x, np.float32))).astype(
        np.float64)


def _promoted_model(aq, sa, wq, sw, bf16_partials: bool):
    """A model of per-K-block promotion run on the CPU from the decoded codes: fp32 partials P_kb
    (exact here), c = fp32(sa sw), acc = fp32(acc + P_kb c) with one rounding per K-block, bf16
    out.  With bf16_partials the planted mistake rounds P_kb and c to bf16 first."""
    dec = oracle.e4m3_decode_all()
    M, K = aq.shape
    N = wq.shape[0]
    KB = K // 128
    A = dec[aq].reshape(M, KB, 128)
    W = dec[wq].reshape(N, KB, 128)
    P = np.einsum("mbk,nbk->mnb", A, W)                     # exact in fp64
    c = (sa.T[:, None, :].astype(np.float32) *
         np.repeat(sw, 128, axis=0)[None, :, :].astype(np.float32)).astype(np.float32)
    acc = np.zeros((M, N), np.float32)
    for b in range(KB):
        p = P[:, :, b].astype(np.float32).astype(np.float64)
        cb = c[:, :, b].astype(np.float64)
        if bf16_partials:
            p, cb = _bf16_round(p), _bf16_round(cb)
        acc = (acc.astype(np.float64) + p * cb).astype(np.float32)   # one rounding (as an FMA)
    return _bf16_round(acc)


def test_tight_bound_admits_fp32_promotion_and_rejects_bf16_partials():
    """The GPU tests' second gate, |out - ref| <= ulp_bf16(|ref|)/2 + (K/128 + 8) 2^-23 absref,
    holds for a faithful fp32 promotion model on every element, and rejects a kernel that rounds
    each K-block partial and each sa*sw to bf16 on a large share of the elements (that mistake
    passes the stated 8e-3 tolerance everywhere)."""
    from helpers import promoted_steps, tight_gemm_bound
    for M, N, K, seed in ((16, 1024, 4096, 0), (64, 512, 512, 1)):
        aq, sa, wq, sw = _quantized_pair(M, N, K, 90 + seed)
        ref, absref = oracle.gemm_w8a8_block(aq, sa, wq, sw)
        bound = tight_gemm_bound(ref, absref, promoted_steps(K))
        good = _promoted_model(aq, sa, wq, sw, False)
        bad = _promoted_model(aq, sa, wq, sw, True)
        assert np.all(np.abs(good - ref) <= bound)
        assert np.all(np.abs(bad - ref) <= oracle.gemm_tolerance(ref, absref))
        assert np.mean(np.abs(bad - ref) > bound) > 0.2
