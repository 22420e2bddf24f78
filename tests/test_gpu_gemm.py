"""GPU parity of the block-scaled W8A8 GEMM (dense and grouped) against the oracle's fp64 reference.

Tolerance (per element): |out - ref| <= 8e-3 * sum_k |dec(a) sa dec(w) sw| + 1 bf16 ulp of |ref|,
and the tight bound of fp32 promotion, |out - ref| <= ulp_bf16(|ref|)/2 + (K/128 + 8) 2^-23 absref.
The GEMM is fed codes and scales produced by the oracle, so the check isolates the GEMM.
Sources: "SGLang ... (PR 21403 analysis)" section 3 (GEMM on the pre-quantized (codes, scale)
pair, bf16 out); "DeepSeek V4 ... (vLLM PR 54894 analysis)" section 3 (batched per-group GEMM).
"""
import numpy as np
import pytest
import torch

import oracle
import fp8_blockwise_w8a8_b200 as fq
from fp8_blockwise_w8a8_b200 import inputs

from helpers import assert_within_gemm_tolerance, dev_f32, dev_u8, host_bf16_f64, promoted_steps

pytestmark = pytest.mark.gpu


def _quantize(a_bits, w_bits, fmt, lds=None):
    lds = (a_bits.shape[0] + 3) // 4 * 4 if lds is None else lds
    aq, sa = oracle.quant_token_1x128(a_bits, lds=lds)
    wq, sw = oracle.quant_weight_block(w_bits, fmt)
    return aq, sa, wq, sw


def _run_dense(aq, sa, wq, sw, fmt, rows=None, pad=0):
    M, K = aq.shape
    N = wq.shape[0]
    out = None
    if pad:
        buf = torch.full((M, N + pad), float("nan"), dtype=torch.bfloat16, device="cuda")
        out = buf[:, :N]
    o = fq.gemm_w8a8_block(dev_u8(aq), dev_f32(sa), dev_u8(wq),
                           dev_f32(sw) if fmt == 0 else dev_u8(sw), fmt, out=out)
    assert fq.check_device_error() == 0
    if pad:
        assert torch.isnan(buf[:, N:].float()).all()        # columns beyond N untouched
    got = host_bf16_f64(o)
    ref, absref = oracle.gemm_w8a8_block(aq, sa, wq, sw, fmt, rows=rows)
    assert_within_gemm_tolerance(got if rows is None else got[rows], ref, absref,
                                 steps=promoted_steps(aq.shape[1]))
    return got, ref


@pytest.mark.parametrize("fmt", [oracle.SCALE_F32, oracle.SCALE_E8M0])
def test_tiny_linear(fmt):
    d = inputs.tiny_linear()
    _run_dense(*_quantize(d["A"], d["W"], fmt), fmt)


@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (127, 256, 256), (129, 384, 640),
                                   (300, 512, 384), (257, 128, 1152)])
def test_ragged_shapes(M, N, K):
    a = inputs.randn_bf16((M, K), 1.0, 40, M + N + K)
    w = inputs.randn_bf16((N, K), 0.02, 41, M + N + K)
    _run_dense(*_quantize(a, w, oracle.SCALE_F32, lds=(M + 7) // 8 * 8), oracle.SCALE_F32,
               pad=8)


def test_identity_blocks_exact():
    """W = identity 128x128 blocks with per-block scales: out = bf16(sa * sw * dec(a))."""
    M, K = 70, 256
    a = inputs.randn_bf16((M, K), 1.0, 42, 0)
    aq, sa = oracle.quant_token_1x128(a, lds=72)
    wq = np.zeros((K, K), np.uint8)
    wq[np.arange(K), np.arange(K)] = 0x38
    sw = np.array([[0.5, 1e9], [1e9, 0.25]], np.float32)
    got, ref = _run_dense(aq, sa, wq, sw, 0)
    # a single product per output: the bf16 result is within one bf16 ulp of the exact value
    assert np.all(np.abs(got - ref) <= oracle.bf16_ulp(ref))


def test_single_nonzero_k_block():
    aq, sa, wq, sw = _quantize(inputs.randn_bf16((130, 384), 1.0, 43, 0),
                               inputs.randn_bf16((256, 384), 0.02, 43, 1), 0)
    aq[:, :128] = 0
    aq[:, 256:] = 0
    sw[:, 0] = 1e6
    sw[:, 2] = 1e6
    _run_dense(aq, sa, wq, sw, 0)


@pytest.mark.parametrize("M,N,K,fmt", [(1000, 9600, 512, oracle.SCALE_F32),
                                       (300, 10240, 256, oracle.SCALE_E8M0),
                                       (512, 19200, 384, oracle.SCALE_F32)])
def test_many_tiles_ragged(M, N, K, fmt):
    """More tiles than SMs (several tiles per persistent CTA), M not a multiple of 128 or 256 and N
    ending in a half 256-column tile, both scale formats."""
    a = inputs.randn_bf16((M, K), 1.0, 42, M + N + K)
    w = inputs.randn_bf16((N, K), 0.02, 43, M + N + K)
    rows = sorted({0, 127, 128, 255, 256, M // 2, M - 1})
    _run_dense(*_quantize(a, w, fmt, lds=(M + 7) // 8 * 8), fmt, rows=rows, pad=8)


def test_decode_full_size_sampled_rows():
    d = inputs.decode_linear()
    aq, sa, wq, sw = _quantize(d["A"], d["W"], 0)
    _run_dense(aq, sa, wq, sw, 0, rows=[0, 1, 63, 64, 126, 127])


def test_prefill_full_size_sampled_rows():
    """Full prefill shape (8192 x 24576 x 4096) on the bench's launch configuration; the oracle
    checks rows from the first, a middle and the last m-tile across all N."""
    d = inputs.prefill_linear()
    aq, sa = oracle.rmsnorm_quant_token(d["X"], d["gamma"], d["eps"])
    wq, sw = oracle.quant_weight_block(d["W"], 0)
    _run_dense(aq, sa, wq, sw, 0, rows=[0, 77, 4095, 4096 + 128, 8191])


# --- grouped ----------------------------------------------------------------------------------

def _run_grouped(aq, sa, wq3, sw3, off, fmt, rows=None):
    o = fq.grouped_gemm_w8a8_block(dev_u8(aq), dev_f32(sa), dev_u8(wq3),
                                   dev_f32(sw3) if fmt == 0 else dev_u8(sw3),
                                   torch.from_numpy(off).cuda(), fmt)
    assert fq.check_device_error() == 0
    got = host_bf16_f64(o)
    ref, absref = oracle.grouped_gemm_w8a8_block(aq, sa, wq3, sw3, off, fmt, rows=rows)
    sel = got if rows is None else got[rows]
    assert_within_gemm_tolerance(sel, ref, absref, "grouped", steps=promoted_steps(aq.shape[1]))
    return got


@pytest.mark.parametrize("fmt", [oracle.SCALE_F32, oracle.SCALE_E8M0])
def test_grouped_small_with_empty_and_ragged_groups(fmt):
    E, N, K = 5, 384, 256
    off = np.array([0, 5, 5, 140, 141, 300], np.int32)
    M = int(off[-1])
    aq, sa = oracle.quant_token_1x128(inputs.randn_bf16((M, K), 1.0, 50, 0))
    wqs, sws = zip(*[oracle.quant_weight_block(inputs.randn_bf16((N, K), 0.02, 50, 1 + e), fmt)
                     for e in range(E)])
    _run_grouped(aq, sa, np.stack(wqs), np.stack(sws), off, fmt)


def test_grouped_moe_full_size_sampled_rows():
    d = inputs.moe()
    off = d["offsets"]
    rng = np.random.default_rng(1)
    experts = [0, 1, 2, 63, 127] + list(rng.choice(128, 4, replace=False))
    rows = sorted({int(off[e]) for e in experts} | {int(off[e + 1]) - 1 for e in experts})
    for a_key, w_key in (("A_gateup", "W_gateup"), ("A_down", "W_down")):
        aq, sa = oracle.quant_token_1x128(d[a_key])
        W = d[w_key]
        E, N, K = W.shape
        wq3, sw3 = oracle.quant_weight_block(W.reshape(E * N, K), 0)
        _run_grouped(aq, sa, wq3.reshape(E, N, K), sw3.reshape(E, N // 128, K // 128), off, 0,
                     rows=rows)
