"""GPU parity of the per-token / per-channel ("PTPC") path against the oracle: row-wise quantization
(bit-exact, with and without RMSNorm) and the per-channel GEMM (per-element tolerance
|out - ref| <= 8e-3 * sum_k |dec(a) dec(w)| sa sw + 1 bf16 ulp).  "SGLang ... (PR 21403
analysis)" sections 1-3: group_size 0 = per token, CHANNEL weight scales, GEMM on
(codes, x_scale) with weight_scale, bf16 out."""
import numpy as np
import pytest
import torch

import oracle
import fp8_blockwise_w8a8_b200 as fq
from fp8_blockwise_w8a8_b200 import inputs

from helpers import (assert_within_gemm_tolerance, dev_bf16, dev_f32, dev_u8, host_bf16_f64,
                     tmem_steps)

pytestmark = pytest.mark.gpu


def _check_rowwise(x, gamma=None, eps=1e-6):
    xd = dev_bf16(x)
    gd = None if gamma is None else dev_bf16(gamma)
    q, s = fq.quant_rowwise(xd, gd, eps)
    assert fq.check_device_error() == 0
    qr, sr = oracle.quant_rowwise(x, gamma, eps)
    assert np.array_equal(q.cpu().numpy(), qr)
    assert np.array_equal(s.cpu().numpy(), sr)


@pytest.mark.parametrize("M,K", [(1, 128), (37, 768), (300, 4096), (64, 16384)])
@pytest.mark.parametrize("norm", [False, True])
def test_quant_rowwise_bit_exact(M, K, norm):
    x = inputs.randn_bf16((M, K), 1.0, 80, M + K)
    g = inputs.randn_bf16((K,), 0.5, 80, K + 1) if norm else None
    _check_rowwise(x, g)


def test_quant_rowwise_zero_and_wide_range_rows():
    x = inputs.randn_bf16((8, 1024), 1.0, 81, 0)
    x[1] = 0                                   # zero row -> s = 1, codes 0
    x[2, ::7] = 0x0001                         # tiny subnormal bf16 values
    x[3, 5] = 0x7F00                           # a huge value: everything else underflows
    x[4] = 0x8000                              # negative zeros
    _check_rowwise(x)


def test_quant_rowwise_prefill_and_per_channel_weight():
    d = inputs.prefill_linear(with_weight=False)
    _check_rowwise(d["X"], d["gamma"], d["eps"])               # per token, fused RMSNorm
    w = inputs.randn_bf16((4096, 4096), 0.02, 82, 0)
    _check_rowwise(w)                                          # per output channel


def _run_gemm(aq, sa, wq, sw, rows=None, pad=0):
    M, K = aq.shape
    N = wq.shape[0]
    out = None
    if pad:
        buf = torch.full((M, N + pad), float("nan"), dtype=torch.bfloat16, device="cuda")
        out = buf[:, :N]
    o = fq.gemm_w8a8_rowwise(dev_u8(aq), dev_f32(sa), dev_u8(wq), dev_f32(sw), out=out)
    assert fq.check_device_error() == 0
    if pad:
        assert torch.isnan(buf[:, N:].float()).all()
    got = host_bf16_f64(o)
    ref, absref = oracle.gemm_w8a8_rowwise(aq, sa, wq, sw, rows=rows)
    assert_within_gemm_tolerance(got if rows is None else got[rows], ref, absref,
                                 steps=tmem_steps(K))
    return got, ref


@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (64, 256, 512), (129, 384, 640),
                                   (300, 512, 384), (257, 1024, 1152)])
def test_gemm_rowwise_ragged(M, N, K):
    aq, sa = oracle.quant_rowwise(inputs.randn_bf16((M, K), 1.0, 83, M + N + K))
    wq, sw = oracle.quant_rowwise(inputs.randn_bf16((N, K), 0.02, 83, M + N + K + 1))
    _run_gemm(aq, sa, wq, sw, pad=8)


def test_gemm_rowwise_identity_is_exact():
    """W = identity codes (1.0) with per-channel scales: out = bf16(sa * sw * dec(a))."""
    M, K = 70, 256
    aq, sa = oracle.quant_rowwise(inputs.randn_bf16((M, K), 1.0, 84, 0))
    wq = np.zeros((K, K), np.uint8)
    wq[np.arange(K), np.arange(K)] = 0x38
    sw = np.linspace(0.25, 4.0, K).astype(np.float32)
    got, ref = _run_gemm(aq, sa, wq, sw)
    assert np.all(np.abs(got - ref) <= 2 * oracle.bf16_ulp(ref))   # two fp32 roundings, one bf16


def test_gemm_rowwise_prefill_full_size_sampled_rows():
    """The bench's PTPC prefill shape (8192 x 24576 x 4096), rows from the first, a middle and the
    last m-tile across all N."""
    d = inputs.prefill_linear()
    aq, sa = oracle.quant_rowwise(d["X"], d["gamma"], d["eps"])
    wq, sw = oracle.quant_rowwise(d["W"])
    _run_gemm(aq, sa, wq, sw, rows=[0, 77, 4095, 4096 + 128, 8191])
