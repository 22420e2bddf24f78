"""GPU parity of the split-K block-scaled GEMM (K-blocks of a tile spread over several CTAs, fp32
partials summed in split order) against the oracle's fp64 reference, with the same per-element
tolerance as the unsplit GEMM: |out - ref| <= 8e-3 * sum_k |dec(a) sa dec(w) sw| + 1 bf16 ulp.
Splitting only reorders the fp32 promotion sum over K-blocks ("SGLang ... (PR 21403 analysis)"
section 3: the GEMM consumes (codes, scale) pairs and writes bf16)."""
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


def _dev(aq, sa, wq, sw, fmt):
    return dev_u8(aq), dev_f32(sa), dev_u8(wq), dev_f32(sw) if fmt == 0 else dev_u8(sw)


@pytest.mark.parametrize("M,N,K,splits", [(1, 128, 256, 2), (70, 384, 640, 5), (128, 512, 1152, 3),
                                          (200, 256, 512, 4), (129, 128, 384, 3)])
@pytest.mark.parametrize("fmt", [oracle.SCALE_F32, oracle.SCALE_E8M0])
def test_splitk_ragged(M, N, K, splits, fmt):
    a = inputs.randn_bf16((M, K), 1.0, 60, M + N + K)
    w = inputs.randn_bf16((N, K), 0.02, 61, M + N + K)
    aq, sa, wq, sw = _quantize(a, w, fmt, lds=(M + 7) // 8 * 8)
    d = _dev(aq, sa, wq, sw, fmt)
    ws = fq.splitk_workspace(M, N, K, splits, device="cuda")
    buf = torch.full((M, N + 8), float("nan"), dtype=torch.bfloat16, device="cuda")
    o = fq.gemm_w8a8_block_splitk(*d, fmt, splits=splits, workspace=ws, out=buf[:, :N])
    assert fq.check_device_error() == 0
    assert torch.isnan(buf[:, N:].float()).all()
    ref, absref = oracle.gemm_w8a8_block(aq, sa, wq, sw, fmt)
    assert_within_gemm_tolerance(host_bf16_f64(o), ref, absref, steps=promoted_steps(K, splits))
    # the same workspace serves the next call, even filled with garbage (every partial is written
    # before it is read); the fixed summation order makes the second result bit-identical
    ws.fill_(0xFF)
    o2 = fq.gemm_w8a8_block_splitk(*d, fmt, splits=splits, workspace=ws)
    assert fq.check_device_error() == 0
    assert torch.equal(o.view(torch.int16), o2.view(torch.int16))


def test_splits_equal_k_blocks_and_single_split():
    M, N, K = 96, 256, 512
    aq, sa, wq, sw = _quantize(inputs.randn_bf16((M, K), 1.0, 62, 0),
                               inputs.randn_bf16((N, K), 0.02, 62, 1), 0)
    d = _dev(aq, sa, wq, sw, 0)
    ref, absref = oracle.gemm_w8a8_block(aq, sa, wq, sw, 0)
    for s in (1, K // 128):
        o = fq.gemm_w8a8_block_splitk(*d, 0, splits=s)
        assert fq.check_device_error() == 0
        assert_within_gemm_tolerance(host_bf16_f64(o), ref, absref, what=f"splits={s}",
                                     steps=promoted_steps(K, s))
    # one split is the unsplit kernel
    o1 = fq.gemm_w8a8_block_splitk(*d, 0, splits=1, workspace=torch.empty(0, device="cuda"))
    o0 = fq.gemm_w8a8_block(*d, 0)
    assert torch.equal(o1.view(torch.int16), o0.view(torch.int16))


def test_decode_long_k_auto_splits_sampled_rows():
    """Decode down projection (128 x 4096 x 12288) with the library's split choice, as the bench
    runs it: long K with few tiles is where splitting pays."""
    M, N, K = 128, 4096, 12288
    assert fq.gemm_splitk_workspace_bytes(M, N, K, 0) > 0       # splits on 148 SMs
    aq, sa, wq, sw = _quantize(inputs.randn_bf16((M, K), 1.0, 64, 0),
                               inputs.randn_bf16((N, K), 0.02, 64, 1), 0)
    dv = _dev(aq, sa, wq, sw, 0)
    ws = fq.splitk_workspace(M, N, K, 0, device="cuda")
    for _ in range(3):   # repeated calls reuse the workspace
        o = fq.gemm_w8a8_block_splitk(*dv, 0, splits=0, workspace=ws)
    assert fq.check_device_error() == 0
    rows = [0, 1, 63, 64, 126, 127]
    ref, absref = oracle.gemm_w8a8_block(aq, sa, wq, sw, 0, rows=rows)
    # the library picks at most one split per K-block
    assert_within_gemm_tolerance(host_bf16_f64(o)[rows], ref, absref,
                                 steps=promoted_steps(K, K // 128))


def test_decode_auto_choice_does_not_split_short_k():
    """128 x 12288 x 4096: splitting was measured not to pay; the library picks one split."""
    assert fq.gemm_splitk_workspace_bytes(128, 12288, 4096, 0) == 0


def test_workspace_too_small_is_rejected():
    M, N, K = 64, 256, 512
    need = fq.gemm_splitk_workspace_bytes(M, N, K, 2)
    assert need == 2 * 128 * 256 * 4
    aq = torch.zeros((M, K), dtype=torch.uint8, device="cuda")
    sa = torch.ones((K // 128, M), dtype=torch.float32, device="cuda")
    wq = torch.zeros((N, K), dtype=torch.uint8, device="cuda")
    sw = torch.ones((N // 128, K // 128), dtype=torch.float32, device="cuda")
    small = torch.zeros(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(fq.Fp8qError):
        fq.gemm_w8a8_block_splitk(aq, sa, wq, sw, 0, splits=2, workspace=small)
