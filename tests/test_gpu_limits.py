"""GPU parity at the size limits the C ABI declares: the block-scaled GEMM at K = 32768 (256
K-blocks, the largest K its scale staging holds) with ragged M and N, the grouped GEMM with 1024
experts (the most it takes), most of them empty, the 1x128 quant at K = 16384 in every scale
format, a 128-row weight 65536 wide, and the batched requant at its 2048-matrix maximum.  Codes
and scales bit-exact; GEMM outputs within both gates (the stated tolerance and the fp32 bound).
Sources: the pages' 128-divisibility rule ("DeepSeek V4 ... (vLLM PR 54894 analysis)", section
2) and the blockwise W8A8 layer of "FP8-RL ...", abstract (i)."""
import numpy as np
import pytest
import torch

import oracle
import fp8_blockwise_w8a8_b200 as fq
from fp8_blockwise_w8a8_b200 import inputs

from helpers import (assert_within_gemm_tolerance, dev_bf16, dev_f32, dev_u8, host_bf16_f64,
                     promoted_steps)

pytestmark = pytest.mark.gpu


def test_gemm_at_the_largest_k():
    M, N, K = 130, 384, 32768
    a = inputs.randn_bf16((M, K), 1.0, 120, 0)
    w = inputs.randn_bf16((N, K), 0.02, 120, 1)
    aq, sa = oracle.quant_token_1x128(a, lds=136)
    wq, sw = oracle.quant_weight_block(w, oracle.SCALE_F32)
    # distinct scales along K so that a K-block indexing slip far into K shows
    sa = (sa * np.ldexp(np.float32(1.0), (np.arange(K // 128) % 7 - 3))[:, None]).astype(np.float32)
    o = fq.gemm_w8a8_block(dev_u8(aq), dev_f32(sa), dev_u8(wq), dev_f32(sw), 0)
    assert fq.check_device_error() == 0
    ref, absref = oracle.gemm_w8a8_block(aq, sa, wq, sw, 0)
    assert_within_gemm_tolerance(host_bf16_f64(o), ref, absref, "K = 32768",
                                 steps=promoted_steps(K))


def test_grouped_gemm_with_the_most_experts():
    E, N, K = 1024, 256, 256
    rng = np.random.default_rng(121)
    counts = np.zeros(E, np.int64)
    live = rng.choice(E, 40, replace=False)
    counts[live] = rng.integers(1, 300, 40)
    counts[E - 1] = 5                                # the last expert has rows
    off = np.zeros(E + 1, np.int32)
    off[1:] = np.cumsum(counts)
    M = int(off[-1])
    aq, sa = oracle.quant_token_1x128(inputs.randn_bf16((M, K), 1.0, 121, 0),
                                      lds=(M + 7) // 8 * 8)
    w = inputs.randn_bf16((E * N, K), 0.02, 121, 1)
    wq, sw = oracle.quant_weight_block(w, oracle.SCALE_F32)
    wq3, sw3 = wq.reshape(E, N, K), sw.reshape(E, N // 128, K // 128)
    o = fq.grouped_gemm_w8a8_block(dev_u8(aq), dev_f32(sa), dev_u8(wq3), dev_f32(sw3),
                                   torch.from_numpy(off).cuda(), 0)
    assert fq.check_device_error() == 0
    ref, absref = oracle.grouped_gemm_w8a8_block(aq, sa, wq3, sw3, off, 0)
    assert_within_gemm_tolerance(host_bf16_f64(o), ref, absref, "1024 experts",
                                 steps=promoted_steps(K))


@pytest.mark.parametrize("fmt", ["f32", "e8m0"])
def test_token_quant_at_the_largest_k(fmt):
    M, K = 300, 16384
    x = inputs.randn_bf16((M, K), 1.0, 122, 0)
    g = inputs.to_bf16_bits(np.random.default_rng(122).uniform(0.5, 1.5, K).astype(np.float32))
    f = fq.scale_format(fmt)
    for gamma in (None, g):
        q_ref, sa_ref = oracle.rmsnorm_quant_token(x, gamma, 1e-6, lds=M, fmt=f)
        sa_dev = torch.zeros((K // 128, M), dtype=torch.float32, device="cuda")
        q, sa = fq.rmsnorm_quant_token(dev_bf16(x), None if gamma is None else dev_bf16(gamma),
                                       1e-6, out_sa=sa_dev, scale_fmt=fmt)
        assert fq.check_device_error() == 0
        assert np.array_equal(q.cpu().numpy(), q_ref)
        assert np.array_equal(sa.cpu().numpy().view(np.uint32), sa_ref.view(np.uint32))


@pytest.mark.parametrize("fmt", [oracle.SCALE_F32, oracle.SCALE_E8M0])
def test_weight_quant_very_wide(fmt):
    w = inputs.randn_bf16((128, 65536), 0.02, 123, fmt)
    q, s = fq.quant_weight_block(dev_bf16(w), fmt)
    assert fq.check_device_error() == 0
    q_ref, s_ref = oracle.quant_weight_block(w, fmt)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy(), s_ref)


def test_weight_batch_at_its_matrix_limit():
    """2048 matrices (the descriptor table's maximum) of 128 x 128 to 256 x 384 in one launch."""
    rng = np.random.default_rng(124)
    shapes = [(128 * int(rng.integers(1, 3)), 128 * int(rng.integers(1, 4))) for _ in range(2048)]
    ws = [inputs.randn_bf16(s, 0.02, 124, i) for i, s in enumerate(shapes)]
    batch = fq.WeightBatch([dev_bf16(w) for w in ws], "f32")
    qs, ss = batch.run()
    assert fq.check_device_error() == 0
    for i in (0, 1, 777, 2046, 2047):
        q_ref, s_ref = oracle.quant_weight_block(ws[i], oracle.SCALE_F32)
        assert np.array_equal(qs[i].cpu().numpy(), q_ref)
        assert np.array_equal(ss[i].cpu().numpy(), s_ref)
