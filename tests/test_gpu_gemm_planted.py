"""Multi-tile GEMM parity with planted scales, every output element checked under both gates (the
stated tolerance and the tight fp32 bound).

Every activation scale sa[m, kb] is multiplied by its own power of two, 2^((3m + 5kb) mod 11 - 5),
and every weight-block scale sw[nb, kb] by its own factor 1 + ((7nb + 3kb) mod 29) / 32, so the
K-blocks of one output weigh differently and a wrong row, K-block, tile, expert, split or head
group in the scale indexing moves that output far outside the tight bound.  Shapes span many
tiles per persistent CTA with ragged edges; the grouped case reaches experts past the hundredth.
Sources: the per-K-block promotion out[m, n] = sum_kb sa[m, kb] sw[nb, kb] P_kb[m, n] of blockwise
W8A8 ("FP8-RL ...", abstract (i); "DeepSeek V4 ... (vLLM PR 54894 analysis)", sections 2-3).
"""
import numpy as np
import pytest
import torch

import oracle
import fp8_blockwise_w8a8_b200 as fq
from fp8_blockwise_w8a8_b200 import inputs

from helpers import (assert_within_gemm_tolerance, dev_f32, dev_u8, host_bf16_f64,
                     promoted_steps, tmem_steps)

pytestmark = pytest.mark.gpu


def _plant_sa(sa):
    KB, lds = sa.shape
    f = (3 * np.arange(lds)[None, :] + 5 * np.arange(KB)[:, None]) % 11 - 5
    return (sa * np.ldexp(np.float32(1.0), f)).astype(np.float32)


def _plant_sw_f32(sw):
    NB, KB = sw.shape[-2:]
    g = 1 + ((7 * np.arange(NB)[:, None] + 3 * np.arange(KB)[None, :]) % 29) / 32
    return (sw * g.astype(np.float32)).astype(np.float32)


def _operands(M, N, K, seed, fmt=oracle.SCALE_F32):
    a = inputs.randn_bf16((M, K), 1.0, seed, 0)
    w = inputs.randn_bf16((N, K), 0.02, seed, 1)
    aq, sa = oracle.quant_token_1x128(a, lds=(M + 7) // 8 * 8)
    wq, sw = oracle.quant_weight_block(w, fmt)
    return aq, _plant_sa(sa), wq, sw


def test_dense_planted_scales_all_rows():
    M, N, K = 1000, 9600, 1024
    aq, sa, wq, sw = _operands(M, N, K, 100)
    sw = _plant_sw_f32(sw)
    o = fq.gemm_w8a8_block(dev_u8(aq), dev_f32(sa), dev_u8(wq), dev_f32(sw), 0)
    assert fq.check_device_error() == 0
    ref, absref = oracle.gemm_w8a8_block(aq, sa, wq, sw, 0)
    assert_within_gemm_tolerance(host_bf16_f64(o), ref, absref, "dense planted",
                                 steps=promoted_steps(K))


def test_dense_planted_e8m0_weight_scales():
    M, N, K = 300, 2560, 1536
    aq, sa, wq, sw = _operands(M, N, K, 101, oracle.SCALE_E8M0)
    NB, KB = sw.shape
    sw = (sw.astype(np.int32) + (7 * np.arange(NB)[:, None] + 3 * np.arange(KB)[None, :]) % 9
          - 4).astype(np.uint8)
    o = fq.gemm_w8a8_block(dev_u8(aq), dev_f32(sa), dev_u8(wq), dev_u8(sw), 1)
    assert fq.check_device_error() == 0
    ref, absref = oracle.gemm_w8a8_block(aq, sa, wq, sw, 1)
    assert_within_gemm_tolerance(host_bf16_f64(o), ref, absref, "dense planted e8m0",
                                 steps=promoted_steps(K))


def test_grouped_planted_scales_experts_past_one_hundred():
    _, off = inputs.moe_routing(tokens=1024, experts=128, topk=8)
    E, N, K = 128, 384, 512
    M = int(off[-1])
    assert all(off[e + 1] > off[e] for e in (100, 110, 127))
    aq, sa = oracle.quant_token_1x128(inputs.randn_bf16((M, K), 1.0, 102, 0),
                                      lds=(M + 7) // 8 * 8)
    sa = _plant_sa(sa)
    w = inputs.randn_bf16((E * N, K), 0.02, 102, 1)
    wq, sw = oracle.quant_weight_block(w, 0)
    wq3 = wq.reshape(E, N, K)
    sw3 = _plant_sw_f32(sw.reshape(E, N // 128, K // 128) *
                        (1 + np.arange(E, dtype=np.float32) / 64)[:, None, None])
    o = fq.grouped_gemm_w8a8_block(dev_u8(aq), dev_f32(sa), dev_u8(wq3), dev_f32(sw3),
                                   torch.from_numpy(off).cuda(), 0)
    assert fq.check_device_error() == 0
    ref, absref = oracle.grouped_gemm_w8a8_block(aq, sa, wq3, sw3, off, 0)
    assert_within_gemm_tolerance(host_bf16_f64(o), ref, absref, "grouped planted",
                                 steps=promoted_steps(K))


@pytest.mark.parametrize("splits", [3, 5])
def test_splitk_planted_scales(splits):
    M, N, K = 200, 1024, 1536
    aq, sa, wq, sw = _operands(M, N, K, 103)
    sw = _plant_sw_f32(sw)
    o = fq.gemm_w8a8_block_splitk(dev_u8(aq), dev_f32(sa), dev_u8(wq), dev_f32(sw), 0,
                                  splits=splits)
    assert fq.check_device_error() == 0
    ref, absref = oracle.gemm_w8a8_block(aq, sa, wq, sw, 0)
    assert_within_gemm_tolerance(host_bf16_f64(o), ref, absref, f"split-K {splits} planted",
                                 steps=promoted_steps(K, splits))


def test_block_diag_planted_scales_all_groups():
    G, M, N_g, K_g = 4, 300, 512, 512
    aq, sa = oracle.quant_token_1x128(inputs.randn_bf16((M, G * K_g), 1.0, 104, 0),
                                      lds=(M + 7) // 8 * 8)
    sa = _plant_sa(sa)
    w = inputs.randn_bf16((G * N_g, K_g), 0.02, 104, 1)
    wq, sw = oracle.quant_weight_block(w, 0)
    wq3 = wq.reshape(G, N_g, K_g)
    sw3 = _plant_sw_f32(sw.reshape(G, N_g // 128, K_g // 128) *
                        np.array([1.0, 3.0, 0.25, 7.0], np.float32)[:, None, None])
    o = fq.gemm_w8a8_block_diag(dev_u8(aq), dev_f32(sa), dev_u8(wq3), dev_f32(sw3), 0)
    assert fq.check_device_error() == 0
    ref, absref = oracle.gemm_w8a8_block_diag(aq, sa, wq3, sw3, 0)
    assert_within_gemm_tolerance(host_bf16_f64(o), ref, absref, "block-diagonal planted",
                                 steps=promoted_steps(K_g))


def test_mx_planted_power_of_two_scales():
    """Hardware block scaling: planted powers of two on both operands (the MX GEMM takes only
    powers of two)."""
    M, N, K = 500, 2048, 1024
    x = inputs.randn_bf16((M, K), 1.0, 105, 0)
    cos = np.ones((1, 1), np.float32)
    aq, sa = oracle.inverse_rope_quant(x.reshape(M, 1, K), np.zeros(M, np.int64), cos, cos, 0,
                                       fmt=1, lds=(M + 3) // 4 * 4)
    sa = _plant_sa(sa)
    wq, sw = oracle.quant_weight_block(inputs.randn_bf16((N, K), 0.02, 105, 1), 1)
    NB, KB = sw.shape
    sw = (sw.astype(np.int32) + (7 * np.arange(NB)[:, None] + 3 * np.arange(KB)[None, :]) % 9
          - 4).astype(np.uint8)
    o = fq.gemm_w8a8_mx(dev_u8(aq), dev_f32(sa), dev_u8(wq), dev_u8(sw))
    assert fq.check_device_error() == 0
    ref, absref = oracle.gemm_w8a8_block(aq, sa, wq, sw, 1)
    assert_within_gemm_tolerance(host_bf16_f64(o), ref, absref, "mx planted",
                                 steps=tmem_steps(K))


def test_rowwise_planted_scales():
    M, N, K = 700, 2560, 512
    aq, sa = oracle.quant_rowwise(inputs.randn_bf16((M, K), 1.0, 106, 0))
    wq, sw = oracle.quant_rowwise(inputs.randn_bf16((N, K), 0.02, 106, 1))
    sa = (sa * np.ldexp(np.float32(1.0), np.arange(M) % 11 - 5)).astype(np.float32)
    sw = (sw * (1 + (np.arange(N) % 29) / 32).astype(np.float32)).astype(np.float32)
    o = fq.gemm_w8a8_rowwise(dev_u8(aq), dev_f32(sa), dev_u8(wq), dev_f32(sw))
    assert fq.check_device_error() == 0
    ref, absref = oracle.gemm_w8a8_rowwise(aq, sa, wq, sw)
    assert_within_gemm_tolerance(host_bf16_f64(o), ref, absref, "rowwise planted",
                                 steps=tmem_steps(K))
