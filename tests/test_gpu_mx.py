"""GPU parity of the hardware block-scaled (MX) W8A8 GEMM: E8M0 weight scales and power-of-two
activation scales applied by the tensor core (tcgen05.mma kind::mxf8f6f4.block_scale), dense and
block-diagonal over head groups, against the oracle's fp64 reference within the GEMM tolerance
|out - ref| <= 8e-3 * sum_k |dec(a) sa dec(w) sw| + 1 bf16 ulp of |ref|.  Operands come from the
oracle's quantizers.  Source: "DeepSeek V4 ... (vLLM PR 54894 analysis)" sections 1-3 (E8M0
scales; the MX-scaled batched GEMM after the inverse-RoPE quant)."""
import numpy as np
import pytest
import torch

import oracle
import fp8_blockwise_w8a8_b200 as fq
from fp8_blockwise_w8a8_b200 import inputs

from helpers import (assert_within_gemm_tolerance, dev_f32, dev_u8, host_bf16_f64,
                     promoted_steps, tmem_steps)

pytestmark = pytest.mark.gpu

E8M0 = oracle.SCALE_E8M0


def _act_e8m0(x_bits, lds=None):
    """1x128 quant with power-of-two scales: the oracle's inverse-RoPE quant with no rotary dims."""
    M, K = x_bits.shape
    cos = np.ones((1, 1), np.float32)
    return oracle.inverse_rope_quant(x_bits.reshape(M, 1, K), np.zeros(M, np.int64), cos, cos, 0,
                                     fmt=1, lds=lds)


def _weights(G, N_g, K_g, seed, std=0.02):
    w = inputs.randn_bf16((G, N_g, K_g), std, seed, 7)
    parts = [oracle.quant_weight_block(w[g], E8M0) for g in range(G)]
    return np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts])


def _run(aq, sa, wq, sw):
    o = fq.gemm_w8a8_mx(dev_u8(aq), dev_f32(sa), dev_u8(wq[0] if wq.shape[0] == 1 else wq),
                        dev_u8(sw[0] if sw.shape[0] == 1 else sw))
    assert fq.check_device_error() == 0
    return host_bf16_f64(o)


@pytest.mark.parametrize("M,N,K", [(1, 256, 128), (200, 384, 512), (129, 1024, 1024),
                                   (256, 128, 2048)])
def test_mx_dense_small(M, N, K):
    x = inputs.randn_bf16((M, K), 1.0, 80, M + N)
    aq, sa = _act_e8m0(x, lds=(M + 3) // 4 * 4)
    wq, sw = _weights(1, N, K, 80 + N)
    got = _run(aq, sa, wq, sw)
    ref, absref = oracle.gemm_w8a8_block(aq, sa, wq[0], sw[0], E8M0)
    assert_within_gemm_tolerance(got, ref, absref, f"mx {M}x{N}x{K}", steps=tmem_steps(K))


def test_mx_wide_scale_range():
    """Rows and weight blocks whose scales span many binades, and all-zero blocks (scale 1)."""
    M, N, K = 160, 512, 768
    x = inputs.bf16_bits_to_f32(inputs.randn_bf16((M, K), 1.0, 81, 0)).copy()
    x[::5] *= 1e12
    x[1::5] *= 1e-12
    x[2, 128:256] = 0.0
    x[3, :, ] *= np.where(np.arange(K) < 384, 1e6, 1e-6).astype(np.float32)
    aq, sa = _act_e8m0(inputs.to_bf16_bits(x), lds=160)
    w = inputs.bf16_bits_to_f32(inputs.randn_bf16((N, K), 0.02, 81, 1)).copy()
    w[:128] *= 1e8
    w[128:256, :128] = 0.0
    wq, sw = oracle.quant_weight_block(inputs.to_bf16_bits(w), E8M0)
    got = _run(aq, sa, wq[None], sw[None])
    ref, absref = oracle.gemm_w8a8_block(aq, sa, wq, sw, E8M0)
    assert_within_gemm_tolerance(got, ref, absref, "mx wide range", steps=tmem_steps(K))


@pytest.mark.parametrize("G,M,N_g,K_g", [(3, 200, 256, 384), (4, 64, 512, 256)])
def test_mx_block_diag_small(G, M, N_g, K_g):
    x = inputs.randn_bf16((M, G * K_g), 1.0, 82, G)
    aq, sa = _act_e8m0(x, lds=(M + 3) // 4 * 4)
    wq, sw = _weights(G, N_g, K_g, 82)
    got = _run(aq, sa, wq, sw)
    ref, absref = oracle.gemm_w8a8_block_diag(aq, sa, wq, sw, E8M0)
    assert_within_gemm_tolerance(got, ref, absref, f"mx diag G={G}", steps=tmem_steps(K_g))


def test_mx_matches_software_promotion_closely():
    """Same operands through the software-promoted block GEMM and the MX GEMM: both within the
    tolerance of the fp64 reference, and within a few bf16 ulp of each other."""
    M, N, K = 256, 512, 1024
    x = inputs.randn_bf16((M, K), 1.0, 83, 0)
    aq, sa = _act_e8m0(x)
    wq, sw = _weights(1, N, K, 83)
    mx = _run(aq, sa, wq, sw)
    sw_f32 = np.ldexp(1.0, sw[0].astype(np.int32) - 127).astype(np.float32)
    sp = host_bf16_f64(fq.gemm_w8a8_block(dev_u8(aq), dev_f32(sa), dev_u8(wq[0]),
                                          dev_f32(sw_f32), 0))
    ref, absref = oracle.gemm_w8a8_block(aq, sa, wq[0], sw[0], E8M0)
    assert_within_gemm_tolerance(sp, ref, absref, "software promotion", steps=promoted_steps(K))
    assert_within_gemm_tolerance(mx, ref, absref, "hardware scaling", steps=tmem_steps(K))
    assert np.all(np.abs(mx - sp) <= 4 * oracle.bf16_ulp(ref) + 2e-3 * absref)


def test_mx_non_power_of_two_scale_is_reported():
    M, N, K = 128, 256, 256
    x = inputs.randn_bf16((M, K), 1.0, 84, 0)
    aq, sa = _act_e8m0(x)
    sa = sa.copy()
    sa[1, 7] *= np.float32(1.5)
    wq, sw = _weights(1, N, K, 84)
    fq.gemm_w8a8_mx(dev_u8(aq), dev_f32(sa), dev_u8(wq[0]), dev_u8(sw[0]))
    assert fq.check_device_error() == fq.FP8Q_ERR_NOT_POW2
    assert fq.check_device_error() == 0


def test_mx_wo_a_full_size_sampled_rows():
    """The page's path at full size: inverse-RoPE quant with E8M0 scales (8192 tokens, 32 heads x
    512, 64 rotary dims) into the MX GEMM over 4 head groups of [1024, 4096]."""
    d = inputs.wo_a()
    G, N_g, K_g = d["W"].shape
    pos = torch.from_numpy(d["positions"]).cuda()
    q, sa = fq.inverse_rope_quant(torch.from_numpy(d["o"].view(np.int16)).view(torch.bfloat16)
                                  .cuda(), pos, dev_f32(d["cos"]), dev_f32(d["sin"]), 64, True,
                                  fq.FP8Q_SCALE_E8M0)
    parts = [oracle.quant_weight_block(d["W"][g], E8M0) for g in range(G)]
    wq = np.stack([p[0] for p in parts])
    sw = np.stack([p[1] for p in parts])
    out = fq.gemm_w8a8_mx(q, sa, dev_u8(wq), dev_u8(sw))
    assert fq.check_device_error() == 0
    T = d["o"].shape[0]
    rows = np.unique(np.concatenate([[0, 127, 128, T - 1],
                                     np.random.default_rng(6).integers(0, T, 60)]))
    aq_r, sa_r = oracle.inverse_rope_quant(d["o"], d["positions"], d["cos"], d["sin"], 64,
                                           True, 1)
    ref, absref = oracle.gemm_w8a8_block_diag(aq_r, sa_r, wq, sw, E8M0, rows=rows)
    got = host_bf16_f64(out[torch.from_numpy(rows).cuda()])
    assert_within_gemm_tolerance(got, ref, absref, "mx wo_a full size", steps=tmem_steps(K_g))


def test_mx_prefill_full_size_sampled_rows():
    d = inputs.prefill_linear()
    M, K = d["X"].shape
    aq, sa = _act_e8m0(d["X"])
    wq, sw = oracle.quant_weight_block(d["W"], E8M0)
    out = fq.gemm_w8a8_mx(dev_u8(aq), dev_f32(sa), dev_u8(wq), dev_u8(sw))
    assert fq.check_device_error() == 0
    rows = np.unique(np.concatenate([[0, 127, 128, M - 1],
                                     np.random.default_rng(7).integers(0, M, 40)]))
    ref, absref = oracle.gemm_w8a8_block(aq, sa, wq, sw, E8M0, rows=rows)
    got = host_bf16_f64(out[torch.from_numpy(rows).cuda()])
    assert_within_gemm_tolerance(got, ref, absref, "mx prefill full size", steps=tmem_steps(K))
