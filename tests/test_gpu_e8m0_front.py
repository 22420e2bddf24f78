"""GPU parity of the front ends with E8M0 (power-of-two) activation scales, the oracle's reading
R12: plain 1x128 token quant, RMSNorm + quant, residual add + RMSNorm + quant and SiLU-and-mul +
quant -- codes, scales (and the updated residual) bit-exact -- and the whole E8M0 prefill linear
layer, RMSNorm + quant -> E8M0 weight requant -> hardware block-scaled GEMM, against the oracle's
fp64 reference under both GEMM gates.

Sources: "DeepSeek V4 performance: FP8 WO_A output projection (vLLM PR 54894 analysis)", sections
1 and 3 (E8M0 scales; group-128 activation quant feeding an MX-scaled GEMM); "SGLang ... (PR 21403
analysis)", section 1 (RMSNorm fused with the FP8 quant).
"""
import numpy as np
import pytest
import torch

import oracle
import fp8_blockwise_w8a8_b200 as fq
from fp8_blockwise_w8a8_b200 import inputs

from helpers import (assert_within_gemm_tolerance, dev_bf16, dev_u8, host_bf16_bits,
                     host_bf16_f64, tmem_steps)

pytestmark = pytest.mark.gpu
E8M0 = oracle.SCALE_E8M0


def _token_case(x, gamma=None, eps=1e-6):
    M, K = x.shape
    lds = max(4, (M + 3) // 4 * 4)
    q_ref, sa_ref = oracle.rmsnorm_quant_token(x, gamma, eps, lds=lds, fmt=E8M0)
    sa_dev = torch.zeros((K // 128, lds), dtype=torch.float32, device="cuda")
    q, sa = fq.rmsnorm_quant_token(dev_bf16(x), None if gamma is None else dev_bf16(gamma), eps,
                                   out_sa=sa_dev, scale_fmt="e8m0")
    assert fq.check_device_error() == 0
    assert np.array_equal(sa.cpu().numpy()[:, :M].view(np.uint32), sa_ref[:, :M].view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), q_ref)


def _gamma(K, seed):
    return inputs.to_bf16_bits(np.random.default_rng(seed).uniform(0.5, 1.5, K).astype(np.float32))


@pytest.mark.parametrize("K", [128, 384, 768, 2048, 4096, 16384])
@pytest.mark.parametrize("M", [1, 37, 301])
def test_token_and_rmsnorm_quant_e8m0(M, K):
    """Plain (whole-row, spread and packed walks) and fused, across row counts and widths."""
    x = inputs.randn_bf16((M, K), 1.0, 110, M + K)
    _token_case(x)
    _token_case(x, _gamma(K, K), 1e-6)


def test_e8m0_wide_range_zeros_and_clamped_scales():
    x = inputs.bf16_bits_to_f32(inputs.randn_bf16((12, 1024), 1.0, 111, 0)).copy()
    x[0] *= 1e30
    x[1] *= 1e-30
    x[2, :128] = 0.0
    x[3, 128:256] = 2.0 ** -126            # scale clamps at 2^-127
    x[4] = 448.0                            # amax / 448 = 1: exactly a power of two
    x[5, ::2] = -0.0
    xb = inputs.to_bf16_bits(x)
    _token_case(xb)
    _token_case(xb, _gamma(1024, 3), 1e-6)


def test_rmsnorm_quant_e8m0_prefill_full():
    d = inputs.prefill_linear(with_weight=False)
    _token_case(d["X"], d["gamma"], d["eps"])


@pytest.mark.parametrize("M,K", [(1, 128), (37, 768), (300, 4096)])
def test_add_rmsnorm_quant_e8m0(M, K):
    x = inputs.randn_bf16((M, K), 1.0, 112, 0)
    r = inputs.randn_bf16((M, K), 3.0, 112, 1)
    g = _gamma(K, 112)
    h_ref, q_ref, sa_ref = oracle.add_rmsnorm_quant(x, r, g, 1e-6, fmt=E8M0)
    rd = dev_bf16(r)
    q, sa = fq.add_rmsnorm_quant(dev_bf16(x), rd, dev_bf16(g), 1e-6, scale_fmt="e8m0")
    assert fq.check_device_error() == 0
    assert np.array_equal(host_bf16_bits(rd), h_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(sa.cpu().numpy()[:, :M].view(np.uint32), sa_ref[:, :M].view(np.uint32))


def test_add_rmsnorm_quant_per_token_e8m0_is_rejected():
    x = dev_bf16(inputs.randn_bf16((4, 256), 1.0, 113, 0))
    r = dev_bf16(inputs.randn_bf16((4, 256), 1.0, 113, 1))
    with pytest.raises(fq.Fp8qError):
        fq.add_rmsnorm_quant(x, r, dev_bf16(_gamma(256, 4)), 1e-6, per_token=True,
                             scale_fmt="e8m0")


@pytest.mark.parametrize("R,I", [(1, 128), (37, 768), (300, 1536), (32768, 768)])
def test_silu_mul_quant_e8m0(R, I):
    h = inputs.randn_bf16((R, 2 * I), 1.0, 114, R + I)
    lds = (R + 3) // 4 * 4
    q, sa = fq.silu_mul_quant(dev_bf16(h), lds=lds, scale_fmt="e8m0")
    assert fq.check_device_error() == 0
    qr, sar = oracle.silu_mul_quant(h, lds=lds, fmt=E8M0)
    assert np.array_equal(q.cpu().numpy(), qr)
    assert np.array_equal(sa.cpu().numpy()[:, :R].view(np.uint32), sar[:, :R].view(np.uint32))


def test_e8m0_prefill_linear_end_to_end():
    """The E8M0 prefill step: RMSNorm + 1x128 quant (E8M0) of X [8192, 4096], E8M0 requant of
    W [24576, 4096], then the hardware block-scaled GEMM; codes and scales bit-exact, the output
    on sampled rows within both GEMM gates."""
    d = inputs.prefill_linear()
    M, K = d["X"].shape
    aq, sa = fq.rmsnorm_quant_token(dev_bf16(d["X"]), dev_bf16(d["gamma"]), d["eps"],
                                    scale_fmt="e8m0")
    wq, sw = fq.quant_weight_block(dev_bf16(d["W"]), "e8m0")
    out = fq.gemm_w8a8_mx(aq, sa, wq, sw)
    assert fq.check_device_error() == 0
    aq_r, sa_r = oracle.rmsnorm_quant_token(d["X"], d["gamma"], d["eps"], lds=sa.shape[1],
                                            fmt=E8M0)
    wq_r, sw_r = oracle.quant_weight_block(d["W"], E8M0)
    assert np.array_equal(aq.cpu().numpy(), aq_r)
    assert np.array_equal(sa.cpu().numpy()[:, :M].view(np.uint32), sa_r[:, :M].view(np.uint32))
    assert np.array_equal(wq.cpu().numpy(), wq_r) and np.array_equal(sw.cpu().numpy(), sw_r)
    rows = np.unique(np.concatenate([[0, 127, 128, M - 1],
                                     np.random.default_rng(8).integers(0, M, 28)]))
    ref, absref = oracle.gemm_w8a8_block(aq_r, sa_r, wq_r, sw_r, E8M0, rows=rows)
    got = host_bf16_f64(out[torch.from_numpy(rows).cuda()])
    assert_within_gemm_tolerance(got, ref, absref, "e8m0 prefill linear", steps=tmem_steps(K))
