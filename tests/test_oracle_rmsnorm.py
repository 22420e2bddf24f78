"""Pins of the oracle's fused RMSNorm + 1x128 token quant.

Sources: "SGLang AMD GPU optimisation: fusing RMSNorm with FP8 per-token quantization (SGLang PR
21403 analysis)", section 1 (RMSNorm with weight and epsilon, fused with the FP8 quant so the
normalised row is never written); torch.nn.RMSNorm documentation linked from that page
(y = x / sqrt(mean(x^2) + eps) * weight).  The rounding steps are the reading stated in the
oracle's header (fp64 sum of squares, fp32 product chain, bf16 output).
"""
import math

import numpy as np
import torch

import oracle
from fp8_blockwise_w8a8_b200 import inputs


def test_constant_rows_closed_form():
    """x_k = c for all k and gamma = 1: mean(x^2) = c^2 exactly, r = 1/sqrt(c^2 + eps)."""
    K = 512
    cs = np.array([1.0, -0.375, 3.5, 1e-3, 0.0, 200.0], np.float32)
    x = inputs.to_bf16_bits(np.repeat(cs[:, None], K, axis=1))
    g = inputs.to_bf16_bits(np.ones(K, np.float32))
    eps = np.float32(1e-6)
    y = inputs.bf16_bits_to_f32(oracle.rmsnorm_bf16(x, g, float(eps)))
    for i, c in enumerate(inputs.bf16_bits_to_f32(x[:, 0])):
        r = np.float32(1.0 / math.sqrt(float(c) * float(c) + float(eps)))
        assert oracle.rms_inverse(x[i], float(eps)) == r
        want = inputs.bf16_bits_to_f32(inputs.to_bf16_bits(np.array([np.float32(c) * r])))[0]
        assert np.all(y[i] == want), (c, y[i][:4], want)


def test_matches_torch_rms_norm_in_fp64():
    """Against torch.nn.functional.rms_norm evaluated in float64, then rounded to bf16: every
    element agrees or differs by one bf16 ulp (double rounding), and nearly all agree."""
    d = inputs.prefill_linear(M=64, K=1024, with_weight=False)
    x, g, eps = d["X"], d["gamma"], d["eps"]
    # add rows with a wide dynamic range
    x[:4] = inputs.to_bf16_bits(inputs.bf16_bits_to_f32(x[:4]) *
                                np.float32(2.0) ** np.arange(-20, 20, 10, dtype=np.float32)[:, None])
    y = oracle.rmsnorm_bf16(x, g, eps)
    xt = torch.from_numpy(inputs.bf16_bits_to_f32(x)).double()
    gt = torch.from_numpy(inputs.bf16_bits_to_f32(g)).double()
    ref = torch.nn.functional.rms_norm(xt, (x.shape[1],), weight=gt, eps=float(np.float32(eps)))
    ref_bits = ref.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    diff = np.abs(y.astype(np.int32) - ref_bits.astype(np.int32))
    assert diff.max() <= 1
    assert (diff == 0).mean() > 0.995


def test_fused_equals_unfused_then_token_quant():
    d = inputs.prefill_linear(M=48, K=768, with_weight=False)
    x, g, eps = d["X"], d["gamma"], d["eps"]
    q1, s1 = oracle.rmsnorm_quant_token(x, g, eps)
    q2, s2 = oracle.quant_token_1x128(oracle.rmsnorm_bf16(x, g, eps))
    assert np.array_equal(q1, q2) and np.array_equal(s1, s2)


def test_gamma_none_is_plain_token_quant():
    d = inputs.tiny_linear()
    q1, s1 = oracle.rmsnorm_quant_token(d["A"], None)
    q2, s2 = oracle.quant_token_1x128(d["A"])
    assert np.array_equal(q1, q2) and np.array_equal(s1, s2)


def test_scale_invariance_by_powers_of_two():
    """RMSNorm output is unchanged when a row is scaled by 2^j (exact in every step while the
    sum of squares dominates eps)."""
    d = inputs.prefill_linear(M=8, K=512, with_weight=False)
    x, g = d["X"], d["gamma"]
    y0 = oracle.rmsnorm_bf16(x, g, 0.0)
    x4 = inputs.to_bf16_bits(inputs.bf16_bits_to_f32(x) * np.float32(16.0))
    assert np.array_equal(oracle.rmsnorm_bf16(x4, g, 0.0), y0)


def test_gamma_is_per_column():
    """A gamma that is zero on one column zeroes exactly that column (pins gamma indexing)."""
    d = inputs.prefill_linear(M=4, K=256, with_weight=False)
    g = d["gamma"].copy()
    g[137] = 0
    y = oracle.rmsnorm_bf16(d["X"], g, 1e-6)
    assert np.all((y[:, 137] & 0x7FFF) == 0)
    assert (y[:, 136] & 0x7FFF).all()
