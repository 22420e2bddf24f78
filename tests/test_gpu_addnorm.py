"""GPU parity of the residual add + RMSNorm + quant against the oracle (reading R11): the updated
residual, the codes and the scales bit-exact, for 1x128 groups and per-token scales.

Source: "SGLang AMD GPU optimisation: fusing RMSNorm with FP8 per-token quantization (SGLang PR
21403 analysis)", section 1 (the fused add_rmsnorm_quant with weight, epsilon and group_size).
"""
import numpy as np
import pytest
import torch

import oracle
import fp8_blockwise_w8a8_b200 as fq
from fp8_blockwise_w8a8_b200 import inputs

from helpers import dev_bf16, host_bf16_bits

pytestmark = pytest.mark.gpu


def _case(x, r, g, per_token, eps=1e-6, ldx=None, ldr=None):
    M, K = x.shape
    h_ref, q_ref, sa_ref = oracle.add_rmsnorm_quant(x, r, g, eps, per_token)
    xd = dev_bf16(x)
    rd = dev_bf16(r)
    if ldx is not None:          # strided rows: the operands sit inside wider buffers
        xw = torch.zeros((M, ldx), dtype=torch.bfloat16, device="cuda")
        xw[:, :K] = xd
        xd = xw[:, :K]
    if ldr is not None:
        rw = torch.full((M, ldr), 7.0, dtype=torch.bfloat16, device="cuda")
        rw[:, :K] = rd
        rd = rw[:, :K]
    x_before = host_bf16_bits(xd)
    q, sa = fq.add_rmsnorm_quant(xd, rd, dev_bf16(g), eps, per_token)
    assert fq.check_device_error() == 0
    assert np.array_equal(host_bf16_bits(xd), x_before)               # x is only read
    assert np.array_equal(host_bf16_bits(rd), h_ref)                  # the new residual
    if ldr is not None:                                               # nothing past K written
        assert torch.all(rw[:, K:] == 7.0)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    sa = sa.cpu().numpy()
    if per_token:
        assert np.array_equal(sa.view(np.uint32), sa_ref.view(np.uint32))
    else:
        assert np.array_equal(sa[:, :M].view(np.uint32), sa_ref[:, :M].view(np.uint32))


@pytest.mark.parametrize("per_token", [False, True])
@pytest.mark.parametrize("M,K", [(1, 128), (37, 768), (64, 4096), (300, 2048), (9, 16384)])
def test_shapes(per_token, M, K):
    x = inputs.randn_bf16((M, K), 1.0, 61, 0)
    r = inputs.randn_bf16((M, K), 3.0, 61, 1)
    g = inputs.to_bf16_bits(inputs.rng_for(61, 2).uniform(0.5, 1.5, K).astype(np.float32))
    _case(x, r, g, per_token)


@pytest.mark.parametrize("per_token", [False, True])
def test_prefill_shape(per_token):
    d = inputs.prefill_linear(with_weight=False)
    r = inputs.randn_bf16(d["X"].shape, 1.0, 62, 0)
    _case(d["X"], r, d["gamma"], per_token, d["eps"])


@pytest.mark.parametrize("per_token", [False, True])
def test_wide_range_cancellation_and_zero_rows(per_token):
    M, K = 24, 1024
    rng = inputs.rng_for(63, 0)
    x = inputs.to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32)
                            * np.exp2(rng.integers(-30, 30, (M, K))).astype(np.float32))
    r = inputs.to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32)
                            * np.exp2(rng.integers(-30, 30, (M, K))).astype(np.float32))
    r[3] = x[3] ^ np.uint16(0x8000)        # h = +0: an all-zero row
    r[4, :512] = x[4, :512] ^ np.uint16(0x8000)   # half the row cancels
    x[5] = 0                               # h = res
    g = inputs.randn_bf16((K,), 0.5, 63, 1)         # signed gamma: signed zero codes
    _case(x, r, g, per_token)


@pytest.mark.parametrize("per_token", [False, True])
def test_strided_rows(per_token):
    M, K = 40, 1024
    x = inputs.randn_bf16((M, K), 1.0, 64, 0)
    r = inputs.randn_bf16((M, K), 1.0, 64, 1)
    g = inputs.randn_bf16((K,), 0.5, 64, 2)
    _case(x, r, g, per_token, ldx=K + 64, ldr=K + 136)


def test_overlapping_residual_is_refused():
    x = torch.zeros((8, 256), dtype=torch.bfloat16, device="cuda")
    g = torch.ones(256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fq.Fp8qError):
        fq.add_rmsnorm_quant(x, x, g)
