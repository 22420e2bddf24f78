"""GPU parity of the SiLU-and-mul + 1x128 quant front end (MoE down projection input): codes and
scales bit-exact against the oracle, whose fp32 exponential the kernel reproduces step by step
(Cody-Waite reduction, degree-7 Taylor polynomial, each operation one IEEE rounding)."""
import numpy as np
import pytest
import torch

import oracle
import fp8_blockwise_w8a8_b200 as fq
from fp8_blockwise_w8a8_b200 import inputs

from helpers import dev_bf16

pytestmark = pytest.mark.gpu


def _check(h, lds=None):
    R = h.shape[0]
    lds = (R + 3) // 4 * 4 if lds is None else lds
    q, sa = fq.silu_mul_quant(dev_bf16(h), lds=lds)
    assert fq.check_device_error() == 0
    qr, sar = oracle.silu_mul_quant(h, lds=lds)
    assert np.array_equal(q.cpu().numpy(), qr)
    assert np.array_equal(sa.cpu().numpy()[:, :R], sar[:, :R])


@pytest.mark.parametrize("R,I", [(1, 128), (37, 768), (300, 1536), (129, 2048)])
@pytest.mark.parametrize("std", [0.5, 4.0])
def test_silu_mul_quant_bit_exact(R, I, std):
    _check(inputs.randn_bf16((R, 2 * I), std, 90, R + I))


def test_silu_mul_quant_special_values():
    h = inputs.randn_bf16((12, 512), 1.0, 91, 0)
    h[0, :256] = 0xC2C8          # gate = -100: e^100 -> silu = -0 (times up)
    h[1, :256] = 0x42C8          # gate = +100
    h[2, :256] = 0xC3B4          # gate = -360: e^360 overflows to inf
    h[3] = 0                     # zeros everywhere: zero block, s = 1
    h[4, 256:] = 0x8000          # up = -0
    h[5, :256:3] = 0x0001        # subnormal gates
    h[6, 256:] = 0x7F00          # huge up: y overflows to inf? bf16(silu*up) saturates in quant
    h[6, :256] = 0x3C00          # small gate keeps y finite
    _check(h)


def test_silu_mul_quant_moe_full_size():
    """The MoE down projection's input: gate/up output [32768, 1536] -> [32768, 768]."""
    h = inputs.randn_bf16((32768, 1536), 1.0, 92, 0)
    _check(h)
