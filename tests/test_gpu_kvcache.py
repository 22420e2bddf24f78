"""GPU parity of the FP8 KV-cache path: per-step per-tensor QKV scales (maxima and scales
bit-exact) and the cache write (Q codes and the K, V cache rows bit-exact against the oracle;
padding slots and all other cache rows untouched; bad slots and scales reported).  Source:
"FP8-RL: ..." abstract, item (ii)."""
import numpy as np
import pytest
import torch

import oracle
import fp8_blockwise_w8a8_b200 as fq
from fp8_blockwise_w8a8_b200 import inputs

from helpers import dev_bf16, dev_f32

pytestmark = pytest.mark.gpu


def _check(d, scales=None):
    Hq, Hkv, D, ns = d["Hq"], d["Hkv"], d["D"], d["num_slots"]
    x = dev_bf16(d["qkv"])
    amax, s = fq.qkv_scales(x, Hq, Hkv, D)
    assert fq.check_device_error() == 0
    amax_r = oracle.qkv_amax(d["qkv"], Hq, Hkv, D)
    s_r = oracle.qkv_scales(amax_r)
    assert np.array_equal(amax.cpu().numpy(), amax_r)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_r.view(np.uint32))
    if scales is not None:
        s = dev_f32(scales)
        s_r = np.asarray(scales, np.float32)
    kc = torch.full((ns, Hkv * D), 0xAA, dtype=torch.uint8, device="cuda")
    vc = torch.full((ns, Hkv * D), 0x55, dtype=torch.uint8, device="cuda")
    q = fq.kv_cache_write(x, Hq, Hkv, D, torch.from_numpy(d["slots"]).cuda(), s, kc, vc)
    assert fq.check_device_error() == 0
    kr = np.full((ns, Hkv * D), 0xAA, np.uint8)
    vr = np.full((ns, Hkv * D), 0x55, np.uint8)
    qr = oracle.kv_cache_write(d["qkv"], Hq, Hkv, D, d["slots"], s_r, kr, vr)
    assert np.array_equal(q.cpu().numpy(), qr)
    assert np.array_equal(kc.cpu().numpy(), kr)
    assert np.array_equal(vc.cpu().numpy(), vr)


@pytest.mark.parametrize("T,Hq,Hkv,D", [(1, 1, 1, 16), (37, 4, 2, 64), (300, 8, 1, 128),
                                        (129, 32, 8, 128)])
def test_kv_cache_small(T, Hq, Hkv, D):
    d = inputs.kv_cache(tokens=T, q_heads=Hq, kv_heads=Hkv, head_dim=D, num_blocks=(T + 40) // 16 + 4)
    _check(d)


def test_kv_cache_full_size():
    _check(inputs.kv_cache())


def test_kv_cache_caller_scales_and_wide_range():
    d = inputs.kv_cache(tokens=200, q_heads=4, kv_heads=2, head_dim=64, num_blocks=20)
    x = inputs.bf16_bits_to_f32(d["qkv"]).copy()
    x[::3] *= 1e-20
    x[1::7] *= 3e4
    d["qkv"] = inputs.to_bf16_bits(x)
    _check(d)
    _check(d, scales=[0.013, 1.5e-6, 2.0 ** -20])      # arbitrary scales, not amax / 448


def test_kv_cache_zero_tensor_and_no_tokens():
    d = inputs.kv_cache(tokens=16, q_heads=2, kv_heads=1, head_dim=32, num_blocks=2)
    d["qkv"] = np.zeros_like(d["qkv"])
    _check(d)
    amax, s = fq.qkv_scales(torch.zeros((0, 128), dtype=torch.bfloat16, device="cuda"), 2, 1, 32)
    assert (amax.cpu().numpy() == 0).all() and (s.cpu().numpy() == 1).all()


def test_kv_cache_bad_slot_and_scale_are_reported():
    d = inputs.kv_cache(tokens=8, q_heads=2, kv_heads=1, head_dim=32, num_blocks=1)
    Hq, Hkv, D = 2, 1, 32
    x = dev_bf16(d["qkv"])
    slots = torch.tensor([0, 1, 2, 16, 3, -1, 4, 5], dtype=torch.int64, device="cuda")  # 16 > 15
    kc = torch.zeros((16, Hkv * D), dtype=torch.uint8, device="cuda")
    vc = torch.zeros_like(kc)
    s = dev_f32(np.array([0.01, 0.01, 0.01], np.float32))
    fq.kv_cache_write(x, Hq, Hkv, D, slots, s, kc, vc)
    assert fq.check_device_error() == fq.FP8Q_ERR_RANGE
    assert fq.check_device_error() == 0
    kr = np.zeros((16, Hkv * D), np.uint8)
    vr = np.zeros_like(kr)
    sl = slots.cpu().numpy().copy()
    sl[3] = -1
    oracle.kv_cache_write(d["qkv"], Hq, Hkv, D, sl, [0.01, 0.01, 0.01], kr, vr)
    assert np.array_equal(kc.cpu().numpy(), kr) and np.array_equal(vc.cpu().numpy(), vr)
    bad = dev_f32(np.array([0.01, 0.0, 0.01], np.float32))
    kc.zero_()
    fq.kv_cache_write(x, Hq, Hkv, D, slots.clamp(max=15), bad, kc, vc)
    assert fq.check_device_error() == fq.FP8Q_ERR_RANGE
    assert not kc.any()                                  # K has a zero scale: not written
