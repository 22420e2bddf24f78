"""GPU parity of the two quantizers against the oracle: bit-exact codes and scales.

Weight blocks: "FP8-RL ..." abstract (i), "DeepSeek V4 ... (vLLM PR 54894 analysis)" sections 1-2.
Token groups / RMSNorm: "... (vLLM PR 54894 analysis)" section 3, "SGLang ... (PR 21403
analysis)" section 1.
"""
import numpy as np
import pytest
import torch

import oracle
import fp8_blockwise_w8a8_b200 as fq
from fp8_blockwise_w8a8_b200 import inputs

from helpers import dev_bf16, host_bf16_bits

pytestmark = pytest.mark.gpu


def _weight_case(w_bits, fmt):
    wq_ref, sw_ref = oracle.quant_weight_block(w_bits, fmt)
    q, s = fq.quant_weight_block(dev_bf16(w_bits), fmt)
    assert fq.check_device_error() == 0
    q = q.cpu().numpy()
    s = s.cpu().numpy()
    assert np.array_equal(s.view(np.uint8) if fmt else s.view(np.uint32),
                          sw_ref.view(np.uint8) if fmt else sw_ref.view(np.uint32))
    assert np.array_equal(q, wq_ref)


@pytest.mark.parametrize("fmt", [oracle.SCALE_F32, oracle.SCALE_E8M0])
def test_weight_tiny_and_decode(fmt):
    _weight_case(inputs.tiny_linear()["W"], fmt)
    _weight_case(inputs.decode_linear(M=8)["W"], fmt)


@pytest.mark.parametrize("fmt", [oracle.SCALE_F32, oracle.SCALE_E8M0])
def test_weight_special_values(fmt):
    rng = np.random.default_rng(5)
    w = inputs.randn_bf16((384, 640), 0.02, 77, 0)
    w[:128, :128] = 0                                            # all-zero block
    w[:128, 128:256] = 0x8000                                    # all -0 block
    w[128:256, :128] = inputs.to_bf16_bits(                      # huge magnitudes
        rng.standard_normal((128, 128)).astype(np.float32) * np.float32(1e37))
    w[256:384, :128] = rng.integers(1, 0x80, (128, 128)).astype(np.uint16) | \
        (rng.integers(0, 2, (128, 128)).astype(np.uint16) << 15)  # bf16 subnormals
    w[128:256, 128:256] = inputs.to_bf16_bits(                   # tiny block: subnormal scale
        rng.standard_normal((128, 128)).astype(np.float32) * np.float32(1e-38))
    w[256:384, 256:384] = 0x8001                                 # negatives that quantize to 0
    w[256, 256] = 0x3F80                                          # ... next to a 1.0
    # exact E4M3 midpoints relative to the block maximum 448 (x/s ties)
    mids = np.array([432, 416 + 8, 1.0625, 2 ** -10, 3 * 2 ** -10, 17, 19], np.float32)
    blk = np.zeros((128, 128), np.float32)
    blk[0, 0] = 448
    blk[1, :mids.size] = mids
    blk[2, :mids.size] = -mids
    w[0:128, 512:640] = inputs.to_bf16_bits(blk)
    _weight_case(w, fmt)


@pytest.mark.parametrize("fmt", [oracle.SCALE_F32, oracle.SCALE_E8M0])
def test_weight_strided(fmt):
    w = inputs.randn_bf16((256, 384), 0.05, 78, 0)
    wd = torch.zeros((256, 520), dtype=torch.bfloat16, device="cuda")
    wd[:, :384] = dev_bf16(w)
    qd = torch.full((256, 400), 0xAB, dtype=torch.uint8, device="cuda")
    q, s = fq.quant_weight_block(wd[:, :384], fmt, out_q=qd[:, :384])
    wq_ref, sw_ref = oracle.quant_weight_block(w, fmt)
    assert np.array_equal(qd[:, :384].cpu().numpy(), wq_ref)
    assert (qd[:, 384:].cpu().numpy() == 0xAB).all()                # padding untouched
    assert np.array_equal(s.cpu().numpy(), sw_ref)


def test_weight_sweep_layer0_and_sampled_layers():
    """Per-step requant of the 36-layer dense model: layer 0 in full, plus sampled blocks of
    three later layers, in both scale formats (same launch configuration the bench times)."""
    rng = np.random.default_rng(0)
    for layer in (0, 17, 35):
        for idx in range(len(inputs.SWEEP_MATRICES)):
            w = inputs.sweep_matrix(layer, idx, "cuda")
            for fmt in (oracle.SCALE_F32, oracle.SCALE_E8M0):
                q, s = fq.quant_weight_block(w, fmt)
                if layer == 0:
                    wq_ref, sw_ref = oracle.quant_weight_block(host_bf16_bits(w), fmt)
                    assert np.array_equal(s.cpu().numpy(), sw_ref)
                    assert np.array_equal(q.cpu().numpy(), wq_ref)
                else:
                    N, K = w.shape
                    for _ in range(8):
                        nb = int(rng.integers(0, N // 128))
                        kb = int(rng.integers(0, K // 128))
                        blk = host_bf16_bits(w[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128])
                        bq, bs = oracle.quant_weight_block(blk, fmt)
                        assert s[nb, kb].item() == bs[0, 0].item()
                        assert np.array_equal(
                            q[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128].cpu().numpy(), bq)
    assert fq.check_device_error() == 0


# --- token groups ------------------------------------------------------------------------------

def _token_case(x_bits, gamma_bits=None, eps=1e-6, lds=None):
    M, K = x_bits.shape
    lds = lds if lds is not None else max(4, (M + 3) // 4 * 4)
    q_ref, sa_ref = oracle.rmsnorm_quant_token(x_bits, gamma_bits, eps, lds=lds)
    g = None if gamma_bits is None else dev_bf16(gamma_bits)
    sa_dev = torch.zeros((K // 128, lds), dtype=torch.float32, device="cuda")
    q, sa = fq.rmsnorm_quant_token(dev_bf16(x_bits), g, eps, out_sa=sa_dev)
    assert fq.check_device_error() == 0
    assert np.array_equal(sa.cpu().numpy()[:, :M].view(np.uint32), sa_ref[:, :M].view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), q_ref)


@pytest.mark.parametrize("M", [1, 3, 64, 127, 129, 600])
def test_token_plain_shapes(M):
    x = inputs.randn_bf16((M, 512), 1.0, 90, M)
    _token_case(x)


def test_token_tiny_decode_and_moe_inputs():
    _token_case(inputs.tiny_linear()["A"])
    _token_case(inputs.decode_linear(N=128)["A"])
    d = inputs.moe(with_weights=False)
    _token_case(d["A_gateup"])
    _token_case(d["A_down"])


@pytest.mark.parametrize("K", [128, 384, 4096, 16384])
def test_rmsnorm_shapes(K):
    x = inputs.randn_bf16((37, K), 1.0, 91, K)
    g = inputs.to_bf16_bits(np.random.default_rng(K).uniform(0.5, 1.5, K).astype(np.float32))
    _token_case(x, g, 1e-6)
    _token_case(x, None)


def test_rmsnorm_prefill_full():
    d = inputs.prefill_linear(with_weight=False)
    _token_case(d["X"], d["gamma"], d["eps"])


def test_rmsnorm_wide_dynamic_range_rows():
    """Rows whose per-block fp64 sums of squares are inexact, so the summation order matters."""
    rng = np.random.default_rng(92)
    x = rng.standard_normal((16, 1024)).astype(np.float32)
    x *= np.float32(2.0) ** rng.integers(-30, 30, size=(16, 1024)).astype(np.float32)
    xb = inputs.to_bf16_bits(x)
    g = inputs.to_bf16_bits(rng.uniform(0.5, 1.5, 1024).astype(np.float32))
    _token_case(xb, g, 1e-6)
    _token_case(xb, g, 0.0)


def test_token_zero_rows_and_sign_of_zero():
    x = np.zeros((4, 256), np.uint16)
    x[1] = 0x8000
    x[2, :128] = 0x8001
    x[2, 5] = 0x4000
    x[3, :] = inputs.to_bf16_bits(np.linspace(-1, 1, 256).astype(np.float32))
    _token_case(x)
    g = np.full(256, 0x3F80, np.uint16)
    _token_case(x, g, 1e-6)


@pytest.mark.parametrize("K", [640, 768, 1920, 2048, 3968])
@pytest.mark.parametrize("M", [1, 37, 301])
def test_token_rows_sharing_a_warp(K, M):
    """Rows of fewer than 32 blocks: several rows per warp (32 // (K / 128) of them), a last
    row group that is cut short by M, with and without RMSNorm."""
    x = inputs.randn_bf16((M, K), 1.0, 93, K + M)
    g = inputs.to_bf16_bits(np.random.default_rng(K).uniform(0.5, 1.5, K).astype(np.float32))
    _token_case(x, g, 1e-6)
    _token_case(x, None)


@pytest.mark.parametrize("M,K", [(2000, 3072), (1111, 5120), (150, 16384)])
def test_token_plain_fewer_rows_than_warps(M, K):
    """Fewer rows than warps: the plain kernel spreads the (row, step) units of all rows over the
    warps, with a unit stride that is not a whole number of rows (a carry from a row's last step
    into the next row) on the full grid."""
    x = inputs.randn_bf16((M, K), 1.0, 95, K + M)
    _token_case(x)


def test_token_strided_rows():
    M, K = 70, 1024
    x = inputs.randn_bf16((M, K + 64), 1.0, 94, 0)
    xs = dev_bf16(x)[:, :K]
    g = inputs.to_bf16_bits(np.random.default_rng(5).uniform(0.5, 1.5, K).astype(np.float32))
    for gamma in (g, None):
        q, sa = fq.rmsnorm_quant_token(xs, None if gamma is None else dev_bf16(gamma), 1e-6)
        assert fq.check_device_error() == 0
        q_ref, sa_ref = oracle.rmsnorm_quant_token(np.ascontiguousarray(x[:, :K]), gamma, 1e-6,
                                                   lds=sa.shape[1])
        assert np.array_equal(q.cpu().numpy(), q_ref)
        assert np.array_equal(sa.cpu().numpy()[:, :M], sa_ref[:, :M])


# --- batched requant ---------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", [oracle.SCALE_F32, oracle.SCALE_E8M0])
def test_weight_batch_mixed_shapes(fmt):
    shapes = [(128, 128), (256, 384), (1024, 4096), (384, 128), (4096, 512), (128, 1152)]
    ws = [inputs.randn_bf16(s, 0.02 * (i + 1), 95, i) for i, s in enumerate(shapes)]
    ws[2] = np.concatenate([ws[2], np.zeros((1024, 64), np.uint16)], axis=1)   # strided rows
    dev = [dev_bf16(w) for w in ws]
    dev[2] = dev[2][:, :4096]
    batch = fq.WeightBatch(dev, fmt)
    qs, ss = batch.run()
    assert fq.check_device_error() == 0
    for w, q, s_ in zip(ws, qs, ss):
        N, K = q.shape
        q_ref, s_ref = oracle.quant_weight_block(np.ascontiguousarray(w[:, :K]), fmt)
        assert np.array_equal(q.cpu().numpy(), q_ref)
        assert np.array_equal(s_.cpu().numpy(), s_ref)


def test_weight_batch_sweep_layer_matches_per_matrix_calls():
    ws = [inputs.sweep_matrix(0, i, "cuda") for i in range(len(inputs.SWEEP_MATRICES))]
    for fmt in ("f32", "e8m0"):
        qs, ss = fq.WeightBatch(ws, fmt).run()
        assert fq.check_device_error() == 0
        for w, q, s_ in zip(ws, qs, ss):
            q1, s1 = fq.quant_weight_block(w, fmt)
            assert torch.equal(q, q1) and torch.equal(s_, s1)


def test_weight_batch_bad_descriptor_is_reported_and_skipped():
    ws = [dev_bf16(inputs.randn_bf16((256, 256), 0.02, 96, i)) for i in range(3)]
    batch = fq.WeightBatch(ws, "f32")
    desc = batch.desc.cpu().numpy().view(fq.WeightBatch._DESC).copy()
    desc[1]["K"] = 200                       # not a multiple of 128
    batch.desc = torch.from_numpy(desc.view(np.uint8).copy()).cuda()
    for q in batch.q:
        q.fill_(0xEE)
    qs, ss = batch.run()
    assert fq.check_device_error() == fq.FP8Q_ERR_SHAPE
    assert (qs[1] == 0xEE).all()
    for i in (0, 2):
        q_ref, s_ref = oracle.quant_weight_block(ws[i].cpu().view(torch.int16).numpy().view(np.uint16), 0)
        assert np.array_equal(qs[i].cpu().numpy(), q_ref) and np.array_equal(ss[i].cpu().numpy(), s_ref)


@pytest.mark.parametrize("K", [768, 4096])
def test_rmsnorm_blocks_with_zeros_and_subnormals(K):
    """Every 128-block of these rows holds a zero, a subnormal or a value 2^-20 below its
    neighbours, so the fused kernel's fast (any-order) block sums are not certified and each block
    is summed again in ascending k; rows of N(0,1) blocks with a few such blocks mixed in take both
    paths within one row."""
    rng = np.random.default_rng(96)
    M = 300
    x = rng.standard_normal((M, K)).astype(np.float32)
    KB = K // 128
    for m in range(M):
        for b in range(KB):
            if m < 150 or rng.random() < 0.25:
                k = b * 128 + int(rng.integers(0, 128))
                x[m, k] = [0.0, -0.0, 1e-40, -3e-39, 2.0 ** -20][int(rng.integers(0, 5))]
    x[7, :128] = 0.0                                  # an all-zero block
    x[8] = 0.0                                        # an all-zero row
    g = inputs.to_bf16_bits(rng.uniform(0.5, 1.5, K).astype(np.float32))
    _token_case(inputs.to_bf16_bits(x), g, 1e-6)
