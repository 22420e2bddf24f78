"""GPU parity of the attention output projection path: the inverse-RoPE + 1x128 quant front end
(codes and scales bit-exact against the oracle, fp32 and E8M0 scales, interleaved and half-split
pairs) and the block-diagonal per-head-group GEMM that consumes it (within the GEMM tolerance
|out - ref| <= 8e-3 * sum_k |dec(a) sa dec(w) sw| + 1 bf16 ulp of |ref|).  Source: "DeepSeek V4
... (vLLM PR 54894 analysis)" sections 2-3."""
import numpy as np
import pytest
import torch

import oracle
import fp8_blockwise_w8a8_b200 as fq
from fp8_blockwise_w8a8_b200 import inputs

from helpers import (assert_within_gemm_tolerance, dev_bf16, dev_f32, dev_u8, host_bf16_f64,
                     promoted_steps)

pytestmark = pytest.mark.gpu


def _dev_rope(d):
    return (torch.from_numpy(d["positions"]).cuda(), dev_f32(d["cos"]), dev_f32(d["sin"]))


def _check_quant(d, R, interleaved, fmt, lds=None, ldo_pad=0):
    o = d["o"]
    T, H, D = o.shape
    lds = max(4, (T + 3) // 4 * 4) if lds is None else lds
    if ldo_pad:
        buf = dev_bf16(np.concatenate([o.reshape(T, H * D),
                                       np.zeros((T, ldo_pad), np.uint16)], axis=1))
        od = buf[:, :H * D].view(T, H, D)
    else:
        od = dev_bf16(o)
    pos, cs, sn = _dev_rope(d)
    q, sa = fq.inverse_rope_quant(od, pos, cs, sn, R, interleaved, fmt, lds=lds)
    assert fq.check_device_error() == 0
    qr, sar = oracle.inverse_rope_quant(o, d["positions"], d["cos"], d["sin"], R, interleaved,
                                        fmt, lds=lds)
    qg = q.cpu().numpy()
    if not np.array_equal(qg, qr):
        bad = np.argwhere(qg != qr)
        raise AssertionError(f"{len(bad)} codes differ; first at {tuple(bad[0])}: "
                             f"{qg[tuple(bad[0])]} vs {qr[tuple(bad[0])]}")
    assert np.array_equal(sa.cpu().numpy()[:, :T], sar[:, :T])


@pytest.mark.parametrize("T,H,D,R", [(1, 1, 128, 64), (37, 4, 192, 64), (300, 8, 128, 32),
                                     (129, 2, 512, 512), (65, 2, 256, 16)])
@pytest.mark.parametrize("interleaved", [True, False])
@pytest.mark.parametrize("fmt", [0, 1])
def test_inverse_rope_quant_bit_exact(T, H, D, R, interleaved, fmt):
    d = inputs.wo_a(tokens=T, heads=H, head_dim=D, rope_dim=R, max_pos=2048, with_weight=False)
    _check_quant(d, R, interleaved, fmt)


def _tie_cases(n, second, seed):
    """n (x_a, x_b, c, s) whose rotated value, with each product rounded to fp32 before the sum,
    is exactly halfway between two bf16 values, while a fused multiply-add would round to the
    other one: a contraction anywhere in the rotation changes the result."""
    r = np.random.default_rng(seed)
    found = []
    while len(found) < n:
        m = 1 << 20
        xa = inputs.bf16_bits_to_f32(inputs.to_bf16_bits(r.standard_normal(m).astype(np.float32)))
        xb = inputs.bf16_bits_to_f32(inputs.to_bf16_bits(r.standard_normal(m).astype(np.float32)))
        c = r.uniform(-1, 1, m).astype(np.float32)
        sn = r.uniform(-1, 1, m).astype(np.float32)
        if not second:
            p1, p2 = xa * c, xb * sn                      # fp32 products
            v = p1 + p2
            fused = (xa.astype(np.float64) * c + p2).astype(np.float32)
        else:
            p1, p2 = xb * c, xa * sn
            v = p1 - p2
            fused = (xb.astype(np.float64) * c - p2).astype(np.float32)
        tie = (v.view(np.uint32) & 0xFFFF) == 0x8000
        differs = inputs.to_bf16_bits(fused) != inputs.to_bf16_bits(v)
        for i in np.flatnonzero(tie & differs & (np.abs(v) > 1e-30)):
            found.append((xa[i], xb[i], c[i], sn[i]))
    return found[:n]


@pytest.mark.parametrize("interleaved", [True, False])
def test_inverse_rope_quant_rounding_ties(interleaved):
    """Every rotated pair sits on a bf16 rounding tie of the separately rounded products."""
    T, H, D, R = 8, 1, 128, 64
    half = R // 2
    cases = _tie_cases(T * half // 2, False, 70) + _tie_cases(T * half // 2, True, 71)
    o = np.zeros((T, H, D), np.float32)
    o[:, :, :D - R] = 0.25
    cos = np.zeros((T, half), np.float32)
    sin = np.zeros((T, half), np.float32)
    for n, (xa, xb, c, sn) in enumerate(cases):
        t, i = divmod(n, half)
        a, b = (2 * i, 2 * i + 1) if interleaved else (i, i + half)
        o[t, 0, D - R + a], o[t, 0, D - R + b] = xa, xb
        cos[t, i], sin[t, i] = c, sn
    d = {"o": inputs.to_bf16_bits(o), "positions": np.arange(T, dtype=np.int64), "cos": cos,
         "sin": sin}
    y = oracle.inverse_rope_bf16(d["o"], d["positions"], cos, sin, R, interleaved)
    assert len(np.unique(y)) > T                       # the cases are in place
    for fmt in (0, 1):
        _check_quant(d, R, interleaved, fmt)


def test_inverse_rope_quant_token_stride_and_wide_range():
    d = inputs.wo_a(tokens=50, heads=4, head_dim=256, rope_dim=64, max_pos=512, with_weight=False)
    o = inputs.bf16_bits_to_f32(d["o"]).copy()
    o[::7] *= 3.0e4                                   # large and tiny magnitudes in one tensor
    o[1::7] *= 1.0e-30
    o[2] = 0.0                                        # an all-zero token
    d["o"] = inputs.to_bf16_bits(o)
    for fmt in (0, 1):
        _check_quant(d, 64, True, fmt, lds=56, ldo_pad=64)


@pytest.mark.parametrize("fmt", [0, 1])
def test_inverse_rope_quant_full_size(fmt):
    d = inputs.wo_a(with_weight=False)                # 8192 tokens x 32 heads x 512
    _check_quant(d, 64, True, fmt)


def test_inverse_rope_quant_without_rotary_dims_is_token_quant():
    x = inputs.randn_bf16((40, 2, 256), 1.0, 60, 0)
    q, sa = fq.inverse_rope_quant(dev_bf16(x), None, None, None, 0)
    assert fq.check_device_error() == 0
    qr, sar = oracle.quant_token_1x128(x.reshape(40, 512), lds=40)
    assert np.array_equal(q.cpu().numpy(), qr)
    assert np.array_equal(sa.cpu().numpy(), sar)


def test_out_of_range_position_skips_the_row_and_reports():
    d = inputs.wo_a(tokens=20, heads=2, head_dim=256, rope_dim=64, max_pos=100, with_weight=False)
    pos = d["positions"].copy()
    pos[3] = -1
    pos[11] = 100
    T, K = 20, 512
    q = torch.full((T, K), 0xAB, dtype=torch.uint8, device="cuda")
    sa = torch.full((K // 128, 20), -7.0, dtype=torch.float32, device="cuda")
    fq.inverse_rope_quant(dev_bf16(d["o"]), torch.from_numpy(pos).cuda(), dev_f32(d["cos"]),
                          dev_f32(d["sin"]), 64, out_q=q, out_sa=sa)
    assert fq.check_device_error() == fq.FP8Q_ERR_RANGE
    assert fq.check_device_error() == 0                # the word is cleared once read
    good = [t for t in range(T) if t not in (3, 11)]
    pos_ok = pos.copy()
    pos_ok[[3, 11]] = 0
    qr, sar = oracle.inverse_rope_quant(d["o"], pos_ok, d["cos"], d["sin"], 64, lds=20)
    qg, sg = q.cpu().numpy(), sa.cpu().numpy()
    assert np.array_equal(qg[good], qr[good]) and np.array_equal(sg[:, good], sar[:, good])
    assert (qg[[3, 11]] == 0xAB).all() and (sg[:, [3, 11]] == -7.0).all()


# ---------------------------------------------------------------------------------------------
# block-diagonal GEMM
# ---------------------------------------------------------------------------------------------

def _weights(G, N_g, K_g, fmt, seed):
    w = inputs.randn_bf16((G, N_g, K_g), 0.02, seed, 7)
    parts = [oracle.quant_weight_block(w[g], fmt) for g in range(G)]
    return np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts])


def _run_diag(aq, sa, wq, sw, fmt):
    o = fq.gemm_w8a8_block_diag(dev_u8(aq), dev_f32(sa), dev_u8(wq),
                                dev_f32(sw) if fmt == 0 else dev_u8(sw), fmt)
    assert fq.check_device_error() == 0
    return host_bf16_f64(o)


@pytest.mark.parametrize("G,M,N_g,K_g", [(3, 200, 256, 384), (1, 130, 512, 256),
                                         (4, 1, 256, 128)])
@pytest.mark.parametrize("fmt", [0, 1])
def test_block_diag_gemm_small(G, M, N_g, K_g, fmt):
    x = inputs.randn_bf16((M, G * K_g), 1.0, 61, M + G)
    aq, sa = oracle.quant_token_1x128(x, lds=(M + 3) // 4 * 4)
    wq, sw = _weights(G, N_g, K_g, fmt, 61)
    got = _run_diag(aq, sa, wq, sw, fmt)
    ref, absref = oracle.gemm_w8a8_block_diag(aq, sa, wq, sw, fmt)
    assert_within_gemm_tolerance(got, ref, absref, f"diag G={G} M={M}", steps=promoted_steps(K_g))


def test_block_diag_with_one_group_is_the_dense_gemm():
    x = inputs.randn_bf16((256, 512), 1.0, 62, 0)
    aq, sa = oracle.quant_token_1x128(x)
    wq, sw = _weights(1, 512, 512, 0, 62)
    a = _run_diag(aq, sa, wq, sw, 0)
    b = host_bf16_f64(fq.gemm_w8a8_block(dev_u8(aq), dev_f32(sa), dev_u8(wq[0]),
                                         dev_f32(sw[0]), 0))
    assert np.array_equal(a, b)


def test_wo_a_path_full_size_sampled_rows():
    """8192 tokens x 32 heads x 512 (64 rotary dims), 4 head groups, 1024 outputs per group:
    inverse-RoPE quant (E8M0 scales) then the block-diagonal GEMM with E8M0 weight scales."""
    d = inputs.wo_a()
    T, H, D = d["o"].shape
    G, N_g, K_g = d["W"].shape
    pos, cs, sn = _dev_rope(d)
    q, sa = fq.inverse_rope_quant(dev_bf16(d["o"]), pos, cs, sn, 64, True, 1)
    parts = [oracle.quant_weight_block(d["W"][g], 1) for g in range(G)]
    wq = np.stack([p[0] for p in parts])
    sw = np.stack([p[1] for p in parts])
    out = fq.gemm_w8a8_block_diag(q, sa, dev_u8(wq), dev_u8(sw), 1)
    assert fq.check_device_error() == 0
    rows = np.unique(np.concatenate([[0, 127, 128, T - 1],
                                     np.random.default_rng(5).integers(0, T, 60)]))
    aq_r, sa_r = oracle.inverse_rope_quant(d["o"], d["positions"], d["cos"], d["sin"], 64,
                                           True, 1)
    ref, absref = oracle.gemm_w8a8_block_diag(aq_r, sa_r, wq, sw, 1, rows=rows)
    got = host_bf16_f64(out[torch.from_numpy(rows).cuda()])
    assert_within_gemm_tolerance(got, ref, absref, "wo_a full size", steps=promoted_steps(K_g))
