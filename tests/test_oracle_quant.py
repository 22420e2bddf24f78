"""Pins of the oracle's block quantization (weight 128x128 blocks, token 1x128 groups).

Sources: "FP8-RL: A Practical and Stable Low-Precision Stack for LLM RL", abstract (i)
(blockwise FP8, weights requantized every step); "DeepSeek V4 performance: FP8 WO_A output
projection (vLLM PR 54894 analysis)" section 1 (E8M0, bias 127, lossless power-of-two rule),
section 2 (scale grid [out/128, in/128]) and section 3 (group-128 activation quant).
The pins are invariants and closed forms that any correct implementation must satisfy, so a
wrong divisor, a floor-vs-ceil exponent, a transposed scale grid or a dropped sign fails.
"""
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from fp8_blockwise_w8a8_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
DEC = None


def dec(codes):
    global DEC
    if DEC is None:
        DEC = oracle.e4m3_decode_all()
    return DEC[np.asarray(codes, dtype=np.uint8)]


def e4m3_half_ulp(v):
    """Half the E4M3 spacing at |v| (v within the finite range)."""
    a = np.abs(v)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    return np.ldexp(0.5, (e - 3).astype(np.int64))


def blocks(a, rb, cb):
    R, C = a.shape
    return a.reshape(R // rb, rb, C // cb, cb).transpose(0, 2, 1, 3)


# --- E8M0 --------------------------------------------------------------------------------------

def test_e8m0_lossless_rule_golden():
    with open(os.path.join(GOLDEN, "e8m0_lossless.txt")) as f:
        rows = [ln.split("#")[0].split() for ln in f if ln.split("#")[0].strip()]
    assert len(rows) >= 8
    for s, b in rows:
        want = None if b == "None" else int(b)
        assert oracle.e8m0_lossless_from_f32(float(s)) == want, s
        if want is not None:
            assert oracle.e8m0_decode(want) == float(s)


def test_e8m0_scales_are_minimal_powers_of_two():
    w = inputs.randn_bf16((256, 640), 0.02, 99, 0)
    wf = inputs.bf16_bits_to_f32(w).astype(np.float64)
    # widen the dynamic range so that the exponents vary across blocks
    w = inputs.to_bf16_bits(wf * np.repeat(np.repeat(
        2.0 ** np.arange(-12, 13, 2.5)[:10].reshape(2, 5), 128, 0), 128, 1))
    q, sw = oracle.quant_weight_block(w, oracle.SCALE_E8M0)
    x = inputs.bf16_bits_to_f32(w).astype(np.float64)
    bx = blocks(x, 128, 128)
    bq = blocks(q, 128, 128)
    for nb in range(sw.shape[0]):
        for kb in range(sw.shape[1]):
            byte = int(sw[nb, kb])
            s = oracle.e8m0_decode(byte)
            amax = Fraction(float(np.abs(bx[nb, kb]).max()))
            # smallest e with amax / 2^e <= 448, by exact rational search
            e = -127
            while amax / Fraction(2) ** e > 448:
                e += 1
            assert byte == e + 127
            # the page's lossless test accepts every scale we emit
            assert oracle.e8m0_lossless_from_f32(s) == byte
            # amax / 2^e lies in (224, 448]; after E4M3 rounding the largest code is in [224, 448]
            assert Fraction(224) < amax / Fraction(2) ** e <= 448
            vmax = np.abs(dec(bq[nb, kb])).max()
            assert 224 <= vmax <= 448


def test_e8m0_zero_block():
    w = np.zeros((128, 256), dtype=np.uint16)
    w[:, 128:] = inputs.randn_bf16((128, 128), 1.0, 5, 0)
    q, sw = oracle.quant_weight_block(w, oracle.SCALE_E8M0)
    assert sw[0, 0] == 127 and not q[:, :128].any()


# --- fp32 block scales -------------------------------------------------------------------------

def _check_fp32_block_quant(x, q, s):
    """Invariants of q = RNEsat(x / s) with s = amax / 448 (fp32) over one block."""
    x = x.astype(np.float64)
    amax = np.abs(x).max()
    if amax == 0:
        assert s == 1.0 and not (q & 0x7F).any()
        return
    # s is the fp32 rounding of amax/448: within half an fp32 ulp of the exact quotient
    exact = amax / 448.0
    assert abs(float(s) - exact) <= np.spacing(np.float32(exact)) / 2 * 1.0000001
    v = dec(q)
    # some element carries the full-scale code 448
    assert np.abs(v).max() == 448.0
    # every code is a nearest E4M3 value to x/s (allowing the fp32 rounding of the quotient)
    t = x / float(s)
    err = np.abs(np.clip(t, -448, 448) - v)
    assert np.all(err <= e4m3_half_ulp(t) * (1 + 2.0 ** -20) + np.abs(t) * 2.0 ** -23)
    # signs agree (zero codes keep the sign of x)
    assert np.all((q >> 7) == (np.signbit(x)).astype(np.uint8))


def test_weight_block_fp32_invariants_and_grid_layout():
    w = inputs.randn_bf16((384, 512), 0.02, 42, 0)
    # make block (1, 2) distinctive: amax 7.0 at a known spot
    w[128 + 5, 256 + 77] = inputs.to_bf16_bits(np.array([7.0], np.float32))[0]
    # block (2, 0) all zero
    w[256:384, 0:128] = 0
    q, sw = oracle.quant_weight_block(w, oracle.SCALE_F32)
    assert sw.shape == (3, 4) and sw.dtype == np.float32
    assert sw[1, 2] == np.float32(7.0) / np.float32(448.0)
    assert q[128 + 5, 256 + 77] == 0x7E
    assert sw[2, 0] == 1.0
    x = inputs.bf16_bits_to_f32(w)
    bx, bq = blocks(x, 128, 128), blocks(q, 128, 128)
    for nb in range(3):
        for kb in range(4):
            _check_fp32_block_quant(bx[nb, kb], bq[nb, kb], sw[nb, kb])


def test_weight_block_rejects_ragged_shapes():
    with pytest.raises(ValueError):
        oracle.quant_weight_block(np.zeros((128, 200), np.uint16))


def test_token_quant_invariants_and_layout():
    d = inputs.tiny_linear()
    a = d["A"]
    q, sa = oracle.quant_token_1x128(a, lds=68)
    assert sa.shape == (4, 68)
    x = inputs.bf16_bits_to_f32(a)
    for m in range(a.shape[0]):
        for kb in range(4):
            _check_fp32_block_quant(x[m, kb * 128:(kb + 1) * 128], q[m, kb * 128:(kb + 1) * 128],
                                    sa[kb, m])
    assert not sa[:, 64:].any()       # padding columns untouched (zero-initialised)


def test_token_quant_zero_row_and_outlier_group():
    x = np.zeros((2, 256), np.float32)
    x[1, :128] = np.linspace(-3, 3, 128)
    x[1, 200] = -1000.0
    q, sa = oracle.quant_token_1x128(inputs.to_bf16_bits(x))
    assert sa[0, 0] == 1.0 and sa[1, 0] == 1.0 and not q[0].any()
    assert sa[1, 1] == np.float32(1000.0) / np.float32(448.0)
    assert q[1, 200] == 0xFE
    assert sa[0, 1] == np.float32(3.0) / np.float32(448.0)


def test_token_quant_equals_weight_quant_on_single_row_blocks():
    """A 1x128 group is a 128x128 block of one distinct row repeated: the scale and codes must
    agree with the weight path on that block."""
    rng = np.random.default_rng(3)
    row = inputs.to_bf16_bits(rng.standard_normal((1, 256)).astype(np.float32))
    q1, sa = oracle.quant_token_1x128(row)
    w = np.repeat(row, 128, axis=0)
    q2, sw = oracle.quant_weight_block(w, oracle.SCALE_F32)
    assert np.array_equal(sa[:, 0], sw[0])
    assert np.array_equal(q1[0], q2[0]) and np.array_equal(q2[0], q2[127])


def test_sweep_qkv_split_equals_fused():
    """128-aligned q/k/v quantized separately equal the stacked matrix quantized at once."""
    qw = inputs.randn_bf16((256, 256), 0.02, 3, 10)
    kw = inputs.randn_bf16((128, 256), 0.02, 3, 11)
    vw = inputs.randn_bf16((128, 256), 0.02, 3, 12)
    fused_q, fused_s = oracle.quant_weight_block(np.concatenate([qw, kw, vw]))
    parts = [oracle.quant_weight_block(t) for t in (qw, kw, vw)]
    assert np.array_equal(fused_q, np.concatenate([p[0] for p in parts]))
    assert np.array_equal(fused_s, np.concatenate([p[1] for p in parts]))
