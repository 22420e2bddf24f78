"""Pins of the oracle's E4M3 codec and bf16 rounding against sources other than the oracle.

The E4M3 format is the OCP FP8 E4M3 element type (dtype float8_e4m3fn in the torchao config of
the veRL torchao-rollout PR page; OCP MX spec linked from the vLLM PR 54894 analysis).
"""
import math
import os

import ml_dtypes
import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _finite_codes():
    return [c for c in range(256) if c not in (0x7F, 0xFF)]


def test_decode_matches_torch_and_ml_dtypes():
    ours = oracle.e4m3_decode_all()
    codes = np.arange(256, dtype=np.uint8)
    t = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    m = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    for c in range(256):
        if math.isnan(ours[c]):
            assert math.isnan(t[c]) and math.isnan(m[c]), hex(c)
        else:
            assert ours[c] == t[c] == m[c], hex(c)
            assert math.copysign(1, ours[c]) == math.copysign(1, t[c]), hex(c)


def test_decode_golden_codes():
    rows = []
    with open(os.path.join(GOLDEN, "e4m3_special_codes.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                code, val = line.split()
                rows.append((int(code, 16), float(val)))
    assert len(rows) >= 10
    for code, val in rows:
        got = oracle.e4m3_decode(code)
        if math.isnan(val):
            assert math.isnan(got), hex(code)
        else:
            assert got == val and math.copysign(1, got) == math.copysign(1, val), hex(code)


def test_format_extremes():
    vals = oracle.e4m3_decode_all()
    finite = vals[~np.isnan(vals)]
    assert finite.size == 254
    assert finite.max() == 448.0 and finite.min() == -448.0
    assert np.min(np.abs(finite[finite != 0])) == 2.0 ** -9


def test_encode_roundtrip_every_finite_code():
    vals = oracle.e4m3_decode_all()
    codes = _finite_codes()
    enc = oracle.e4m3_encode(np.array([vals[c] for c in codes], dtype=np.float32))
    assert list(enc) == codes


def test_encode_midpoints_go_to_even_code():
    vals = oracle.e4m3_decode_all()
    for c in range(0, 126):          # positive neighbours c, c+1
        mid = (vals[c] + vals[c + 1]) / 2
        assert np.float32(mid) == mid     # midpoints are exact in fp32
        even = c if c % 2 == 0 else c + 1
        assert oracle.e4m3_encode([mid])[0] == even, hex(c)
        assert oracle.e4m3_encode([-mid])[0] == even | 0x80, hex(c)
        # just off the midpoint goes to the nearer neighbour
        below = np.nextafter(np.float32(mid), np.float32(0))
        above = np.nextafter(np.float32(mid), np.float32(1e9))
        assert oracle.e4m3_encode([below])[0] == c
        assert oracle.e4m3_encode([above])[0] == c + 1


def test_encode_saturates():
    big = np.array([448.0, 448.0001, 463.99, 464.0, 500.0, 1e6, 3.4e38], dtype=np.float32)
    assert list(oracle.e4m3_encode(big)) == [0x7E] * len(big)
    assert list(oracle.e4m3_encode(-big)) == [0xFE] * len(big)


def test_encode_sign_of_zero_kept():
    assert list(oracle.e4m3_encode([0.0, -0.0, -1e-30, 1e-30, -2.0 ** -10])) == \
        [0x00, 0x80, 0x80, 0x00, 0x80]


def test_encode_exhaustive_against_table_search():
    """Every finite fp32 bit pattern (2^32 - 2^24 of them) against an independent nearest-value
    search over the sorted table of E4M3 values (C, multi-threaded)."""
    bad, first = oracle.e4m3_encode_exhaustive_check()
    assert bad == 0, f"{bad} mismatches, first at bits {first:#010x}"


def _torch_rnesat(v: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(v.astype(np.float32)).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def test_encode_matches_torch_cast_on_boundaries_and_random_bits():
    vals = oracle.e4m3_decode_all()
    pts = []
    for c in range(0, 127):
        for v in (vals[c], (vals[c] + vals[min(c + 1, 126)]) / 2):
            f = np.float32(v)
            for d in range(-4, 5):
                g = f
                step = np.float32(1e9) if d > 0 else np.float32(0)
                for _ in range(abs(d)):
                    g = np.nextafter(g, step)
                pts.append(g)
    pts = np.array(pts, dtype=np.float32)
    pts = np.concatenate([pts, -pts])
    rng = np.random.default_rng(123)
    bits = rng.integers(0, 2 ** 32, size=4_000_000, dtype=np.uint64).astype(np.uint32)
    bits = bits[((bits >> 23) & 0xFF) != 0xFF]
    rand = bits.view(np.float32)
    # random patterns concentrated in the E4M3 range too
    scaled = (rng.standard_normal(4_000_000) * 100).astype(np.float32)
    for v in (pts, rand, scaled):
        assert np.array_equal(oracle.e4m3_encode(v), _torch_rnesat(v))


def test_encode_matches_ml_dtypes_in_range():
    rng = np.random.default_rng(7)
    v = (rng.standard_normal(2_000_000) * 50).astype(np.float32)
    v = np.clip(v, -448, 448)
    ref = v.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(oracle.e4m3_encode(v), ref)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(11)
    bits = rng.integers(0, 2 ** 32, size=2_000_000, dtype=np.uint64).astype(np.uint32)
    bits = bits[((bits >> 23) & 0xFF) != 0xFF]
    # avoid the few patterns that overflow bf16 to infinity: the oracle never rounds them
    v = bits.view(np.float32)
    v = v[np.abs(v) < 3.3e38]
    t = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.f32_to_bf16(v), t)
    # exact ties
    ties = (np.arange(1, 5000, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    t = torch.from_numpy(ties).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.f32_to_bf16(ties), t)
