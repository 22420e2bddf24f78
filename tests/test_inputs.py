"""The seeded input generators: deterministic, right shapes, routing well formed."""
import numpy as np

from fp8_blockwise_w8a8_b200 import inputs


def test_deterministic():
    a = inputs.tiny_linear()
    b = inputs.tiny_linear()
    assert np.array_equal(a["A"], b["A"]) and np.array_equal(a["W"], b["W"])
    assert a["A"].shape == (64, 512) and a["W"].shape == (256, 512)
    x = inputs.bf16_bits_to_f32(a["A"])
    assert np.abs(x).max() > 20          # the x20 outliers are present


def test_decode_outlier_channels():
    d = inputs.decode_linear(M=8, N=128, K=4096)
    x = np.abs(inputs.bf16_bits_to_f32(d["A"]))
    assert len(d["outlier_channels"]) == 20
    assert x[:, d["outlier_channels"]].mean() > 10 * x.mean() / 2


def test_moe_routing_properties():
    tok, off = inputs.moe_routing()
    assert off[0] == 0 and off[-1] == 4096 * 8 and np.all(np.diff(off) >= 0)
    assert tok.size == 4096 * 8
    counts = np.diff(off)
    assert counts.max() > 20 * max(counts.min(), 1)          # Zipf skew
    for e in (0, 64, 127):
        seg = tok[off[e]:off[e + 1]]
        assert np.all(np.diff(seg) > 0)                     # a token picks an expert once
    per_tok = np.bincount(tok, minlength=4096)
    assert np.all(per_tok == 8)


def test_sweep_shapes():
    assert inputs.sweep_elements() == 6_945_767_424
    w = inputs.sweep_matrix(0, 1, "cpu")
    assert tuple(w.shape) == (1024, 4096)
