"""Pins of the oracle's FP8 KV-cache path (reading R10: per-step per-tensor QKV scales, E4M3 codes
written at per-token cache slots): the maxima against numpy, the scale rule, the 448 code at each
tensor's maximum, every code against a brute-force nearest search over all finite E4M3 values
(ties to the even code), and the slot semantics (negative slots write nothing, other rows stay
untouched).  Every code of every tensor is also checked against numpy's IEEE fp32 quotient
encoded by ml_dtypes' E4M3 cast (round to nearest even, clamped to +-448), which catches a
reciprocal-multiply slip that a sample of a few hundred elements would miss."""
import ml_dtypes
import numpy as np

import oracle
from fp8_blockwise_w8a8_b200 import inputs


def _small(T=40, Hq=4, Hkv=2, D=64, num_slots=96):
    d = inputs.kv_cache(tokens=T, q_heads=Hq, kv_heads=Hkv, head_dim=D, num_blocks=num_slots // 16)
    return d


def _parts(d):
    x = inputs.bf16_bits_to_f32(d["qkv"])
    wq, wkv = d["Hq"] * d["D"], d["Hkv"] * d["D"]
    return x[:, :wq], x[:, wq:wq + wkv], x[:, wq + wkv:]


def test_amax_and_scales():
    d = _small()
    amax = oracle.qkv_amax(d["qkv"], d["Hq"], d["Hkv"], d["D"])
    for a, part in zip(amax, _parts(d)):
        assert a == np.abs(part).max()
    s = oracle.qkv_scales(amax)
    assert np.array_equal(s, (amax / np.float32(448.0)).astype(np.float32))
    assert np.array_equal(oracle.qkv_scales(np.zeros(3, np.float32)), np.ones(3, np.float32))


def _nearest_codes(v):
    """Brute force: the E4M3 code whose value is nearest each fp32 v (ties to the even code),
    saturating at +-448."""
    vals = oracle.e4m3_decode_all()
    finite = np.array([c for c in range(256) if np.isfinite(vals[c])])
    fv = vals[finite]
    out = np.empty(v.size, np.uint8)
    for i, x in enumerate(np.asarray(v, np.float64).ravel()):
        x = min(max(x, -448.0), 448.0)
        dist = np.abs(fv - x)
        best = finite[dist == dist.min()]
        if best.size > 1:
            best = best[(best & 1) == 0]
            if best.size > 1:              # +0 and -0: keep the sign of x
                best = best[(best >= 128) == (np.signbit(x))]
        out[i] = best[0]
    return out


def test_codes_against_brute_force_and_slots():
    d = _small()
    Hq, Hkv, D, ns = d["Hq"], d["Hkv"], d["D"], d["num_slots"]
    s = oracle.qkv_scales(oracle.qkv_amax(d["qkv"], Hq, Hkv, D))
    kc = np.full((ns, Hkv * D), 0xAA, np.uint8)
    vc = np.full((ns, Hkv * D), 0xAA, np.uint8)
    slots = d["slots"].copy()
    slots[[3, 17]] = -1
    qc = oracle.kv_cache_write(d["qkv"], Hq, Hkv, D, slots, s, kc, vc)
    q, k, v = _parts(d)
    rng = np.random.default_rng(0)
    for codes, x, sc in ((qc, q, s[0]), (kc[slots[slots >= 0]], k[slots >= 0], s[1]),
                         (vc[slots[slots >= 0]], v[slots >= 0], s[2])):
        idx = rng.choice(x.size, 400, replace=False)
        quot = (x.ravel()[idx] / sc).astype(np.float32)
        assert np.array_equal(codes.ravel()[idx], _nearest_codes(quot))
        # every element: IEEE fp32 division (numpy), then ml_dtypes' E4M3 rounding
        every = np.clip((x / np.float32(sc)).astype(np.float32), -448, 448)
        assert np.array_equal(codes, every.astype(ml_dtypes.float8_e4m3fn).view(np.uint8))
        # the tensor's maximum lands on the largest code
        i = np.argmax(np.abs(x))
        assert codes.ravel()[i] & 0x7F == 0x7E
    untouched = np.setdiff1d(np.arange(ns), slots[slots >= 0])
    assert (kc[untouched] == 0xAA).all() and (vc[untouched] == 0xAA).all()


def test_full_size_every_code_and_negative_control():
    """The bench's KV workload (8192 tokens, 32 + 2 x 8 heads of 128): all codes of Q, K and V
    against the independent chain; the reciprocal-multiply slip must change some of them."""
    d = inputs.kv_cache()
    Hq, Hkv, D, ns = d["Hq"], d["Hkv"], d["D"], d["num_slots"]
    s = oracle.qkv_scales(oracle.qkv_amax(d["qkv"], Hq, Hkv, D))
    kc = np.zeros((ns, Hkv * D), np.uint8)
    vc = np.zeros((ns, Hkv * D), np.uint8)
    slots = d["slots"]
    qc = oracle.kv_cache_write(d["qkv"], Hq, Hkv, D, slots, s, kc, vc)
    q, k, v = _parts(d)
    live = slots >= 0
    planted = 0
    for codes, x, sc in ((qc, q, s[0]), (kc[slots[live]], k[live], s[1]),
                         (vc[slots[live]], v[live], s[2])):
        t = np.clip((x / np.float32(sc)).astype(np.float32), -448, 448)
        assert np.array_equal(codes, t.astype(ml_dtypes.float8_e4m3fn).view(np.uint8))
        inv = np.float32(1.0) / np.float32(sc)
        slip = np.clip((x * inv).astype(np.float32), -448, 448)
        planted += int(np.count_nonzero(
            codes != slip.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)))
    assert planted > 0


def test_negative_slot_only_writes_q():
    d = _small(T=4)
    Hq, Hkv, D, ns = d["Hq"], d["Hkv"], d["D"], d["num_slots"]
    s = np.array([0.01, 0.02, 0.005], np.float32)
    kc = np.zeros((ns, Hkv * D), np.uint8)
    vc = np.zeros((ns, Hkv * D), np.uint8)
    qc = oracle.kv_cache_write(d["qkv"], Hq, Hkv, D, np.full(4, -1), s, kc, vc)
    assert not kc.any() and not vc.any()
    assert qc.any()
