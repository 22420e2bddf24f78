"""Pins of the oracle's decode attention over the FP8 KV cache (its reading R13): each check is a
fact the definition fixes independently of how the oracle sums -- a single position returns its
value row, equal keys average the values, two keys weigh their values by the logistic of their
score gap, a large gap selects the argmax row exactly, query head h reads kv head h / (Hq / Hkv),
the block table (not the physical slot order) decides which rows a sequence sees, and the scales
enter as the products the definition states.

Source: "FP8-RL ...", abstract, item (ii) (FP8 KV cache with per-step QKV scale recalibration; the
attention arithmetic is the plain scaled dot-product reading R13).
"""
import math

import numpy as np

import oracle

DEC = oracle.e4m3_decode_all()


def _codes(shape, rng, lo=0x08, hi=0x6E):
    """Random finite E4M3 codes of both signs with magnitudes from 2^-6 to 240."""
    c = rng.integers(lo, hi + 1, size=shape).astype(np.uint8)
    return c | (rng.integers(0, 2, size=shape).astype(np.uint8) << 7)


def _case(B=3, Hq=8, Hkv=2, D=64, bs=4, L=(5, 9, 1), seed=0):
    rng = np.random.default_rng(seed)
    maxb = max(-(-l // bs) for l in L)
    nblocks = B * maxb + 3
    perm = rng.permutation(nblocks)[:B * maxb].reshape(B, maxb).astype(np.int32)
    k = _codes((nblocks * bs, Hkv * D), rng)
    v = _codes((nblocks * bs, Hkv * D), rng)
    q = _codes((B, Hq * D), rng, hi=0x40)
    return q, k, v, perm, np.array(L, np.int32)


def test_single_position_returns_its_value_row():
    q, k, v, bt, _ = _case()
    sl = np.array([1, 1, 1], np.int32)
    s3 = (0.5, 0.25, 3.0)
    out, absref, _ = oracle.attention_decode(q, k, v, s3, bt, sl, 8, 2, 64, 4)
    for b in range(3):
        slot = bt[b, 0] * 4
        for h in range(8):
            g = h // 4
            np.testing.assert_array_equal(out[b, h * 64:(h + 1) * 64],
                                          3.0 * DEC[v[slot, g * 64:(g + 1) * 64]])
    assert np.all(absref >= np.abs(out))


def test_equal_keys_average_the_values():
    q, k, v, bt, sl = _case(L=(7, 12, 3))
    k[:] = k[0]                                      # every position has the same key
    out, _, _ = oracle.attention_decode(q, k, v, (1.0, 1.0, 2.0), bt, sl, 8, 2, 64, 4)
    for b, L in enumerate(sl):
        slots = [bt[b, j // 4] * 4 + j % 4 for j in range(L)]
        for h in range(8):
            g = h // 4
            mean = DEC[v[slots, g * 64:(g + 1) * 64]].mean(axis=0)
            np.testing.assert_allclose(out[b, h * 64:(h + 1) * 64], 2.0 * mean, rtol=1e-14,
                                       atol=1e-300)


def test_two_keys_weigh_by_the_logistic_of_the_score_gap():
    """Query and keys nonzero in dimension 0 only: z_j = c * dec(q_0) * dec(k_j0)."""
    D, bs = 32, 2
    q = np.zeros((1, D), np.uint8)
    q[0, 0] = 0x38                                   # 1.0
    k = np.zeros((2, D), np.uint8)
    k[0, 0], k[1, 0] = 0x40, 0x48                    # 2.0, 4.0
    v = np.zeros((2, D), np.uint8)
    v[0, :] = 0x38                                   # 1.0
    v[1, :] = 0xB8                                   # -1.0
    bt = np.zeros((1, 1), np.int32)
    sl = np.array([2], np.int32)
    sm, sq, sk, sv = 0.375, 0.5, 1.5, 0.75
    out, _, zabs = oracle.attention_decode(q, k, v, (sq, sk, sv), bt, sl, 1, 1, D, bs, sm)
    c = sm * sq * sk
    p0 = 1.0 / (1.0 + math.exp(c * 4.0 - c * 2.0))
    np.testing.assert_allclose(out[0], sv * (p0 - (1.0 - p0)), rtol=1e-14)
    assert zabs[0, 0] == c * 4.0


def test_large_gap_selects_the_argmax_row_exactly():
    q, k, v, bt, sl = _case(B=1, L=(10,), seed=3)
    Hq, Hkv, D = 8, 2, 64
    k[:] = 0x00                                      # every score 0 ...
    j_star = 6
    slot = bt[0, j_star // 4] * 4 + j_star % 4
    q[:] = 0x38                                      # ... except at j* where q.k = 64 * 448
    k[slot, :] = 0x7E
    out, _, _ = oracle.attention_decode(q, k, v, (1.0, 1.0, 1.0), bt, sl, Hq, Hkv, D, 4, 1.0)
    for h in range(Hq):
        g = h // 4
        np.testing.assert_array_equal(out[0, h * D:(h + 1) * D], DEC[v[slot, g * D:(g + 1) * D]])


def test_query_head_h_reads_kv_head_h_over_group_size():
    """GQA with Hq = 8, Hkv = 2 equals multi-head attention whose 8 kv heads repeat each of the
    two, four times (head h -> kv head h // 4, not h % 2)."""
    q, k, v, bt, sl = _case()
    D = 64
    out, _, _ = oracle.attention_decode(q, k, v, (1.0, 0.5, 1.0), bt, sl, 8, 2, D, 4)
    rep = lambda c: np.concatenate([np.tile(c[:, g * D:(g + 1) * D], 4) for g in range(2)], axis=1)
    out_mha, _, _ = oracle.attention_decode(q, rep(k), rep(v), (1.0, 0.5, 1.0), bt, sl, 8, 8, D, 4)
    np.testing.assert_array_equal(out, out_mha)
    wrong = lambda c: np.concatenate([c] * 4, axis=1)        # kv head h % 2
    out_wrong, _, _ = oracle.attention_decode(q, wrong(k), wrong(v), (1.0, 0.5, 1.0), bt, sl, 8, 8,
                                              D, 4)
    assert not np.allclose(out, out_wrong)


def test_the_block_table_decides_which_rows_a_sequence_sees():
    """The same logical sequences stored in other physical blocks give identical outputs; a
    shuffled table (other rows) does not."""
    q, k, v, bt, sl = _case(seed=5)
    bs = 4
    out, _, _ = oracle.attention_decode(q, k, v, (1.0, 1.0, 1.0), bt, sl, 8, 2, 64, bs)
    nblocks = k.shape[0] // bs
    perm = np.random.default_rng(9).permutation(nblocks)       # move block i to block perm[i]
    k2, v2 = np.empty_like(k), np.empty_like(v)
    for i in range(nblocks):
        k2[perm[i] * bs:(perm[i] + 1) * bs] = k[i * bs:(i + 1) * bs]
        v2[perm[i] * bs:(perm[i] + 1) * bs] = v[i * bs:(i + 1) * bs]
    out2, _, _ = oracle.attention_decode(q, k2, v2, (1.0, 1.0, 1.0), perm[bt].astype(np.int32), sl,
                                         8, 2, 64, bs)
    np.testing.assert_array_equal(out, out2)
    out3, _, _ = oracle.attention_decode(q, k, v, (1.0, 1.0, 1.0), bt[::-1].copy(), sl, 8, 2,
                                         64, bs)
    assert not np.allclose(out, out3)


def test_scales_enter_as_stated():
    q, k, v, bt, sl = _case(seed=7)
    base, _, _ = oracle.attention_decode(q, k, v, (0.5, 0.25, 1.0), bt, sl, 8, 2, 64, 4, 0.125)
    dbl, _, _ = oracle.attention_decode(q, k, v, (0.5, 0.25, 2.0), bt, sl, 8, 2, 64, 4, 0.125)
    np.testing.assert_array_equal(dbl, 2.0 * base)                       # o is linear in s_v
    swp, _, _ = oracle.attention_decode(q, k, v, (0.25, 0.5, 1.0), bt, sl, 8, 2, 64, 4, 0.125)
    np.testing.assert_array_equal(swp, base)                             # only s_q s_k matters
    mov, _, _ = oracle.attention_decode(q, k, v, (1.0, 0.25, 1.0), bt, sl, 8, 2, 64, 4, 0.0625)
    np.testing.assert_array_equal(mov, base)                             # ... times sm_scale
    flat, _, _ = oracle.attention_decode(q, k, v, (0.5, 0.25, 1.0), bt, sl, 8, 2, 64, 4, 0.0)
    assert not np.allclose(flat, base)                                   # sm_scale is used


def test_empty_sequence_gives_zero():
    q, k, v, bt, _ = _case()
    out, absref, zabs = oracle.attention_decode(q, k, v, (1.0, 1.0, 1.0), bt,
                                                np.array([0, 3, 0], np.int32), 8, 2, 64, 4)
    assert not out[0].any() and not out[2].any() and out[1].any()
    assert not absref[0].any() and zabs[0].max() == 0.0
