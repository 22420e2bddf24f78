"""GPU parity of the decode attention over the FP8 KV cache (fp8q_attention_decode) against the
oracle's fp64 reading R13, on caches and query codes quantized by the oracle: every head-group
size the kernel takes (Hq / Hkv = 1, 2, 4, 8), context lengths that fill, cross and fall short
of the 128-position tile and the split chunk (0, 1, 127, 128, 129, long), block sizes 1, 7 and 16,
block tables in random order, and bad block ids and lengths (recorded, not read).

The gate follows from the kernel's arithmetic: a score is a sum of D exact fp16 products in fp32
then one scale multiply, so |dz| <= (D + 2) 2^-24 zabs (zabs = |c| sum_d |dec q dec k|); the weights
move by at most 2|dz| relatively; they enter the value sums as fp16 (the tensor core's operand type:
at most 2^-11 relative); the value sums, the softmax sums, the chunk merge and exp2 add at most
(L + 16) 2^-23 of absref (= s_v sum_j p_j |dec v_j|); the bf16 rounding adds half an ulp:
    |out - ref| <= ulp_bf16(|ref|) / 2 + absref * (2^-11 + 2 (D + 2) 2^-24 zabs + (L + 16) 2^-23).

Source: "FP8-RL ...", abstract, item (ii) (FP8 KV cache; plain scaled dot-product attention).
"""
import numpy as np
import pytest
import torch

import oracle
import fp8_blockwise_w8a8_b200 as fq
from fp8_blockwise_w8a8_b200 import inputs

from helpers import host_bf16_f64

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def _quantize(d):
    """Codes and scales of the workload, by the oracle: the cache rows as K|V rows (no Q part),
    the query rows as Q|0|0 rows; the scales from the maxima of both."""
    Hq, Hkv, D = d["Hq"], d["Hkv"], d["D"]
    q, k, v = _bits(d["q"]), _bits(d["k"]), _bits(d["v"])
    S = k.shape[0]
    cache_rows = np.concatenate([k, v], axis=1)
    zkv = np.zeros((q.shape[0], Hkv * D), np.uint16)
    query_rows = np.concatenate([q, zkv, zkv], axis=1)
    a_c = oracle.qkv_amax(cache_rows, 0, Hkv, D)
    a_q = oracle.qkv_amax(query_rows, Hq, Hkv, D)
    s3 = oracle.qkv_scales(np.maximum(a_c, a_q))
    kc = np.zeros((S, Hkv * D), np.uint8)
    vc = np.zeros((S, Hkv * D), np.uint8)
    oracle.kv_cache_write(cache_rows, 0, Hkv, D, np.arange(S), s3, kc, vc)
    qc = oracle.kv_cache_write(query_rows, Hq, Hkv, D, -np.ones(q.shape[0]), s3, kc, vc)
    return qc, kc, vc, s3


def _run(qc, kc, vc, s3, bt, sl, Hq, Hkv, bs, max_seq_len, sm_scale=None):
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    o = fq.attention_decode(dev(qc), dev(kc), dev(vc), dev(np.asarray(s3, np.float32)), dev(bt),
                            dev(sl), Hq, Hkv, bs, max_seq_len, sm_scale=sm_scale)
    return o


def _check(o, qc, kc, vc, s3, bt, sl, Hq, Hkv, D, bs, sm_scale=None, rows=None):
    ref, absref, zabs = oracle.attention_decode(qc, kc, vc, s3, bt, sl, Hq, Hkv, D, bs, sm_scale)
    got = host_bf16_f64(o)
    rows = np.arange(qc.shape[0]) if rows is None else np.asarray(rows)
    L = np.clip(sl, 0, None).astype(np.float64)[:, None]
    zb = np.repeat(zabs, D, axis=1)
    bound = (oracle.bf16_ulp(np.abs(ref)) / 2 +
             absref * (2.0 ** -11 + 2 * (D + 2) * 2.0 ** -24 * zb + (L + 16) * 2.0 ** -23))
    err = np.abs(got[rows] - ref[rows])
    bad = err > bound[rows]
    assert not bad.any(), (f"{bad.sum()} of {bad.size} outside the bound; worst excess "
                           f"{(err - bound[rows]).max():.3e}")
    return ref


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (8, 4), (32, 8), (32, 4)])
def test_group_sizes_and_ragged_lengths(Hq, Hkv):
    d = inputs.decode_attention(Hq=Hq, Hkv=Hkv, seed=20 + Hq + Hkv,
                                lengths=[0, 1, 127, 128, 129, 700, 333])
    qc, kc, vc, s3 = _quantize(d)
    bt, sl = d["block_table"], d["seq_lens"]
    o = _run(qc, kc, vc, s3, bt, sl, Hq, Hkv, 16, 700)
    assert fq.check_device_error() == 0
    out = _check(o, qc, kc, vc, s3, bt, sl, Hq, Hkv, 128, 16)
    assert not host_bf16_f64(o)[0].any()                     # L = 0: zeros
    assert np.abs(out[1:]).max() > 0


@pytest.mark.parametrize("bs", [1, 7])
def test_block_sizes(bs):
    d = inputs.decode_attention(B=5, Hq=8, Hkv=2, block_size=bs, lmin=50, lmax=300, seed=30 + bs)
    qc, kc, vc, s3 = _quantize(d)
    o = _run(qc, kc, vc, s3, d["block_table"], d["seq_lens"], 8, 2, bs, d["max_seq_len"])
    assert fq.check_device_error() == 0
    _check(o, qc, kc, vc, s3, d["block_table"], d["seq_lens"], 8, 2, 128, bs)


def test_long_context_many_chunks_and_explicit_scale():
    """Two long sequences over many split chunks, and a non-default softmax scale."""
    d = inputs.decode_attention(B=2, Hq=16, Hkv=4, lmin=9000, lmax=12000, seed=40)
    qc, kc, vc, s3 = _quantize(d)
    o = _run(qc, kc, vc, s3, d["block_table"], d["seq_lens"], 16, 4, 16, d["max_seq_len"],
             sm_scale=0.25)
    assert fq.check_device_error() == 0
    _check(o, qc, kc, vc, s3, d["block_table"], d["seq_lens"], 16, 4, 128, 16, sm_scale=0.25)


def test_bad_block_ids_and_lengths_are_recorded():
    """A block id outside the cache and a length beyond max_seq_len record FP8Q_ERR_RANGE; the
    other sequences are unaffected, the too-long one is clamped to max_seq_len, and the one with
    the bad block stays finite (its positions in that block are skipped, nothing is read)."""
    d = inputs.decode_attention(B=3, Hq=8, Hkv=2, lmin=40, lmax=60, seed=50)
    qc, kc, vc, s3 = _quantize(d)
    bt = d["block_table"].copy()
    bt[1, 0] = 10 ** 6                                       # outside the cache
    sl = d["seq_lens"].copy()
    sl[2] = 10 ** 5                                          # beyond max_seq_len
    max_len = int(d["seq_lens"].max())
    o = _run(qc, kc, vc, s3, bt, sl, 8, 2, 16, max_len)
    assert fq.check_device_error() == 9                      # FP8Q_ERR_RANGE
    assert fq.check_device_error() == 0                      # the read cleared it
    ok_lens = np.array([sl[0], 0, max_len], np.int32)        # row 2 as clamped
    _check(o, qc, kc, vc, s3, d["block_table"], ok_lens, 8, 2, 128, 16, rows=[0, 2])
    assert np.isfinite(host_bf16_f64(o)[1]).all()


def test_decode_batch_full_size_sampled_sequences():
    """The bench's decode step (64 sequences, lengths U[512, 4096], 32 / 8 heads): sequences
    0, 17, 40 and 63 against the oracle."""
    d = inputs.decode_attention()
    qc, kc, vc, s3 = _quantize(d)
    o = _run(qc, kc, vc, s3, d["block_table"], d["seq_lens"], 32, 8, 16, d["max_seq_len"])
    assert fq.check_device_error() == 0
    rows = [0, 17, 40, 63]
    sub = np.zeros_like(d["seq_lens"])
    sub[rows] = d["seq_lens"][rows]
    _check(o, qc, kc, vc, s3, d["block_table"], sub, 32, 8, 128, 16, rows=rows)
