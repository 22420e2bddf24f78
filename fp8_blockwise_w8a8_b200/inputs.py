"""Seeded synthetic inputs for the blockwise FP8 W8A8 linear layer.

This module is shared by the tests, the benchmark and the oracle-side checks.  It draws random
numbers and rounds them to bf16 -- nothing else: it holds none of the quantization or GEMM
arithmetic, and it imports neither the CUDA binding nor the oracle.

bf16 tensors are returned as numpy ``uint16`` bit patterns (host) or torch ``bfloat16`` tensors
(device generator).  Recipes (per-tensor seed = 1000 * workload_seed + tensor_id):

* tiny linear      A [64, 512] ~ N(0,1), 1% of entries x20; W [256, 512] ~ N(0, 0.02); seed 0
* decode linear    A [128, 4096] ~ N(0,1), 20 (0.5%) channels x30; W [12288, 4096] ~ N(0,0.02);
                   seed 1
* prefill linear   X [8192, 4096] ~ N(0,1); gamma ~ U(0.5, 1.5); eps 1e-6;
                   W [24576, 4096] ~ N(0, 0.02); seed 2
* requant sweep    36 layers of {q 4096x4096, k/v 1024x4096, o 4096x4096, gate/up 12288x4096,
                   down 4096x12288} ~ N(0, 0.02), drawn per matrix with torch's generator on the
                   chosen device; seed 3
* MoE              4096 tokens, hidden 2048, 128 experts, top-8 distinct experts per token with
                   p_i proportional to rank^-1.1 over a seeded permutation of expert ids
                   (Gumbel-top-k); rows sorted by expert; gate/up input = the token rows
                   gathered in routed order; down input ~ N(0,1) [routed, 768];
                   W_gateup [128, 1536, 2048], W_down [128, 2048, 768] ~ N(0, 0.02); seed 4
* attention output projection (wo_a): o [8192, 32 heads, 512] ~ N(0,1) with the last 64 dims
                   of each head the rotary part; positions ~ U[0, 16384); cos/sin caches
                   [16384, 32] of the angle p * 10000^(-2i/64), computed in float64 and rounded
                   to fp32; 4 head groups, W_wo_a [4, 1024, 8 * 512] ~ N(0, 0.02); seed 5
* FP8 KV cache     QKV activations [8192 tokens, (32 + 2 x 8) heads x 128]: Q ~ N(0,1), K ~ N(0,1)
                   with 4 channels per head x 8, V ~ N(0, 0.5); a paged cache of 1024 blocks x 16
                   slots; each token gets a distinct random slot, 2 % of them -1 (padding, not
                   cached); seed 6
* decode attention over the FP8 KV cache: a batch of B = 64 sequences (one query token each),
                   context lengths ~ U[512, 4096]; a paged cache of block_size 16 whose blocks
                   are dealt to the sequences in a seeded random order (plus 8 spare blocks);
                   32 query heads, 8 kv heads, head_dim 128; Q ~ N(0,1), K ~ N(0,1) with 4
                   channels per head x 8, V ~ N(0, 0.5) for every cache slot, drawn with torch's
                   generator on the chosen device (bf16); seed 7.  A Llama/Qwen-8B-class decode
                   step; the pages give no shapes.
"""
import numpy as np
import torch


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 array -> bf16 bit patterns (uint16), round-to-nearest-even via torch on the CPU."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(a, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def rng_for(seed: int, tensor_id: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(1000 * seed + tensor_id))


def randn_bf16(shape, std: float, seed: int, tensor_id: int) -> np.ndarray:
    r = rng_for(seed, tensor_id)
    return to_bf16_bits(r.standard_normal(shape, dtype=np.float32) * np.float32(std))


# --- workloads ---------------------------------------------------------------------------------

def tiny_linear():
    seed = 0
    r = rng_for(seed, 0)
    a = r.standard_normal((64, 512), dtype=np.float32)
    mask = r.random((64, 512)) < 0.01
    a = np.where(mask, a * np.float32(20.0), a)
    return {"A": to_bf16_bits(a), "W": randn_bf16((256, 512), 0.02, seed, 1)}


def decode_linear(M: int = 128, N: int = 12288, K: int = 4096):
    seed = 1
    r = rng_for(seed, 0)
    a = r.standard_normal((M, K), dtype=np.float32)
    n_out = int(round(0.005 * K))
    ch = r.choice(K, size=n_out, replace=False)
    a[:, ch] *= np.float32(30.0)
    return {"A": to_bf16_bits(a), "W": randn_bf16((N, K), 0.02, seed, 1), "outlier_channels": ch}


def prefill_linear(M: int = 8192, N: int = 24576, K: int = 4096, with_weight: bool = True):
    seed = 2
    x = randn_bf16((M, K), 1.0, seed, 0)
    r = rng_for(seed, 1)
    gamma = to_bf16_bits(r.uniform(0.5, 1.5, size=K).astype(np.float32))
    out = {"X": x, "gamma": gamma, "eps": 1e-6}
    if with_weight:
        out["W"] = randn_bf16((N, K), 0.02, seed, 2)
    return out


SWEEP_LAYERS = 36
SWEEP_MATRICES = (("q", 4096, 4096), ("k", 1024, 4096), ("v", 1024, 4096), ("o", 4096, 4096),
                  ("gate", 12288, 4096), ("up", 12288, 4096), ("down", 4096, 12288))


def sweep_matrix(layer: int, index: int, device="cpu") -> torch.Tensor:
    """One weight of the 36-layer requant sweep as a bf16 torch tensor on ``device``."""
    seed = 3
    name, n, k = SWEEP_MATRICES[index]
    g = torch.Generator(device=device)
    g.manual_seed(1000 * seed + layer * len(SWEEP_MATRICES) + index)
    w = torch.randn((n, k), generator=g, device=device, dtype=torch.float32) * 0.02
    return w.to(torch.bfloat16)


def sweep_elements() -> int:
    return SWEEP_LAYERS * sum(n * k for _, n, k in SWEEP_MATRICES)


def moe_routing(tokens: int = 4096, experts: int = 128, topk: int = 8, alpha: float = 1.1,
                seed: int = 4):
    """Zipf-skewed top-k routing.  Returns (token index per routed row sorted by expert,
    group offsets int32 [experts + 1])."""
    r = rng_for(seed, 0)
    perm = r.permutation(experts)                   # expert id -> popularity rank
    rank = np.empty(experts, dtype=np.int64)
    rank[perm] = np.arange(experts)
    logp = -alpha * np.log(rank + 1.0)
    gumbel = -np.log(-np.log(r.random((tokens, experts))))
    choice = np.argsort(-(logp[None, :] + gumbel), axis=1)[:, :topk]  # distinct per token
    tok = np.repeat(np.arange(tokens), topk)
    exp = choice.reshape(-1)
    order = np.lexsort((tok, exp))                  # by expert, then token
    counts = np.bincount(exp, minlength=experts)
    off = np.zeros(experts + 1, dtype=np.int32)
    off[1:] = np.cumsum(counts)
    return tok[order].astype(np.int64), off


def moe(tokens: int = 4096, hidden: int = 2048, experts: int = 128, topk: int = 8,
        ffn: int = 768, with_weights: bool = True):
    seed = 4
    tok, off = moe_routing(tokens, experts, topk, 1.1, seed)
    x = randn_bf16((tokens, hidden), 1.0, seed, 1)
    out = {"tok": tok, "offsets": off, "X": x, "A_gateup": x[tok],
           "A_down": randn_bf16((tok.size, ffn), 1.0, seed, 2)}
    if with_weights:
        out["W_gateup"] = randn_bf16((experts, 2 * ffn, hidden), 0.02, seed, 3)
        out["W_down"] = randn_bf16((experts, hidden, ffn), 0.02, seed, 4)
    return out


def rope_caches(max_pos: int, rope_dim: int, base: float = 10000.0):
    """fp32 cos/sin tables [max_pos, rope_dim / 2] of the angles p * base^(-2i / rope_dim)."""
    inv_freq = base ** (-np.arange(0, rope_dim, 2, dtype=np.float64) / rope_dim)
    ang = np.arange(max_pos, dtype=np.float64)[:, None] * inv_freq[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def wo_a(tokens: int = 8192, heads: int = 32, head_dim: int = 512, rope_dim: int = 64,
         groups: int = 4, out_per_group: int = 1024, max_pos: int = 16384,
         with_weight: bool = True):
    seed = 5
    r = rng_for(seed, 1)
    cos, sin = rope_caches(max_pos, rope_dim)
    out = {"o": randn_bf16((tokens, heads, head_dim), 1.0, seed, 0),
           "positions": r.integers(0, max_pos, tokens).astype(np.int64),
           "cos": cos, "sin": sin}
    if with_weight:
        out["W"] = randn_bf16((groups, out_per_group, heads // groups * head_dim), 0.02, seed, 2)
    return out


def kv_cache(tokens: int = 8192, q_heads: int = 32, kv_heads: int = 8, head_dim: int = 128,
             num_blocks: int = 1024, block_size: int = 16):
    seed = 6
    r = rng_for(seed, 1)
    D = head_dim
    q = r.standard_normal((tokens, q_heads * D)).astype(np.float32)
    k = r.standard_normal((tokens, kv_heads, D)).astype(np.float32)
    outl = r.choice(D, size=4, replace=False)
    k[:, :, outl] *= 8.0
    v = (0.5 * r.standard_normal((tokens, kv_heads * D))).astype(np.float32)
    qkv = to_bf16_bits(np.concatenate([q, k.reshape(tokens, -1), v], axis=1))
    num_slots = num_blocks * block_size
    slots = r.permutation(num_slots)[:tokens].astype(np.int64)
    slots[r.random(tokens) < 0.02] = -1
    return {"qkv": qkv, "slots": slots, "num_slots": num_slots, "Hq": q_heads, "Hkv": kv_heads,
            "D": D}


def decode_attention(B: int = 64, Hq: int = 32, Hkv: int = 8, D: int = 128,
                     block_size: int = 16, lmin: int = 512, lmax: int = 4096, seed: int = 7,
                     device="cpu", lengths=None):
    """The decode-attention workload: bf16 q [B, Hq*D], k and v [num_slots, Hkv*D] (torch, on
    ``device``), int32 block_table [B, max_blocks] and seq_lens [B] (numpy).  ``lengths``
    replaces the drawn context lengths."""
    r = rng_for(seed, 0)
    seq_lens = r.integers(lmin, lmax + 1, size=B).astype(np.int32)
    if lengths is not None:
        seq_lens = np.asarray(lengths, np.int32)
        B = seq_lens.size
    nblk = -(-seq_lens // block_size)
    max_blocks = int(nblk.max()) if B else 1
    num_blocks = int(nblk.sum()) + 8
    order = r.permutation(num_blocks).astype(np.int32)
    block_table = np.zeros((B, max(max_blocks, 1)), np.int32)
    at = 0
    for b in range(B):
        block_table[b, :nblk[b]] = order[at:at + nblk[b]]
        at += nblk[b]
    num_slots = num_blocks * block_size
    g = torch.Generator(device=device)
    g.manual_seed(1000 * seed + 1)
    q = torch.randn((B, Hq * D), generator=g, device=device)
    k = torch.randn((num_slots, Hkv, D), generator=g, device=device)
    outl = torch.from_numpy(r.choice(D, size=4, replace=False)).to(device)
    k[:, :, outl] *= 8.0
    v = 0.5 * torch.randn((num_slots, Hkv * D), generator=g, device=device)
    return {"q": q.to(torch.bfloat16), "k": k.reshape(num_slots, Hkv * D).to(torch.bfloat16),
            "v": v.to(torch.bfloat16), "block_table": block_table, "seq_lens": seq_lens,
            "num_slots": num_slots, "block_size": block_size, "Hq": Hq, "Hkv": Hkv, "D": D,
            "max_seq_len": int(seq_lens.max()) if B else 0}
