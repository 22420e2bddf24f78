"""Blockwise FP8 (E4M3) W8A8 linear layer on B200 (sm_100a).

Thin torch-facing binding over the C ABI of ``libfp8q.so`` (declared in include/fp8q.h).  These
functions only marshal arguments -- tensors become device pointers, the current torch CUDA stream
becomes the launch stream, missing outputs are allocated with torch -- and every step of the
computation runs in the library's CUDA kernels.  There is no CPU or PyTorch fallback: a missing
library or a non-sm_100 device raises.

    quant_weight_block(w, fmt)                 bf16 [N, K] -> (codes u8 [N, K], scales [N/128, K/128])
    rmsnorm_quant_token(x, gamma, eps)         bf16 [M, K] -> (codes u8 [M, K], sa f32 [K/128, lds])
    gemm_w8a8_block(aq, sa, wq, sw, fmt)       -> bf16 [M, N]
    gemm_w8a8_block_splitk(aq, sa, wq, sw, ...) -> bf16 [M, N], K split over CTAs (small M)
    grouped_gemm_w8a8_block(aq, sa, wq, sw, offsets, fmt) -> bf16 [M, N]
"""
import numpy as np
import torch

from . import _lib
from ._lib import (FP8Q_ERR_ALIGN, FP8Q_ERR_ARCH, FP8Q_ERR_ARG, FP8Q_ERR_LAUNCH, FP8Q_ERR_NULL,
                   FP8Q_ERR_NOT_POW2, FP8Q_ERR_RANGE, FP8Q_ERR_SHAPE, FP8Q_ERR_TIMEOUT, FP8Q_OK, FP8Q_SCALE_E8M0, FP8Q_SCALE_F32,
                   Fp8qError)

import ctypes

__all__ = ["quant_weight_block", "rmsnorm_quant_token", "add_rmsnorm_quant", "gemm_w8a8_block",
           "gemm_w8a8_block_splitk", "gemm_splitk_workspace_bytes", "splitk_workspace",
           "quant_rowwise", "gemm_w8a8_rowwise", "silu_mul_quant", "inverse_rope_quant",
           "gemm_w8a8_block_diag", "gemm_w8a8_mx", "qkv_scales", "kv_cache_write", "WeightBatch",
           "selftest_timeout", "attention_decode", "attention_decode_workspace_bytes",
           "grouped_gemm_w8a8_block", "check_device_error", "Fp8qError", "FP8Q_SCALE_F32",
           "FP8Q_SCALE_E8M0", "scale_format"]


def scale_format(fmt) -> int:
    if fmt in (FP8Q_SCALE_F32, "f32", "fp32", torch.float32):
        return FP8Q_SCALE_F32
    if fmt in (FP8Q_SCALE_E8M0, "e8m0", torch.uint8):
        return FP8Q_SCALE_E8M0
    raise ValueError(f"unknown scale format {fmt!r}")


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _ld(t: torch.Tensor) -> int:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("expected a 2-D tensor with unit stride along its last dimension")
    return t.stride(0)


def quant_weight_block(w: torch.Tensor, fmt="f32", out_q=None, out_s=None, stream=None):
    """bf16 W [N, K] -> (E4M3 codes uint8 [N, K], block scales [N/128, K/128] fp32 or E8M0)."""
    f = scale_format(fmt)
    N, K = w.shape
    q = torch.empty((N, K), dtype=torch.uint8, device=w.device) if out_q is None else out_q
    s = (torch.empty((N // 128, K // 128), device=w.device,
                     dtype=torch.float32 if f == FP8Q_SCALE_F32 else torch.uint8)
         if out_s is None else out_s)
    st = _lib.lib().fp8q_quant_weight_block(_ptr(w), N, K, _ld(w), _ptr(q), _ld(q), _ptr(s), f,
                                            _stream(stream))
    _lib.check(st, "fp8q_quant_weight_block")
    return q, s


class WeightBatch:
    """A fixed list of bf16 weights [N_i, K_i] requantized together in one launch
    (fp8q_quant_weight_block_batched).  Builds the output codes and scales once and a device
    table of descriptors; run() requantizes every weight into them (e.g. once per step, after
    the weights changed in place)."""

    _DESC = np.dtype([("w", "<u8"), ("q", "<u8"), ("s", "<u8"), ("N", "<i8"), ("K", "<i8"),
                      ("ldw", "<i8"), ("ldq", "<i8"), ("off", "<i8")])

    def __init__(self, weights, fmt="f32"):
        self.fmt = scale_format(fmt)
        self.weights = list(weights)
        if not self.weights:
            raise ValueError("empty weight list")
        dev = self.weights[0].device
        sdt = torch.float32 if self.fmt == FP8Q_SCALE_F32 else torch.uint8
        self.q, self.s = [], []
        desc = np.zeros(len(self.weights), self._DESC)
        off = 0
        for i, w in enumerate(self.weights):
            N, K = w.shape
            q = torch.empty((N, K), dtype=torch.uint8, device=dev)
            sc = torch.empty((N // 128, K // 128), dtype=sdt, device=dev)
            self.q.append(q)
            self.s.append(sc)
            desc[i] = (w.data_ptr(), q.data_ptr(), sc.data_ptr(), N, K, _ld(w), _ld(q), off)
            off += (N // 128) * (K // 128)
        self.total_blocks = off
        self.desc = torch.from_numpy(desc.view(np.uint8).copy()).to(dev)

    def run(self, stream=None):
        st = _lib.lib().fp8q_quant_weight_block_batched(_ptr(self.desc), len(self.weights),
                                                        self.total_blocks, self.fmt,
                                                        _stream(stream))
        _lib.check(st, "fp8q_quant_weight_block_batched")
        return self.q, self.s


def rmsnorm_quant_token(x: torch.Tensor, gamma=None, eps: float = 1e-6, lds=None, out_q=None,
                        out_sa=None, stream=None, scale_fmt="f32"):
    """bf16 X [M, K] -> (codes uint8 [M, K], sa fp32 [K/128, lds]); sa[kb, m] is the scale of
    row m, K-block kb.  gamma=None: plain 1x128 token quant without RMSNorm.  scale_fmt "e8m0":
    power-of-two scales (stored as fp32) through fp8q_rmsnorm_quant_token_fmt."""
    f = scale_format(scale_fmt)
    M, K = x.shape
    if lds is None:
        lds = max(4, (M + 3) // 4 * 4)
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device) if out_q is None else out_q
    sa = (torch.empty((K // 128, lds), dtype=torch.float32, device=x.device)
          if out_sa is None else out_sa)
    if f == FP8Q_SCALE_F32:
        st = _lib.lib().fp8q_rmsnorm_quant_token(_ptr(x), _ptr(gamma), float(eps), M, K, _ld(x),
                                                 _ptr(q), _ld(q), _ptr(sa), sa.stride(0),
                                                 _stream(stream))
        _lib.check(st, "fp8q_rmsnorm_quant_token")
    else:
        st = _lib.lib().fp8q_rmsnorm_quant_token_fmt(_ptr(x), _ptr(gamma), float(eps), M, K,
                                                     _ld(x), _ptr(q), _ld(q), _ptr(sa),
                                                     sa.stride(0), f, _stream(stream))
        _lib.check(st, "fp8q_rmsnorm_quant_token_fmt")
    return q, sa


def gemm_w8a8_block(aq: torch.Tensor, sa: torch.Tensor, wq: torch.Tensor, sw: torch.Tensor,
                    fmt=None, out=None, stream=None):
    """Codes aq [M, K] (scales sa [K/128, lds]) x codes wq [N, K] (scales sw [N/128, K/128])
    -> bf16 [M, N]."""
    f = scale_format(sw.dtype if fmt is None else fmt)
    M, K = aq.shape
    N = wq.shape[0]
    o = torch.empty((M, N), dtype=torch.bfloat16, device=aq.device) if out is None else out
    st = _lib.lib().fp8q_gemm_w8a8_block(_ptr(aq), _ld(aq), _ptr(sa), sa.stride(0), _ptr(wq),
                                         _ld(wq), _ptr(sw), f, M, N, K, _ptr(o), _ld(o),
                                         _stream(stream))
    _lib.check(st, "fp8q_gemm_w8a8_block")
    return o


def gemm_splitk_workspace_bytes(M: int, N: int, K: int, splits: int = 0) -> int:
    """Bytes of split-K workspace for these sizes (splits=0: the library's choice)."""
    b = ctypes.c_int64(0)
    st = _lib.lib().fp8q_gemm_splitk_workspace_bytes(M, N, K, int(splits), ctypes.byref(b))
    _lib.check(st, "fp8q_gemm_splitk_workspace_bytes")
    return b.value


def splitk_workspace(M: int, N: int, K: int, splits: int = 0, device=None) -> torch.Tensor:
    """A workspace for gemm_w8a8_block_splitk (no initialisation needed); reusable by later calls
    in stream order."""
    n = gemm_splitk_workspace_bytes(M, N, K, splits)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def gemm_w8a8_block_splitk(aq: torch.Tensor, sa: torch.Tensor, wq: torch.Tensor,
                           sw: torch.Tensor, fmt=None, splits: int = 0, workspace=None, out=None,
                           stream=None):
    """gemm_w8a8_block with K split over several CTAs per output tile.  `workspace` is a uint8
    device tensor of gemm_splitk_workspace_bytes(M, N, K, splits) bytes, reused across calls on
    one stream; None allocates a fresh one."""
    f = scale_format(sw.dtype if fmt is None else fmt)
    M, K = aq.shape
    N = wq.shape[0]
    if workspace is None:
        workspace = splitk_workspace(M, N, K, splits, device=aq.device)
    o = torch.empty((M, N), dtype=torch.bfloat16, device=aq.device) if out is None else out
    st = _lib.lib().fp8q_gemm_w8a8_block_splitk(_ptr(aq), _ld(aq), _ptr(sa), sa.stride(0),
                                                _ptr(wq), _ld(wq), _ptr(sw), f, M, N, K, _ptr(o),
                                                _ld(o), int(splits), _ptr(workspace),
                                                workspace.numel() * workspace.element_size(),
                                                _stream(stream))
    _lib.check(st, "fp8q_gemm_w8a8_block_splitk")
    return o


def attention_decode_workspace_bytes(B: int, Hq: int, Hkv: int, D: int, max_seq_len: int) -> int:
    b = ctypes.c_int64(0)
    st = _lib.lib().fp8q_attention_decode_workspace_bytes(B, Hq, Hkv, D, max_seq_len,
                                                          ctypes.byref(b))
    _lib.check(st, "fp8q_attention_decode_workspace_bytes")
    return b.value


def attention_decode(q_codes: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                     scale3: torch.Tensor, block_table: torch.Tensor, seq_lens: torch.Tensor,
                     Hq: int, Hkv: int, block_size: int, max_seq_len: int, sm_scale=None,
                     workspace=None, out=None, stream=None):
    """Decode attention over the FP8 KV cache (fp8q_attention_decode): q_codes uint8 [B, Hq*D],
    caches uint8 [slots, Hkv*D], scale3 fp32 [3] (s_q, s_k, s_v), block_table int32 [B, max
    blocks], seq_lens int32 [B] -> bf16 [B, Hq*D].  sm_scale defaults to 1/sqrt(D)."""
    B = q_codes.shape[0]
    D = k_cache.shape[1] // Hkv
    if sm_scale is None:
        sm_scale = 1.0 / float(np.sqrt(D))
    if workspace is None:
        n = attention_decode_workspace_bytes(B, Hq, Hkv, D, max_seq_len)
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q_codes.device)
    o = torch.empty((B, Hq * D), dtype=torch.bfloat16, device=q_codes.device) if out is None else out
    st = _lib.lib().fp8q_attention_decode(
        _ptr(q_codes), _ld(q_codes), _ptr(k_cache), _ptr(v_cache), k_cache.shape[0],
        _ptr(scale3), _ptr(block_table), block_table.shape[1], _ptr(seq_lens), B, Hq, Hkv, D,
        block_size, max_seq_len, float(sm_scale), _ptr(o), _ld(o), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _lib.check(st, "fp8q_attention_decode")
    return o


def grouped_gemm_w8a8_block(aq: torch.Tensor, sa: torch.Tensor, wq: torch.Tensor,
                            sw: torch.Tensor, group_offsets: torch.Tensor, fmt=None, out=None,
                            stream=None):
    """Rows [off[e], off[e+1]) of aq times expert e's codes wq[e] ([E, N, K], scales
    sw [E, N/128, K/128]) -> bf16 [M, N].  group_offsets: int32 [E+1] on the device."""
    f = scale_format(sw.dtype if fmt is None else fmt)
    M, K = aq.shape
    E, N, K2 = wq.shape
    if K2 != K:
        raise ValueError("K mismatch")
    if wq.stride(2) != 1 or wq.stride(0) != N * wq.stride(1):
        raise ValueError("wq must be [E, N, K] with expert stride N * ldw")
    if group_offsets.dtype != torch.int32 or group_offsets.numel() != E + 1:
        raise ValueError("group_offsets must be int32 [E + 1]")
    o = torch.empty((M, N), dtype=torch.bfloat16, device=aq.device) if out is None else out
    st = _lib.lib().fp8q_grouped_gemm_w8a8_block(_ptr(aq), _ld(aq), _ptr(sa), sa.stride(0),
                                                 _ptr(wq), wq.stride(1), _ptr(sw), f,
                                                 _ptr(group_offsets), E, M, N, K, _ptr(o),
                                                 _ld(o), _stream(stream))
    _lib.check(st, "fp8q_grouped_gemm_w8a8_block")
    return o


def silu_mul_quant(h: torch.Tensor, lds=None, out_q=None, out_sa=None, stream=None,
                   scale_fmt="f32"):
    """h = [gate | up] bf16 [R, 2I] -> (codes uint8 [R, I] of bf16(silu(gate) * up),
    sa fp32 [I/128, lds]): the front end of an MoE down projection.  scale_fmt "e8m0":
    power-of-two scales stored as fp32."""
    f = scale_format(scale_fmt)
    R, I2 = h.shape
    I = I2 // 2
    if lds is None:
        lds = max(4, (R + 3) // 4 * 4)
    q = torch.empty((R, I), dtype=torch.uint8, device=h.device) if out_q is None else out_q
    sa = (torch.empty((I // 128, lds), dtype=torch.float32, device=h.device)
          if out_sa is None else out_sa)
    st = _lib.lib().fp8q_silu_mul_quant(_ptr(h), R, I, _ld(h), _ptr(q), _ld(q), _ptr(sa),
                                        sa.stride(0), f, _stream(stream))
    _lib.check(st, "fp8q_silu_mul_quant")
    return q, sa


def inverse_rope_quant(o: torch.Tensor, positions: torch.Tensor, cos_cache: torch.Tensor,
                       sin_cache: torch.Tensor, rope_dim: int, interleaved: bool = True,
                       fmt=FP8Q_SCALE_F32, lds=None, out_q=None, out_sa=None, stream=None):
    """Attention output o bf16 [T, H, D] (token stride o.stride(0); heads contiguous) ->
    (codes uint8 [T, H*D], sa fp32 [H*D/128, lds]): inverse RoPE of the last rope_dim dims of
    each head at the tokens' positions (int64 [T]; fp32 cos/sin caches [max_pos, rope_dim/2]),
    then 1x128 quant; fmt SCALE_E8M0 gives power-of-two scales (stored as fp32)."""
    T, H, D = o.shape
    if o.stride(2) != 1 or o.stride(1) != D:
        raise ValueError("o must have contiguous heads: strides (ldo, D, 1)")
    K = H * D
    if lds is None:
        lds = max(4, (T + 3) // 4 * 4)
    q = torch.empty((T, K), dtype=torch.uint8, device=o.device) if out_q is None else out_q
    sa = (torch.empty((K // 128, lds), dtype=torch.float32, device=o.device)
          if out_sa is None else out_sa)
    max_pos = cos_cache.shape[0] if cos_cache is not None else 0
    if rope_dim > 0:
        for t, name in ((cos_cache, "cos_cache"), (sin_cache, "sin_cache")):
            if (t.dtype != torch.float32 or not t.is_contiguous()
                    or tuple(t.shape) != (max_pos, rope_dim // 2)):
                raise ValueError(f"{name} must be contiguous fp32 [max_pos, rope_dim/2]")
        if positions.dtype != torch.int64 or positions.numel() != T or not positions.is_contiguous():
            raise ValueError("positions must be a contiguous int64 tensor of T entries")
    f = scale_format(fmt)
    st = _lib.lib().fp8q_inverse_rope_quant(
        _ptr(o), o.stride(0), _ptr(positions), _ptr(cos_cache), _ptr(sin_cache), max_pos, T, H,
        D, int(rope_dim), int(bool(interleaved)), f, _ptr(q), _ld(q), _ptr(sa), sa.stride(0),
        _stream(stream))
    _lib.check(st, "fp8q_inverse_rope_quant")
    return q, sa


def gemm_w8a8_block_diag(aq: torch.Tensor, sa: torch.Tensor, wq: torch.Tensor, sw: torch.Tensor,
                         fmt=None, out=None, stream=None):
    """Per-group (block-diagonal) GEMM: codes aq [M, G*K_g] (scales sa [G*K_g/128, lds]) with
    weights wq [G, N_g, K_g] (scales sw [G, N_g/128, K_g/128]) -> bf16 [M, G*N_g], group g's
    columns from A's g-th K-slice and W[g]."""
    f = scale_format(sw.dtype if fmt is None else fmt)
    G, N_g, K_g = wq.shape
    M = aq.shape[0]
    if wq.stride(0) != N_g * wq.stride(1) or wq.stride(2) != 1:
        raise ValueError("wq must be [G, N_g, ldw] with group stride N_g * ldw")
    o = torch.empty((M, G * N_g), dtype=torch.bfloat16, device=aq.device) if out is None else out
    st = _lib.lib().fp8q_gemm_w8a8_block_diag(_ptr(aq), _ld(aq), _ptr(sa), sa.stride(0),
                                              _ptr(wq), wq.stride(1), _ptr(sw), f, G, M, N_g,
                                              K_g, _ptr(o), _ld(o), _stream(stream))
    _lib.check(st, "fp8q_gemm_w8a8_block_diag")
    return o


def gemm_w8a8_mx(aq: torch.Tensor, sa: torch.Tensor, wq: torch.Tensor, sw: torch.Tensor,
                 out=None, stream=None):
    """Hardware block-scaled GEMM for power-of-two scales: codes aq [M, G*K_g] with fp32
    power-of-two scales sa [G*K_g/128, lds], weights wq [N, K] (G = 1) or [G, N_g, K_g] with E8M0
    bytes sw [N/128, K/128] or [G, N_g/128, K_g/128] -> bf16 [M, G*N_g]."""
    if sw.dtype != torch.uint8:
        raise ValueError("sw must hold E8M0 bytes (torch.uint8)")
    if wq.dim() == 2:
        G, (N_g, K_g) = 1, wq.shape
        ldw = _ld(wq)
    else:
        G, N_g, K_g = wq.shape
        if wq.stride(0) != N_g * wq.stride(1) or wq.stride(2) != 1:
            raise ValueError("wq must be [G, N_g, ldw] with group stride N_g * ldw")
        ldw = wq.stride(1)
    M = aq.shape[0]
    o = torch.empty((M, G * N_g), dtype=torch.bfloat16, device=aq.device) if out is None else out
    st = _lib.lib().fp8q_gemm_w8a8_mx(_ptr(aq), _ld(aq), _ptr(sa), sa.stride(0), _ptr(wq), ldw,
                                      _ptr(sw), G, M, N_g, K_g, _ptr(o), _ld(o), _stream(stream))
    _lib.check(st, "fp8q_gemm_w8a8_mx")
    return o


def qkv_scales(qkv: torch.Tensor, Hq: int, Hkv: int, D: int, out_amax=None, out_scales=None,
               stream=None):
    """Per-step recalibration of the FP8 KV-cache scales: QKV activations bf16
    [T, (Hq + 2 Hkv) D] -> (amax fp32 [3], scales fp32 [3]) for Q, K, V."""
    T = qkv.shape[0]
    a = torch.empty(3, dtype=torch.float32, device=qkv.device) if out_amax is None else out_amax
    s = torch.empty(3, dtype=torch.float32, device=qkv.device) if out_scales is None else out_scales
    st = _lib.lib().fp8q_qkv_scales(_ptr(qkv), T, _ld(qkv), Hq, Hkv, D, _ptr(a), _ptr(s),
                                    _stream(stream))
    _lib.check(st, "fp8q_qkv_scales")
    return a, s


def kv_cache_write(qkv: torch.Tensor, Hq: int, Hkv: int, D: int, slots: torch.Tensor,
                   scales: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                   out_q=None, quantize_q: bool = True, stream=None):
    """Quantize Q (returned, uint8 [T, Hq D], unless quantize_q is False) and write the E4M3
    codes of K and V into rows slots[t] of k_cache / v_cache (uint8, [num_slots, Hkv D] or any
    contiguous view of it, e.g. [blocks, block_size, Hkv, D])."""
    T = qkv.shape[0]
    for c, name in ((k_cache, "k_cache"), (v_cache, "v_cache")):
        if c.dtype != torch.uint8 or not c.is_contiguous() or c.numel() % (Hkv * D):
            raise ValueError(f"{name} must be a contiguous uint8 tensor of whole Hkv*D rows")
    if slots.dtype != torch.int64 or slots.numel() != T or not slots.is_contiguous():
        raise ValueError("slots must be a contiguous int64 tensor of T entries")
    num_slots = k_cache.numel() // (Hkv * D)
    q = None
    if quantize_q:
        q = torch.empty((T, Hq * D), dtype=torch.uint8, device=qkv.device) if out_q is None else out_q
    st = _lib.lib().fp8q_kv_cache_write(_ptr(qkv), T, _ld(qkv), Hq, Hkv, D, _ptr(slots),
                                        num_slots, _ptr(scales), _ptr(q),
                                        q.stride(0) if q is not None else 0, _ptr(k_cache),
                                        _ptr(v_cache), _stream(stream))
    _lib.check(st, "fp8q_kv_cache_write")
    return q


def quant_rowwise(x: torch.Tensor, gamma=None, eps: float = 1e-6, out_q=None, out_s=None,
                  stream=None):
    """bf16 [R, K] -> (codes uint8 [R, K], scales fp32 [R]): one scale per row (per token, or per
    output channel for a weight); gamma: RMSNorm first."""
    R, K = x.shape
    q = torch.empty((R, K), dtype=torch.uint8, device=x.device) if out_q is None else out_q
    s = torch.empty((R,), dtype=torch.float32, device=x.device) if out_s is None else out_s
    st = _lib.lib().fp8q_quant_rowwise(_ptr(x), _ptr(gamma), float(eps), R, K, _ld(x), _ptr(q),
                                       _ld(q), _ptr(s), _stream(stream))
    _lib.check(st, "fp8q_quant_rowwise")
    return q, s


def add_rmsnorm_quant(x: torch.Tensor, residual: torch.Tensor, gamma: torch.Tensor,
                      eps: float = 1e-6, per_token: bool = False, out_q=None, out_sa=None,
                      lds: int = None, stream=None, scale_fmt="f32"):
    """Residual add + RMSNorm + quant: residual <- bf16(x + residual) (in place), then the codes
    of RMSNorm(residual) with 1x128 scales (sa fp32 [K/128, lds], K-block-major; scale_fmt
    "e8m0": powers of two stored as fp32) or, per_token, one fp32 scale per row (sa [M]).
    Returns (codes, sa)."""
    f = scale_format(scale_fmt)
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device) if out_q is None else out_q
    if per_token:
        sa = torch.empty((M,), dtype=torch.float32, device=x.device) if out_sa is None else out_sa
        lds = 0
    else:
        if lds is None:
            lds = max(4, (M + 3) // 4 * 4)
        sa = (torch.empty((K // 128, lds), dtype=torch.float32, device=x.device)
              if out_sa is None else out_sa)
        lds = sa.stride(0)
    st = _lib.lib().fp8q_add_rmsnorm_quant(_ptr(x), _ld(x), _ptr(residual), _ld(residual),
                                           _ptr(gamma), float(eps), M, K, 1 if per_token else 0,
                                           f, _ptr(q), _ld(q), _ptr(sa), lds, _stream(stream))
    _lib.check(st, "fp8q_add_rmsnorm_quant")
    return q, sa


def gemm_w8a8_rowwise(aq: torch.Tensor, sa: torch.Tensor, wq: torch.Tensor, sw: torch.Tensor,
                      out=None, stream=None):
    """Per-token x per-channel GEMM: codes aq [M, K] (scales sa [M]) x codes wq [N, K] (scales
    sw [N]) -> bf16 [M, N]."""
    M, K = aq.shape
    N = wq.shape[0]
    o = torch.empty((M, N), dtype=torch.bfloat16, device=aq.device) if out is None else out
    st = _lib.lib().fp8q_gemm_w8a8_rowwise(_ptr(aq), _ld(aq), _ptr(sa), _ptr(wq), _ld(wq),
                                           _ptr(sw), M, N, K, _ptr(o), _ld(o), _stream(stream))
    _lib.check(st, "fp8q_gemm_w8a8_rowwise")
    return o


def selftest_timeout(limit_ns: int = 1_000_000, stream=None):
    """Launch the bounded-wait self-test kernel (a wait that nothing completes, given up after
    limit_ns); fp8q_check_device_error then reports FP8Q_ERR_TIMEOUT."""
    st = _lib.lib().fp8q_selftest_timeout(int(limit_ns), _stream(stream))
    _lib.check(st, "fp8q_selftest_timeout")


def check_device_error(stream=None) -> int:
    """Synchronize the stream and return (and clear) the device error word."""
    return _lib.lib().fp8q_check_device_error(_stream(stream))
