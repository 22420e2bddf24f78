"""CPU oracle for the blockwise FP8 (E4M3) W8A8 linear layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package.  The CUDA library and its Python binding never do, and this package never imports
them: the two share no code.  Arrays are numpy: bf16 tensors travel as ``uint16`` bit patterns,
E4M3 codes and E8M0 scale bytes as ``uint8``.

The arithmetic lives in ``fp8q_oracle.c`` (plain C, fp64 for the GEMM reference); this module is
argument marshalling.  See the C file's header for the definitions and readings it follows.

Parity status: every function here is pinned by ``tests/test_oracle_*.py`` against library
decoders/encoders, closed forms, brute force and invariants; none is "parity unpinned".
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        L.oracle_e4m3_decode.restype = ctypes.c_double
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_e8m0_lossless_from_f32.restype = ctypes.c_int
        L.oracle_e8m0_lossless_from_f32.argtypes = [ctypes.c_float]
        L.oracle_e8m0_decode.restype = ctypes.c_double
        L.oracle_e8m0_decode.argtypes = [ctypes.c_uint8]
        L.oracle_quant_weight_block.restype = None
        L.oracle_quant_weight_block.argtypes = [P, I64, I64, I64, P, I64, P, ctypes.c_int]
        L.oracle_quant_token_1x128.restype = None
        L.oracle_quant_token_1x128.argtypes = [P, I64, I64, I64, P, I64, P, I64, ctypes.c_int]
        L.oracle_rmsnorm_bf16.restype = None
        L.oracle_rmsnorm_bf16.argtypes = [P, P, ctypes.c_float, I64, I64, I64, P, I64]
        L.oracle_rmsnorm_quant_token.restype = None
        L.oracle_rmsnorm_quant_token.argtypes = [P, P, ctypes.c_float, I64, I64, I64, P, I64,
                                                 P, I64, ctypes.c_int]
        L.oracle_gemm_w8a8_block_rows.restype = None
        L.oracle_gemm_w8a8_block_rows.argtypes = [P, I64, P, I64, P, I64, P, ctypes.c_int,
                                                  I64, I64, P, I64, P, P]
        L.oracle_grouped_gemm_w8a8_block_rows.restype = None
        L.oracle_grouped_gemm_w8a8_block_rows.argtypes = [P, I64, P, I64, P, I64, P,
                                                          ctypes.c_int, P, I64, I64, I64, P,
                                                          I64, P, P]
        L.oracle_e4m3_encode_array.restype = None
        L.oracle_exp_constants.restype = None
        L.oracle_exp_constants.argtypes = [P, ctypes.c_int]
        L.oracle_exp_f32.argtypes = [ctypes.c_float]
        L.oracle_exp_f32.restype = ctypes.c_float
        L.oracle_silu_f32.argtypes = [ctypes.c_float]
        L.oracle_silu_f32.restype = ctypes.c_float
        L.oracle_silu_mul_quant.argtypes = [P, I64, I64, I64, P, I64, P, I64, ctypes.c_int]
        L.oracle_silu_mul_quant.restype = None
        L.oracle_silu_mul_bf16.argtypes = [P, I64, I64, I64, P]
        L.oracle_silu_mul_bf16.restype = None
        L.oracle_inverse_rope_bf16.argtypes = [P, P, P, P, I64, I64, I64, I64, ctypes.c_int, P]
        L.oracle_inverse_rope_bf16.restype = None
        L.oracle_inverse_rope_quant.argtypes = [P, P, P, P, I64, I64, I64, I64, ctypes.c_int,
                                                ctypes.c_int, P, P, I64]
        L.oracle_inverse_rope_quant.restype = None
        L.oracle_qkv_amax.argtypes = [P, I64, I64, I64, I64, I64, P]
        L.oracle_qkv_amax.restype = None
        L.oracle_qkv_scales.argtypes = [P, P]
        L.oracle_qkv_scales.restype = None
        L.oracle_kv_cache_write.argtypes = [P, I64, I64, I64, I64, I64, P, P, P, I64, P, P]
        L.oracle_kv_cache_write.restype = None
        L.oracle_attention_decode.argtypes = [P, I64, P, P, P, P, I64, P, I64, I64, I64, I64,
                                              I64, ctypes.c_float, P, P, P]
        L.oracle_attention_decode.restype = None
        L.oracle_quant_rowwise.argtypes = [P, P, ctypes.c_float, I64, I64, I64, P, I64, P]
        L.oracle_quant_rowwise.restype = None
        L.oracle_add_rmsnorm_quant.argtypes = [P, I64, P, I64, P, ctypes.c_float, I64, I64,
                                               ctypes.c_int, ctypes.c_int, P, I64, P, I64]
        L.oracle_add_rmsnorm_quant.restype = None
        L.oracle_gemm_w8a8_rowwise_rows.argtypes = [P, I64, P, P, I64, P, I64, I64, P, I64, P, P]
        L.oracle_gemm_w8a8_rowwise_rows.restype = None
        L.oracle_e4m3_encode_array.argtypes = [P, I64, P]
        L.oracle_f32_to_bf16_array.restype = None
        L.oracle_f32_to_bf16_array.argtypes = [P, I64, P]
        L.oracle_rms_inverse.restype = ctypes.c_float
        L.oracle_rms_inverse.argtypes = [P, I64, ctypes.c_float]
        L.oracle_e4m3_encode_exhaustive_check.restype = I64
        L.oracle_e4m3_encode_exhaustive_check.argtypes = [ctypes.POINTER(ctypes.c_uint32)]
        L.oracle_num_threads.restype = ctypes.c_int
        L.oracle_num_threads.argtypes = []
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {a.dtype}")
    return a


SCALE_F32 = 0
SCALE_E8M0 = 1


def num_threads() -> int:
    return lib().oracle_num_threads()


# --- codec ------------------------------------------------------------------------------------

def e4m3_decode(code: int) -> float:
    return lib().oracle_e4m3_decode(int(code))


def e4m3_decode_all() -> np.ndarray:
    """Value of each of the 256 codes (fp64; NaN for 0x7F and 0xFF)."""
    return np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)


def e4m3_encode(values) -> np.ndarray:
    v = np.ascontiguousarray(np.asarray(values, dtype=np.float32).ravel())
    out = np.empty(v.shape, dtype=np.uint8)
    lib().oracle_e4m3_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def f32_to_bf16(values) -> np.ndarray:
    v = np.ascontiguousarray(np.asarray(values, dtype=np.float32).ravel())
    out = np.empty(v.shape, dtype=np.uint16)
    lib().oracle_f32_to_bf16_array(_ptr(v), v.size, _ptr(out))
    return out


def e8m0_lossless_from_f32(s: float):
    r = lib().oracle_e8m0_lossless_from_f32(float(s))
    return None if r < 0 else r


def e8m0_decode(byte: int) -> float:
    return lib().oracle_e8m0_decode(int(byte))


def e4m3_encode_exhaustive_check():
    first = ctypes.c_uint32(0)
    bad = lib().oracle_e4m3_encode_exhaustive_check(ctypes.byref(first))
    return bad, first.value


# --- hot-path operations ----------------------------------------------------------------------

def quant_weight_block(w_bf16: np.ndarray, fmt: int = SCALE_F32):
    """W bf16 [N, K] (uint16 bits) -> (codes uint8 [N, K], scales [N/128, K/128])."""
    w = _c(w_bf16, np.uint16)
    N, K = w.shape
    if N % 128 or K % 128:
        raise ValueError("N and K must be multiples of 128")
    q = np.empty((N, K), dtype=np.uint8)
    sw = np.empty((N // 128, K // 128), dtype=np.float32 if fmt == SCALE_F32 else np.uint8)
    lib().oracle_quant_weight_block(_ptr(w), N, K, K, _ptr(q), K, _ptr(sw), int(fmt))
    return q, sw


def quant_token_1x128(x_bf16: np.ndarray, lds: int = None, fmt: int = SCALE_F32):
    """X bf16 [M, K] -> (codes [M, K], sa fp32 [K/128, lds]) with sa[kb, m] the scale: amax/448
    (fmt SCALE_F32) or the E8M0 power of two stored as fp32 (fmt SCALE_E8M0, reading R12)."""
    x = _c(x_bf16, np.uint16)
    M, K = x.shape
    lds = M if lds is None else lds
    q = np.empty((M, K), dtype=np.uint8)
    sa = np.zeros((K // 128, lds), dtype=np.float32)
    lib().oracle_quant_token_1x128(_ptr(x), M, K, K, _ptr(q), K, _ptr(sa), lds, int(fmt))
    return q, sa


def rmsnorm_bf16(x_bf16: np.ndarray, gamma_bf16: np.ndarray, eps: float = 1e-6):
    x = _c(x_bf16, np.uint16)
    g = _c(gamma_bf16, np.uint16)
    M, K = x.shape
    y = np.empty((M, K), dtype=np.uint16)
    lib().oracle_rmsnorm_bf16(_ptr(x), _ptr(g), float(eps), M, K, K, _ptr(y), K)
    return y


def rmsnorm_quant_token(x_bf16: np.ndarray, gamma_bf16=None, eps: float = 1e-6,
                        lds: int = None, fmt: int = SCALE_F32):
    """Fused RMSNorm + 1x128 token quant (gamma None: plain token quant); fmt as
    quant_token_1x128."""
    x = _c(x_bf16, np.uint16)
    M, K = x.shape
    lds = M if lds is None else lds
    q = np.empty((M, K), dtype=np.uint8)
    sa = np.zeros((K // 128, lds), dtype=np.float32)
    if gamma_bf16 is None:
        gp = None
    else:
        g = _c(gamma_bf16, np.uint16)
        gp = _ptr(g)
    lib().oracle_rmsnorm_quant_token(_ptr(x), gp, float(eps), M, K, K, _ptr(q), K, _ptr(sa),
                                     lds, int(fmt))
    return q, sa


def rms_inverse(x_row_bf16: np.ndarray, eps: float = 1e-6) -> float:
    x = _c(x_row_bf16, np.uint16)
    return lib().oracle_rms_inverse(_ptr(x), x.size, float(eps))


def gemm_w8a8_block(aq, sa, wq, sw, sw_fmt: int = SCALE_F32, rows=None):
    """fp64 reference (ref, absref), each [len(rows), N]; rows default to all of M."""
    aq = _c(aq, np.uint8)
    wq = _c(wq, np.uint8)
    sa = _c(sa, np.float32)
    sw = _c(sw, np.float32 if sw_fmt == SCALE_F32 else np.uint8)
    M, K = aq.shape
    N = wq.shape[0]
    rows = np.arange(M, dtype=np.int64) if rows is None else _c(np.asarray(rows, np.int64),
                                                                 np.int64)
    ref = np.empty((rows.size, N), dtype=np.float64)
    absref = np.empty((rows.size, N), dtype=np.float64)
    lib().oracle_gemm_w8a8_block_rows(_ptr(aq), K, _ptr(sa), sa.shape[1], _ptr(wq), K, _ptr(sw),
                                      int(sw_fmt), N, K, _ptr(rows), rows.size, _ptr(ref),
                                      _ptr(absref))
    return ref, absref


def grouped_gemm_w8a8_block(aq, sa, wq, sw, group_offsets, sw_fmt: int = SCALE_F32, rows=None):
    """Grouped reference: wq [E, N, K], sw [E, N/128, K/128], group_offsets int32 [E+1]."""
    aq = _c(aq, np.uint8)
    wq = _c(wq, np.uint8)
    sa = _c(sa, np.float32)
    sw = _c(sw, np.float32 if sw_fmt == SCALE_F32 else np.uint8)
    off = _c(np.asarray(group_offsets, np.int32), np.int32)
    M, K = aq.shape
    E, N, _ = wq.shape
    rows = np.arange(M, dtype=np.int64) if rows is None else _c(np.asarray(rows, np.int64),
                                                                 np.int64)
    ref = np.empty((rows.size, N), dtype=np.float64)
    absref = np.empty((rows.size, N), dtype=np.float64)
    lib().oracle_grouped_gemm_w8a8_block_rows(_ptr(aq), K, _ptr(sa), sa.shape[1], _ptr(wq), K,
                                              _ptr(sw), int(sw_fmt), _ptr(off), E, N, K,
                                              _ptr(rows), rows.size, _ptr(ref), _ptr(absref))
    return ref, absref


def gemm_w8a8_block_diag(aq, sa, wq, sw, sw_fmt: int = SCALE_F32, rows=None):
    """Block-diagonal reference [DSv4-WOA sections 2-3: a batched GEMM over head groups]:
    wq [G, N_g, K_g], sw [G, N_g/128, K_g/128]; group g multiplies the K-slice
    [g K_g, (g+1) K_g) of aq (scales: sa's K-blocks [g K_g/128, ...)) by wq[g] and fills the
    output columns [g N_g, (g+1) N_g).  Each group is one call of the plain block GEMM."""
    aq = _c(aq, np.uint8)
    sa = _c(sa, np.float32)
    G, N_g, K_g = wq.shape
    KB = K_g // 128
    M = aq.shape[0]
    nrows = M if rows is None else len(rows)
    ref = np.empty((nrows, G * N_g), dtype=np.float64)
    absref = np.empty((nrows, G * N_g), dtype=np.float64)
    for g in range(G):
        r, a = gemm_w8a8_block(aq[:, g * K_g:(g + 1) * K_g], sa[g * KB:(g + 1) * KB], wq[g],
                               sw[g], sw_fmt, rows)
        ref[:, g * N_g:(g + 1) * N_g] = r
        absref[:, g * N_g:(g + 1) * N_g] = a
    return ref, absref


def exp_f32(x: float) -> float:
    """e^x in fp32 by the method of reading R8 (Cody-Waite reduction, degree-7 Taylor)."""
    return float(lib().oracle_exp_f32(float(x)))


def exp_constants() -> np.ndarray:
    """The exponential's constants: [1/ln 2, c1, c2, 1/7!, 1/6!, ..., 1/1!, 1/0!] as fp32."""
    out = np.zeros(11, np.float32)
    lib().oracle_exp_constants(_ptr(out), 11)
    return out


def silu_f32(g: float) -> float:
    return float(lib().oracle_silu_f32(float(g)))


def silu_mul_bf16(h_bf16: np.ndarray) -> np.ndarray:
    """y = bf16(silu(gate) * up) of reading R8 for h = [gate | up] bf16 [R, 2I]."""
    h = _c(h_bf16, np.uint16)
    R, I2 = h.shape
    y = np.empty((R, I2 // 2), np.uint16)
    lib().oracle_silu_mul_bf16(_ptr(h), R, I2 // 2, I2, _ptr(y))
    return y


def silu_mul_quant(h_bf16: np.ndarray, lds: int = None, fmt: int = SCALE_F32):
    """SiLU-and-mul then 1x128 token quant (reading R8): codes [R, I] and sa [I/128, lds]; fmt as
    quant_token_1x128."""
    h = _c(h_bf16, np.uint16)
    R, I2 = h.shape
    I = I2 // 2
    lds = R if lds is None else lds
    q = np.empty((R, I), np.uint8)
    sa = np.zeros((I // 128, lds), np.float32)
    lib().oracle_silu_mul_quant(_ptr(h), R, I, I2, _ptr(q), I, _ptr(sa), lds, int(fmt))
    return q, sa


def inverse_rope_bf16(o_bf16: np.ndarray, positions, cos_cache, sin_cache, rope_dim: int,
                      interleaved: bool = True):
    """The bf16 inverse RoPE of reading R9: o [T, H, D] -> y [T, H*D]."""
    o = _c(o_bf16, np.uint16)
    T, H, D = o.shape
    pos = _c(np.asarray(positions), np.int64)
    c = _c(cos_cache, np.float32)
    sn = _c(sin_cache, np.float32)
    y = np.empty((T, H * D), np.uint16)
    lib().oracle_inverse_rope_bf16(_ptr(o), _ptr(pos), _ptr(c), _ptr(sn), T, H, D, rope_dim,
                                   int(interleaved), _ptr(y))
    return y


def inverse_rope_quant(o_bf16: np.ndarray, positions, cos_cache, sin_cache, rope_dim: int,
                       interleaved: bool = True, fmt: int = 0, lds: int = None):
    """Inverse RoPE + 1x128 quant (reading R9): codes [T, H*D] and sa [H*D/128, lds]
    (fmt 0: fp32 amax/448 scales; fmt 1: E8M0 powers of two stored as fp32)."""
    o = _c(o_bf16, np.uint16)
    T, H, D = o.shape
    lds = T if lds is None else lds
    pos = _c(np.asarray(positions), np.int64)
    c = _c(cos_cache, np.float32)
    sn = _c(sin_cache, np.float32)
    q = np.empty((T, H * D), np.uint8)
    sa = np.zeros((H * D // 128, lds), np.float32)
    lib().oracle_inverse_rope_quant(_ptr(o), _ptr(pos), _ptr(c), _ptr(sn), T, H, D, rope_dim,
                                    int(interleaved), int(fmt), _ptr(q), _ptr(sa), lds)
    return q, sa


def qkv_amax(qkv_bf16: np.ndarray, Hq: int, Hkv: int, D: int) -> np.ndarray:
    """Per-tensor absolute maxima (Q, K, V) of a QKV activation [T, (Hq + 2 Hkv) D] (R10)."""
    x = _c(qkv_bf16, np.uint16)
    a = np.zeros(3, np.float32)
    lib().oracle_qkv_amax(_ptr(x), x.shape[0], x.shape[1], Hq, Hkv, D, _ptr(a))
    return a


def qkv_scales(amax3) -> np.ndarray:
    """Per-tensor scales of reading R10: amax / 448 in fp32, 1 for an all-zero tensor."""
    a = _c(np.asarray(amax3, np.float32), np.float32)
    s = np.zeros(3, np.float32)
    lib().oracle_qkv_scales(_ptr(a), _ptr(s))
    return s


def kv_cache_write(qkv_bf16: np.ndarray, Hq: int, Hkv: int, D: int, slots, scales3,
                   k_cache: np.ndarray, v_cache: np.ndarray) -> np.ndarray:
    """Writes K and V codes into rows slots[t] of k_cache / v_cache (uint8 [num_slots, Hkv D],
    updated in place; negative slots skipped) and returns the Q codes [T, Hq D]."""
    x = _c(qkv_bf16, np.uint16)
    T = x.shape[0]
    sl = _c(np.asarray(slots, np.int64), np.int64)
    sc = _c(np.asarray(scales3, np.float32), np.float32)
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    assert k_cache.dtype == np.uint8 and v_cache.dtype == np.uint8
    q = np.zeros((T, Hq * D), np.uint8)
    lib().oracle_kv_cache_write(_ptr(x), T, x.shape[1], Hq, Hkv, D, _ptr(sl), _ptr(sc), _ptr(q),
                                Hq * D, _ptr(k_cache), _ptr(v_cache))
    return q


def attention_decode(q_codes, k_cache, v_cache, scales3, block_table, seq_lens, Hq: int,
                     Hkv: int, D: int, block_size: int, sm_scale=None):
    """Decode attention over the FP8 KV cache, reading R13: q_codes [B, Hq*D] uint8, caches
    [slots, Hkv*D] uint8, scales3 (s_q, s_k, s_v), block_table [B, max_blocks] int32, seq_lens
    [B] int32; sm_scale defaults to 1/sqrt(D) (as fp32).  Returns (out [B, Hq*D] fp64, absref
    [B, Hq*D] = s_v sum_j p_j |dec(v_j)|, zabs [B, Hq] = the largest |scale| sum_d |dec(q)
    dec(k_j)|)."""
    q = _c(q_codes, np.uint8)
    kc, vc = _c(k_cache, np.uint8), _c(v_cache, np.uint8)
    sc = _c(np.asarray(scales3, np.float32), np.float32)
    bt = _c(block_table, np.int32)
    sl = _c(seq_lens, np.int32)
    B = q.shape[0]
    if sm_scale is None:
        sm_scale = float(np.float32(1.0) / np.sqrt(np.float32(D)))
    out = np.zeros((B, Hq * D), np.float64)
    absref = np.zeros((B, Hq * D), np.float64)
    zabs = np.zeros((B, Hq), np.float64)
    lib().oracle_attention_decode(_ptr(q), q.shape[1], _ptr(kc), _ptr(vc), _ptr(sc), _ptr(bt),
                                  bt.shape[1], _ptr(sl), B, Hq, Hkv, D, block_size,
                                  float(sm_scale), _ptr(out), _ptr(absref), _ptr(zabs))
    return out, absref, zabs


def quant_rowwise(x_bf16: np.ndarray, gamma_bf16=None, eps: float = 1e-6):
    """Per-token (or per-channel) quantization, reading R7: codes uint8 [R, K] and one fp32 scale
    per row; with gamma, each row is RMS-normalised first (reading R4)."""
    x = _c(x_bf16, np.uint16)
    R, K = x.shape
    q = np.empty((R, K), np.uint8)
    s = np.empty(R, np.float32)
    g = None if gamma_bf16 is None else _c(gamma_bf16, np.uint16)
    lib().oracle_quant_rowwise(_ptr(x), None if g is None else _ptr(g), float(eps), R, K, K,
                               _ptr(q), K, _ptr(s))
    return q, s


def add_rmsnorm_quant(x_bf16: np.ndarray, res_bf16: np.ndarray, gamma_bf16: np.ndarray,
                      eps: float = 1e-6, per_token: bool = False, lds: int = None,
                      fmt: int = SCALE_F32):
    """Residual add + RMSNorm + quant, reading R11: h = bf16(fp32(x) + fp32(res)); returns
    (h, codes, scales) -- h the updated residual, scales [K/128, lds] K-block-major (1x128 groups)
    or [M] (per_token).  fmt (1x128 groups only) as quant_token_1x128.  The inputs are not
    modified."""
    if per_token and fmt != SCALE_F32:
        raise ValueError("per-token scales are fp32 only")
    x = _c(x_bf16, np.uint16)
    h = np.array(_c(res_bf16, np.uint16), copy=True)
    g = _c(gamma_bf16, np.uint16)
    M, K = x.shape
    if h.shape != (M, K):
        raise ValueError("x and res differ in shape")
    q = np.empty((M, K), np.uint8)
    if per_token:
        lds = 0
        sa = np.empty(M, np.float32)
    else:
        lds = M if lds is None else lds
        sa = np.zeros((K // 128, lds), np.float32)
    lib().oracle_add_rmsnorm_quant(_ptr(x), K, _ptr(h), K, _ptr(g), float(eps), M, K,
                                   1 if per_token else 0, int(fmt), _ptr(q), K, _ptr(sa), lds)
    return h, q, sa


def gemm_w8a8_rowwise(aq, sa, wq, sw, rows=None):
    """Per-channel GEMM reference (reading R7) in fp64 on the selected rows: (ref, absref)."""
    aq = _c(aq, np.uint8)
    wq = _c(wq, np.uint8)
    sa = _c(sa, np.float32)
    sw = _c(sw, np.float32)
    M, K = aq.shape
    N = wq.shape[0]
    r = np.arange(M, dtype=np.int64) if rows is None else _c(np.asarray(rows), np.int64)
    ref = np.empty((len(r), N), np.float64)
    absref = np.empty((len(r), N), np.float64)
    lib().oracle_gemm_w8a8_rowwise_rows(_ptr(aq), K, _ptr(sa), _ptr(wq), K, _ptr(sw), N, K,
                                        _ptr(r), len(r), _ptr(ref), _ptr(absref))
    return ref, absref


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """One bf16 ulp at |x| (2^(floor(log2|x|) - 7)); 2^-133 at zero and in the subnormal range."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    ulp = np.ldexp(1.0, (e - 7).astype(np.int64))
    return np.where(a >= 2.0 ** -126, ulp, 2.0 ** -133)


def gemm_tolerance(ref: np.ndarray, absref: np.ndarray) -> np.ndarray:
    """Per-element bound |out - ref| <= 8e-3 * absref + one bf16 ulp of |ref|."""
    return 8e-3 * absref + bf16_ulp(ref)
