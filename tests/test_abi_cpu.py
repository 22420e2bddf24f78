"""The C-ABI library builds for sm_100a, loads without a GPU, exports exactly what include/fp8q.h
declares, and rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

from fp8_blockwise_w8a8_b200 import _lib, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "fp8q.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(fp8q_\w+)\s*\(", text, re.M)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.lib()


def test_exports_match_header(L):
    names = declared_functions()
    assert names == sorted(_lib.SIGNATURES), names
    for n in names:
        assert hasattr(L, n), n
    assert L.fp8q_abi_version() >> 16 == 1


def test_status_strings(L):
    for s in range(11):
        assert len(_lib.status_string(s)) >= 2
    assert _lib.status_string(99) == "unknown status"


P = ctypes.c_void_p
FAKE = 1 << 20          # a 16-byte aligned non-null address; never dereferenced on these paths


def test_weight_quant_host_checks(L):
    f = L.fp8q_quant_weight_block
    assert f(FAKE, 128, 200, 200, FAKE, 208, FAKE, 0, None) == _lib.FP8Q_ERR_SHAPE
    assert f(FAKE, 100, 128, 128, FAKE, 128, FAKE, 0, None) == _lib.FP8Q_ERR_SHAPE
    assert f(FAKE, 128, 128, 64, FAKE, 128, FAKE, 0, None) == _lib.FP8Q_ERR_SHAPE
    assert f(FAKE, 128, 128, 128, FAKE, 128, FAKE, 2, None) == _lib.FP8Q_ERR_ARG
    assert f(None, 128, 128, 128, FAKE, 128, FAKE, 0, None) == _lib.FP8Q_ERR_NULL
    assert f(FAKE + 2, 128, 128, 128, FAKE, 128, FAKE, 0, None) == _lib.FP8Q_ERR_ALIGN
    assert f(FAKE, 128, 128, 132, FAKE, 128, FAKE, 0, None) == _lib.FP8Q_ERR_ALIGN
    assert f(FAKE, 0, 128, 128, FAKE, 128, FAKE, 0, None) == _lib.FP8Q_OK      # empty: no-op


def test_token_quant_fmt_host_checks(L):
    f = L.fp8q_rmsnorm_quant_token_fmt
    assert f(FAKE, None, 1e-6, 4, 128, 128, FAKE, 128, FAKE, 4, 2, None) == _lib.FP8Q_ERR_ARG
    assert f(FAKE, None, 1e-6, 4, 100, 100, FAKE, 112, FAKE, 4, 1, None) == _lib.FP8Q_ERR_SHAPE
    assert f(None, None, 1e-6, 4, 128, 128, FAKE, 128, FAKE, 4, 1, None) == _lib.FP8Q_ERR_NULL
    assert f(FAKE, None, 1e-6, 4, 128, 128, FAKE, 128, FAKE + 4, 4, 1, None) == _lib.FP8Q_ERR_ALIGN
    assert f(None, None, 1e-6, 0, 128, 128, None, 128, None, 4, 1, None) == _lib.FP8Q_OK
    import torch
    if not torch.cuda.is_available():
        assert f(FAKE, FAKE, 1e-6, 4, 128, 128, FAKE, 128, FAKE, 4, 1, None) == _lib.FP8Q_ERR_ARCH


def test_attention_decode_host_checks(L):
    q = L.fp8q_attention_decode_workspace_bytes
    b = ctypes.c_int64(-1)
    assert q(2, 8, 2, 128, 300, ctypes.byref(b)) == _lib.FP8Q_OK
    assert b.value == 2 * 2 * 5 * 4 * 130 * 4     # 5 chunks of 64 positions, 4 heads per group
    assert q(2, 8, 2, 64, 300, ctypes.byref(b)) == _lib.FP8Q_ERR_SHAPE      # D != 128
    assert q(2, 12, 8, 128, 300, ctypes.byref(b)) == _lib.FP8Q_ERR_SHAPE    # Hq % Hkv
    assert q(2, 24, 8, 128, 300, ctypes.byref(b)) == _lib.FP8Q_ERR_SHAPE    # group of 3
    assert q(2, 8, 2, 128, 300, None) == _lib.FP8Q_ERR_NULL
    assert q(65536, 8, 2, 128, 300, ctypes.byref(b)) == _lib.FP8Q_ERR_SHAPE   # grid z
    f = L.fp8q_attention_decode
    ws = 1 << 22

    def call(**kw):
        a = dict(q=FAKE, ldq=1024, k=FAKE, v=FAKE, slots=64, s3=FAKE, bt=FAKE, maxb=4, sl=FAKE,
                 B=2, Hq=8, Hkv=2, D=128, bs=16, maxlen=64, sm=0.088, out=FAKE, ldo=1024,
                 ws=FAKE, wsb=ws)
        a.update(kw)
        return f(a["q"], a["ldq"], a["k"], a["v"], a["slots"], a["s3"], a["bt"], a["maxb"],
                 a["sl"], a["B"], a["Hq"], a["Hkv"], a["D"], a["bs"], a["maxlen"], a["sm"],
                 a["out"], a["ldo"], a["ws"], a["wsb"], None)
    assert call(D=64) == _lib.FP8Q_ERR_SHAPE
    assert call(maxlen=65) == _lib.FP8Q_ERR_SHAPE               # beyond max_blocks * block_size
    assert call(ldq=512) == _lib.FP8Q_ERR_SHAPE
    assert call(B=0, q=None, out=None, ws=None) == _lib.FP8Q_OK
    assert call(q=None) == _lib.FP8Q_ERR_NULL
    assert call(q=FAKE + 8) == _lib.FP8Q_ERR_ALIGN
    assert call(ldq=1032) == _lib.FP8Q_ERR_ALIGN
    assert call(wsb=16) == _lib.FP8Q_ERR_SHAPE                 # workspace too small
    assert call(slots=2 ** 31) == _lib.FP8Q_ERR_SHAPE          # slots beyond int32
    import torch
    if not torch.cuda.is_available():
        assert call() == _lib.FP8Q_ERR_ARCH


def test_token_quant_host_checks(L):
    f = L.fp8q_rmsnorm_quant_token
    assert f(FAKE, None, 1e-6, 4, 100, 100, FAKE, 112, FAKE, 4, None) == _lib.FP8Q_ERR_SHAPE
    assert f(FAKE, None, 1e-6, 4, 32768, 32768, FAKE, 32768, FAKE, 4, None) == _lib.FP8Q_ERR_SHAPE
    assert f(FAKE, None, 1e-6, 8, 128, 128, FAKE, 128, FAKE, 4, None) == _lib.FP8Q_ERR_SHAPE
    assert f(FAKE, None, 1e-6, 4, 128, 128, FAKE, 128, FAKE, 6, None) == _lib.FP8Q_ERR_ALIGN
    assert f(FAKE, FAKE + 8, 1e-6, 4, 128, 128, FAKE, 128, FAKE, 4, None) == _lib.FP8Q_ERR_ALIGN
    assert f(None, None, 1e-6, 4, 128, 128, FAKE, 128, FAKE, 4, None) == _lib.FP8Q_ERR_NULL
    assert f(None, None, 1e-6, 0, 128, 128, None, 128, None, 4, None) == _lib.FP8Q_OK


def test_gemm_host_checks(L):
    g = L.fp8q_gemm_w8a8_block
    ok = dict(aq=FAKE, lda=256, sa=FAKE, lds=64, wq=FAKE, ldw=256, sw=FAKE, fmt=0, M=64, N=128,
              K=256, out=FAKE, ldo=128)

    def call(**kw):
        a = dict(ok, **kw)
        return g(a["aq"], a["lda"], a["sa"], a["lds"], a["wq"], a["ldw"], a["sw"], a["fmt"],
                 a["M"], a["N"], a["K"], a["out"], a["ldo"], None)
    assert call(N=100) == _lib.FP8Q_ERR_SHAPE
    assert call(K=200, lda=208, ldw=208) == _lib.FP8Q_ERR_SHAPE
    assert call(lds=32) == _lib.FP8Q_ERR_SHAPE
    assert call(M=-1) == _lib.FP8Q_ERR_SHAPE
    assert call(fmt=5) == _lib.FP8Q_ERR_ARG
    assert call(sa=None) == _lib.FP8Q_ERR_NULL
    assert call(lda=264) == _lib.FP8Q_ERR_ALIGN
    assert call(out=FAKE + 4) == _lib.FP8Q_ERR_ALIGN
    assert call(M=0, aq=None, sa=None, out=None) == _lib.FP8Q_OK
    gg = L.fp8q_grouped_gemm_w8a8_block
    assert gg(FAKE, 256, FAKE, 64, FAKE, 256, FAKE, 0, FAKE, 0, 64, 128, 256, FAKE, 128,
              None) == _lib.FP8Q_ERR_SHAPE
    assert gg(FAKE, 256, FAKE, 64, FAKE, 256, FAKE, 0, None, 4, 64, 128, 256, FAKE, 128,
              None) == _lib.FP8Q_ERR_NULL


def test_size_limits_are_rejected_on_the_host(L):
    """K beyond 32768 (256 K-blocks of staged scales), more than 1024 experts, K beyond 16384 for
    the token quant, more than 2048 matrices in a batch."""
    g = L.fp8q_gemm_w8a8_block
    K = 32768 + 128
    assert g(FAKE, K, FAKE, 64, FAKE, K, FAKE, 0, 64, 256, K, FAKE, 256, None) == _lib.FP8Q_ERR_SHAPE
    gg = L.fp8q_grouped_gemm_w8a8_block
    assert gg(FAKE, 256, FAKE, 64, FAKE, 256, FAKE, 0, FAKE, 1025, 64, 256, 256, FAKE, 256,
              None) == _lib.FP8Q_ERR_SHAPE
    t = L.fp8q_rmsnorm_quant_token
    assert t(FAKE, None, 1e-6, 4, 16512, 16512, FAKE, 16512, FAKE, 4, None) == _lib.FP8Q_ERR_SHAPE
    b = L.fp8q_quant_weight_block_batched
    assert b(FAKE, 2049, 2049, 0, None) == _lib.FP8Q_ERR_SHAPE


def test_valid_call_without_gpu_reports_arch(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    f = L.fp8q_quant_weight_block
    assert f(FAKE, 128, 128, 128, FAKE, 128, FAKE, 0, None) == _lib.FP8Q_ERR_ARCH


def test_splitk_host_checks(L):
    g = L.fp8q_gemm_w8a8_block_splitk
    ok = dict(aq=FAKE, lda=512, sa=FAKE, lds=64, wq=FAKE, ldw=512, sw=FAKE, fmt=0, M=64, N=256,
              K=512, out=FAKE, ldo=256, splits=2, ws=FAKE, wsb=1 << 30)

    def call(**kw):
        a = dict(ok, **kw)
        return g(a["aq"], a["lda"], a["sa"], a["lds"], a["wq"], a["ldw"], a["sw"], a["fmt"],
                 a["M"], a["N"], a["K"], a["out"], a["ldo"], a["splits"], a["ws"], a["wsb"], None)
    assert call(splits=-1) == _lib.FP8Q_ERR_ARG
    assert call(splits=5) == _lib.FP8Q_ERR_ARG          # more splits than K-blocks
    assert call(N=100) == _lib.FP8Q_ERR_SHAPE
    assert call(lda=520) == _lib.FP8Q_ERR_ALIGN
    assert call(M=0, aq=None, sa=None, out=None, ws=None) == _lib.FP8Q_OK
    q = L.fp8q_gemm_splitk_workspace_bytes
    b = ctypes.c_int64(-1)
    assert q(64, 256, 512, 2, ctypes.byref(b)) == _lib.FP8Q_OK
    assert b.value == 2 * 128 * 256 * 4
    assert q(300, 768, 4096, 3, ctypes.byref(b)) == _lib.FP8Q_OK
    assert b.value == 9 * 3 * 128 * 256 * 4           # 9 tiles x 3 splits of fp32 partials
    assert q(64, 256, 512, 1, ctypes.byref(b)) == _lib.FP8Q_OK and b.value == 0
    assert q(64, 256, 512, 5, ctypes.byref(b)) == _lib.FP8Q_ERR_ARG
    assert q(64, 200, 512, 2, ctypes.byref(b)) == _lib.FP8Q_ERR_SHAPE
    assert q(64, 256, 512, 2, None) == _lib.FP8Q_ERR_NULL


def test_splitk_noalloc_host_checks(L):
    g = L.fp8q_gemm_w8a8_block_splitk_noalloc
    a = (FAKE, 512, FAKE, 64, FAKE, 512, FAKE, 0)
    assert g(*a, 64, 256, 512, FAKE, 256, -1, None) == _lib.FP8Q_ERR_ARG
    assert g(*a, 64, 256, 512, FAKE, 256, 5, None) == _lib.FP8Q_ERR_ARG
    assert g(*a, 64, 200, 512, FAKE, 256, 2, None) == _lib.FP8Q_ERR_SHAPE
    assert g(*a, 0, 256, 512, None, 256, 2, None) == _lib.FP8Q_OK


def test_rowwise_host_checks(L):
    f = L.fp8q_quant_rowwise
    assert f(FAKE, None, 1e-6, 4, 100, 100, FAKE, 112, FAKE, None) == _lib.FP8Q_ERR_SHAPE
    assert f(FAKE, None, 1e-6, 4, 32768, 32768, FAKE, 32768, FAKE, None) == _lib.FP8Q_ERR_SHAPE
    assert f(FAKE, None, 1e-6, 4, 128, 128, FAKE, 128, FAKE + 2, None) == _lib.FP8Q_ERR_ALIGN
    assert f(FAKE, FAKE + 8, 1e-6, 4, 128, 128, FAKE, 128, FAKE, None) == _lib.FP8Q_ERR_ALIGN
    assert f(None, None, 1e-6, 4, 128, 128, FAKE, 128, FAKE, None) == _lib.FP8Q_ERR_NULL
    assert f(None, None, 1e-6, 0, 128, 128, None, 128, None, None) == _lib.FP8Q_OK
    g = L.fp8q_gemm_w8a8_rowwise
    a = dict(aq=FAKE, lda=256, sa=FAKE, wq=FAKE, ldw=256, sw=FAKE, M=64, N=128, K=256, out=FAKE,
             ldo=128)

    def call(**kw):
        b = dict(a, **kw)
        return g(b["aq"], b["lda"], b["sa"], b["wq"], b["ldw"], b["sw"], b["M"], b["N"], b["K"],
                 b["out"], b["ldo"], None)
    assert call(N=100) == _lib.FP8Q_ERR_SHAPE
    assert call(K=200, lda=208, ldw=208) == _lib.FP8Q_ERR_SHAPE
    assert call(sw=None) == _lib.FP8Q_ERR_NULL
    assert call(sa=FAKE + 2) == _lib.FP8Q_ERR_ALIGN
    assert call(lda=264) == _lib.FP8Q_ERR_ALIGN
    assert call(M=0, aq=None, sa=None, out=None) == _lib.FP8Q_OK


def test_add_rmsnorm_quant_host_checks(L):
    f = L.fp8q_add_rmsnorm_quant
    R2 = FAKE + (1 << 24)                 # a residual that does not overlap x
    ok = dict(x=FAKE, ldx=256, res=R2, ldr=256, g=FAKE, M=8, K=256, pt=0, fmt=0, q=FAKE,
              ldq=256, sa=FAKE, lds=8)

    def call(**kw):
        b = dict(ok, **kw)
        return f(b["x"], b["ldx"], b["res"], b["ldr"], b["g"], 1e-6, b["M"], b["K"], b["pt"],
                 b["fmt"], b["q"], b["ldq"], b["sa"], b["lds"], None)
    assert call(K=200, ldx=208, ldr=208, ldq=208) == _lib.FP8Q_ERR_SHAPE   # K % 128
    assert call(K=32768, ldx=32768, ldr=32768, ldq=32768) == _lib.FP8Q_ERR_SHAPE
    assert call(lds=4) == _lib.FP8Q_ERR_SHAPE                              # lds < M
    assert call(ldr=128) == _lib.FP8Q_ERR_SHAPE                            # ldr < K
    assert call(pt=2) == _lib.FP8Q_ERR_ARG
    assert call(fmt=2) == _lib.FP8Q_ERR_ARG
    assert call(pt=1, lds=0, fmt=1) == _lib.FP8Q_ERR_ARG                   # per-token: fp32 only
    assert call(g=None) == _lib.FP8Q_ERR_NULL                              # gamma is required
    assert call(res=None) == _lib.FP8Q_ERR_NULL
    assert call(ldr=260) == _lib.FP8Q_ERR_ALIGN
    assert call(res=R2 + 4) == _lib.FP8Q_ERR_ALIGN
    assert call(lds=10) == _lib.FP8Q_ERR_ALIGN                             # 1x128: lds % 4
    assert call(pt=1, lds=0, sa=FAKE + 2) == _lib.FP8Q_ERR_ALIGN
    assert call(res=FAKE + 256) == _lib.FP8Q_ERR_ARG                       # x and res overlap
    assert call(M=0, x=None, res=None, g=None, q=None, sa=None) == _lib.FP8Q_OK
    import torch
    if not torch.cuda.is_available():     # valid arguments reach the device query
        assert call() == _lib.FP8Q_ERR_ARCH
        assert call(fmt=1) == _lib.FP8Q_ERR_ARCH
        assert call(pt=1, lds=0) == _lib.FP8Q_ERR_ARCH


def test_silu_mul_quant_host_checks(L):
    f = L.fp8q_silu_mul_quant
    assert f(FAKE, 4, 100, 200, FAKE, 112, FAKE, 4, 0, None) == _lib.FP8Q_ERR_SHAPE   # I % 128
    assert f(FAKE, 4, 128, 200, FAKE, 128, FAKE, 4, 0, None) == _lib.FP8Q_ERR_SHAPE   # ldh < 2I
    assert f(FAKE, 8, 128, 256, FAKE, 128, FAKE, 4, 0, None) == _lib.FP8Q_ERR_SHAPE   # lds < R
    assert f(FAKE, 4, 128, 260, FAKE, 128, FAKE, 4, 0, None) == _lib.FP8Q_ERR_ALIGN   # ldh % 8
    assert f(None, 4, 128, 256, FAKE, 128, FAKE, 4, 0, None) == _lib.FP8Q_ERR_NULL
    assert f(FAKE, 4, 128, 256, FAKE, 128, FAKE, 4, 3, None) == _lib.FP8Q_ERR_ARG    # format
    assert f(None, 0, 128, 256, None, 128, None, 4, 1, None) == _lib.FP8Q_OK


def test_inverse_rope_quant_host_checks(L):
    f = L.fp8q_inverse_rope_quant
    ok = dict(o=FAKE, ldo=1024, pos=FAKE, cos=FAKE, sin=FAKE, max_pos=64, T=8, H=2, D=512, R=64,
              il=1, fmt=0, q=FAKE, ldq=1024, sa=FAKE, lds=8)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["o"], a["ldo"], a["pos"], a["cos"], a["sin"], a["max_pos"], a["T"], a["H"],
                 a["D"], a["R"], a["il"], a["fmt"], a["q"], a["ldq"], a["sa"], a["lds"], None)
    assert call(fmt=2) == _lib.FP8Q_ERR_ARG
    assert call(il=2) == _lib.FP8Q_ERR_ARG
    assert call(D=100, ldo=200, ldq=208) == _lib.FP8Q_ERR_SHAPE          # D % 8
    assert call(H=1, D=192, ldo=192, ldq=192) == _lib.FP8Q_ERR_SHAPE      # H*D % 128
    assert call(R=60) == _lib.FP8Q_ERR_SHAPE                              # rope_dim % 8
    assert call(R=520) == _lib.FP8Q_ERR_SHAPE                             # rope_dim > D
    assert call(R=40, il=0) == _lib.FP8Q_ERR_SHAPE                        # halves: % 16
    assert call(ldo=1000) == _lib.FP8Q_ERR_SHAPE
    assert call(lds=4) == _lib.FP8Q_ERR_SHAPE
    assert call(max_pos=0) == _lib.FP8Q_ERR_SHAPE
    assert call(pos=None) == _lib.FP8Q_ERR_NULL
    assert call(cos=FAKE + 4) == _lib.FP8Q_ERR_ALIGN
    assert call(pos=FAKE + 4) == _lib.FP8Q_ERR_ALIGN
    assert call(ldo=1028) == _lib.FP8Q_ERR_ALIGN
    assert call(T=0, o=None, q=None, sa=None, pos=None) == _lib.FP8Q_OK
    import torch
    if not torch.cuda.is_available():   # valid arguments reach the device check (never launched)
        assert call() == _lib.FP8Q_ERR_ARCH
        assert call(R=0, pos=None, cos=None, sin=None, max_pos=0) == _lib.FP8Q_ERR_ARCH


def test_block_diag_gemm_host_checks(L):
    g = L.fp8q_gemm_w8a8_block_diag
    ok = dict(aq=FAKE, lda=1024, sa=FAKE, lds=64, wq=FAKE, ldw=512, sw=FAKE, fmt=0, G=2, M=64,
              N_g=256, K_g=512, out=FAKE, ldo=512)

    def call(**kw):
        a = dict(ok, **kw)
        return g(a["aq"], a["lda"], a["sa"], a["lds"], a["wq"], a["ldw"], a["sw"], a["fmt"],
                 a["G"], a["M"], a["N_g"], a["K_g"], a["out"], a["ldo"], None)
    assert call(N_g=128, ldo=256) == _lib.FP8Q_ERR_SHAPE                  # N_g % 256
    assert call(G=0) == _lib.FP8Q_ERR_SHAPE
    assert call(lda=768) == _lib.FP8Q_ERR_SHAPE                           # lda < G K_g
    assert call(ldo=256) == _lib.FP8Q_ERR_SHAPE                           # ldo < G N_g
    assert call(K_g=200, ldw=208) == _lib.FP8Q_ERR_SHAPE
    assert call(fmt=3) == _lib.FP8Q_ERR_ARG
    assert call(sw=None) == _lib.FP8Q_ERR_NULL
    assert call(lda=1032) == _lib.FP8Q_ERR_ALIGN
    assert call(M=0, aq=None, sa=None, out=None) == _lib.FP8Q_OK


def test_mx_gemm_host_checks(L):
    g = L.fp8q_gemm_w8a8_mx
    ok = dict(aq=FAKE, lda=1024, sa=FAKE, lds=64, wq=FAKE, ldw=512, sw=FAKE, G=2, M=64, N_g=256,
              K_g=512, out=FAKE, ldo=512)

    def call(**kw):
        a = dict(ok, **kw)
        return g(a["aq"], a["lda"], a["sa"], a["lds"], a["wq"], a["ldw"], a["sw"], a["G"],
                 a["M"], a["N_g"], a["K_g"], a["out"], a["ldo"], None)
    assert call(N_g=128, ldo=256) == _lib.FP8Q_ERR_SHAPE                  # groups: N_g % 256
    assert call(G=1, N_g=100, ldo=128) == _lib.FP8Q_ERR_SHAPE             # N % 128
    assert call(K_g=200, ldw=208) == _lib.FP8Q_ERR_SHAPE
    assert call(lda=768) == _lib.FP8Q_ERR_SHAPE
    assert call(lds=32) == _lib.FP8Q_ERR_SHAPE
    assert call(sw=None) == _lib.FP8Q_ERR_NULL
    assert call(sa=FAKE + 2) == _lib.FP8Q_ERR_ALIGN
    assert call(ldo=516) == _lib.FP8Q_ERR_ALIGN
    assert call(M=0, aq=None, sa=None, out=None) == _lib.FP8Q_OK


def test_kv_cache_host_checks(L):
    f = L.fp8q_qkv_scales
    assert f(FAKE, 8, 6144, 32, 8, 100, FAKE, FAKE, None) == _lib.FP8Q_ERR_SHAPE     # D % 8
    assert f(FAKE, 8, 6000, 32, 8, 128, FAKE, FAKE, None) == _lib.FP8Q_ERR_SHAPE     # ld
    assert f(FAKE, 8, 6144, 32, 8, 128, None, FAKE, None) == _lib.FP8Q_ERR_NULL
    assert f(FAKE, 8, 6148, 32, 8, 128, FAKE, FAKE, None) == _lib.FP8Q_ERR_ALIGN     # ld % 8
    w = L.fp8q_kv_cache_write
    ok = dict(x=FAKE, T=8, ld=6144, Hq=32, Hkv=8, D=128, slots=FAKE, ns=64, s=FAKE, q=FAKE,
              ldq=4096, k=FAKE, v=FAKE)

    def call(**kw):
        a = dict(ok, **kw)
        return w(a["x"], a["T"], a["ld"], a["Hq"], a["Hkv"], a["D"], a["slots"], a["ns"], a["s"],
                 a["q"], a["ldq"], a["k"], a["v"], None)
    assert call(D=72, ld=72 * 48, ldq=72 * 32) == _lib.FP8Q_ERR_SHAPE            # D % 16
    assert call(ldq=4000) == _lib.FP8Q_ERR_SHAPE
    assert call(ns=-1) == _lib.FP8Q_ERR_SHAPE
    assert call(slots=None) == _lib.FP8Q_ERR_NULL
    assert call(k=None) == _lib.FP8Q_ERR_NULL
    assert call(slots=FAKE + 4) == _lib.FP8Q_ERR_ALIGN
    assert call(q=FAKE + 4) == _lib.FP8Q_ERR_ALIGN
    assert call(T=0, x=None, slots=None, s=None, q=None, k=None, v=None) == _lib.FP8Q_OK


def test_weight_batch_host_checks(L):
    f = L.fp8q_quant_weight_block_batched
    assert f(FAKE, 3, 100, 5, None) == _lib.FP8Q_ERR_ARG
    assert f(FAKE, 4096, 100, 0, None) == _lib.FP8Q_ERR_SHAPE
    assert f(FAKE, 3, -1, 0, None) == _lib.FP8Q_ERR_SHAPE
    assert f(None, 3, 100, 0, None) == _lib.FP8Q_ERR_NULL
    assert f(FAKE + 4, 3, 100, 0, None) == _lib.FP8Q_ERR_ALIGN
    assert f(None, 0, 0, 1, None) == _lib.FP8Q_OK


def test_selftest_timeout_host_checks(L):
    f = L.fp8q_selftest_timeout
    assert f(0, None) == _lib.FP8Q_ERR_ARG
    assert f(200_000_000, None) == _lib.FP8Q_ERR_ARG
    import torch
    if not torch.cuda.is_available():
        assert f(1_000_000, None) == _lib.FP8Q_ERR_ARCH
