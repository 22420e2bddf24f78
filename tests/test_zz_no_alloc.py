"""The split-K GEMM entry point that allocates nothing (its scratch is a fixed buffer in the
library's own device memory), called through the C ABI and compared with the workspace entry
point it mirrors and with the oracle.  Two calls in a row check that each call leaves the
scratch ready for the next.  Collected last; also meant to pass alone in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from fp8_blockwise_w8a8_b200 import _lib, inputs

from helpers import assert_within_gemm_tolerance, dev_f32, dev_u8, host_bf16_f64, promoted_steps

pytestmark = pytest.mark.gpu


def _operands(M, N, K, seed, fmt=oracle.SCALE_F32):
    a = inputs.randn_bf16((M, K), 1.0, seed, 0)
    w = inputs.randn_bf16((N, K), 0.02, seed, 1)
    lds = (M + 3) // 4 * 4
    aq, sa = oracle.quant_token_1x128(a, lds=lds)
    wq, sw = oracle.quant_weight_block(w, fmt)
    return aq, sa, wq, sw


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _call_noalloc(L, d, M, N, K, out, splits, fmt=_lib.FP8Q_SCALE_F32):
    aq, sa, wq, sw = d
    return L.fp8q_gemm_w8a8_block_splitk_noalloc(
        aq.data_ptr(), aq.stride(0), sa.data_ptr(), sa.stride(0), wq.data_ptr(), wq.stride(0),
        sw.data_ptr(), fmt, M, N, K, out.data_ptr(), out.stride(0), splits, _stream())


def _call_workspace(L, d, M, N, K, out, splits, fmt=_lib.FP8Q_SCALE_F32):
    aq, sa, wq, sw = d
    nbytes = ctypes.c_int64(0)
    assert L.fp8q_gemm_splitk_workspace_bytes(M, N, K, splits, ctypes.byref(nbytes)) == 0
    ws = torch.empty(max(16, nbytes.value), dtype=torch.uint8, device="cuda")
    st = L.fp8q_gemm_w8a8_block_splitk(
        aq.data_ptr(), aq.stride(0), sa.data_ptr(), sa.stride(0), wq.data_ptr(), wq.stride(0),
        sw.data_ptr(), fmt, M, N, K, out.data_ptr(), out.stride(0), splits, ws.data_ptr(),
        ws.numel(), _stream())
    return st


@pytest.mark.parametrize("M,N,K,splits,rows", [
    (100, 2048, 1024, 4, None),                              # 8 tiles x 4 splits, all rows
    (128, 12288, 4096, 3, [0, 1, 63, 64, 126, 127]),         # decode shape, 48 tiles x 3
    (128, 4096, 12288, 0, [0, 77, 127]),                     # the library's choice: 8 splits
])
def test_noalloc_matches_workspace_entry_twice(M, N, K, splits, rows):
    L = _lib.lib()
    aq, sa, wq, sw = _operands(M, N, K, 70 + splits)
    d = (dev_u8(aq), dev_f32(sa), dev_u8(wq), dev_f32(sw))
    ref_out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    assert _call_workspace(L, d, M, N, K, ref_out, splits) == _lib.FP8Q_OK
    assert L.fp8q_check_device_error(_stream()) == _lib.FP8Q_OK
    ref, absref = oracle.gemm_w8a8_block(aq, sa, wq, sw, oracle.SCALE_F32, rows=rows)
    expect = host_bf16_f64(ref_out)
    sel = slice(None) if rows is None else rows
    for _ in range(2):
        out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _call_noalloc(L, d, M, N, K, out, splits) == _lib.FP8Q_OK
        assert L.fp8q_check_device_error(_stream()) == _lib.FP8Q_OK
        got = host_bf16_f64(out)
        # against the workspace entry point: within the GEMM tolerance (in fact bit-identical,
        # since both run the same kernel with the same split order)
        steps = promoted_steps(K, splits if splits else K // 128)
        assert_within_gemm_tolerance(got[sel], expect[sel], absref, what="vs workspace entry",
                                     steps=steps)
        assert np.array_equal(got, expect)
        assert_within_gemm_tolerance(got[sel], ref, absref, what="vs oracle", steps=steps)


def test_noalloc_e8m0_weight_scales_twice():
    """E8M0 weight scales through the same scratch: decode shape, 3 splits."""
    L = _lib.lib()
    M, N, K, splits = 128, 12288, 4096, 3
    E8M0 = oracle.SCALE_E8M0
    aq, sa, wq, sw = _operands(M, N, K, 77, E8M0)
    d = (dev_u8(aq), dev_f32(sa), dev_u8(wq), dev_u8(sw))
    ref_out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    assert _call_workspace(L, d, M, N, K, ref_out, splits, E8M0) == _lib.FP8Q_OK
    assert L.fp8q_check_device_error(_stream()) == _lib.FP8Q_OK
    rows = [0, 1, 64, 127]
    ref, absref = oracle.gemm_w8a8_block(aq, sa, wq, sw, E8M0, rows=rows)
    expect = host_bf16_f64(ref_out)
    for _ in range(2):
        out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _call_noalloc(L, d, M, N, K, out, splits, E8M0) == _lib.FP8Q_OK
        assert L.fp8q_check_device_error(_stream()) == _lib.FP8Q_OK
        got = host_bf16_f64(out)
        assert np.array_equal(got, expect)
        assert_within_gemm_tolerance(got[rows], ref, absref, what="e8m0 vs oracle",
                                     steps=promoted_steps(K, splits))


def test_noalloc_rejects_problems_beyond_its_scratch():
    L = _lib.lib()
    M, N, K = 128, 24576, 4096                 # 96 tiles x 3 splits = 288 > 192 tile-splits
    aq = torch.zeros((M, K), dtype=torch.uint8, device="cuda")
    sa = torch.ones((K // 128, M), dtype=torch.float32, device="cuda")
    wq = torch.zeros((N, K), dtype=torch.uint8, device="cuda")
    sw = torch.ones((N // 128, K // 128), dtype=torch.float32, device="cuda")
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    st = _call_noalloc(L, (aq, sa, wq, sw), M, N, K, out, 3)
    assert st == _lib.FP8Q_ERR_TOO_LARGE
    assert "static" in _lib.status_string(st)
