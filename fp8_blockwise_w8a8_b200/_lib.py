"""ctypes declarations of the C ABI in include/fp8q.h (libfp8q.so, built in-tree).

Loading fails loudly when the library is missing: there is no fallback implementation.
"""
import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfp8q.so")

FP8Q_OK = 0
FP8Q_ERR_NULL = 1
FP8Q_ERR_SHAPE = 2
FP8Q_ERR_ALIGN = 3
FP8Q_ERR_ARCH = 4
FP8Q_ERR_LAUNCH = 5
FP8Q_ERR_TIMEOUT = 6
FP8Q_ERR_ARG = 7
FP8Q_ERR_TOO_LARGE = 8
FP8Q_ERR_RANGE = 9
FP8Q_ERR_NOT_POW2 = 10

FP8Q_SCALE_F32 = 0
FP8Q_SCALE_E8M0 = 1

# Every symbol include/fp8q.h declares, with (restype, argtypes).
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
SIGNATURES = {
    "fp8q_quant_weight_block": (_I, [_P, _I64, _I64, _I64, _P, _I64, _P, _I, _P]),
    "fp8q_rmsnorm_quant_token": (_I, [_P, _P, ctypes.c_float, _I64, _I64, _I64, _P, _I64, _P,
                                      _I64, _P]),
    "fp8q_rmsnorm_quant_token_fmt": (_I, [_P, _P, ctypes.c_float, _I64, _I64, _I64, _P, _I64, _P,
                                          _I64, _I, _P]),
    "fp8q_gemm_w8a8_block": (_I, [_P, _I64, _P, _I64, _P, _I64, _P, _I, _I64, _I64, _I64, _P,
                                  _I64, _P]),
    "fp8q_gemm_w8a8_block_splitk": (_I, [_P, _I64, _P, _I64, _P, _I64, _P, _I, _I64, _I64, _I64,
                                         _P, _I64, _I, _P, _I64, _P]),
    "fp8q_gemm_w8a8_block_splitk_noalloc": (_I, [_P, _I64, _P, _I64, _P, _I64, _P, _I, _I64, _I64,
                                                 _I64, _P, _I64, _I, _P]),
    "fp8q_gemm_splitk_workspace_bytes": (_I, [_I64, _I64, _I64, _I, ctypes.POINTER(_I64)]),
    "fp8q_grouped_gemm_w8a8_block": (_I, [_P, _I64, _P, _I64, _P, _I64, _P, _I, _P, _I64, _I64,
                                          _I64, _I64, _P, _I64, _P]),
    "fp8q_silu_mul_quant": (_I, [_P, _I64, _I64, _I64, _P, _I64, _P, _I64, _I, _P]),
    "fp8q_inverse_rope_quant": (_I, [_P, _I64, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, _I, _I,
                                     _P, _I64, _P, _I64, _P]),
    "fp8q_gemm_w8a8_block_diag": (_I, [_P, _I64, _P, _I64, _P, _I64, _P, _I, _I64, _I64, _I64,
                                       _I64, _P, _I64, _P]),
    "fp8q_gemm_w8a8_mx": (_I, [_P, _I64, _P, _I64, _P, _I64, _P, _I64, _I64, _I64, _I64, _P,
                               _I64, _P]),
    "fp8q_qkv_scales": (_I, [_P, _I64, _I64, _I64, _I64, _I64, _P, _P, _P]),
    "fp8q_quant_weight_block_batched": (_I, [_P, _I64, _I64, _I, _P]),
    "fp8q_kv_cache_write": (_I, [_P, _I64, _I64, _I64, _I64, _I64, _P, _I64, _P, _P, _I64, _P, _P,
                                 _P]),
    "fp8q_quant_rowwise": (_I, [_P, _P, ctypes.c_float, _I64, _I64, _I64, _P, _I64, _P, _P]),
    "fp8q_gemm_w8a8_rowwise": (_I, [_P, _I64, _P, _P, _I64, _P, _I64, _I64, _I64, _P, _I64, _P]),
    "fp8q_add_rmsnorm_quant": (_I, [_P, _I64, _P, _I64, _P, ctypes.c_float, _I64, _I64, _I, _I,
                                    _P, _I64, _P, _I64, _P]),
    "fp8q_selftest_timeout": (_I, [_I64, _P]),
    "fp8q_check_device_error": (_I, [_P]),
    "fp8q_status_string": (ctypes.c_char_p, [_I]),
    "fp8q_attention_decode": (_I, [_P, _I64, _P, _P, _I64, _P, _P, _I64, _P, _I64, _I64, _I64,
                                   _I64, _I64, _I64, ctypes.c_float, _P, _I64, _P, _I64, _P]),
    "fp8q_attention_decode_workspace_bytes": (_I, [_I64, _I64, _I64, _I64, _I64, _P]),
    "fp8q_abi_version": (_I, []),
}

_lib = None


class Fp8qError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = status_string(status) if _lib is not None else str(status)
        super().__init__(f"{where}: status {status} ({msg})")


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libfp8q.so is not built ({LIB_PATH}); run `python -m fp8_blockwise_w8a8_b200.build`"
                " (there is no non-CUDA fallback)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().fp8q_status_string(int(status)).decode()


def check(status: int, where: str) -> None:
    if status != FP8Q_OK:
        raise Fp8qError(status, where)
