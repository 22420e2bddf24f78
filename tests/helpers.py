"""Shared test helpers: moving oracle-side numpy arrays to and from torch device tensors, and the
GEMM tolerance comparisons.  No arithmetic of the method lives here."""
import numpy as np
import torch

import oracle


def dev_bf16(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def dev_u8(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def dev_f32(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def host_bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def host_bf16_f64(t: torch.Tensor) -> np.ndarray:
    bits = host_bf16_bits(t).astype(np.uint32) << 16
    return bits.view(np.float32).astype(np.float64)


def promoted_steps(K: int, splits: int = 1) -> int:
    """fp32 rounding steps of a GEMM that promotes each 128-wide K-block: one fused multiply-add
    per K-block, the split partials' sum, and a constant for the scale product and the tensor
    core's own accumulation inside a K-block."""
    return K // 128 + (splits - 1 if splits > 1 else 0) + 8


def tmem_steps(K: int) -> int:
    """fp32 rounding steps of a GEMM that accumulates all of K in tensor memory (four K=32 MMAs
    per 128-wide K-block), then applies its scales once."""
    return 2 * (K // 128) + 8


def tight_gemm_bound(ref: np.ndarray, absref: np.ndarray, steps: int) -> np.ndarray:
    """The bound that follows from fp32 arithmetic: each of the kernel's fp32 roundings costs at
    most 2^-24 of a partial sum bounded by absref = sum_k |dec(a) sa dec(w) sw|, and the final
    rounding to bf16 at most half a bf16 ulp.  With a factor 2 of margin:
    |out - ref| <= ulp_bf16(|ref|) / 2 + steps * 2^-23 * absref.
    Rounding each K-block partial or each sa*sw to bf16 violates it on a third or more of the
    elements of random operands (tests/test_oracle_gemm.py plants that mistake)."""
    return 0.5 * oracle.bf16_ulp(ref) + steps * 2.0 ** -23 * absref


def assert_within_gemm_tolerance(out: np.ndarray, ref: np.ndarray, absref: np.ndarray, what="",
                                 *, steps: int):
    """Two gates, element by element: the stated tolerance |out - ref| <= 8e-3 * absref + one
    bf16 ulp of |ref|, and the tight bound of the kernel's fp32 arithmetic (tight_gemm_bound)."""
    err = np.abs(out - ref)
    assert np.isfinite(out).all(), what
    for name, tol in (("stated tolerance", oracle.gemm_tolerance(ref, absref)),
                      (f"fp32 bound ({steps} steps)", tight_gemm_bound(ref, absref, steps))):
        bad = err > tol
        if bad.any():
            i = np.argwhere(bad)[0]
            raise AssertionError(
                f"{what}: {bad.sum()} of {bad.size} outside the {name}; first at {tuple(i)}: "
                f"out={out[tuple(i)]!r} ref={ref[tuple(i)]!r} tol={tol[tuple(i)]!r} "
                f"absref={absref[tuple(i)]!r}")
