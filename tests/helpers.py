"""Shared test helpers: moving oracle-side numpy arrays to and from torch device tensors, and the
GEMM tolerance comparison.  No arithmetic of the method lives here."""
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


def assert_within_gemm_tolerance(out: np.ndarray, ref: np.ndarray, absref: np.ndarray, what=""):
    """|out - ref| <= 8e-3 * sum|a sa w sw| + one bf16 ulp of |ref|, element by element."""
    err = np.abs(out - ref)
    tol = oracle.gemm_tolerance(ref, absref)
    bad = err > tol
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(
            f"{what}: {bad.sum()} of {bad.size} outside tolerance; first at {tuple(i)}: "
            f"out={out[tuple(i)]!r} ref={ref[tuple(i)]!r} tol={tol[tuple(i)]!r}")
    assert np.isfinite(out).all(), what
