"""Helpers of the GPU parity tests: moving arrays, status words and the float
tolerance used against the oracle."""
from __future__ import annotations

import numpy as np
import torch

# Float bound: max relative error 1e-3 against the oracle's fp32
# dequant epilogue.
REL_TOL = 1e-3


def dev(a, dtype=None) -> torch.Tensor:
    t = a if isinstance(a, torch.Tensor) else torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.contiguous().cuda()


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.cpu().numpy()


def new_status() -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def status_word(st: torch.Tensor) -> int:
    torch.cuda.synchronize()
    return int(st.item())


def bf16_half_ulp(ref: np.ndarray) -> np.ndarray:
    """Half a bf16 ulp at |ref| (8 significant bits): the rounding error a
    correct bf16 store may add on top of the float32 result."""
    a = np.abs(ref.astype(np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (e - 8), 2.0 ** -133)


def assert_close(got, ref, D, bf16: bool = False, what: str = ""):
    """|got - ref| <= 1e-3 * D (+ half a bf16 ulp for bf16 outputs), elementwise.
    D is the magnitude of the summands that form ref (so that cancellation in
    ref does not make the bound vanish)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    bound = REL_TOL * np.asarray(D, np.float64) + 1e-30
    if bf16:
        bound = bound + bf16_half_ulp(ref)
    err = np.abs(got - ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err / bound), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; "
                             f"worst at {i}: got {got[i]!r} ref {ref[i]!r} bound {bound[i]!r}")


def rotated_magnitude(pre: np.ndarray, B: int) -> np.ndarray:
    """Summand magnitude of (pre R) with R = blockdiag(H_B)/sqrt(B): every
    output of a block is +-c times each input of the block, so D = c*sum|pre|."""
    rows, cols = pre.shape
    a = np.abs(pre.astype(np.float64)).reshape(rows, cols // B, B).sum(-1, keepdims=True)
    return np.broadcast_to(a / np.sqrt(B), (rows, cols // B, B)).reshape(rows, cols)
