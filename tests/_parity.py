"""Helpers for the GPU parity tests: move seeded inputs to the device, run the
CUDA path through the binding, compare with the oracle.

Acceptance per output element (bf16 output, fp32 accumulation):
    |y - y_ref| <= 2**-7 * |y_ref| + 1e-3 * A,   A = sum_k |w_hat[n,k] * v[k]|
"""
from __future__ import annotations

import numpy as np
import torch

REL_TOL = 2.0 ** -7
ABS_COEF = 1e-3


def dev_bf16(a: np.ndarray) -> torch.Tensor:
    a = np.ascontiguousarray(a, dtype=np.uint16)
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()


def dev_u32(a: np.ndarray) -> torch.Tensor:
    a = np.ascontiguousarray(a, dtype=np.uint32)
    return torch.from_numpy(a.view(np.int32)).cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 device tensor -> numpy uint16 bit patterns."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_values(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def empty_bf16(*shape, fill_bits: int = 0x7FC1) -> torch.Tensor:
    """Output buffer pre-filled with a NaN sentinel so unwritten rows show."""
    t = torch.empty(shape, dtype=torch.int16, device="cuda")
    t.fill_(np.int16(np.uint16(fill_bits).view(np.int16)))
    return t.view(torch.bfloat16)


def check(y_bits: np.ndarray, y_ref: np.ndarray, a_ref: np.ndarray, what: str = ""):
    """Asserts the tolerance element-wise; returns the worst error/bound ratio."""
    y = bf16_values(y_bits)
    assert y.shape == y_ref.shape, (y.shape, y_ref.shape)
    assert np.all(np.isfinite(y)), f"{what}: non-finite outputs"
    err = np.abs(y - y_ref)
    bound = REL_TOL * np.abs(y_ref) + ABS_COEF * a_ref
    bad = err > bound
    if bad.any():
        idx = np.argwhere(bad)[:5]
        det = [(tuple(i), y[tuple(i)], y_ref[tuple(i)], bound[tuple(i)]) for i in idx]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside tolerance; "
                             f"first (index, y, y_ref, bound): {det}")
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(bound > 0, err / bound, 0.0)
    return float(ratio.max()) if ratio.size else 0.0


def sample_rows(N: int, count: int, seed: int) -> np.ndarray:
    """First, last and random rows: covers both tile edges and the interior."""
    rng = np.random.default_rng(seed)
    fixed = [0, 1, N // 2, N - 2, N - 1]
    rnd = rng.choice(N, size=min(count, N), replace=False)
    rows = np.unique(np.concatenate([np.array(fixed), rnd]) % N)
    return rows.astype(np.int32)
