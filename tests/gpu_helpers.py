"""Shared helpers of the GPU parity tests: host<->device copies of numpy
arrays and the output tolerance check."""
import numpy as np
import torch

import oracle

DEV = "cuda"


def to_dev(a: np.ndarray) -> torch.Tensor:
    """numpy array -> CUDA tensor with the same bytes (uint16 becomes int16)."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).to(DEV)


def empty(shape, dtype) -> torch.Tensor:
    return torch.empty(shape, dtype=dtype, device=DEV)


def host(t: torch.Tensor, dtype=None) -> np.ndarray:
    a = t.detach().cpu().numpy()
    if dtype is not None:
        a = a.view(dtype)
    return a


def bf16_out(shape) -> torch.Tensor:
    # poisoned with NaN bit patterns so an unwritten output cannot pass
    return torch.full(shape, -1, dtype=torch.int16, device=DEV)


def check_tol(gpu_bits: np.ndarray, oracle_bits: np.ndarray, abssum: np.ndarray, what: str):
    """|gpu - oracle| <= 1e-2 |oracle| + 1e-3 sum|a*w|, element by element."""
    g = oracle.bf16_to_f32(gpu_bits).astype(np.float64)
    o = oracle.bf16_to_f32(oracle_bits).astype(np.float64)
    assert np.all(np.isfinite(g)), f"{what}: non-finite GPU output"
    tol = oracle.tolerance(oracle_bits, abssum)
    err = np.abs(g - o)
    bad = err > tol
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside tolerance; first at {tuple(i)}: "
                             f"gpu={g[tuple(i)]} oracle={o[tuple(i)]} tol={tol[tuple(i)]}")
    return float((err / np.maximum(tol, 1e-30)).max())
