"""Seeded synthetic inputs shaped like the pages' workloads.

This module only draws random numbers: it holds none of the method's
arithmetic, and both the CUDA path (tests, benchmark) and the CPU oracle take
their inputs from it.  Every tensor comes from its own numpy PCG64 stream,
keyed by ``(seed, tensor_id)``, so a tensor does not depend on which others
were drawn before it.  BF16 tensors are returned as ``uint16`` bit patterns
(numpy has no bfloat16); the FP32 -> BF16 step is torch's round-to-nearest-even
cast.

Distributions (the workloads of the linear layers the pages serve):
  * weights  : N(0, 0.02)
  * activations : N(0, 1), or Student-t(nu=4), optionally with 1% of the K
    channels ("outlier channels") scaled by 20.
"""
from __future__ import annotations

import numpy as np
import torch


def rng(seed: int, tensor_id: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(tensor_id)])


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """FP32 array -> BF16 bit patterns (uint16), round-to-nearest-even."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def outlier_channels(k: int, seed: int, tensor_id: int, frac: float = 0.01) -> np.ndarray:
    """Indices of the ``frac`` share of the K channels that carry outliers."""
    count = max(1, int(round(frac * k)))
    return np.sort(rng(seed, tensor_id + 500_000).permutation(k)[:count])


def _fill_chunks(shape, draw) -> np.ndarray:
    """Draw a large FP32 tensor row-block by row-block (bounded host memory)."""
    rows, k = shape
    out = np.empty((rows, k), np.uint16)
    step = max(1, (1 << 24) // max(k, 1))
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        out[r0:r1] = to_bf16_bits(draw(r1 - r0))
    return out


def normal_bf16(shape, std: float, seed: int, tensor_id: int) -> np.ndarray:
    g = rng(seed, tensor_id)
    return _fill_chunks(shape, lambda r: g.standard_normal((r, shape[1]), dtype=np.float32) * np.float32(std))


def student_t_bf16(shape, nu: float, seed: int, tensor_id: int,
                   outlier_frac: float = 0.0, outlier_scale: float = 20.0) -> np.ndarray:
    g = rng(seed, tensor_id)
    cols = outlier_channels(shape[1], seed, tensor_id, outlier_frac) if outlier_frac > 0 else None

    def draw(r):
        x = g.standard_t(nu, size=(r, shape[1])).astype(np.float32)
        if cols is not None:
            x[:, cols] *= np.float32(outlier_scale)
        return x
    return _fill_chunks(shape, draw)


def normal_outliers_bf16(shape, std: float, seed: int, tensor_id: int,
                         outlier_frac: float = 0.01, outlier_scale: float = 20.0) -> np.ndarray:
    g = rng(seed, tensor_id)
    cols = outlier_channels(shape[1], seed, tensor_id, outlier_frac)

    def draw(r):
        x = g.standard_normal((r, shape[1]), dtype=np.float32) * np.float32(std)
        x[:, cols] *= np.float32(outlier_scale)
        return x
    return _fill_chunks(shape, draw)


def uniform_bytes(shape, seed: int, tensor_id: int, low: int = 0, high: int = 256) -> np.ndarray:
    """Uniform integers in [low, high) as uint8."""
    return rng(seed, tensor_id).integers(low, high, size=shape, dtype=np.uint16).astype(np.uint8)


def uniform_int8(shape, seed: int, tensor_id: int, low: int = -127, high: int = 128) -> np.ndarray:
    return rng(seed, tensor_id).integers(low, high, size=shape, dtype=np.int16).astype(np.int8)


def uniform_f32(shape, seed: int, tensor_id: int, low: float, high: float) -> np.ndarray:
    return rng(seed, tensor_id).uniform(low, high, size=shape).astype(np.float32)


# Workload recipes (shapes of the pages' linear layers) ------------------------

def w4a4_inputs(m: int, n: int, k: int, seed: int = 0, heavy_tailed: bool = True):
    """A: BF16 [m,k] (Student-t(4) with 1% outlier channels x20, or N(0,1));
    W: BF16 [n,k] N(0, 0.02).  Returns (A bits, W bits)."""
    if heavy_tailed:
        a = student_t_bf16((m, k), 4.0, seed, 1, outlier_frac=0.01, outlier_scale=20.0)
    else:
        a = normal_bf16((m, k), 1.0, seed, 1)
    w = normal_bf16((n, k), 0.02, seed, 2)
    return a, w


def gemv_inputs(m: int, n: int, k: int, seed: int = 0):
    """in: BF16 [m,k] N(0,1); W: BF16 [n,k] N(0,0.02) (to be row-quantised)."""
    return normal_bf16((m, k), 1.0, seed, 3), normal_bf16((n, k), 0.02, seed, 4)


def w4a8_inputs(m: int, n: int, k: int, seed: int = 0):
    """A: BF16 [m,k] N(0,1) with 1% outlier channels x20; W: BF16 [n,k]
    N(0,0.02) (to be NVFP4-quantised, then requantised to int8)."""
    return normal_outliers_bf16((m, k), 1.0, seed, 5), normal_bf16((n, k), 0.02, seed, 6)


def blockfp8_inputs(m: int, n: int, k: int, seed: int = 0):
    """A: BF16 [m,k] N(0,1); W: BF16 [n,k] N(0,0.02) (to be block-FP8
    quantised with one scale per 128x128 block)."""
    return normal_bf16((m, k), 1.0, seed, 7), normal_bf16((n, k), 0.02, seed, 8)
