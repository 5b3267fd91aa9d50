"""Structured operands whose products are exact in FP32, for bit-exact
full-K parity of the three tensor-core GEMMs.

Each activation row has exactly one non-zero element per quantisation block
along K (one per 16 for NVFP4, one per 32 for the int8 per-32 format, one per
32-wide MMA step for row-scaled FP8), at a seeded random position inside the
block, with a small value; weights take a handful of small codes, and every
scale is a power of two.  Every product and every partial sum is then a
multiple of a power of two far below 2^24 units, so an FP32 accumulation in
any order gives the exact sum, and the single BF16 rounding of the GPU and of
the oracle (round-to-nearest-even of that exact sum) agree bit for bit.  The
typical output stays within 8 significant bits, so losing a single block
(a K step, a scale column, a stage of a late persistent round) changes the
BF16 result of most outputs.

Only random draws live here (through synth's seeded streams); the products
themselves come from the oracle.
"""
import numpy as np

from int8_gemm_gemv_b200 import synth

# E2M1 codes: 1 = 0.5, 2 = 1.0, 3 = 1.5; bit 3 = sign.  E4M3 bytes: 0x30 =
# 0.5, 0x38 = 1.0, 0x3C = 1.5, 0x40 = 2.0; bit 7 = sign.


def _one_per_block(rows, k, block, seed, tid):
    """Positions [rows, k/block] of the one non-zero element of each block."""
    return synth.rng(seed, tid).integers(0, block, size=(rows, k // block))


def _signs(shape, seed, tid):
    return synth.rng(seed, tid).integers(0, 2, size=shape).astype(np.uint8)


def w4a4_sparse(m, n, k, seed):
    """NVFP4 operands: A rows with one +-0.5 / +-1 per 16-block and block
    scales 1 or 2; W codes in {0, +-0.5, +-1, +-1.5} with block scales 0.5 or
    1.  Returns (a_packed, a_sf, w_packed, w_sf)."""
    pos = _one_per_block(m, k, 16, seed, 901)
    mag = synth.rng(seed, 902).integers(1, 3, size=pos.shape).astype(np.uint8)  # codes 1, 2
    sgn = _signs(pos.shape, seed, 903)
    codes = np.zeros((m, k), np.uint8)
    cols = np.arange(k // 16)[None, :] * 16 + pos
    codes[np.arange(m)[:, None], cols] = mag | (sgn << 3)
    a_packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    a_sf = np.where(synth.rng(seed, 904).integers(0, 2, size=(m, k // 16)) == 1, 0x40, 0x38).astype(np.uint8)
    wc = synth.rng(seed, 905).integers(0, 4, size=(n, k)).astype(np.uint8) | (_signs((n, k), seed, 906) << 3)
    w_packed = (wc[:, 0::2] | (wc[:, 1::2] << 4)).astype(np.uint8)
    w_sf = np.where(synth.rng(seed, 907).integers(0, 2, size=(n, k // 16)) == 1, 0x38, 0x30).astype(np.uint8)
    return a_packed, a_sf, w_packed, w_sf


def fp8_sparse(m, n, k, seed):
    """Row-scaled FP8 operands: A rows with one +-0.5 / +-1 per 32 K; W bytes
    in {0, +-0.5, +-1, +-1.5}; row scales powers of two.  Returns
    (a, a_scale, w, w_scale)."""
    pos = _one_per_block(m, k, 32, seed, 911)
    mag = np.where(synth.rng(seed, 912).integers(0, 2, size=pos.shape) == 1, 0x38, 0x30).astype(np.uint8)
    a = np.zeros((m, k), np.uint8)
    cols = np.arange(k // 32)[None, :] * 32 + pos
    a[np.arange(m)[:, None], cols] = mag | (_signs(pos.shape, seed, 913) << 7)
    wmag = np.array([0x00, 0x30, 0x38, 0x3C], np.uint8)[synth.rng(seed, 914).integers(0, 4, size=(n, k))]
    w = (wmag | (_signs((n, k), seed, 915) << 7)).astype(np.uint8)
    a_scale = np.ldexp(np.float32(1.0), synth.rng(seed, 916).integers(-3, 1, size=m)).astype(np.float32)
    w_scale = np.ldexp(np.float32(1.0), synth.rng(seed, 917).integers(-2, 1, size=n)).astype(np.float32)
    return a, a_scale, w, w_scale


def int8_sparse(m, n, k, seed):
    """int8 per-32 operands: A rows with one +-1 per 32-block; W in -2..2;
    per-32 scales 0.5 or 1 on both sides.  Returns (a, w, a_scale, w_scale)."""
    pos = _one_per_block(m, k, 32, seed, 921)
    a = np.zeros((m, k), np.int8)
    cols = np.arange(k // 32)[None, :] * 32 + pos
    a[np.arange(m)[:, None], cols] = np.where(_signs(pos.shape, seed, 922) == 1, -1, 1).astype(np.int8)
    w = synth.rng(seed, 923).integers(-2, 3, size=(n, k)).astype(np.int8)
    a_scale = np.where(synth.rng(seed, 924).integers(0, 2, size=(m, k // 32)) == 1, 1.0, 0.5).astype(np.float32)
    w_scale = np.where(synth.rng(seed, 925).integers(0, 2, size=(n, k // 32)) == 1, 1.0, 0.5).astype(np.float32)
    return a, w, a_scale, w_scale


def int8_saturated(m, n, k, seed):
    """int8 per-32 operands at the ends of the code range: each 32-block of a
    row (of A or of W) is all -128, all 127, or a seeded mix of the two, and
    every scale is 1.  A block's exact int32 partial then reaches +-2^19
    (32 * 128 * 128 = 524288 for two all -128 blocks, -520192 for -128 against
    127), the largest magnitude the format allows.  With K <= 1024 every sum
    stays below 2^24 and is exact in FP32.  Returns (a, w, a_scale, w_scale)."""
    assert k <= 1024 and k % 32 == 0

    def side(rows, tid):
        kind = synth.rng(seed, tid).integers(0, 3, size=(rows, k // 32))
        mix = np.where(synth.rng(seed, tid + 1).integers(0, 2, size=(rows, k)) == 1, -128, 127)
        kind_k = np.repeat(kind, 32, axis=1)
        v = np.where(kind_k == 0, -128, np.where(kind_k == 1, 127, mix))
        return v.astype(np.int8)

    a = side(m, 931)
    w = side(n, 933)
    return a, w, np.ones((m, k // 32), np.float32), np.ones((n, k // 32), np.float32)
