"""The int8 per-32 GEMM's convert-free fold, checked exhaustively on the host.

The kernel never converts an int32 partial to FP32.  Before each 32-wide K
block, an FP16 tensor-core MMA over a constant tile (every element 768,
K = 16, FP32 accumulate) writes C = 16 * 768^2 into every accumulator word;
the block's int8 MMA then adds its exact int32 partial p to those same 32
bits, read as an int32.  The fold reads the word back as FP32 and subtracts
C.  This test replays those steps in numpy:

- 768 is exact in FP16, and every partial sum k * 768^2 (k <= 16) is exact
  in FP32, so the offset MMA writes exactly C, whatever order it adds in;
- every partial a block can produce, from 32 * (-128) * 127 to
  32 * (-128) * (-128), read back through the offset, gives p exactly;
- a partial just outside that range would leave the binade where FP32
  encodings are consecutive integers, which is why the range matters.

The arithmetic is that of the kernel (FP32 bit patterns, an int32 add, one
FP32 subtraction); nothing here calls the library."""
import numpy as np

OFFSET = np.float32(16 * 768 * 768)  # 9 * 2^20
P_MIN, P_MAX = 32 * (-128) * 127, 32 * (-128) * (-128)


def fold_readback(p):
    """The word the fold sees after the offset MMA and the int8 MMA, as FP32,
    minus the offset (one FP32 subtraction)."""
    word = np.full(p.shape, OFFSET, np.float32).view(np.int32)
    word = (word.astype(np.int64) + p).astype(np.int32)  # the int8 MMA's int32 accumulate
    return (word.view(np.float32) - OFFSET).astype(np.float32)


def test_offset_mma_writes_exact_constant():
    h = np.float16(768)
    assert float(h) == 768.0
    prod = np.float32(h) * np.float32(h)
    assert float(prod) == 768.0 ** 2
    # every prefix sum of the sixteen equal products is exact in FP32, so any
    # accumulation order inside the MMA gives the same word
    acc = np.float32(0)
    for k in range(16):
        acc = np.float32(acc + prod)
        assert float(acc) == (k + 1) * 768.0 ** 2
    assert acc == OFFSET
    assert OFFSET.view(np.uint32) == 0x4B100000


def test_every_block_partial_reads_back_exactly():
    p = np.arange(P_MIN, P_MAX + 1, dtype=np.int64)
    got = fold_readback(p)
    assert np.array_equal(got.astype(np.int64), p)
    assert np.all(got.astype(np.float64) == p.astype(np.float64))


def test_partials_of_saturated_blocks():
    for a, w in ((-128, -128), (-128, 127), (127, 127), (127, -128), (0, 0)):
        p = np.array([32 * a * w], np.int64)
        assert int(fold_readback(p)[0]) == 32 * a * w


def test_range_is_what_makes_it_exact():
    # The binade [2^23, 2^24) holds the offset with room 2^19 on each side;
    # past 2^24 the spacing is 2 and odd partials would be lost.
    assert OFFSET - 2 ** 19 >= 2 ** 23 and OFFSET + 2 ** 19 < 2 ** 24
    beyond = np.array([2 ** 24 - int(OFFSET) + 1], np.int64)  # reaches 2^24 + 1
    assert int(fold_readback(beyond)[0]) != int(beyond[0])
