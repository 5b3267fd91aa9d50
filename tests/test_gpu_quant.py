"""GPU parity of the quantisers and requantisers: every code and scale must be
bit-identical to the CPU oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import int8_gemm_gemv_b200 as bsq
import oracle
from int8_gemm_gemv_b200 import synth
from gpu_helpers import empty, host, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _no_timeouts():
    yield
    assert bsq.debug_take_timeouts() == 0


def gpu_nvfp4(x_bits, scale2):
    m, k = x_bits.shape
    packed, sf = empty((m, k // 2), torch.uint8), empty((m, k // 16), torch.uint8)
    bsq.quantize_bf16_to_nvfp4(to_dev(x_bits), packed, sf, scale2, m, k)
    torch.cuda.synchronize()
    return host(packed), host(sf)


def special_rows():
    """Rows that exercise ties, signed zeros, zero blocks, saturation and
    the worked examples."""
    rows = [
        [6, -3, 1.5, 0.5, 0, 2, -4, 1, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, -0.25],
        [3, 1, -0.5, 0.125, 0.375, 2.25, -1.75, 0, 0, 0, 0, 0, 0, 0, 0, -3],
        [0] * 16,
        [6144, -2688, 448, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0],
        [1e-30, -1e-30, 0, -0.0, 1e-38, -1e-39, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0],
        [-6, -5, -3.5, -2.5, -1.75, -1.25, -0.75, -0.25, -0.1, 0.1, 3e4, -3e4, 1, 2, 4, 6],
    ]
    return synth.to_bf16_bits(np.array(rows, np.float32).reshape(3, 32))


@pytest.mark.parametrize("case", ["cfg1_act", "cfg1_weight", "ragged", "special", "cfg3_act"])
def test_quant_nvfp4_bitexact(case):
    if case == "cfg1_act":
        x, s2 = synth.normal_bf16((16, 512), 1.0, 0, 1), 1.0
    elif case == "cfg1_weight":
        x = synth.normal_bf16((256, 512), 0.02, 0, 2)
        s2 = float(np.float32(oracle.amax_bf16(x)) / np.float32(6 * 448))
    elif case == "ragged":
        x, s2 = synth.student_t_bf16((37, 1040), 4.0, 1, 9, outlier_frac=0.02), 1.0
    elif case == "special":
        x, s2 = special_rows(), 1.0
    else:
        x, s2 = synth.student_t_bf16((4096, 5120), 4.0, 0, 1, outlier_frac=0.01), 1.0
    gp, gs = gpu_nvfp4(x, s2)
    op, os_ = oracle.quant_nvfp4(x, s2)
    assert np.array_equal(gs, os_), f"scales differ at {np.argwhere(gs != os_)[:4]}"
    assert np.array_equal(gp, op), f"codes differ at {np.argwhere(gp != op)[:4]}"


def test_quant_nvfp4_largest_activation_shape_sampled_rows():
    """16384 x 5120 activations (the largest W4A4 configuration): every
    sampled row bit-exact."""
    x = synth.student_t_bf16((16384, 5120), 4.0, 0, 11, outlier_frac=0.01)
    gp, gs = gpu_nvfp4(x, 1.0)
    rows = np.array([0, 1, 4095, 4096, 8191, 12345, 16383])
    op, os_ = oracle.quant_nvfp4(x[rows], 1.0)
    assert np.array_equal(gs[rows], os_) and np.array_equal(gp[rows], op)


def test_quant_nvfp4_weight_scale2_from_device_amax():
    x = synth.normal_bf16((512, 1024), 0.02, 3, 2)
    amax = empty((1,), torch.float32)
    bsq.bsq_amax_bf16(to_dev(x), x.size, amax)
    torch.cuda.synchronize()
    assert float(amax.item()) == oracle.amax_bf16(x)
    s2 = float(np.float32(amax.item()) / np.float32(6 * 448))
    gp, gs = gpu_nvfp4(x, s2)
    op, os_ = oracle.quant_nvfp4(x, s2)
    assert np.array_equal(gs, os_) and np.array_equal(gp, op)


@pytest.mark.parametrize("shape", [(5120, 5120), (33, 1040), (3, 16)])
def test_quant_rowwise_fp8_bitexact(shape):
    x = synth.normal_bf16(shape, 0.02, 0, 4)
    q, s = empty(shape, torch.uint8), empty((shape[0],), torch.float32)
    bsq.quant_rowwise_fp8(to_dev(x), q, s, shape[0], shape[1])
    torch.cuda.synchronize()
    oq, os_ = oracle.quant_rowwise_fp8(x)
    assert np.array_equal(host(s), os_)
    assert np.array_equal(host(q), oq)


def test_quant_rowwise_fp8_activation_rows_and_zero_row():
    x = synth.normal_bf16((8192, 5120), 1.0, 0, 7)
    x[5] = 0
    q, s = empty(x.shape, torch.uint8), empty((8192,), torch.float32)
    bsq.quant_rowwise_fp8(to_dev(x), q, s, 8192, 5120)
    torch.cuda.synchronize()
    rows = np.array([0, 5, 1, 4095, 8191])
    oq, os_ = oracle.quant_rowwise_fp8(x[rows])
    assert np.array_equal(host(s)[rows], os_) and np.array_equal(host(q)[rows], oq)
    assert host(s)[5] == 0 and not host(q)[5].any()


def test_quant_blockfp8_bitexact():
    x = synth.normal_bf16((10240, 5120), 0.02, 0, 8)
    q, S = empty(x.shape, torch.uint8), empty((80, 40), torch.float32)
    bsq.quant_blockfp8(to_dev(x), q, S, 10240, 5120)
    torch.cuda.synchronize()
    for r0 in (0, 10240 - 256):
        oq, oS = oracle.quant_blockfp8(x[r0:r0 + 256])
        assert np.array_equal(host(S)[r0 // 128:r0 // 128 + 2], oS)
        assert np.array_equal(host(q)[r0:r0 + 256], oq)


def test_requant_blockfp8_to_rowwise_bitexact_and_passthrough():
    x = synth.normal_bf16((10240, 5120), 0.02, 0, 8)
    w, S = oracle.quant_blockfp8(x[:1024])
    dw, dS = to_dev(w), to_dev(S)
    q, s = empty(w.shape, torch.uint8), empty((w.shape[0],), torch.float32)
    n0 = bsq.debug_launch_count()
    wu, su = bsq.requant_blockfp8_to_rowwise(bsq.BSQ_FP8_BLOCK_SCALED, dw, dS, w.shape[0], 5120, q, s)
    assert bsq.debug_launch_count() == n0 + 1
    assert (wu, su) == (q.data_ptr(), s.data_ptr())
    torch.cuda.synchronize()
    oq, os_ = oracle.requant_blockfp8_to_rowwise(w, S)
    assert np.array_equal(host(s), os_)
    assert np.array_equal(host(q), oq)
    # an already row-wise pair comes back untouched: same pointers, no launch
    before = host(q).copy()
    wu2, su2 = bsq.requant_blockfp8_to_rowwise(bsq.BSQ_FP8_PER_ROW, q, s, w.shape[0], 5120, None, None)
    assert (wu2, su2) == (q.data_ptr(), s.data_ptr())
    assert bsq.debug_launch_count() == n0 + 1
    torch.cuda.synchronize()
    assert np.array_equal(host(q), before)


@pytest.mark.parametrize("nk", [(256, 128), (128, 384), (128, 49280)])
def test_requant_blockfp8_to_rowwise_row_lengths(nk):
    # one-block rows, an odd number of blocks, and rows longer than the
    # shared-memory row buffer (the register path); row 3 is all zero
    n, k = nk
    x = synth.normal_bf16((n, k), 0.02, 0, 11)
    x[3, :] = 0
    w, S = oracle.quant_blockfp8(x)
    q, s = empty(w.shape, torch.uint8), empty((n,), torch.float32)
    bsq.requant_blockfp8_to_rowwise(bsq.BSQ_FP8_BLOCK_SCALED, to_dev(w), to_dev(S), n, k, q, s)
    torch.cuda.synchronize()
    oq, os_ = oracle.requant_blockfp8_to_rowwise(w, S)
    assert np.array_equal(host(s), os_)
    assert np.array_equal(host(q), oq)
    assert bsq.debug_take_timeouts() == 0


@pytest.mark.parametrize("shape", [(5120, 17408), (40, 1056)])
def test_requant_w_nvfp4_int8_bitexact(shape):
    x = synth.normal_bf16(shape, 0.02, 0, 6)
    s2 = float(np.float32(oracle.amax_bf16(x)) / np.float32(6 * 448))
    rows = np.arange(shape[0]) if shape[0] < 100 else np.array([0, 1, 2, 777, shape[0] - 1])
    op, os_ = oracle.quant_nvfp4(x[rows], s2)
    # the GPU requantises the whole weight; quantise it on the oracle side
    # only for the rows compared (rows are independent)
    fp, fs = oracle.quant_nvfp4(x, s2) if shape[0] < 100 else (None, None)
    if fp is None:
        fp = np.zeros((shape[0], shape[1] // 2), np.uint8)
        fs = np.zeros((shape[0], shape[1] // 16), np.uint8)
        fp[rows], fs[rows] = op, os_
    n, k = shape
    q, s = empty(shape, torch.int8), empty((n, k // 32), torch.float32)
    bsq.requant_w_nvfp4_int8(to_dev(fp), to_dev(fs), s2, q, s, n, k)
    torch.cuda.synchronize()
    oq, oscale = oracle.requant_w_nvfp4_int8(fp[rows], fs[rows], s2)
    assert np.array_equal(host(s)[rows], oscale)
    assert np.array_equal(host(q)[rows], oq)


@pytest.mark.parametrize("shape", [(2048, 17408), (7, 96)])
def test_quant_act_int8_bitexact(shape):
    x = synth.normal_outliers_bf16(shape, 1.0, 0, 5)
    if shape[0] > 100:
        x[3] = 0
    m, k = shape
    q, s = empty(shape, torch.int8), empty((m, k // 32), torch.float32)
    bsq.quant_act_int8_per32(to_dev(x), q, s, m, k)
    torch.cuda.synchronize()
    rows = np.arange(m) if m < 100 else np.array([0, 3, 1000, m - 1])
    oq, os_ = oracle.quant_act_int8_per32(x[rows])
    assert np.array_equal(host(s)[rows], os_)
    assert np.array_equal(host(q)[rows], oq)


def test_amax_exact_and_empty():
    x = synth.student_t_bf16((333, 1000), 4.0, 2, 1)
    amax = empty((1,), torch.float32)
    bsq.bsq_amax_bf16(to_dev(x), x.size, amax)
    torch.cuda.synchronize()
    assert float(amax.item()) == oracle.amax_bf16(x)
    bsq.bsq_amax_bf16(None, 0, amax)
    torch.cuda.synchronize()
    assert float(amax.item()) == 0.0


# ---------------------------------------------------------------------------
# Rounding boundaries.  The kernels decide most codes from two products that
# bracket the quotient and divide exactly only where the bracket straddles a
# boundary between two codes; these rows put quotients exactly on the
# boundaries (ties) and one BF16 step either side of them.

def _e4m3_values():
    sub = [m * 2.0 ** -9 for m in range(0, 8)]
    nrm = [(1 + m / 8) * 2.0 ** (e - 7) for e in range(1, 16) for m in range(8) if not (e == 15 and m == 7)]
    return np.array(sub + nrm, np.float64)


def _bf16_exact(v):
    b = synth.to_bf16_bits(np.asarray(v, np.float32))
    back = (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.array_equal(back, np.asarray(v, np.float64)), "boundary value not exact in BF16"
    return b


def _neighbours(v):
    """v and the BF16 values one step below and above it (v > 0)."""
    b = synth.to_bf16_bits(np.asarray(v, np.float32)).astype(np.int32)
    out = np.stack([b - 1, b, b + 1], -1).reshape(-1).astype(np.uint16)
    return (out.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def e4m3_boundary_rows(scales, k=256):
    """One row per scale s: amax 448 s, then s times every E4M3 midpoint
    and its BF16 neighbours, with alternating signs."""
    vals = _e4m3_values()
    mids = (vals[:-1] + vals[1:]) / 2
    rows = []
    for s in scales:
        body = _neighbours(mids * s)
        body = body * np.where(np.arange(body.size) % 2 == 0, 1.0, -1.0)
        row = np.concatenate([[448.0 * s], body])
        row = np.resize(row, k)
        row[0] = 448.0 * s
        _bf16_exact(row[:1])
        rows.append(row)
    return synth.to_bf16_bits(np.array(rows, np.float32))


def test_quant_rowwise_fp8_rounding_boundaries():
    x = e4m3_boundary_rows([1.0, 3.0, 0.75, 2.0 ** -6], k=1024)
    m, k = x.shape
    q, s = empty(x.shape, torch.uint8), empty((m,), torch.float32)
    bsq.quant_rowwise_fp8(to_dev(x), q, s, m, k)
    torch.cuda.synchronize()
    oq, os_ = oracle.quant_rowwise_fp8(x)
    assert np.array_equal(host(s), os_)
    assert np.array_equal(host(q), oq), f"codes differ at {np.argwhere(host(q) != oq)[:4]}"


def test_quant_blockfp8_rounding_boundaries():
    rows = e4m3_boundary_rows([1.0, 3.0], k=256)
    x = np.repeat(rows, 128, axis=0)  # 256 x 256: 2 x 2 blocks, amax 448 s in each
    x = np.ascontiguousarray(x)
    q, S = empty(x.shape, torch.uint8), empty((2, 2), torch.float32)
    bsq.quant_blockfp8(to_dev(x), q, S, 256, 256)
    torch.cuda.synchronize()
    oq, oS = oracle.quant_blockfp8(x)
    assert np.array_equal(host(S), oS)
    assert np.array_equal(host(q), oq)


def test_quant_act_int8_rounding_boundaries():
    blocks = []
    for s in (1.0, 2.0, 0.5):
        halves = (np.arange(0, 127) + 0.5) * s
        body = _neighbours(halves) * np.where(np.arange(3 * 127) % 2 == 0, 1.0, -1.0)
        for c in range(0, body.size, 31):
            blk = np.zeros(32)
            blk[0] = 127.0 * s
            seg = body[c:c + 31]
            blk[1:1 + seg.size] = seg
            blocks.append(blk)
    while len(blocks) % 8:
        blocks.append(blocks[0])
    x = synth.to_bf16_bits(np.array(blocks, np.float32).reshape(-1, 256))
    m, k = x.shape
    q, s = empty(x.shape, torch.int8), empty((m, k // 32), torch.float32)
    bsq.quant_act_int8_per32(to_dev(x), q, s, m, k)
    torch.cuda.synchronize()
    oq, os_ = oracle.quant_act_int8_per32(x)
    assert np.array_equal(host(s), os_)
    assert np.array_equal(host(q), oq), f"codes differ at {np.argwhere(host(q) != oq)[:4]}"


def test_quant_nvfp4_scale_rounding_boundaries():
    """Block amaxes at 6 x (every E4M3 midpoint up to 448), so that the scale
    quotient amax / (6 scale2) is a tie, with E2M1 midpoints inside."""
    vals = _e4m3_values()
    mids = ((vals[:-1] + vals[1:]) / 2)[8:]  # normal range
    blocks = []
    for mu in mids:
        amax = 6.0 * mu
        blk = np.array([amax, -0.25, 0.75, -1.25, 1.75, -2.5, 3.5, -5.0, 0.5, 1, 2, 3, 4, -6, 0.3, 0.1]) * mu
        blk[0] = amax
        blocks.append(blk)
    n = len(blocks) // 4 * 4
    x = synth.to_bf16_bits(np.array(blocks[:n], np.float32).reshape(-1, 64))
    gp, gs = gpu_nvfp4(x, 1.0)
    op, os_ = oracle.quant_nvfp4(x, 1.0)
    assert np.array_equal(gs, os_), f"scales differ at {np.argwhere(gs != os_)[:4]}"
    assert np.array_equal(gp, op), f"codes differ at {np.argwhere(gp != op)[:4]}"


@pytest.mark.parametrize("scale2", [1.0, 0.75, 0.625, 2.0 ** -3, float(np.float32(1 / 3)), 1e-3])
def test_quant_nvfp4_divisor_classes(scale2):
    """The block divisor d = e4m3(sf) * scale2 has few significant bits for
    scale2 = 1, 0.75, 2^-3 (exact ties are then common and the kernel snaps
    to the boundary) and many for 0.625 (7 bits with some scales), 1/3 and
    1e-3 (the bracketed path).  Tie-heavy rows scaled by scale2 and
    Student-t rows, bit-exact against the oracle."""
    ties = (special_rows().astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    body = synth.student_t_bf16((64, 1024), 4.0, 4, 3, outlier_frac=0.01)
    x = np.concatenate([synth.to_bf16_bits(np.resize(ties * scale2, (3, 1024)).astype(np.float32)), body])
    gp, gs = gpu_nvfp4(x, scale2)
    op, os_ = oracle.quant_nvfp4(x, scale2)
    assert np.array_equal(gs, os_), f"scales differ at {np.argwhere(gs != os_)[:4]}"
    assert np.array_equal(gp, op), f"codes differ at {np.argwhere(gp != op)[:4]}"


def test_quant_nvfp4_every_scale_at_every_boundary():
    """Every finite positive E4M3 block scale, forced by a block whose
    largest element is exactly 6 times its value (activation path, scale2 =
    1), with the other fifteen elements on E2M1 code boundaries (exact ties),
    on code values, and one BF16 step either side of a boundary, both signs:
    the kernels' division-free code rule must give the oracle's codes bit for
    bit for every divisor it meets."""
    mags = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0]
    rows = []
    for code in range(1, 127):
        v = np.float32(oracle.e4m3_value(code))
        base = [np.float32(6.0) * v] + [np.float32(b) * v for b in mags]
        for sign in (1.0, -1.0):
            for step in (0, 1, -1):
                blk = np.array(base[:1] + base[1:], np.float32)
                body = blk[1:] * np.float32(sign)
                bits = synth.to_bf16_bits(body).astype(np.int32)
                if step:
                    # one BF16 step away from zero (+1) or towards it (-1)
                    bits = bits + step
                body = oracle.bf16_to_f32(bits.astype(np.uint16))
                block = np.zeros(16, np.float32)
                block[0] = blk[0]
                block[1:1 + len(body)] = body
                rows.append(block)
    x = synth.to_bf16_bits(np.stack(rows).reshape(-1, 32))
    # the forced block maxima are exact in BF16, so every block's scale is its code
    gp, gs = gpu_nvfp4(x, 1.0)
    op, os_ = oracle.quant_nvfp4(x, 1.0)
    assert np.array_equal(gs, os_), f"scales differ at {np.argwhere(gs != os_)[:4]}"
    assert np.array_equal(gp, op), f"codes differ at {np.argwhere(gp != op)[:4]}"
    assert len(set(gs.ravel().tolist())) >= 126
