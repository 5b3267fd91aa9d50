"""Bit-exact full-K parity of the three tensor-core GEMMs at their benchmark
shapes, on structured operands whose partial sums are exact in FP32
(tests/exact_inputs.py): W4A4 4096 x 17408 x 5120 (gemm_fp4.rs, `w4a4_gemm`),
row-scaled FP8 8192 x 10240 x 5120 (dispatch_proj_rowwise.rs,
`cublas_fp8_rowwise_proj`) and int8 per-32 2048 x 5120 x 17408
(gemm_dense_int8.rs, `int8_gemm_faith2_prefill`).  Sampled rows, across all
N columns and so across every persistent round, must equal the oracle bit for
bit: a lost K block, scale block or stage changes the BF16 result.

The CPU tests at the end check, on the oracle alone, that this design has the
power claimed: one dropped block changes most outputs of its row."""
import numpy as np
import pytest
import torch

import int8_gemm_gemv_b200 as bsq
import oracle
from exact_inputs import fp8_sparse, int8_saturated, int8_sparse, w4a4_sparse
from gpu_helpers import bf16_out, host, to_dev


def sample_rows(m, count, seed):
    g = np.random.default_rng(seed)
    r = set([0, m - 1, 127, 128, 255, 256, m // 2])
    r.update(g.integers(0, m, count).tolist())
    return np.array(sorted(r), np.int64)


def _assert_bits(got, ob, what):
    bad = got != ob
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outputs differ; first at {i}: "
                             f"gpu={oracle.bf16_to_f32(got[i])} oracle={oracle.bf16_to_f32(ob[i])}")


@pytest.mark.gpu
def test_w4a4_full_k_bit_exact():
    m, n, k = 4096, 17408, 5120
    ap, asf, wp, wsf = w4a4_sparse(m, n, k, seed=1)
    out = bf16_out((m, n))
    bsq.w4a4_gemm(to_dev(ap), to_dev(asf), to_dev(wp), to_dev(wsf), out, 1.0, 1.0, m, n, k)
    torch.cuda.synchronize()
    assert bsq.debug_take_timeouts() == 0
    rows = sample_rows(m, 10, 1)
    ob, ex, _ = oracle.w4a4_gemm(ap, asf, wp, wsf, 1.0, 1.0, rows=rows)
    _assert_bits(host(out, np.uint16)[rows], ob, "w4a4 4096x17408x5120 exact")


@pytest.mark.gpu
def test_fp8_gemm_full_k_bit_exact():
    m, n, k = 8192, 10240, 5120
    a, sa, w, sw = fp8_sparse(m, n, k, seed=2)
    out = bf16_out((m, n))
    bsq.fp8_gemm_rowscale(to_dev(a), to_dev(sa), to_dev(w), to_dev(sw), out, m, n, k)
    torch.cuda.synchronize()
    assert bsq.debug_take_timeouts() == 0
    rows = sample_rows(m, 10, 2)
    ob, _, _ = oracle.fp8_gemm_rowscale(a, sa, w, sw, rows=rows)
    _assert_bits(host(out, np.uint16)[rows], ob, "fp8 gemm 8192x10240x5120 exact")


@pytest.mark.gpu
def test_int8_full_k_bit_exact():
    m, n, k = 2048, 5120, 17408
    a, w, sa, sw = int8_sparse(m, n, k, seed=3)
    out = bf16_out((m, n))
    bsq.int8_blockscaled_gemm(to_dev(a), to_dev(w), to_dev(sa), to_dev(sw), out, m, n, k)
    torch.cuda.synchronize()
    assert bsq.debug_take_timeouts() == 0
    rows = sample_rows(m, 10, 3)
    ob, _, _ = oracle.int8_blockscaled_gemm(a, w, sa, sw, rows=rows)
    _assert_bits(host(out, np.uint16)[rows], ob, "int8 2048x5120x17408 exact")


@pytest.mark.gpu
def test_int8_ws_full_k_bit_exact():
    """The workspace form at the benchmark shape: 640 tiles on 148 SMs, so the
    last 48 tiles (output columns 4736..5119) are split along K into three
    pieces each.  Exact sums regardless of order, so bit-exact; every sampled
    row crosses the split tiles."""
    m, n, k = 2048, 5120, 17408
    a, w, sa, sw = int8_sparse(m, n, k, seed=3)
    out = bf16_out((m, n))
    nbytes = bsq.int8_gemm_workspace_bytes()
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    bsq.int8_blockscaled_gemm_ws(to_dev(a), to_dev(w), to_dev(sa), to_dev(sw), out, ws, nbytes, m, n, k)
    torch.cuda.synchronize()
    assert bsq.debug_take_timeouts() == 0
    rows = sample_rows(m, 10, 3)
    ob, _, _ = oracle.int8_blockscaled_gemm(a, w, sa, sw, rows=rows)
    _assert_bits(host(out, np.uint16)[rows], ob, "int8 ws 2048x5120x17408 exact")


@pytest.mark.gpu
@pytest.mark.parametrize("mnk", [(200, 300, 640), (2048, 1280, 256), (129, 136, 1024)])
def test_int8_saturated_blocks_bit_exact(mnk):
    """Blocks of all -128 and all 127 codes: every block partial is as large
    as the format allows (up to 2^19 in magnitude), through the plain call
    and the workspace form (whose last round splits at 2048 x 1280 x 256).
    Unit scales keep every sum exact, so the result is bit-exact."""
    m, n, k = mnk
    a, w, sa, sw = int8_saturated(m, n, k, seed=7)
    ob, _, _ = oracle.int8_blockscaled_gemm(a, w, sa, sw)
    out = bf16_out((m, n))
    bsq.int8_blockscaled_gemm(to_dev(a), to_dev(w), to_dev(sa), to_dev(sw), out, m, n, k)
    torch.cuda.synchronize()
    _assert_bits(host(out, np.uint16), ob, f"int8 saturated {mnk}")
    nbytes = bsq.int8_gemm_workspace_bytes()
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    out2 = bf16_out((m, n))
    bsq.int8_blockscaled_gemm_ws(to_dev(a), to_dev(w), to_dev(sa), to_dev(sw), out2, ws, nbytes, m, n, k)
    torch.cuda.synchronize()
    _assert_bits(host(out2, np.uint16), ob, f"int8 ws saturated {mnk}")
    assert bsq.debug_take_timeouts() == 0


# --------------------------------------------- power of the design (CPU) ---

def _changed_share(before, after):
    return float(np.mean(before != after))


def test_w4a4_design_sees_one_dropped_block():
    m, n, k = 8, 512, 5120
    ap, asf, wp, wsf = w4a4_sparse(m, n, k, seed=4)
    ob, ex, _ = oracle.w4a4_gemm(ap, asf, wp, wsf, 1.0, 1.0)
    # exact partial sums: the double result is a multiple of 1/8 (1/8 = 0.5 x
    # 0.5 x 0.5, the smallest product of codes and scales)
    assert np.all(ex * 8 == np.round(ex * 8))
    for blk in (0, 137, 319):  # first, middle and last 16-block of K
        ap2 = ap.copy()
        ap2[:, blk * 8:(blk + 1) * 8] = 0  # drop one 16-element block of every row
        ob2, _, _ = oracle.w4a4_gemm(ap2, asf, wp, wsf, 1.0, 1.0)
        assert _changed_share(ob, ob2) > 0.6, blk
    asf2 = asf.copy()
    asf2[:, 200] = np.where(asf[:, 200] == 0x38, 0x40, 0x38)  # one scale block of every row: 1 <-> 2
    ob3, _, _ = oracle.w4a4_gemm(ap, asf2, wp, wsf, 1.0, 1.0)
    assert _changed_share(ob, ob3) > 0.6


def test_fp8_design_sees_one_dropped_step():
    m, n, k = 8, 512, 5120
    a, sa, w, sw = fp8_sparse(m, n, k, seed=5)
    ob, ex, _ = oracle.fp8_gemm_rowscale(a, sa, w, sw)
    for step in (0, 80, 159):
        a2 = a.copy()
        a2[:, step * 32:(step + 1) * 32] = 0
        ob2, _, _ = oracle.fp8_gemm_rowscale(a2, sa, w, sw)
        assert _changed_share(ob, ob2) > 0.6, step


def test_int8_design_sees_one_dropped_block():
    m, n, k = 8, 512, 17408
    a, w, sa, sw = int8_sparse(m, n, k, seed=6)
    ob, ex, _ = oracle.int8_blockscaled_gemm(a, w, sa, sw)
    assert np.all(ex * 4 == np.round(ex * 4))
    for blk in (0, 271, 543):
        a2 = a.copy()
        a2[:, blk * 32:(blk + 1) * 32] = 0
        ob2, _, _ = oracle.int8_blockscaled_gemm(a2, w, sa, sw)
        assert _changed_share(ob, ob2) > 0.6, blk
    sw2 = sw.copy()
    sw2[:, 300] = np.where(sw[:, 300] == 1.0, 0.5, 1.0).astype(np.float32)
    ob3, _, _ = oracle.int8_blockscaled_gemm(a, w, sa, sw2)
    assert _changed_share(ob, ob3) > 0.4
