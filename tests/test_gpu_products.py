"""GPU parity of the products (W4A4 GEMM, FP8 GEMV, FP8 GEMM, int8 per-32
GEMM) against the CPU oracle on identical quantised codes:
|gpu - oracle| <= 1e-2 |oracle| + 1e-3 sum|a*w|, element by element.  Sizes
span several tiles with ragged edges; the full configurations run in the
launch configuration the benchmark times, checked on sampled rows."""
import numpy as np
import pytest
import torch

import int8_gemm_gemv_b200 as bsq
import oracle
from int8_gemm_gemv_b200 import synth
from gpu_helpers import bf16_out, check_tol, empty, host, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _no_timeouts():
    yield
    assert bsq.debug_take_timeouts() == 0


def sample_rows(m, count=16, seed=0):
    g = np.random.default_rng(seed)
    r = set([0, m - 1, min(m - 1, 127), min(m - 1, 128)])
    r.update(g.integers(0, m, count).tolist())
    return np.array(sorted(r), np.int64)


# ------------------------------------------------------------------ W4A4 ---

def nvfp4_from_oracle(m, n, k, seed, heavy=True):
    a_bf, w_bf = synth.w4a4_inputs(m, n, k, seed=seed, heavy_tailed=heavy)
    sb2 = float(np.float32(oracle.amax_bf16(w_bf)) / np.float32(6 * 448))
    ap, asf = oracle.quant_nvfp4(a_bf, 1.0)
    wp, wsf = oracle.quant_nvfp4(w_bf, sb2)
    return ap, asf, wp, wsf, 1.0, sb2


def nvfp4_random(m, n, k, seed):
    ap = synth.uniform_bytes((m, k // 2), seed, 11)
    wp = synth.uniform_bytes((n, k // 2), seed, 12)
    asf = synth.uniform_bytes((m, k // 16), seed, 13, 0x20, 0x60)
    wsf = synth.uniform_bytes((n, k // 16), seed, 14, 0x20, 0x60)
    return ap, asf, wp, wsf, 1.0, 2.0**-7


def run_w4a4(ap, asf, wp, wsf, sa2, sb2):
    m, n, k = ap.shape[0], wp.shape[0], ap.shape[1] * 2
    out = bf16_out((m, n))
    bsq.w4a4_gemm(to_dev(ap), to_dev(asf), to_dev(wp), to_dev(wsf), out, sa2, sb2, m, n, k)
    torch.cuda.synchronize()
    return host(out, np.uint16)


@pytest.mark.parametrize("mnk", [(16, 256, 512), (200, 300, 512), (129, 520, 768), (1, 8, 256), (300, 1000, 1024),
                                 (257, 510, 1536)])
def test_w4a4_small_and_ragged(mnk):
    m, n, k = mnk
    args = nvfp4_from_oracle(m, n, k, seed=1)
    g = run_w4a4(*args)
    ob, _, ab = oracle.w4a4_gemm(*args)
    check_tol(g, ob, ab, f"w4a4 {mnk}")


@pytest.mark.parametrize("m", [1, 2, 31, 32, 33, 64, 65, 100, 128])
def test_w4a4_small_m_swapped(m):
    """M <= 128 runs the swapped-operand kernel (weights as the MMA's M
    operand, activations padded to 32, 64 or 128 columns); ragged N."""
    n, k = 1984, 5120
    args = nvfp4_from_oracle(m, n, k, seed=3)
    g = run_w4a4(*args)
    ob, _, ab = oracle.w4a4_gemm(*args)
    check_tol(g, ob, ab, f"w4a4 small {m}x{n}x{k}")


@pytest.mark.parametrize("mnk", [(4, 17408, 5120), (5, 1001, 512), (128, 130, 256), (3, 24, 768)])
def test_w4a4_small_m_shapes(mnk):
    m, n, k = mnk
    args = nvfp4_from_oracle(m, n, k, seed=4)
    g = run_w4a4(*args)
    ob, _, ab = oracle.w4a4_gemm(*args)
    check_tol(g, ob, ab, f"w4a4 small {mnk}")


@pytest.mark.parametrize("m", [16, 300])
def test_w4a4_device_scale2_chain(m):
    """Weight scale2 formed on the device (amax -> scale2 -> codes) and read
    by the GEMM from device memory: codes, scales and scale2 equal the host
    form; the GEMM output equals the host-scale call bit for bit."""
    n, k = 768, 1024
    a_bf, w_bf = synth.w4a4_inputs(m, n, k, seed=7, heavy_tailed=True)
    wd = to_dev(w_bf)
    amax = empty((1,), torch.float32)
    bsq.bsq_amax_bf16(wd, w_bf.size, amax)
    wp, wsf = empty((n, k // 2), torch.uint8), empty((n, k // 16), torch.uint8)
    s2 = empty((1,), torch.float32)
    bsq.quantize_bf16_to_nvfp4_devscale(wd, wp, wsf, amax, s2, n, k)
    torch.cuda.synchronize()
    s2_host = float(np.float32(oracle.amax_bf16(w_bf)) / np.float32(6 * 448))
    assert float(s2.item()) == s2_host
    owp, owsf = oracle.quant_nvfp4(w_bf, s2_host)
    assert np.array_equal(host(wp), owp) and np.array_equal(host(wsf), owsf)
    ap, asf = oracle.quant_nvfp4(a_bf, 1.0)
    out_dev = bf16_out((m, n))
    bsq.w4a4_gemm_devscale(to_dev(ap), to_dev(asf), wp, wsf, out_dev, 1.0, s2, m, n, k)
    out_host = bf16_out((m, n))
    bsq.w4a4_gemm(to_dev(ap), to_dev(asf), wp, wsf, out_host, 1.0, s2_host, m, n, k)
    torch.cuda.synchronize()
    assert np.array_equal(host(out_dev, np.uint16), host(out_host, np.uint16))
    ob, _, ab = oracle.w4a4_gemm(ap, asf, owp, owsf, 1.0, s2_host)
    check_tol(host(out_dev, np.uint16), ob, ab, f"w4a4 devscale m={m}")


def test_nvfp4_device_scale2_all_zero():
    x = np.zeros((4, 64), np.uint16)
    amax = empty((1,), torch.float32)
    xd = to_dev(x)
    bsq.bsq_amax_bf16(xd, x.size, amax)
    p, sf = empty((4, 32), torch.uint8), empty((4, 4), torch.uint8)
    s2 = empty((1,), torch.float32)
    bsq.quantize_bf16_to_nvfp4_devscale(xd, p, sf, amax, s2, 4, 64)
    torch.cuda.synchronize()
    assert float(s2.item()) == 0.0 and not host(p).any() and not host(sf).any()


@pytest.mark.parametrize("amax", [float("nan"), float("inf"), 1e-36])
def test_nvfp4_device_scale2_rejected_amax(amax):
    """An amax whose scale2 (amax / 2688) the host form rejects -- NaN,
    infinite, or non-zero below 2688 * FLT_MIN -- quantises like an all-zero
    tensor (scale2 0, zero scales and codes), the GEMM then gives zeros, and
    flag bit 1 is raised once."""
    m, n, k = 16, 64, 256
    x = synth.normal_bf16((n, k), 0.02, 0, 8)
    xd = to_dev(x)
    amax_dev = torch.tensor([amax], dtype=torch.float32, device="cuda")
    p = torch.full((n, k // 2), 0x55, dtype=torch.uint8, device="cuda")
    sf = torch.full((n, k // 16), 0x55, dtype=torch.uint8, device="cuda")
    s2 = torch.full((1,), 1.0, dtype=torch.float32, device="cuda")
    bsq.quantize_bf16_to_nvfp4_devscale(xd, p, sf, amax_dev, s2, n, k)
    torch.cuda.synchronize()
    assert float(s2.item()) == 0.0 and not host(p).any() and not host(sf).any()
    assert bsq.debug_take_timeouts() == 2
    ap, asf = oracle.quant_nvfp4(synth.normal_bf16((m, k), 1.0, 0, 9), 1.0)
    out = bf16_out((m, n))
    bsq.w4a4_gemm_devscale(to_dev(ap), to_dev(asf), p, sf, out, 1.0, s2, m, n, k)
    torch.cuda.synchronize()
    assert np.all(oracle.bf16_to_f32(host(out, np.uint16)) == 0.0)


def test_w4a4_structured_one_hot():
    """One-hot activation rows pick single weight elements: checks nibble
    order, scale placement per row and per 16-block, and the M/N tiling."""
    m, n, k = 256, 512, 512
    g = np.random.default_rng(5)
    a = np.zeros((m, k), np.uint8)
    cols = g.integers(0, k, m)
    a[np.arange(m), cols] = 2  # 1.0
    ap = (a[:, 0::2] | (a[:, 1::2] << 4)).astype(np.uint8)
    asf = synth.uniform_bytes((m, k // 16), 5, 1, 0x30, 0x48)
    wp = synth.uniform_bytes((n, k // 2), 5, 2)
    wsf = synth.uniform_bytes((n, k // 16), 5, 3, 0x30, 0x48)
    got = run_w4a4(ap, asf, wp, wsf, 1.0, 1.0)
    ob, ex, ab = oracle.w4a4_gemm(ap, asf, wp, wsf, 1.0, 1.0)
    check_tol(got, ob, ab, "w4a4 one-hot")
    # each product is exact in FP32 and BF16 keeps 8 bits: exact match
    # whenever the exact value is BF16-representable
    exact_rep = oracle.bf16_to_f32(ob).astype(np.float64) == ex
    assert np.array_equal(got[exact_rep], ob[exact_rep])


def test_w4a4_realistic_mid():
    args = nvfp4_from_oracle(512, 2048, 5120, seed=0)
    g = run_w4a4(*args)
    rows = sample_rows(512, 24)
    ob, _, ab = oracle.w4a4_gemm(*args, rows=rows)
    check_tol(g[rows], ob, ab, "w4a4 512x2048x5120")


@pytest.mark.parametrize("m", [4096, 512, 16384])
def test_w4a4_full_size(m):
    n, k = 17408, 5120
    args = nvfp4_random(m, n, k, seed=2)
    g = run_w4a4(*args)
    rows = sample_rows(m, 12)
    ob, _, ab = oracle.w4a4_gemm(*args, rows=rows)
    check_tol(g[rows], ob, ab, f"w4a4 {m}x{n}x{k}")


# ------------------------------------------------------------------ GEMV ---

def run_gemv(inp, wq, ws):
    m, k = inp.shape
    n = wq.shape[0]
    out = bf16_out((m, n))
    bsq.fp8_gemv_rowscale(to_dev(inp), to_dev(wq), to_dev(ws), out, m, n, k)
    torch.cuda.synchronize()
    return host(out, np.uint16)


@pytest.fixture(scope="module")
def gemv_weight():
    _, w_bf = synth.gemv_inputs(1, 5120, 5120, seed=0)
    return oracle.quant_rowwise_fp8(w_bf)


@pytest.mark.parametrize("m", [1, 2, 3, 8, 9, 16])
def test_gemv_cfg2(gemv_weight, m):
    wq, ws = gemv_weight
    inp = synth.normal_bf16((m, 5120), 1.0, 0, 3)
    g = run_gemv(inp, wq, ws)
    ob, _, ab = oracle.fp8_gemv_rowscale(inp, wq, ws)
    check_tol(g, ob, ab, f"gemv m={m}")


def test_gemv_activation_range(gemv_weight):
    """The GEMV runs its activations through FP16 with a per-row power of two,
    so rows far from 1 in magnitude must still match the oracle: a row
    scaled by 2^100, one by 2^-100, an all-zero row, and a row whose largest
    element is 2^20 times its others; each row's result must also equal the
    same row computed alone (the scale is per row)."""
    wq, ws = gemv_weight
    base = synth.normal_bf16((4, 5120), 1.0, 2, 7)
    x = oracle.bf16_to_f32(base).astype(np.float32)
    x[0] *= np.float32(2.0**100)
    x[1] *= np.float32(2.0**-100)
    x[2] = 0.0
    x[3, 17] = np.float32(2.0**20)
    inp = synth.to_bf16_bits(x)
    g = run_gemv(inp, wq, ws)
    ob, _, ab = oracle.fp8_gemv_rowscale(inp, wq, ws)
    check_tol(g, ob, ab, "gemv activation range")
    assert np.all(oracle.bf16_to_f32(g[2]) == 0.0)
    for r in range(4):
        assert np.array_equal(run_gemv(inp[r:r + 1].copy(), wq, ws), g[r:r + 1]), r


def test_gemv_row_independent_of_batch(gemv_weight):
    """A row computed alone, or in a batch of 2, 8 or 16, gives the same bits
    (fp8_gemv_batch.rs: the batched kernels are bit-identical per row)."""
    wq, ws = gemv_weight
    inp = synth.normal_bf16((16, 5120), 1.0, 1, 3)
    full = run_gemv(inp, wq, ws)
    for m in (1, 2, 8, 15):
        part = run_gemv(inp[:m].copy(), wq, ws)
        assert np.array_equal(part, full[:m]), m


@pytest.mark.parametrize("nk", [(1000, 1040), (17, 16), (4095, 64)])
def test_gemv_ragged(nk):
    n, k = nk
    inp, w_bf = synth.gemv_inputs(16, n, k, seed=2)
    wq, ws = oracle.quant_rowwise_fp8(w_bf)
    for m in (1, 5, 16):
        g = run_gemv(inp[:m].copy(), wq, ws)
        ob, _, ab = oracle.fp8_gemv_rowscale(inp[:m], wq, ws)
        check_tol(g, ob, ab, f"gemv {m}x{n}x{k}")


def run_gemv_bs(inp, wq, S):
    m, k = inp.shape
    n = wq.shape[0]
    out = bf16_out((m, n))
    bsq.fp8_gemv_blockscaled(to_dev(inp), to_dev(wq), to_dev(S), out, m, n, k)
    torch.cuda.synchronize()
    return host(out, np.uint16)


@pytest.mark.parametrize("mnk", [(1, 5120, 5120), (2, 5120, 5120), (4, 5120, 5120), (16, 1024, 1024),
                                 (3, 256, 128), (9, 1152, 1920), (2, 8192, 5120)])
def test_gemv_blockscaled(mnk):
    """Block-scaled FP8 weights (the block FP8 format, per-128x128 scales)."""
    m, n, k = mnk
    inp, w_bf = synth.gemv_inputs(m, n, k, seed=5)
    wq, S = oracle.quant_blockfp8(w_bf)
    g = run_gemv_bs(inp, wq, S)
    ob, _, ab = oracle.fp8_gemv_blockscaled(inp, wq, S)
    check_tol(g, ob, ab, f"gemv block-scaled {mnk}")


def test_gemv_blockscaled_row_independent_of_batch():
    inp, w_bf = synth.gemv_inputs(16, 1024, 2048, seed=6)
    wq, S = oracle.quant_blockfp8(w_bf)
    all16 = run_gemv_bs(inp, wq, S)
    for m in (1, 4):
        part = run_gemv_bs(inp[:m].copy(), wq, S)
        assert np.array_equal(part, all16[:m])


# lm_head-sized N: many tile groups per CTA, ragged N, K % 64 != 0 (one copy
# per 64-byte chunk) and K % 64 == 0 (one copy per slot)
@pytest.mark.parametrize("nkm", [(75781, 80, 1), (75781, 80, 9), (80000, 128, 2), (80000, 128, 16)])
def test_gemv_large_n_ragged(nkm):
    n, k, m = nkm
    inp, w_bf = synth.gemv_inputs(m, n, k, seed=9)
    wq, ws = oracle.quant_rowwise_fp8(w_bf)
    g = run_gemv(inp, wq, ws)
    ob, _, ab = oracle.fp8_gemv_rowscale(inp, wq, ws)
    check_tol(g, ob, ab, f"gemv large n {m}x{n}x{k}")


@pytest.mark.parametrize("n", [256, 76800])
def test_gemv_every_code_exact(n):
    """Every finite E4M3 byte, each picked out by a one-hot activation row
    with row scale 1: the output is the code's value, exact in BF16, so the
    E4M3 conversion inside the kernel must match the oracle bit for bit
    (one tile group per CTA at n = 256, many at n = 76800)."""
    k, m = 256, 16
    codes = np.arange(256, dtype=np.uint8)
    codes[codes == 0x7F] = 0x7E
    codes[codes == 0xFF] = 0xFE
    wq = np.empty((n, k), np.uint8)
    for r in range(n):  # a different rotation per row, so every code meets every one-hot column
        wq[r] = np.roll(codes, r % 256)
    ws = np.ones(n, np.float32)
    inp = np.zeros((m, k), np.uint16)
    hot = np.random.default_rng(3).choice(k, m, replace=False)
    inp[np.arange(m), hot] = 0x3F80  # 1.0
    g = run_gemv(inp, wq, ws)
    ob, _, _ = oracle.fp8_gemv_rowscale(inp, wq, ws)
    assert np.array_equal(g, ob)


@pytest.mark.parametrize("mn", [(3, 76800), (11, 76800)])
def test_gemv_blockscaled_large_n(mn):
    m, n = mn
    k = 256
    inp, w_bf = synth.gemv_inputs(m, n, k, seed=10)
    wq, S = oracle.quant_blockfp8(w_bf)
    g = run_gemv_bs(inp, wq, S)
    ob, _, ab = oracle.fp8_gemv_blockscaled(inp, wq, S)
    check_tol(g, ob, ab, f"gemv block-scaled large n {m}x{n}x{k}")


def test_gemv_large_n_independent_of_batch():
    n, k = 76800, 512
    inp, w_bf = synth.gemv_inputs(16, n, k, seed=11)
    wq, ws = oracle.quant_rowwise_fp8(w_bf)
    full = run_gemv(inp, wq, ws)
    for m in (1, 8, 9):
        part = run_gemv(inp[:m].copy(), wq, ws)
        assert np.array_equal(part, full[:m]), m


def test_gemv_lm_head_shape():
    n, k = 151936, 5120
    wq = synth.uniform_bytes((n, k), 0, 21, 0, 0x7F) | (synth.uniform_bytes((n, k), 0, 22, 0, 2) << 7)
    ws = synth.uniform_f32((n,), 0, 23, 1e-4, 1e-3)
    inp = synth.normal_bf16((2, k), 1.0, 0, 24)
    g = run_gemv(inp, wq, ws)
    cols = sample_rows(n, 200, seed=3)
    ob, _, ab = oracle.fp8_gemv_rowscale(inp, wq[cols], ws[cols])
    check_tol(g[:, cols], ob, ab, "gemv lm_head")


# -------------------------------------------------------------- FP8 GEMM ---

def run_fp8_gemm(a, sa, w, sw):
    m, k = a.shape
    n = w.shape[0]
    out = bf16_out((m, n))
    bsq.fp8_gemm_rowscale(to_dev(a), to_dev(sa), to_dev(w), to_dev(sw), out, m, n, k)
    torch.cuda.synchronize()
    return host(out, np.uint16)


@pytest.mark.parametrize("mnk", [(23, 256, 256), (300, 520, 1040), (128, 256, 128)])
def test_fp8_gemm_small_and_ragged(mnk):
    m, n, k = mnk
    a_bf, w_bf = synth.blockfp8_inputs(m, n, k, seed=1)
    a, sa = oracle.quant_rowwise_fp8(a_bf)
    w, sw = oracle.quant_rowwise_fp8(w_bf)
    g = run_fp8_gemm(a, sa, w, sw)
    ob, _, ab = oracle.fp8_gemm_rowscale(a, sa, w, sw)
    check_tol(g, ob, ab, f"fp8 gemm {mnk}")


def test_fp8_gemm_full_size():
    m, n, k = 8192, 10240, 5120
    a = synth.uniform_bytes((m, k), 0, 31, 0, 0x7F) | (synth.uniform_bytes((m, k), 0, 32, 0, 2) << 7)
    w = synth.uniform_bytes((n, k), 0, 33, 0, 0x7F) | (synth.uniform_bytes((n, k), 0, 34, 0, 2) << 7)
    sa = synth.uniform_f32((m,), 0, 35, 1e-3, 1e-2)
    sw = synth.uniform_f32((n,), 0, 36, 1e-5, 1e-4)
    g = run_fp8_gemm(a, sa, w, sw)
    rows = sample_rows(m, 12)
    ob, _, ab = oracle.fp8_gemm_rowscale(a, sa, w, sw, rows=rows)
    check_tol(g[rows], ob, ab, "fp8 gemm 8192x10240x5120")


# -------------------------------------------------------------- int8 GEMM --

def run_int8(a, w, sa, sw):
    m, k = a.shape
    n = w.shape[0]
    out = bf16_out((m, n))
    bsq.int8_blockscaled_gemm(to_dev(a), to_dev(w), to_dev(sa), to_dev(sw), out, m, n, k)
    torch.cuda.synchronize()
    return host(out, np.uint16)


# (128, 20224, 128) has 158 tiles: more than one per SM, so some CTAs take a
# second tile; (2048, 1280, 256) has 160 (a short second round), and
# (2000, 1280, 384) the same with a ragged last row tile.
@pytest.mark.parametrize("mnk", [(64, 128, 128), (200, 300, 640), (129, 136, 1024), (1, 130, 256), (77, 131, 384),
                                 (128, 20224, 128), (64, 128, 512), (2048, 1280, 256), (2000, 1280, 384)])
def test_int8_small_and_ragged(mnk):
    m, n, k = mnk
    a_bf, w_bf = synth.w4a8_inputs(m, n, k, seed=1)
    s2 = float(np.float32(oracle.amax_bf16(w_bf)) / np.float32(6 * 448))
    wp, wsf = oracle.quant_nvfp4(w_bf, s2)
    w, sw = oracle.requant_w_nvfp4_int8(wp, wsf, s2)
    a, sa = oracle.quant_act_int8_per32(a_bf)
    g = run_int8(a, w, sa, sw)
    ob, _, ab = oracle.int8_blockscaled_gemm(a, w, sa, sw)
    check_tol(g, ob, ab, f"int8 {mnk}")


def run_int8_ws(a, w, sa, sw, ws=None):
    m, k = a.shape
    n = w.shape[0]
    out = bf16_out((m, n))
    nbytes = bsq.int8_gemm_workspace_bytes()
    if ws is None:
        ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    bsq.int8_blockscaled_gemm_ws(to_dev(a), to_dev(w), to_dev(sa), to_dev(sw), out, ws, nbytes, m, n, k)
    torch.cuda.synchronize()
    return host(out, np.uint16)


# With the workspace a last round of at most a third (a half) of the SMs'
# tiles is split along K: (2048, 1280, 256) leaves 12 tiles for 148 SMs, two
# pieces each (K has two blocks of 128); (2000, 1280, 384) three pieces; the
# others take no split and must equal the plain call bit for bit.
@pytest.mark.parametrize("mnk", [(2048, 1280, 256), (2000, 1280, 384), (64, 128, 512), (200, 300, 640)])
def test_int8_ws_matches_oracle(mnk):
    m, n, k = mnk
    a_bf, w_bf = synth.w4a8_inputs(m, n, k, seed=4)
    s2 = float(np.float32(oracle.amax_bf16(w_bf)) / np.float32(6 * 448))
    wp, wsf = oracle.quant_nvfp4(w_bf, s2)
    w, sw = oracle.requant_w_nvfp4_int8(wp, wsf, s2)
    a, sa = oracle.quant_act_int8_per32(a_bf)
    g = run_int8_ws(a, w, sa, sw)
    ob, _, ab = oracle.int8_blockscaled_gemm(a, w, sa, sw)
    check_tol(g, ob, ab, f"int8 ws {mnk}")
    if mnk in ((64, 128, 512), (200, 300, 640)):
        assert np.array_equal(g, run_int8(a, w, sa, sw))
    assert bsq.debug_take_timeouts() == 0


def test_int8_ws_reuse_and_determinism():
    """Two calls on one workspace (the first leaves its counters at zero)
    give the same bits, and a third on a fresh workspace too."""
    m, n, k = 2000, 1280, 384
    a_bf, w_bf = synth.w4a8_inputs(m, n, k, seed=5)
    s2 = float(np.float32(oracle.amax_bf16(w_bf)) / np.float32(6 * 448))
    wp, wsf = oracle.quant_nvfp4(w_bf, s2)
    w, sw = oracle.requant_w_nvfp4_int8(wp, wsf, s2)
    a, sa = oracle.quant_act_int8_per32(a_bf)
    ws = torch.zeros(bsq.int8_gemm_workspace_bytes(), dtype=torch.uint8, device="cuda")
    g1 = run_int8_ws(a, w, sa, sw, ws)
    g2 = run_int8_ws(a, w, sa, sw, ws)
    g3 = run_int8_ws(a, w, sa, sw)
    assert np.array_equal(g1, g2) and np.array_equal(g1, g3)
    assert bsq.debug_take_timeouts() == 0


def test_int8_prefill_two_launches():
    m, n, k = 96, 256, 512
    a_bf, w_bf = synth.w4a8_inputs(m, n, k, seed=3)
    w = synth.uniform_int8((n, k), 3, 40)
    sw = synth.uniform_f32((n, k // 32), 3, 41, 1e-4, 1e-3)
    out = bf16_out((m, n))
    a_i8, a_s = empty((m, k), torch.int8), empty((m, k // 32), torch.float32)
    n0 = bsq.debug_launch_count()
    bsq.int8_w4a8_prefill(to_dev(a_bf), to_dev(w), to_dev(sw), a_i8, a_s, out, m, n, k)
    assert bsq.debug_launch_count() == n0 + 2
    torch.cuda.synchronize()
    a, sa = oracle.quant_act_int8_per32(a_bf)
    assert np.array_equal(host(a_i8), a) and np.array_equal(host(a_s), sa)
    ob, _, ab = oracle.int8_blockscaled_gemm(a, w, sa, sw)
    check_tol(host(out, np.uint16), ob, ab, "int8 prefill")


def test_int8_full_size():
    m, n, k = 2048, 5120, 17408
    a = synth.uniform_int8((m, k), 0, 42)
    w = synth.uniform_int8((n, k), 0, 43)
    sa = synth.uniform_f32((m, k // 32), 0, 44, 1e-3, 1e-1)
    sw = synth.uniform_f32((n, k // 32), 0, 45, 1e-5, 1e-4)
    g = run_int8(a, w, sa, sw)
    rows = sample_rows(m, 10)
    ob, _, ab = oracle.int8_blockscaled_gemm(a, w, sa, sw, rows=rows)
    check_tol(g[rows], ob, ab, "int8 2048x5120x17408")
