"""Pins of the CPU oracle against things other than itself.

Every check here compares the oracle with an independent source: the
format specifications (golden tables), hand-worked examples, torch's own
FP8/BF16 casts, numpy's FP32 arithmetic and integer/float64 matmuls,
exact-rational brute force, and invariants of the method.  No GPU.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from int8_gemm_gemv_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_table(name, hexkeys=False):
    out = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, v = line.split()
        out[int(k, 16) if hexkeys else int(k)] = float(v)
    return out


E2M1 = _golden_table("e2m1_grid.txt")
E2M1_GRID = [Fraction(E2M1[i]) for i in range(8)]


def torch_e4m3_decode(codes):
    t = torch.from_numpy(np.asarray(codes, np.uint8).copy()).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def torch_e4m3_encode(x_f32):
    """torch's RNE cast; valid for |x| <= 448 (no saturation in torch)."""
    t = torch.from_numpy(np.asarray(x_f32, np.float32).copy()).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def bf16(x):
    return synth.to_bf16_bits(np.asarray(x, np.float32))


def f32(b):
    return synth.bf16_bits_to_f32(b)


def brute_e2m1(v: float) -> int:
    """Nearest E2M1 code by exact rational search; ties to the even index;
    saturating; sign kept."""
    sign = 8 if math.copysign(1.0, v) < 0 else 0
    a = abs(Fraction(v)) if math.isfinite(v) else Fraction(10**9)
    if a >= 6:
        return sign | 7
    best, bestd = 0, abs(a)
    for i in range(1, 8):
        d = abs(E2M1_GRID[i] - a)
        if d < bestd or (d == bestd and i % 2 == 0):
            best, bestd = i, d
    return sign | best


# ---------------------------------------------------------------- codecs ---

def test_e2m1_table_matches_spec():
    for c in range(16):
        got = oracle.e2m1_value(c)
        assert got == E2M1[c] and math.copysign(1, got) == math.copysign(1, E2M1[c])


def test_e4m3_points_match_spec():
    for c, v in _golden_table("e4m3_points.txt", hexkeys=True).items():
        got = oracle.e4m3_value(c)
        if math.isnan(v):
            assert math.isnan(got)
        else:
            assert got == v and math.copysign(1, got) == math.copysign(1, v), hex(c)


def test_e4m3_table_matches_torch_decode():
    ref = torch_e4m3_decode(np.arange(256))
    for c in range(256):
        got = oracle.e4m3_value(c)
        if math.isnan(ref[c]):
            assert math.isnan(got)
        else:
            assert got == ref[c], hex(c)


def test_e4m3_encode_decode_roundtrip():
    for c in range(256):
        if c & 0x7F == 0x7F:
            continue
        assert oracle.e4m3_encode(oracle.e4m3_value(c)) == c, hex(c)


def test_e4m3_encode_matches_torch_rne():
    g = np.random.default_rng(11)
    # dense sweep over every binade plus exact midpoints between codes
    vals = list(g.uniform(-448, 448, 4000).astype(np.float32))
    vals += list((g.standard_normal(4000) * 2.0 ** g.integers(-12, 8, 4000)).astype(np.float32))
    mags = [oracle.e4m3_value(c) for c in range(0x7F)]
    mids = [(mags[i] + mags[i + 1]) / 2 for i in range(len(mags) - 1)]
    vals += [np.float32(m) for m in mids] + [np.float32(-m) for m in mids]
    vals = np.array(vals, np.float32)
    ref = torch_e4m3_encode(vals)
    for v, r in zip(vals, ref):
        assert oracle.e4m3_encode(float(v)) == r, float(v)


def test_e4m3_encode_saturates():
    for v in [448.0, 449.0, 463.9, 464.0, 480.0, 1e6, float("inf")]:
        assert oracle.e4m3_encode(v) == 0x7E
        assert oracle.e4m3_encode(-v) == 0xFE
    assert oracle.e4m3_encode(-0.0) == 0x80
    assert oracle.e4m3_encode(-1e-30) == 0x80  # rounds to zero, keeps sign


def test_e2m1_encode_matches_brute_force():
    g = np.random.default_rng(12)
    vals = list(g.uniform(-8, 8, 3000).astype(np.float32))
    grid = [float(x) for x in E2M1_GRID]
    vals += [np.float32((grid[i] + grid[i + 1]) / 2) for i in range(7)]
    vals += [np.float32(-(grid[i] + grid[i + 1]) / 2) for i in range(7)]
    vals += [np.float32(x) for x in grid] + [np.float32(7.0), np.float32(-0.0), np.float32(-0.1)]
    for v in vals:
        assert oracle.e2m1_encode(float(v)) == brute_e2m1(float(v)), float(v)


def test_e2m1_ties_to_even():
    expect = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for v, code in expect.items():
        assert oracle.e2m1_encode(v) == code
        assert oracle.e2m1_encode(-v) == (code | 8)


def test_bf16_encode_matches_torch_on_f32():
    g = np.random.default_rng(13)
    x = np.concatenate([g.standard_normal(5000).astype(np.float32),
                        (g.standard_normal(2000) * 1e-39).astype(np.float32),  # subnormals
                        np.array([1 + 2**-8, 1 + 3 * 2**-8, -(1 + 2**-8), 3.0e38], np.float32)])
    ref = bf16(x)
    for v, r in zip(x, ref):
        assert oracle.bf16_encode(float(v)) == r, float(v)


def test_bf16_encode_from_double_is_single_rounding():
    # 1 + 2^-8 + 2^-30: just above the midpoint of two BF16 neighbours; a
    # double -> float -> bf16 path would see the exact midpoint and go even.
    v = 1.0 + 2.0**-8 + 2.0**-30
    assert oracle.bf16_value(oracle.bf16_encode(v)) == 1.0 + 2.0**-7
    assert oracle.bf16_value(oracle.bf16_encode(1.0 + 2.0**-8)) == 1.0
    assert oracle.bf16_value(oracle.bf16_encode(-(1.0 + 2.0**-8 + 2.0**-30))) == -(1.0 + 2.0**-7)


# --------------------------------------------------------- hand examples ---

def _worked(kind):
    for line in open(os.path.join(GOLDEN, "worked_quant.txt")):
        line = line.strip()
        if line.startswith(kind + " "):
            fields = dict(f.split("=", 1) for f in line.split()[1:])
            yield fields


def test_nvfp4_worked_examples():
    n = 0
    for f in _worked("nvfp4"):
        x = np.array([float(v) for v in f["x"].split(",")], np.float32)
        assert np.all(f32(bf16(x)) == x)
        packed, sf = oracle.quant_nvfp4(bf16(x)[None, :], float(f["scale2"]))
        assert sf[0, 0] == int(f["sf"], 16)
        assert list(packed[0]) == [int(b, 16) for b in f["packed"].split(",")]
        n += 1
    assert n == 5


def test_rowfp8_worked_examples():
    n = 0
    for f in _worked("rowfp8"):
        x = np.array([float(v) for v in f["x"].split(",")], np.float32)
        q, s = oracle.quant_rowwise_fp8(bf16(x)[None, :])
        assert s[0] == float(f["s"])
        assert list(q[0]) == [int(b, 16) for b in f["q"].split(",")]
        n += 1
    assert n == 2


def test_int8_worked_examples():
    n = 0
    for f in _worked("int8"):
        x = np.array([float(v) for v in f["x"].split(",")], np.float32)
        q, s = oracle.quant_act_int8_per32(bf16(x)[None, :])
        assert s[0, 0] == float(f["s"])
        assert list(q[0]) == [int(v) for v in f["q"].split(",")]
        n += 1
    assert n == 2


# ------------------------------------------------------------ quantisers ---

def _decode_nvfp4(packed, sf, scale2):
    rows, k = packed.shape[0], packed.shape[1] * 2
    codes = np.empty((rows, k), np.uint8)
    codes[:, 0::2] = packed & 15
    codes[:, 1::2] = packed >> 4
    grid = np.array([E2M1[i] for i in range(16)])
    s = torch_e4m3_decode(sf).reshape(rows, k // 16)
    return codes, grid[codes] * np.repeat(s, 16, axis=1) * scale2


def test_nvfp4_exact_blocks_recovered():
    """Blocks whose values are e2m1 * s with amax = 6s (scale2 = 1) give the
    scale code of s and the codes back exactly (sign of zero included)."""
    g = np.random.default_rng(21)
    for sc in list(range(1, 0x7F)):
        s = oracle.e4m3_value(sc)
        codes = g.integers(0, 16, 16).astype(np.uint8)
        codes[g.integers(0, 16)] = 7 | (8 * g.integers(0, 2))
        vals = np.array([E2M1[c] for c in codes], np.float64) * s
        x = bf16(vals.astype(np.float32))
        assert np.all(f32(x) == vals)
        packed, sf = oracle.quant_nvfp4(x[None, :], 1.0)
        assert sf[0, 0] == sc
        got = np.empty(16, np.uint8)
        got[0::2], got[1::2] = packed[0] & 15, packed[0] >> 4
        assert np.array_equal(got, codes), (hex(sc), codes, got)


@pytest.mark.parametrize("scale2", [1.0, 0.25, 3.0e-4, 7.3e-6])
def test_nvfp4_brute_force_per_element(scale2):
    """Scale code = torch's RNE E4M3 of the FP32 quotient amax/(6*scale2)
    (saturated at 448); each element code = nearest E2M1 (exact rational
    search) of the FP32 quotient x/d, d = e4m3(sf)*scale2."""
    x = synth.student_t_bf16((8, 256), 4.0, 3, 1, outlier_frac=0.05)
    x = bf16(f32(x) * np.float32(scale2 * 40))
    packed, sf = oracle.quant_nvfp4(x, scale2)
    xf = f32(x).reshape(8, 16, 16)
    t = np.float32(6.0) * np.float32(scale2)
    amax = np.abs(xf).max(axis=2)
    q = (amax / t).astype(np.float32)
    exp_sf = np.where(q >= 448, 0x7E, torch_e4m3_encode(np.minimum(q, 448)))
    assert np.array_equal(sf.reshape(8, 16), exp_sf)
    codes = np.empty((8, 256), np.uint8)
    codes[:, 0::2], codes[:, 1::2] = packed & 15, packed >> 4
    sdec = torch_e4m3_decode(sf).reshape(8, 16)
    for r in range(8):
        for b in range(16):
            if sdec[r, b] == 0:
                assert np.all(codes[r, b * 16:(b + 1) * 16] == 0)
                continue
            d = np.float32(sdec[r, b]) * np.float32(scale2)
            for i in range(16):
                v = np.float32(xf[r, b, i]) / d
                assert codes[r, b * 16 + i] == brute_e2m1(float(v))


def test_nvfp4_forced_scale_sweep():
    """For every finite positive scale code c: a block whose amax is
    6*e4m3(c) (scale2 = 1) is given scale code c."""
    g = np.random.default_rng(22)
    for c in range(1, 0x7F):
        amax = 6.0 * oracle.e4m3_value(c)
        vals = g.uniform(-1, 1, 16) * amax
        vals[g.integers(0, 16)] = amax * (1 if g.integers(0, 2) else -1)
        x = bf16(vals.astype(np.float32))
        if np.abs(f32(x)).max() != amax:
            continue
        _, sf = oracle.quant_nvfp4(x[None, :], 1.0)
        assert sf[0, 0] == c


def test_nvfp4_requantise_idempotent():
    """Dequantise -> quantise reproduces codes and scales for blocks whose
    largest code is +-6 (scale2 a power of two, so every step is exact)."""
    for scale2 in [1.0, 2.0**-10]:
        x = synth.normal_bf16((16, 512), 1.0, 4, 2)
        x = bf16(f32(x) * np.float32(scale2 * 100))
        packed, sf = oracle.quant_nvfp4(x, scale2)
        codes, deq = _decode_nvfp4(packed, sf, scale2)
        x2 = bf16(deq.astype(np.float32))
        assert np.all(f32(x2) == deq)
        p2, sf2 = oracle.quant_nvfp4(x2, scale2)
        c2, _ = _decode_nvfp4(p2, sf2, scale2)
        blk_max = (codes & 7).reshape(16, 32, 16).max(axis=2)
        ok = blk_max == 7
        assert ok.mean() > 0.5
        assert np.array_equal(sf.reshape(16, 32)[ok], sf2.reshape(16, 32)[ok])
        cb, c2b = codes.reshape(16, 32, 16), c2.reshape(16, 32, 16)
        # a +0 element of the dequantised tensor comes back as +0 whatever its
        # original sign, so compare magnitudes and non-zero signs
        assert np.array_equal((cb & 7)[ok], (c2b & 7)[ok])
        nz = (cb[ok] & 7) != 0
        assert np.array_equal(cb[ok][nz], c2b[ok][nz])


def test_nvfp4_error_bound():
    """Every element lands within half a grid step of x/d (or saturates)."""
    x = synth.student_t_bf16((8, 512), 4.0, 5, 1, outlier_frac=0.02)
    packed, sf = oracle.quant_nvfp4(x, 1.0)
    codes, deq = _decode_nvfp4(packed, sf, 1.0)
    d = np.repeat(torch_e4m3_decode(sf).reshape(8, 32), 16, axis=1)
    xf = f32(x).astype(np.float64)
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    gap = np.array([.5, .5, .5, .5, 1, 1, 2, 2])  # spacing above each grid point
    mag = np.abs(xf / d)
    idx = (codes & 7).astype(np.int64)
    err = np.abs(mag - grid[idx])
    half = np.maximum(gap[idx], np.where(idx > 0, gap[np.maximum(idx - 1, 0)], 0.5)) / 2
    assert np.all((err <= half + 1e-6) | (mag >= 6))


def test_nvfp4_zero_and_weight_scale2():
    x = np.zeros((2, 32), np.uint16)
    packed, sf = oracle.quant_nvfp4(x, 1.0)
    assert not packed.any() and not sf.any()
    w = synth.normal_bf16((64, 256), 0.02, 0, 2)
    scale2 = oracle.amax_bf16(w) / (6.0 * 448.0)
    packed, sf = oracle.quant_nvfp4(w, np.float32(scale2))
    # the block holding the tensor's amax gets (about) the top scale 448
    assert torch_e4m3_decode(sf).max() >= 416


def _torch_amax(bits: np.ndarray) -> float:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy()).view(torch.bfloat16)
    return float(t.to(torch.float32).abs().max().item()) if t.numel() else 0.0


def test_amax_bf16_matches_torch_abs_max():
    """The weight scale2 of gemm_fp4.rs (weight_scale_2 = amax / (6*448))
    rests on amax = max |x| over the whole tensor.  Pinned two-sided against
    torch's BF16 decode + abs + max: the largest magnitude negative and in
    the last element (a missing abs or a skipped tail under-estimates it), a
    positive maximum at index 0, BF16 subnormals only, -0 and +0 only, a
    single element, and seeded random tensors of odd lengths."""
    g = np.random.default_rng(11)
    cases = []
    x = synth.normal_bf16((1, 1001), 1.0, 3, 9).ravel().copy()
    xf = f32(x)
    big = np.float32(-2.0 * np.abs(xf).max())
    x[-1] = bf16(big).reshape(-1)[0]
    cases.append((x, abs(float(big))))
    y = synth.normal_bf16((1, 777), 0.5, 4, 9).ravel().copy()
    y[0] = bf16(np.float32(9.5)).reshape(-1)[0]
    cases.append((y, 9.5))
    sub = (g.integers(1, 0x7F, 257).astype(np.uint16) | (g.integers(0, 2, 257).astype(np.uint16) << 15))
    cases.append((sub, None))
    cases.append((np.array([0x8000, 0x0000, 0x8000], np.uint16), 0.0))
    cases.append((bf16(np.float32([-3.25])).reshape(-1), 3.25))
    for n in (15, 16, 17, 4095):
        cases.append((synth.normal_bf16((1, n), 0.02, 5, n).ravel().copy(), None))
    for bits, expect in cases:
        got = oracle.amax_bf16(bits)
        ref = _torch_amax(bits)
        assert got == ref, (got, ref)
        if expect is not None:
            assert got == expect
    # the subnormal-only case is a real subnormal maximum, not a flush to 0
    assert oracle.amax_bf16(sub) > 0.0


def test_rowfp8_matches_torch_cast():
    x = synth.normal_bf16((16, 384), 0.02, 1, 4)
    q, s = oracle.quant_rowwise_fp8(x)
    xf = f32(x)
    amax = np.abs(xf).max(axis=1)
    assert np.array_equal(s, (amax / np.float32(448.0)).astype(np.float32))
    ref = torch_e4m3_encode(xf / s[:, None])
    assert np.array_equal(q, ref)
    # the amax element maps to +-448
    for r in range(16):
        i = int(np.argmax(np.abs(xf[r])))
        assert q[r, i] & 0x7F == 0x7E


def test_blockfp8_matches_torch_cast():
    x = synth.normal_bf16((256, 384), 0.02, 2, 8)
    q, S = oracle.quant_blockfp8(x)
    xf = f32(x)
    for bi in range(2):
        for bj in range(3):
            blk = xf[bi * 128:(bi + 1) * 128, bj * 128:(bj + 1) * 128]
            s = np.float32(np.abs(blk).max()) / np.float32(448.0)
            assert S[bi, bj] == s
            ref = torch_e4m3_encode(blk / s)
            assert np.array_equal(q[bi * 128:(bi + 1) * 128, bj * 128:(bj + 1) * 128], ref)


def test_int8_act_matches_numpy():
    x = synth.normal_outliers_bf16((8, 256), 1.0, 3, 5)
    q, s = oracle.quant_act_int8_per32(x)
    xf = f32(x).reshape(8, 8, 32)
    amax = np.abs(xf).max(axis=2)
    es = (amax / np.float32(127.0)).astype(np.float32)
    assert np.array_equal(s, es)
    eq = np.clip(np.rint(xf / es[..., None]), -127, 127).astype(np.int8)
    assert np.array_equal(q.reshape(8, 8, 32), eq)
    assert np.all(np.abs(q.reshape(8, 8, 32).astype(int)).max(axis=2) == 127)


def test_int8_zero_block():
    q, s = oracle.quant_act_int8_per32(np.zeros((1, 64), np.uint16))
    assert not q.any() and not s.any()


def test_requant_w_nvfp4_int8_matches_numpy():
    w = synth.normal_bf16((32, 512), 0.02, 4, 6)
    scale2 = np.float32(oracle.amax_bf16(w) / (6.0 * 448.0))
    packed, sf = oracle.quant_nvfp4(w, scale2)
    q, s = oracle.requant_w_nvfp4_int8(packed, sf, scale2)
    codes, _ = _decode_nvfp4(packed, sf, 1.0)
    grid = np.array([E2M1[i] for i in range(16)], np.float32)
    sdec = np.repeat(torch_e4m3_decode(sf).astype(np.float32).reshape(32, 32), 16, axis=1)
    v = (grid[codes] * sdec).astype(np.float32) * scale2
    v = v.astype(np.float32).reshape(32, 16, 32)
    amax = np.abs(v).max(axis=2)
    es = (amax / np.float32(127.0)).astype(np.float32)
    assert np.array_equal(s, es)
    with np.errstate(invalid="ignore", divide="ignore"):
        eq = np.where(es[..., None] == 0, 0, np.clip(np.rint(v / es[..., None]), -127, 127))
    assert np.array_equal(q.reshape(32, 16, 32), eq.astype(np.int8))


def test_requant_w_nvfp4_int8_pm6_blocks_are_pm127():
    """Two 16-halves sharing one scale with codes in {0, +-6} map to exactly
    +-127 and 0."""
    g = np.random.default_rng(23)
    codes = g.choice([0, 7, 15], size=(4, 64)).astype(np.uint8)
    codes[:, ::32] = 7
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    sf = np.full((4, 4), 0x3A, np.uint8)  # 1.25
    q, s = oracle.requant_w_nvfp4_int8(packed, sf, 0.5)
    exp = np.where(codes == 7, 127, np.where(codes == 15, -127, 0))
    assert np.array_equal(q.astype(int), exp)
    assert np.all(s == np.float32(6 * 1.25 * 0.5) / np.float32(127))


def test_blockfp8_to_rowwise_matches_torch():
    x = synth.normal_bf16((256, 256), 0.02, 5, 8)
    w, S = oracle.quant_blockfp8(x)
    q, s = oracle.requant_blockfp8_to_rowwise(w, S)
    deq = (torch_e4m3_decode(w).astype(np.float32) *
           np.repeat(np.repeat(S, 128, axis=0), 128, axis=1)).astype(np.float32)
    b = bf16(deq)  # the BF16 transient
    rq, rs = oracle.quant_rowwise_fp8(b)
    bf = f32(b)
    assert np.array_equal(rs, (np.abs(bf).max(axis=1) / np.float32(448)).astype(np.float32))
    assert np.array_equal(q, rq) and np.array_equal(s, rs)
    assert np.array_equal(q, torch_e4m3_encode(bf / rs[:, None]))


def test_blockfp8_to_rowwise_power_of_two_scales_is_identity():
    """Equal power-of-two block scales on a row whose amax code is +-448:
    the requant gives back the input codes and that scale."""
    g = np.random.default_rng(24)
    w = g.integers(0, 0x7F, size=(128, 256)).astype(np.uint8) | (g.integers(0, 2, size=(128, 256)) * 0x80).astype(np.uint8)
    w[:, 7] = 0x7E
    S = np.full((1, 2), 2.0**-9, np.float32)
    q, s = oracle.requant_blockfp8_to_rowwise(w, S)
    assert np.array_equal(q, w) and np.all(s == np.float32(2.0**-9))


# ---------------------------------------------------------------- products ---

def _pack(codes):
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


def test_w4a4_brute_force_all_code_pairs():
    """M=N=1, K=16, one non-zero element each: the product of every pair of
    the 16 x 16 codes, with scales, equals the golden-table product."""
    g = np.random.default_rng(31)
    for ca in range(16):
        for cw in range(16):
            pos = int(g.integers(0, 16))
            a = np.zeros((1, 16), np.uint8)
            w = np.zeros((1, 16), np.uint8)
            a[0, pos], w[0, pos] = ca, cw
            sfa, sfw = np.uint8(g.integers(0x20, 0x50)), np.uint8(g.integers(0x20, 0x50))
            sa2, sb2 = 1.0, 0.5
            _, ex, _ = oracle.w4a4_gemm(_pack(a), np.array([[sfa]]), _pack(w), np.array([[sfw]]), sa2, sb2)
            want = (E2M1[ca] * torch_e4m3_decode([sfa])[0] * E2M1[cw] * torch_e4m3_decode([sfw])[0] * sa2 * sb2)
            assert ex[0, 0] == want


def test_w4a4_unit_scales_is_integer_matmul():
    g = np.random.default_rng(32)
    a = g.integers(0, 16, size=(5, 64)).astype(np.uint8)
    w = g.integers(0, 16, size=(7, 64)).astype(np.uint8)
    ones_a = np.full((5, 4), 0x38, np.uint8)
    ones_w = np.full((7, 4), 0x38, np.uint8)
    grid = np.array([E2M1[i] for i in range(16)])
    _, ex, ab = oracle.w4a4_gemm(_pack(a), ones_a, _pack(w), ones_w, 1.0, 1.0)
    assert np.array_equal(ex, grid[a] @ grid[w].T)
    assert np.array_equal(ab, np.abs(grid[a]) @ np.abs(grid[w]).T)


def test_w4a4_nibble_order_one_hot():
    """Element 1 (high nibble of byte 0) of A multiplies element 1 of W."""
    a = np.zeros((1, 32), np.uint8)
    a[0, 1] = 2  # 1.0
    w = np.zeros((2, 32), np.uint8)
    w[0, 0] = 7  # 6.0 at element 0
    w[1, 1] = 5  # 3.0 at element 1
    s = np.full((1, 2), 0x38, np.uint8)
    _, ex, _ = oracle.w4a4_gemm(_pack(a), s, _pack(w), np.full((2, 2), 0x38, np.uint8), 1.0, 1.0)
    assert list(ex[0]) == [0.0, 3.0]


def test_w4a4_random_matches_float64_matmul():
    a_bf, w_bf = synth.w4a4_inputs(16, 48, 512, seed=0)
    sa2 = 1.0
    sb2 = np.float32(oracle.amax_bf16(w_bf) / (6 * 448))
    ap, asf = oracle.quant_nvfp4(a_bf, sa2)
    wp, wsf = oracle.quant_nvfp4(w_bf, sb2)
    _, adq = _decode_nvfp4(ap, asf, 1.0)
    _, wdq = _decode_nvfp4(wp, wsf, 1.0)
    ob, ex, ab = oracle.w4a4_gemm(ap, asf, wp, wsf, sa2, sb2)
    ref = (adq @ wdq.T) * float(sa2) * float(sb2)
    assert np.allclose(ex, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    assert np.allclose(ab, (np.abs(adq) @ np.abs(wdq).T) * float(sa2) * float(sb2), rtol=1e-12)
    # the BF16 output is torch's RNE cast of the exact value (exact values
    # here are FP32-representable up to rounding far below BF16's step)
    assert np.mean(ob == bf16(ex.astype(np.float32))) > 0.999
    # quantisation error of the whole layer stays small against the BF16 inputs
    ref_bf = f32(a_bf).astype(np.float64) @ f32(w_bf).astype(np.float64).T
    rel = np.linalg.norm(ex - ref_bf) / np.linalg.norm(ref_bf)
    assert rel < 0.2


def test_w4a4_row_subset():
    a_bf, w_bf = synth.w4a4_inputs(8, 16, 256, seed=1)
    ap, asf = oracle.quant_nvfp4(a_bf, 1.0)
    wp, wsf = oracle.quant_nvfp4(w_bf, 0.001)
    full = oracle.w4a4_gemm(ap, asf, wp, wsf, 1.0, 0.001)
    sub = oracle.w4a4_gemm(ap, asf, wp, wsf, 1.0, 0.001, rows=np.array([5, 2]))
    for f, s in zip(full, sub):
        assert np.array_equal(f[[5, 2]], s)


def test_fp8_gemv_matches_float64_and_identity():
    inp, w_bf = synth.gemv_inputs(16, 40, 256, seed=0)
    wq, ws = oracle.quant_rowwise_fp8(w_bf)
    ob, ex, ab = oracle.fp8_gemv_rowscale(inp, wq, ws)
    ref = (f32(inp).astype(np.float64) @ torch_e4m3_decode(wq).reshape(40, 256).T) * ws.astype(np.float64)
    assert np.allclose(ex, ref, rtol=1e-12, atol=1e-15)
    # one-hot rows with unit scale: output = input (BF16-exact already)
    eye = np.zeros((256, 256), np.uint8)
    eye[np.arange(256), np.arange(256)] = 0x38
    ob, ex, _ = oracle.fp8_gemv_rowscale(inp, eye, np.ones(256, np.float32))
    assert np.array_equal(ob, inp)
    # a row's result does not depend on the batch it is computed in
    ob1, _, _ = oracle.fp8_gemv_rowscale(inp[3:4], wq, ws)
    ob16, _, _ = oracle.fp8_gemv_rowscale(inp, wq, ws)
    assert np.array_equal(ob1[0], ob16[3])


def _e4m3_tab():
    return np.array([oracle.e4m3_value(c) for c in range(256)])


def test_fp8_gemv_blockscaled_matches_float64_blocks():
    """Block scales: each 128 x 128 weight block's products carry that
    block's scale (fp8_gemv_batch.rs, `w8a16_gemv_batch4`).  Checked against
    an independent float64 sum built block by block, with distinct scales
    per row block and per K block, so a swapped or dropped index fails."""
    m, n, k = 3, 256, 384
    inp = synth.normal_bf16((m, k), 1.0, 0, 21)
    w = synth.uniform_bytes((n, k), 21, 2, 0x00, 0x7F)  # finite E4M3 codes
    S = np.array([[0.5, 2.0, 0.125], [3.0, 0.25, 1.5]], np.float32)
    ob, ex, ab = oracle.fp8_gemv_blockscaled(inp, w, S)
    x = (inp.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    wv = _e4m3_tab()[w]
    ref = np.zeros((m, n))
    for nb in range(2):
        for kb in range(3):
            ref[:, nb * 128:(nb + 1) * 128] += S[nb, kb] * (
                x[:, kb * 128:(kb + 1) * 128] @ wv[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128].T)
    assert np.allclose(ex, ref, rtol=1e-12, atol=1e-12)
    assert np.array_equal(ob, np.array([[oracle.bf16_encode(v) for v in row] for row in ref], np.uint16))
    assert np.all(ab >= np.abs(ex) - 1e-9)


def test_fp8_gemv_blockscaled_uniform_scale_is_rowscale():
    """With one scale per 128-row block and no change along K, the block
    form reduces to the row-scaled GEMV with those row scales."""
    m, n, k = 2, 256, 256
    inp = synth.normal_bf16((m, k), 1.0, 0, 22)
    w = synth.uniform_bytes((n, k), 22, 2, 0x00, 0x7F)
    S = np.array([[0.75, 0.75], [4.0, 4.0]], np.float32)
    _, ex_b, _ = oracle.fp8_gemv_blockscaled(inp, w, S)
    rs = np.repeat(S[:, 0], 128).astype(np.float32)
    _, ex_r, _ = oracle.fp8_gemv_rowscale(inp, w, rs)
    assert np.allclose(ex_b, ex_r, rtol=1e-12, atol=1e-12)


def test_int8_gemm_matches_integer_blocks():
    g = np.random.default_rng(33)
    a = g.integers(-127, 128, size=(6, 128)).astype(np.int8)
    w = g.integers(-127, 128, size=(9, 128)).astype(np.int8)
    sa = g.uniform(0.01, 1, size=(6, 4)).astype(np.float32)
    sw = g.uniform(0.01, 1, size=(9, 4)).astype(np.float32)
    _, ex, ab = oracle.int8_blockscaled_gemm(a, w, sa, sw)
    ref = np.zeros((6, 9))
    refab = np.zeros((6, 9))
    for b in range(4):
        p = a[:, b * 32:(b + 1) * 32].astype(np.int64) @ w[:, b * 32:(b + 1) * 32].astype(np.int64).T
        pa = np.abs(a[:, b * 32:(b + 1) * 32].astype(np.int64)) @ np.abs(w[:, b * 32:(b + 1) * 32].astype(np.int64)).T
        s = sa[:, b:b + 1].astype(np.float64) * sw[:, b].astype(np.float64)[None, :]
        ref += p * s
        refab += pa * s
    assert np.allclose(ex, ref, rtol=1e-13) and np.allclose(ab, refab, rtol=1e-13)


def test_fp8_gemm_rowscale_matches_float64():
    g = np.random.default_rng(34)
    a = g.integers(0, 0x7F, size=(5, 96)).astype(np.uint8) | (g.integers(0, 2, (5, 96)) * 0x80).astype(np.uint8)
    w = g.integers(0, 0x7F, size=(7, 96)).astype(np.uint8)
    sa = g.uniform(0.001, 0.1, 5).astype(np.float32)
    sw = g.uniform(0.001, 0.1, 7).astype(np.float32)
    _, ex, _ = oracle.fp8_gemm_rowscale(a, sa, w, sw)
    ref = (torch_e4m3_decode(a).reshape(5, 96) @ torch_e4m3_decode(w).reshape(7, 96).T)
    ref = ref * sa[:, None].astype(np.float64) * sw[None, :].astype(np.float64)
    assert np.allclose(ex, ref, rtol=1e-12)


def test_tolerance_helper_rejects_planted_error():
    """The tolerance of the parity tests catches a dropped K block."""
    a_bf, w_bf = synth.w4a4_inputs(8, 32, 512, seed=2)
    ap, asf = oracle.quant_nvfp4(a_bf, 1.0)
    wp, wsf = oracle.quant_nvfp4(w_bf, 0.0001)
    ob, ex, ab = oracle.w4a4_gemm(ap, asf, wp, wsf, 1.0, 0.0001)
    ap2 = ap.copy()
    ap2[:, 0:8] = 0  # drop the first 16-block of K
    ob2, _, _ = oracle.w4a4_gemm(ap2, asf, wp, wsf, 1.0, 0.0001)
    tol = oracle.tolerance(ob, ab)
    diff = np.abs(oracle.bf16_to_f32(ob2).astype(np.float64) - oracle.bf16_to_f32(ob))
    assert np.any(diff > tol)
