"""The NVFP4 quantiser's division-free E2M1 rule for short divisors, checked
exhaustively on the host.

For a divisor d with at most 6 significant bits the kernels find the E2M1
code of RN(x / d) (round to nearest even, saturating at 6; the element code
definition of the NVFP4 recipe) without dividing: p = RN(x * r) with r the
hardware reciprocal estimate of d, m = p rounded to a multiple of 1/4 by
adding and subtracting 3 * 2^20, and the FMA residual e = x - m * d; the code
is that of m when e is +0 and that of p otherwise.  This test replays those
FP32 steps in numpy for every finite BF16 x, every E4M3 scale and several
scale2 values, with r anywhere within one ulp of 1/d (the estimate's error
bound), and compares with the code of the exact quotient."""
import numpy as np

MAGS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_exact(q64):
    """E2M1 code (sign in bit 3) of a float64 value, ties to the even code,
    saturating at 6."""
    a = np.abs(q64)
    hi = np.clip(np.searchsorted(MAGS, a), 0, 7)
    lo = np.clip(hi - 1, 0, 7)
    dlo, dhi = a - MAGS[lo], MAGS[hi] - a
    pick = np.where(dlo < dhi, lo, np.where(dhi < dlo, hi, np.where(lo % 2 == 0, lo, hi)))
    pick = np.where(a >= 6, 7, pick)
    return (pick | (np.signbit(q64).astype(np.int64) << 3)).astype(np.uint8)


def snap_rule(x, d, r):
    c = np.float32(3 * 2 ** 20)
    with np.errstate(over="ignore", invalid="ignore"):
        p = (x * r).astype(np.float32)
        m = ((p + c).astype(np.float32) - c).astype(np.float32)
        # one FMA: m * d is exact here, so the float64 difference is exact
        # before its single rounding to FP32
        e = (x.astype(np.float64) - m.astype(np.float64) * np.float64(d)).astype(np.float32)
    q = np.where(e.view(np.uint32) == 0, m, p)
    return e2m1_exact(q.astype(np.float64))


def e4m3_value(code):
    e, mant = (code >> 3) & 15, code & 7
    return mant / 8 * 2.0 ** -6 if e == 0 else (1 + mant / 8) * 2.0 ** (e - 7)


def test_snap_rule_matches_exact_quotient_for_every_bf16():
    bits = np.arange(65536, dtype=np.uint32) << 16
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    checked = 0
    for scale2 in (1.0, 0.5, 2.0 ** -20, 1.5, 3 * 2.0 ** -10):
        for code in range(1, 127):
            d = np.float32(np.float32(e4m3_value(code)) * np.float32(scale2))
            if (int(d.view(np.uint32)) & ((1 << 18) - 1)) or not (2.0 ** -60 <= d <= 2.0 ** 60):
                continue  # the rule's domain: at most 6 significant bits
            ref = e2m1_exact(x.astype(np.float64) / np.float64(d))
            r0 = np.float32(1.0) / d
            for ulps in (-1, 0, 1):
                r = (r0.view(np.uint32) + np.uint32(ulps) if ulps >= 0 else r0.view(np.uint32) - np.uint32(1))
                got = snap_rule(x, d, r.view(np.float32))
                bad = np.flatnonzero(got != ref)
                assert bad.size == 0, (scale2, code, ulps, x[bad[:4]], got[bad[:4]], ref[bad[:4]])
            checked += 1
    assert checked > 400


def test_snap_rule_needs_the_residual():
    """Without the residual test (codes of p alone) exact ties go wrong: the
    check above is not vacuous."""
    d = np.float32(1.125)  # 1/d is inexact
    x = np.array([0.25 * 1.125 * 2 ** k for k in range(-1, 3)] + [5 * 1.125], np.float32)
    r = np.float32(1.0) / d
    ref = e2m1_exact(x.astype(np.float64) / np.float64(d))
    wrong = 0
    for ulps in (-1, 1):
        rr = (r.view(np.uint32) + np.uint32(1) if ulps > 0 else r.view(np.uint32) - np.uint32(1)).view(np.float32)
        p = (x * rr).astype(np.float32)
        wrong += int(np.sum(e2m1_exact(p.astype(np.float64)) != ref))
        assert np.array_equal(snap_rule(x, d, rr), ref)
    assert wrong > 0
