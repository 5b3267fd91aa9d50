// Device code of the division-free quantisers, shared by the quantiser
// kernels (quant.cu) and the fused quantise + W4A4 GEMM (gemm_w4a4.cu): the
// codes of correctly rounded FP32 quotients found without dividing, and the
// NVFP4 quantisation of one 16-element block.  sm_100a only.
#pragma once

#include "bsq_common.cuh"

namespace bsq {
namespace qc {

__device__ __forceinline__ uint4 ld_nc_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Largest magnitude (as BF16 bits, sign cleared) of 8 packed BF16 values.
// For finite values the unsigned order of the magnitude bits is the order
// of the magnitudes.
__device__ __forceinline__ uint32_t amax_bits_8(const uint4 &v) {
    uint32_t a = __vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu);
    uint32_t b = __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu);
    uint32_t m = __vmaxu2(a, b);
    return max(m & 0xFFFFu, m >> 16);
}

__device__ __forceinline__ float lo_bf16(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_bf16(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint8_t f32_to_e4m3(float x) {
    return static_cast<uint8_t>(f32x2_to_e4m3x2(x, 0.0f) & 0xFF);
}

// Two E2M1 codes (one byte, element 2j in the low nibble) -> two FP32.
__device__ __forceinline__ float2 e2m1x2_to_f32x2(uint32_t byte) {
    uint32_t h2;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.u8.u32 t, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
        : "=r"(h2)
        : "r"(byte));
    __half2 h = *reinterpret_cast<__half2 *>(&h2);
    return __half22float2(h);
}

// Two E4M3 codes (low byte first) -> two FP32 (exact: every E4M3 value is an
// FP16 value).
__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint32_t pair) {
    uint32_t h2;
    asm("{\n\t.reg .b16 t;\n\t"
        "cvt.u16.u32 t, %1;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
        : "=r"(h2)
        : "r"(pair));
    __half2 h = *reinterpret_cast<__half2 *>(&h2);
    return __half22float2(h);
}

// ---------------------------------------------------------------------------
// Codes of RN(x / d) without a division.
//
// Every code map used here (nearest E2M1 and nearest E4M3 with saturation,
// nearest integer clamped to +-127; ties to even) is monotone in its FP32
// argument and gives one code per value.  For d in [2^-60, 2^60] let r be
// rcp.approx(d) (within 2^-23 of 1/d, relative), rl = RN(r (1 - 2^-16)) and
// rh = RN(r (1 + 2^-16)).  Then RN(x rl) and RN(x rh) lie 2^-16 +- 2^-22 of
// x/d away from it (relative), on opposite sides, while RN(x/d) is within
// 2^-24 of it: RN(x/d) lies between the two products.  Quotients below
// 2^-126, where relative bounds fail, round to a signed zero code in every
// map, and so do the products then.  Hence:
//   * both products give the same code: it is the code of RN(x/d);
//   * they give two codes, necessarily adjacent (the bracket is far narrower
//     than any gap between code boundaries).  The boundary m between them
//     has few significant bits (3 for E2M1, 5 for E4M3; a half-integer for
//     int8) and lies within 2^-15 of the products, so rounding a product to
//     that many bits recovers it.  Then rho = x - m d is exact in one FMA
//     (x and m d agree to 15 bits and their lowest bits lie no further
//     apart than 24 bits), and (m of at most 8 bits) RN(x/d) = m exactly
//     when |x|/d - |m| lies in [-h_in, h_out], h_out half an ulp of |m| and
//     h_in the same except a quarter ulp where |m| is a power of two.  In
//     that case the code map breaks the tie at m itself; otherwise the sign
//     of rho picks the code above or below m.  All comparisons are exact:
//     h d is a power-of-two multiple of d, normal in this range of d.
// So the code of the correctly rounded quotient is found without dividing.
//
// Divisors with few significant bits need no bracket (see `snapped`).
struct Bracket {
    float r, lo, hi;
    bool ok;
};

__device__ __forceinline__ Bracket bracket_of(float d) {
    Bracket b;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(b.r) : "f"(d));
    b.ok = d >= 0x1p-60f && d <= 0x1p60f;
    b.lo = __fmul_rn(b.r, 1.0f - 0x1p-16f);
    b.hi = __fmul_rn(b.r, 1.0f + 0x1p-16f);
    return b;
}

// p rounded to B significant bits (round half up on the magnitude).
template <int B>
__device__ __forceinline__ float round_to_bits(float p) {
    constexpr uint32_t half = 1u << (23 - B);
    return __uint_as_float((__float_as_uint(p) + half) & ~(2u * half - 1u));
}

// Divisors with few significant bits.  Let x be BF16 (8 significant bits),
// d have at most SB significant bits and every code boundary at most MB, with
// SB + MB <= 9.  For x near 2^e and any MB-bit m with m d near x, x - m d is
// a multiple of 2^(e-9), so x/d either equals m or lies at least 2^-10
// (relative) from it.  p = RN(x r), r = rcp.approx(d), is within 2^-22 of
// x/d.  So when p lies within 2^-12 of its rounding m to MB bits, x/d = m
// exactly and RN(x/d) = m (the code map then breaks a tie at m itself);
// otherwise no MB-bit number, and so no boundary, lies between p and
// RN(x/d), and p has the code of RN(x/d).  is_short<SB> tests the bits of d.
template <int MB>
__device__ __forceinline__ float snapped(float p) {
    const float m = round_to_bits<MB>(p);
    const uint32_t ulps = __float_as_uint(p) - __float_as_uint(m) + 2048u;  // p, m share a sign
    return ulps <= 4096u ? m : p;
}

template <int bits>
__device__ __forceinline__ bool is_short(float d) {
    return (__float_as_uint(d) & ((1u << (24 - bits)) - 1u)) == 0u;
}

// The half-integer nearest p (|p| < 2^21).
__device__ __forceinline__ float nearest_half_integer(float p) {
    const float a = __fadd_rn(__fadd_rn(__fadd_rn(fabsf(p), -0.5f), 12582912.0f), -12582912.0f);
    return copysignf(__fadd_rn(a, 0.5f), p);
}

// A value whose code is the code of RN(x/d), for x/d next to the code
// boundary m (see above).
__device__ __forceinline__ float boundary_resolved(float x, float d, float m) {
    const float rho = __fmaf_rn(-m, d, x);
    if (rho == 0.0f) return m;  // x/d = m exactly
    const uint32_t mb = __float_as_uint(m) & 0x7FFFFFFFu;
    const float h_out = __fmul_rn(__uint_as_float(mb & 0x7F800000u), 0x1p-24f);
    const float h_in = (mb & 0x7FFFFFu) ? h_out : __fmul_rn(h_out, 0.5f);
    const float a = x < 0.0f ? -rho : rho;  // sign of |x|/d - |m|
    if (a <= __fmul_rn(h_out, d) && a >= -__fmul_rn(h_in, d)) return m;
    return __fmul_rn(m, a > 0.0f ? 1.0f + 0x1p-10f : 1.0f - 0x1p-10f);
}

// Codes (E2M1 or E4M3, by B) of a pair of quotients from their bracket ends:
// p0, p1 the low-end products, lo/hi the code pairs of the two ends (FMT
// bits per code).
template <int B, int FMT>
__device__ __forceinline__ void pair_boundaries(float x0, float x1, float d, float &p0, float &p1, uint32_t lo,
                                                uint32_t hi) {
    constexpr uint32_t mask = (1u << FMT) - 1u;
    if ((lo ^ hi) & mask) p0 = boundary_resolved(x0, d, round_to_bits<B>(p0));
    if ((lo ^ hi) >> FMT) p1 = boundary_resolved(x1, d, round_to_bits<B>(p1));
}

// E4M3 code of RN(x / d) for a BF16 x (the NVFP4 block scale).
__device__ __forceinline__ uint8_t e4m3_of_quotient(float x, float d, const Bracket &br) {
    if (!br.ok) return f32_to_e4m3(__fdiv_rn(x, d));
    if (is_short<4>(d)) return f32_to_e4m3(snapped<5>(__fmul_rn(x, br.r)));
    const float pl = __fmul_rn(x, br.lo), ph = __fmul_rn(x, br.hi);
    const uint32_t b2 = f32x2_to_e4m3x2(pl, ph);
    if ((b2 & 0xFFu) == (b2 >> 8)) return (uint8_t)(b2 & 0xFFu);
    return f32_to_e4m3(boundary_resolved(x, d, round_to_bits<5>(pl)));
}

__device__ __forceinline__ uint64_t f32x2_pack(float lo, float hi) {
    return (uint64_t)__float_as_uint(lo) | ((uint64_t)__float_as_uint(hi) << 32);
}

// E2M1 codes (one byte, element 0 in the low nibble) of RN(x0 / d) and
// RN(x1 / d) for the BF16 pair w and a divisor d of at most 6 significant
// bits, given rr = (r, r) for r = rcp.approx(d) and nd = (-d, -d).
// Every E2M1 code boundary (1/4, 3/4, 5/4, 7/4, 5/2, 7/2, 5) is a multiple
// of 1/4 below 8.  Let p = RN(x r), within 2^-22 of x/d, and m = p rounded
// to a multiple of 1/4 (adding and subtracting 3 * 2^20, exact for
// |p| < 2^21).  The FMA residual x - m d is exact whenever it is zero, and
// it is +0 exactly when x = m d with x non-zero or x = +0 (-0 gives -0):
//   * x/d a non-zero multiple of 1/4: then m = x/d, the residual is +0 and
//     m is the quotient itself (the code map breaks a tie at m);
//   * otherwise x/d is no code boundary and, by the argument given for
//     `snapped` (8-bit x, 6-bit d, 3-bit boundaries), lies at least 2^-10
//     (relative) from every boundary, so p has its code; the residual is
//     non-zero or -0 (x = -0, p = -0), and p is kept.
// An infinite p gives a NaN residual and keeps p.  The arithmetic is packed
// FP32 pairs, leaving the integer pipe to the selects and the packing.
__device__ __forceinline__ uint32_t e2m1x2_short(uint32_t w, uint64_t rr, uint64_t nd) {
    const uint64_t xx = f32x2_pack(lo_bf16(w), hi_bf16(w));
    const uint64_t cc = f32x2_pack(3145728.0f, 3145728.0f), ncc = f32x2_pack(-3145728.0f, -3145728.0f);
    uint64_t pp, mm, ee;
    asm("mul.rn.f32x2 %0, %3, %4;\n\t"
        "add.rn.f32x2 %1, %0, %5;\n\t"
        "add.rn.f32x2 %1, %1, %6;\n\t"
        "fma.rn.f32x2 %2, %1, %7, %3;"
        : "=&l"(pp), "=&l"(mm), "=l"(ee)
        : "l"(xx), "l"(rr), "l"(cc), "l"(ncc), "l"(nd));
    const uint32_t e0 = (uint32_t)ee, e1 = (uint32_t)(ee >> 32);
    const float q0 = __uint_as_float(e0 == 0u ? (uint32_t)mm : (uint32_t)pp);
    const float q1 = __uint_as_float(e1 == 0u ? (uint32_t)(mm >> 32) : (uint32_t)(pp >> 32));
    return f32x2_to_e2m1x2(q0, q1);
}

// Eight x / d quotients (packed BF16 x) -> eight E2M1 nibbles in one 32-bit
// word, element 0 in the lowest nibble.
__device__ __forceinline__ uint32_t nvfp4_codes_8(const uint4 &v, float d, const Bracket &br) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t out = 0;
    if (br.ok && is_short<6>(d)) {
        const uint64_t rr = f32x2_pack(br.r, br.r), nd = f32x2_pack(-d, -d);
#pragma unroll
        for (int j = 0; j < 4; j++) out |= e2m1x2_short(w[j], rr, nd) << (8 * j);
        return out;
    }
    if (br.ok) {
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const float e0 = lo_bf16(w[j]), e1 = hi_bf16(w[j]);
            float p0 = __fmul_rn(e0, br.lo), p1 = __fmul_rn(e1, br.lo);
            uint32_t lo = f32x2_to_e2m1x2(p0, p1);
            const uint32_t hi = f32x2_to_e2m1x2(__fmul_rn(e0, br.hi), __fmul_rn(e1, br.hi));
            if (lo != hi) {
                pair_boundaries<3, 4>(e0, e1, d, p0, p1, lo, hi);
                lo = f32x2_to_e2m1x2(p0, p1);
            }
            out |= lo << (8 * j);
        }
        return out;
    }
#pragma unroll
    for (int j = 0; j < 4; j++) {
        float lo = __fdiv_rn(lo_bf16(w[j]), d);
        float hi = __fdiv_rn(hi_bf16(w[j]), d);
        out |= f32x2_to_e2m1x2(lo, hi) << (8 * j);
    }
    return out;
}

// The NVFP4 quantisation of one 16-element block (gemm_fp4.rs,
// `quantize_bf16_to_nvfp4`): v0, v1 hold its 16 BF16 values; t6 = 6 * scale2
// (and t6b its bracket).  sc = E4M3(amax / t6) (RNE, satfinite; 0 for an
// all-zero block or when zero_all), codes = E2M1(x / (e4m3(sc) * scale2))
// packed two per byte, element 2j in the low nibble.
__device__ __forceinline__ void nvfp4_block(const uint4 &v0, const uint4 &v1, float scale2, float t6,
                                            const Bracket &t6b, bool zero_all, uint2 &codes, uint8_t &sc) {
    const uint32_t mx = max(amax_bits_8(v0), amax_bits_8(v1));
    sc = (mx == 0 || zero_all) ? (uint8_t)0 : e4m3_of_quotient(__uint_as_float(mx << 16), t6, t6b);
    const float sfv = e4m3_to_f32(sc);
    codes = make_uint2(0u, 0u);
    if (sfv != 0.0f) {
        const float d = __fmul_rn(sfv, scale2);
        const Bracket br = bracket_of(d);
        codes.x = nvfp4_codes_8(v0, d, br);
        codes.y = nvfp4_codes_8(v1, d, br);
    }
}

}  // namespace qc
}  // namespace bsq
