// Quantisers and requantisers of libbsq (all HBM-bound, one pass over the
// input, 16-byte vector loads, packed stores).
//
//   NVFP4           gemm_fp4.rs, `quantize_bf16_to_nvfp4`
//   row-wise FP8    quantize_fns.rs, `quantize_to_fp8`; dispatch_proj_rowwise.rs,
//                   `quant_rowwise_fp8`
//   block FP8       the block-scaled weight format of dispatch_proj_rowwise.rs
//   block -> row    dispatch_proj_rowwise.rs, `requant_weight_rowwise_fp8_cached`
//                   (dequant + row quant fused; the BF16 transient stays in
//                   registers)
//   NVFP4 -> int8   gemm_dense_int8.rs, `requant_w_nvfp4_int8`
//   BF16 -> int8    gemm_dense_int8.rs, `int8_gemm_faith2_prefill` step (a)
//
// Every pinned FP32 step uses an explicit round-to-nearest intrinsic so the
// compiler cannot contract or reorder it.  The per-element quotients x / d
// are not divided out one by one: a bracket of two products decides the code
// and the exact division runs only where the bracket straddles a rounding
// boundary (see `Bracket`).
#include <cfloat>

#include "quant_codes.cuh"

namespace bsq {

namespace {

using namespace qc;

// Grid-stride quantisers take this many independent units per thread and
// pass, so several loads per thread are in flight at once.
constexpr int kQuantUnroll = 2;

// Flags of this file's kernels, read and cleared by take_timeouts_quant: bit
// 0, a bounded wait of the bulk-copy requant ran out; bit 1, the device-
// scale2 NVFP4 quantiser met an amax whose scale2 the host form rejects.
static __device__ unsigned int g_quant_timeouts;

// One thread per 16-element block: two 16-byte loads, the block amax in
// registers, eight code bytes and one scale byte stored.
__global__ void __launch_bounds__(256) k_quant_nvfp4(const uint4 *__restrict__ in, uint2 *__restrict__ packed,
                                                     uint8_t *__restrict__ sf, float scale2, float t6,
                                                     const float *__restrict__ amax_dev,
                                                     float *__restrict__ scale2_out, int64_t nblocks) {
    // a GEMM launched after this kernel with programmatic stream
    // serialization may start its prologue now; it reads these outputs only
    // after griddepcontrol.wait, i.e. after this grid has completed
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    bool zero_all = false;
    if (amax_dev != nullptr) {
        // the weight's scale2 from its device amax, the same FP32 steps as
        // on the host: scale2 = amax / (6 * 448), t6 = 6 * scale2
        const float amax = __ldg(amax_dev);
        scale2 = __fdiv_rn(amax, 2688.0f);
        // The host form accepts only a finite scale2 >= FLT_MIN.  A scale2 it
        // would reject (an amax that is NaN, infinite, or below 2688 *
        // FLT_MIN but not 0) gives what an all-zero tensor gives -- scale2
        // 0, every scale and code 0 -- and sets flag bit 1.
        if (amax != 0.0f && !(scale2 >= FLT_MIN && scale2 <= FLT_MAX)) {
            zero_all = true;
            scale2 = 0.0f;
            if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(&g_quant_timeouts, 2u);
        }
        t6 = __fmul_rn(6.0f, scale2);
        if (scale2_out != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *scale2_out = scale2;
    }
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const Bracket t6b = bracket_of(t6);
    // kQuantUnroll blocks per thread and pass, all loads issued first
    for (int64_t b0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b0 < nblocks; b0 += kQuantUnroll * stride) {
        uint4 v[kQuantUnroll][2];
#pragma unroll
        for (int u = 0; u < kQuantUnroll; u++) {
            const int64_t b = b0 + u * stride;
            v[u][0] = v[u][1] = make_uint4(0u, 0u, 0u, 0u);
            if (b < nblocks) {
                v[u][0] = ld_nc_v4(in + 2 * b);
                v[u][1] = ld_nc_v4(in + 2 * b + 1);
            }
        }
#pragma unroll
        for (int u = 0; u < kQuantUnroll; u++) {
            const int64_t b = b0 + u * stride;
            if (b >= nblocks) break;
            // an all-zero block has scale code 0 (also when scale2 is 0: an
            // all-zero tensor's device amax)
            uint2 codes;
            uint8_t sc;
            nvfp4_block(v[u][0], v[u][1], scale2, t6, t6b, zero_all, codes, sc);
            packed[b] = codes;
            sf[b] = sc;
        }
    }
}

// ---------------------------------------------------------------------------
// Block-wide max of a non-negative value held as float bits.
template <int NT>
__device__ __forceinline__ uint32_t block_max_u32(uint32_t v, uint32_t *red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < NT / 32 ? red[lane] : 0u;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
        if (lane == 0) red[0] = v;
    }
    __syncthreads();
    v = red[0];
    __syncthreads();
    return v;
}

// Eight E4M3 codes of x / s (RNE, satfinite) packed little-endian; `br` is
// bracket_of(s).
__device__ __forceinline__ uint2 e4m3_codes_8(const float (&x)[8], float s, const Bracket &br) {
    uint32_t w[4];
    if (br.ok) {
#pragma unroll
        for (int j = 0; j < 4; j++) {
            float p0 = __fmul_rn(x[2 * j], br.lo), p1 = __fmul_rn(x[2 * j + 1], br.lo);
            w[j] = f32x2_to_e4m3x2(p0, p1);
            const uint32_t hi = f32x2_to_e4m3x2(__fmul_rn(x[2 * j], br.hi), __fmul_rn(x[2 * j + 1], br.hi));
            if (w[j] != hi) {
                pair_boundaries<5, 8>(x[2 * j], x[2 * j + 1], s, p0, p1, w[j], hi);
                w[j] = f32x2_to_e4m3x2(p0, p1);
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < 4; j++) w[j] = f32x2_to_e4m3x2(__fdiv_rn(x[2 * j], s), __fdiv_rn(x[2 * j + 1], s));
    }
    return make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
}

__device__ __forceinline__ void unpack_bf16_8(const uint4 &v, float (&x)[8]) {
    x[0] = lo_bf16(v.x); x[1] = hi_bf16(v.x); x[2] = lo_bf16(v.y); x[3] = hi_bf16(v.y);
    x[4] = lo_bf16(v.z); x[5] = hi_bf16(v.z); x[6] = lo_bf16(v.w); x[7] = hi_bf16(v.w);
}

__device__ __forceinline__ uint2 row_codes_8(const uint4 &v, float s, const Bracket &br) {
    if (s == 0.0f) return make_uint2(0, 0);
    float f[8];
    unpack_bf16_8(v, f);
    return e4m3_codes_8(f, s, br);
}

__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

// Max over the CTA of a non-negative value held as float bits; one barrier
// (the CTA handles a single row, so `red` is not reused).
template <int NT>
__device__ __forceinline__ uint32_t cta_max_once(uint32_t v, uint32_t *red) {
    v = warp_max_u32(v);
    if (NT == 32) return v;
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    v = red[0];
#pragma unroll
    for (int i = 1; i < NT / 32; i++) v = max(v, red[i]);
    return v;
}

// Row-wise FP8: one CTA of kRowThreads per row.  Pass 1 finds the row amax
// with the row's 16-byte chunks kept in registers (kRowKeep per thread, so
// rows of up to kRowThreads * kRowKeep * 8 elements; longer rows are read
// again in pass 2), pass 2 writes the codes.
constexpr int kRowThreads = 128;
constexpr int kRowKeep = 5;

__global__ void __launch_bounds__(kRowThreads) k_quant_rowwise_fp8(const uint16_t *__restrict__ in,
                                                                   uint8_t *__restrict__ q,
                                                                   float *__restrict__ scale, int k) {
    __shared__ uint32_t red[kRowThreads / 32];
    const int64_t row = blockIdx.x;
    const int t = threadIdx.x;
    const uint16_t *x = in + row * k;
    const int nch = k >> 3;
    uint4 keep[kRowKeep];
    uint32_t mx = 0;
#pragma unroll
    for (int i = 0; i < kRowKeep; i++) {
        const int c = t + kRowThreads * i;
        keep[i] = c < nch ? ld_nc_v4(x + c * 8) : make_uint4(0, 0, 0, 0);
        mx = max(mx, amax_bits_8(keep[i]));
    }
    for (int c = t + kRowThreads * kRowKeep; c < nch; c += kRowThreads)
        mx = max(mx, amax_bits_8(ld_nc_v4(x + c * 8)));
    mx = cta_max_once<kRowThreads>(mx, red);
    const float s = __fdiv_rn(__uint_as_float(mx << 16), 448.0f);
    if (t == 0) scale[row] = s;
    const Bracket br = bracket_of(s);
    uint8_t *qr = q + row * k;
#pragma unroll
    for (int i = 0; i < kRowKeep; i++) {
        const int c = t + kRowThreads * i;
        if (c < nch) *reinterpret_cast<uint2 *>(qr + c * 8) = row_codes_8(keep[i], s, br);
    }
    for (int c = t + kRowThreads * kRowKeep; c < nch; c += kRowThreads)
        *reinterpret_cast<uint2 *>(qr + c * 8) = row_codes_8(ld_nc_v4(x + c * 8), s, br);
}

// One CTA per 128x128 block; 256 threads x 64 elements.
__global__ void __launch_bounds__(256) k_quant_blockfp8(const uint16_t *__restrict__ in, uint8_t *__restrict__ q,
                                                        float *__restrict__ scale, int k) {
    __shared__ uint32_t red[32];
    const int bj = blockIdx.x, bi = blockIdx.y;
    // thread t: row (t / 2) of the block, 64 columns starting at (t & 1) * 64
    const int r = threadIdx.x >> 1, c0 = (threadIdx.x & 1) * 64;
    const uint16_t *x = in + ((int64_t)bi * 128 + r) * k + (int64_t)bj * 128 + c0;
    uint4 v[8];
    uint32_t mx = 0;
#pragma unroll
    for (int i = 0; i < 8; i++) {
        v[i] = ld_nc_v4(x + i * 8);
        mx = max(mx, amax_bits_8(v[i]));
    }
    mx = block_max_u32<256>(mx, red);
    const float s = __fdiv_rn(__uint_as_float(mx << 16), 448.0f);
    if (threadIdx.x == 0) scale[(int64_t)bi * gridDim.x + bj] = s;
    const Bracket br = bracket_of(s);
    uint8_t *qo = q + ((int64_t)bi * 128 + r) * k + (int64_t)bj * 128 + c0;
#pragma unroll
    for (int i = 0; i < 8; i++) {
        uint2 out = make_uint2(0, 0);
        if (s != 0.0f) {
            float f[8];
            unpack_bf16_8(v[i], f);
            out = e4m3_codes_8(f, s, br);
        }
        *reinterpret_cast<uint2 *>(qo + i * 8) = out;
    }
}

// Block-scaled FP8 -> BF16 transient -> row-wise FP8.  The transient
// b = BF16(RN(e4m3(w) * S)) of a 16-code chunk is held packed (eight BF16x2
// words) between the amax pass and the code pass; it is never stored.
struct Bf16x16 {
    uint4 a, b;  // elements 0-7, 8-15
};

__device__ __forceinline__ Bf16x16 dequant_16(const uint4 &w, float S) {
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < 8; j++) {
        const float2 f = e4m3x2_to_f32x2((ws[j >> 1] >> (16 * (j & 1))) & 0xFFFFu);  // exact
        o[j] = pack_bf16x2(__fmul_rn(f.x, S), __fmul_rn(f.y, S));
    }
    return {make_uint4(o[0], o[1], o[2], o[3]), make_uint4(o[4], o[5], o[6], o[7])};
}

__device__ __forceinline__ uint4 requant_codes_16(const Bf16x16 &t, float s, const Bracket &br) {
    if (s == 0.0f) return make_uint4(0, 0, 0, 0);
    float lo[8], hi[8];
    unpack_bf16_8(t.a, lo);
    unpack_bf16_8(t.b, hi);
    const uint2 a = e4m3_codes_8(lo, s, br), b = e4m3_codes_8(hi, s, br);
    return make_uint4(a.x, a.y, b.x, b.y);
}

// One CTA of kReqThreads per row, the row's transients kept in registers
// (kReqKeep chunks per thread; longer rows are dequantised again).
constexpr int kReqThreads = 256;
constexpr int kReqKeep = 2;

__global__ void __launch_bounds__(kReqThreads) k_requant_blockfp8_to_rowwise(const uint8_t *__restrict__ w,
                                                                             const float *__restrict__ bscale,
                                                                             uint8_t *__restrict__ q,
                                                                             float *__restrict__ scale, int k) {
    __shared__ uint32_t red[kReqThreads / 32];
    const int64_t row = blockIdx.x;
    const int t = threadIdx.x;
    const int kb = k >> 7;
    const float *srow = bscale + (row >> 7) * kb;  // one scale per 128 codes = 8 chunks
    const uint8_t *wr = w + row * k;
    const int nch = k >> 4;
    Bf16x16 keep[kReqKeep];
    uint32_t mx = 0;
#pragma unroll
    for (int i = 0; i < kReqKeep; i++) {
        const int c = t + kReqThreads * i;
        keep[i] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
        if (c < nch) keep[i] = dequant_16(ld_nc_v4(wr + c * 16), __ldg(srow + (c >> 3)));
        mx = max(mx, max(amax_bits_8(keep[i].a), amax_bits_8(keep[i].b)));
    }
    for (int c = t + kReqThreads * kReqKeep; c < nch; c += kReqThreads) {
        const Bf16x16 d = dequant_16(ld_nc_v4(wr + c * 16), __ldg(srow + (c >> 3)));
        mx = max(mx, max(amax_bits_8(d.a), amax_bits_8(d.b)));
    }
    mx = cta_max_once<kReqThreads>(mx, red);
    const float s = __fdiv_rn(__uint_as_float(mx << 16), 448.0f);
    if (t == 0) scale[row] = s;
    const Bracket br = bracket_of(s);
    uint8_t *qr = q + row * k;
#pragma unroll
    for (int i = 0; i < kReqKeep; i++) {
        const int c = t + kReqThreads * i;
        if (c < nch) *reinterpret_cast<uint4 *>(qr + c * 16) = requant_codes_16(keep[i], s, br);
    }
    for (int c = t + kReqThreads * kReqKeep; c < nch; c += kReqThreads)
        *reinterpret_cast<uint4 *>(qr + c * 16) =
            requant_codes_16(dequant_16(ld_nc_v4(wr + c * 16), __ldg(srow + (c >> 3))), s, br);
}

// Rows of up to kReqSmemMaxK codes: one CTA of kReqRowThreads per row.  One
// bulk copy brings the whole row into shared memory, so every CTA has its
// row in flight at once and many rows are in flight per SM; pass 1 finds the
// amax of the BF16 transient, pass 2 writes the codes, both from shared
// memory.
constexpr int kReqRowThreads = 64;
constexpr int kReqSmemMaxK = 48 * 1024;

__global__ void __launch_bounds__(kReqRowThreads) k_requant_blockfp8_rows_smem(const uint8_t *__restrict__ w,
                                                                              const float *__restrict__ bscale,
                                                                              uint8_t *__restrict__ q,
                                                                              float *__restrict__ scale, int k) {
    extern __shared__ __align__(16) uint8_t srow[];
    __shared__ uint64_t bar;
    __shared__ uint32_t red[kReqRowThreads / 32];
    __shared__ float ssc[kReqSmemMaxK / 128];
    const int64_t row = blockIdx.x;
    const int t = threadIdx.x;
    if (t == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (t == 0) {
        mbar_arrive_expect_tx(&bar, (uint32_t)k);
        bulk_load_g2s(srow, w + row * k, (uint32_t)k, &bar);
    }
    // the row's block scales (one per 128 codes = 8 chunks), while the row is in flight
    const int kb = k >> 7;
    const float *srs = bscale + (row >> 7) * kb;
    for (int i = t; i < kb; i += kReqRowThreads) ssc[i] = __ldg(srs + i);
    __syncthreads();
    const int nch = k >> 4;
    // a copy that has not landed within the wait limit is reported through
    // the timeout flag; the whole CTA leaves together
    if (!__syncthreads_and(mbar_wait(&bar, 0, &g_quant_timeouts))) return;
    const uint4 *sv = reinterpret_cast<const uint4 *>(srow);
    uint32_t mx = 0;
    for (int c = t; c < nch; c += kReqRowThreads) {
        const Bf16x16 d = dequant_16(sv[c], ssc[c >> 3]);
        mx = max(mx, max(amax_bits_8(d.a), amax_bits_8(d.b)));
    }
    mx = cta_max_once<kReqRowThreads>(mx, red);
    const float s = __fdiv_rn(__uint_as_float(mx << 16), 448.0f);
    if (t == 0) scale[row] = s;
    const Bracket br = bracket_of(s);
    uint4 *qr = reinterpret_cast<uint4 *>(q + row * k);
    for (int c = t; c < nch; c += kReqRowThreads) qr[c] = requant_codes_16(dequant_16(sv[c], ssc[c >> 3]), s, br);
}

// ---------------------------------------------------------------------------
// int8 per-32 blocks, one thread per block.

// Nearest integer (ties to even) of q clamped to [-127, 127], as the low
// byte of the FP32 sum t + 1.5 * 2^23: in [2^23, 2^24) one unit is one ulp,
// so the round-to-nearest addition rounds t itself.  Clamping before
// rounding equals clamping after, the bounds being integers.
__device__ __forceinline__ uint32_t int8_code_bits(float q) {
    const float t = fminf(fmaxf(q, -127.0f), 127.0f);
    return __float_as_uint(__fadd_rn(t, 12582912.0f));
}

// Eight int8 codes of v / s packed little-endian (element 0 in the lowest
// byte); `br` is bracket_of(s), s = RN(amax / 127) with |v| <= amax.  In the
// bracketed range of s every product |v| r(1 +- 2^-16) stays below 127.5,
// so the codes need no clamp: the low byte of RN(p + 1.5 * 2^23) is the
// nearest integer of p (ties to even) in two's complement.
__device__ __forceinline__ uint2 int8_codes_8(const float (&v)[8], float s, const Bracket &br) {
    if (s == 0.0f) return make_uint2(0u, 0u);
    uint32_t c[8];
    if (br.ok) {
        uint32_t h[8], diff = 0;
#pragma unroll
        for (int i = 0; i < 8; i++) {
            c[i] = __float_as_uint(__fadd_rn(__fmul_rn(v[i], br.lo), 12582912.0f));
            h[i] = __float_as_uint(__fadd_rn(__fmul_rn(v[i], br.hi), 12582912.0f));
            diff |= c[i] ^ h[i];
        }
        if (diff != 0) {
#pragma unroll
            for (int i = 0; i < 8; i++)
                if (c[i] != h[i])
                    c[i] = int8_code_bits(
                        boundary_resolved(v[i], s, nearest_half_integer(__fmul_rn(v[i], br.lo))));
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; i++) c[i] = int8_code_bits(__fdiv_rn(v[i], s));
    }
    // low bytes of c[0..3] and c[4..7]
    const uint32_t w0 = __byte_perm(__byte_perm(c[0], c[1], 0x0040), __byte_perm(c[2], c[3], 0x0040), 0x5410);
    const uint32_t w1 = __byte_perm(__byte_perm(c[4], c[5], 0x0040), __byte_perm(c[6], c[7], 0x0040), 0x5410);
    return make_uint2(w0, w1);
}

// NVFP4 -> int8 requant: two threads per 32-block, one 16-element NVFP4
// block each.  A block's values take only eight magnitudes,
// v(e) = RN(RN(e2m1(e) * sf) * scale2), and the int8 code map is odd
// (RN, rint and the clamp are symmetric).  So each thread codes the eight
// magnitudes once and looks its sixteen codes up by nibble with byte
// permutes: magnitude bits select from the table, the sign bit selects the
// negated table.  The block amax is v at the largest magnitude present.
__global__ void __launch_bounds__(256) k_requant_w_nvfp4_int8(const uint2 *__restrict__ packed,
                                                              const uint8_t *__restrict__ sf, float scale2,
                                                              uint4 *__restrict__ q, float *__restrict__ scale,
                                                              int64_t nblocks16) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t h = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; h < nblocks16; h += stride) {
        const uint2 p = __ldg(packed + h);
        const float sfv = e4m3_to_f32(__ldg(sf + h));
        // largest magnitude code present (per-byte maxima of both nibbles)
        const uint32_t mags = __vmaxu4(__vmaxu4(p.x & 0x07070707u, (p.x >> 4) & 0x07070707u),
                                       __vmaxu4(p.y & 0x07070707u, (p.y >> 4) & 0x07070707u));
        const uint32_t mmax = max(max(mags & 0xFFu, (mags >> 8) & 0xFFu), max((mags >> 16) & 0xFFu, mags >> 24));
        // v(e) for e = 0..7, as four pairs
        float v[8];
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const float2 e = e2m1x2_to_f32x2((uint32_t)((2 * j + 1) << 4 | (2 * j)));
            v[2 * j] = __fmul_rn(__fmul_rn(e.x, sfv), scale2);
            v[2 * j + 1] = __fmul_rn(__fmul_rn(e.y, sfv), scale2);
        }
        const float vmax = mmax == 0 ? 0.0f : mmax == 1 ? v[1] : mmax == 2 ? v[2] : mmax == 3 ? v[3]
                         : mmax == 4 ? v[4] : mmax == 5 ? v[5] : mmax == 6 ? v[6] : v[7];
        const float amax = fmaxf(fabsf(vmax), __shfl_xor_sync(__activemask(), fabsf(vmax), 1));
        const float s = __fdiv_rn(amax, 127.0f);
        // table of the eight magnitudes' codes (bytes 0..7) and its negation
        const uint2 t = int8_codes_8(v, s, bracket_of(s));
        const uint2 tn = make_uint2(__vsub4(0u, t.x), __vsub4(0u, t.y));
        uint32_t w[4];
#pragma unroll
        for (int g = 0; g < 4; g++) {
            const uint32_t n = ((g < 2 ? p.x : p.y) >> (16 * (g & 1))) & 0xFFFFu;  // elements 4g..4g+3
            const uint32_t sel = n & 0x7777u;
            const uint32_t pos = __byte_perm(t.x, t.y, sel), neg = __byte_perm(tn.x, tn.y, sel);
            const uint32_t neg_mask = __byte_perm(0x0000FF00u, 0u, (n >> 3) & 0x1111u);
            w[g] = (pos & ~neg_mask) | (neg & neg_mask);
        }
        q[h] = make_uint4(w[0], w[1], w[2], w[3]);
        if ((h & 1) == 0) scale[h >> 1] = s;
    }
}

// Activations -> int8: four threads to each 32-element block, eight
// elements per thread; the block amax is a two-step shuffle of magnitude
// bits inside the quad, and the quad's first thread stores the block scale.
// The grid stride is a multiple of four, so a quad stays together to the
// last iteration.
__global__ void __launch_bounds__(256) k_quant_act_int8_per32(const uint16_t *__restrict__ a, uint2 *__restrict__ q,
                                                              float *__restrict__ scale, int64_t ngroups) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    // kQuantUnroll groups per thread and pass, all loads issued first; a
    // quad's four groups are in or out of range together (ngroups % 4 == 0)
    for (int64_t h0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; h0 < ngroups; h0 += kQuantUnroll * stride) {
        uint4 x[kQuantUnroll];
#pragma unroll
        for (int u = 0; u < kQuantUnroll; u++) {
            const int64_t h = h0 + u * stride;
            x[u] = h < ngroups ? ld_nc_v4(a + h * 8) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kQuantUnroll; u++) {
            const int64_t h = h0 + u * stride;
            if (h >= ngroups) break;
            float v[8];
            unpack_bf16_8(x[u], v);
            uint32_t mx = amax_bits_8(x[u]);
            const unsigned mask = __activemask();
            mx = max(mx, __shfl_xor_sync(mask, mx, 1));
            mx = max(mx, __shfl_xor_sync(mask, mx, 2));
            const float s = __fdiv_rn(__uint_as_float(mx << 16), 127.0f);
            q[h] = int8_codes_8(v, s, bracket_of(s));
            if ((h & 3) == 0) scale[h >> 2] = s;
        }
    }
}

__global__ void __launch_bounds__(256) k_amax_bf16(const uint16_t *__restrict__ x, int64_t count,
                                                   uint32_t *__restrict__ out) {
    __shared__ uint32_t red[32];
    uint32_t mx = 0;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t nvec = count >> 3;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nvec; i += stride)
        mx = max(mx, amax_bits_8(ld_nc_v4(x + i * 8)));
    for (int64_t i = nvec * 8 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride)
        mx = max(mx, static_cast<uint32_t>(x[i] & 0x7FFF));
    mx = block_max_u32<256>(mx, red);
    if (threadIdx.x == 0) atomicMax(out, mx << 16);
}

int grid_for(int64_t work, int threads) {
    const int64_t want = (work + threads - 1) / threads;
    const int64_t cap = (int64_t)sm_count() * (2048 / threads) * 4;
    return static_cast<int>(want < cap ? (want > 0 ? want : 1) : cap);
}

}  // namespace

cudaError_t launch_quant_nvfp4(const uint16_t *in, uint8_t *packed, uint8_t *scale, float scale2,
                               const float *amax_dev, float *scale2_out, int m, int k, cudaStream_t s) {
    const int64_t nblocks = (int64_t)m * k / 16;
    const float t6 = 6.0f * scale2;
    k_quant_nvfp4<<<grid_for((nblocks + kQuantUnroll - 1) / kQuantUnroll, 256), 256, 0, s>>>(reinterpret_cast<const uint4 *>(in),
                                                         reinterpret_cast<uint2 *>(packed), scale, scale2, t6,
                                                         amax_dev, scale2_out, nblocks);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_quant_rowwise_fp8(const uint16_t *in, uint8_t *q, float *scale, int rows, int k,
                                     cudaStream_t s) {
    k_quant_rowwise_fp8<<<rows, kRowThreads, 0, s>>>(in, q, scale, k);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_quant_blockfp8(const uint16_t *in, uint8_t *q, float *scale, int n, int k, cudaStream_t s) {
    k_quant_blockfp8<<<dim3(k / 128, n / 128), 256, 0, s>>>(in, q, scale, k);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_requant_blockfp8_to_rowwise(const uint8_t *w, const float *bscale, int n, int k, uint8_t *q,
                                               float *scale, cudaStream_t s) {
    if (k <= kReqSmemMaxK)
        k_requant_blockfp8_rows_smem<<<n, kReqRowThreads, k, s>>>(w, bscale, q, scale, k);
    else
        k_requant_blockfp8_to_rowwise<<<n, kReqThreads, 0, s>>>(w, bscale, q, scale, k);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_requant_w_nvfp4_int8(const uint8_t *packed, const uint8_t *sf, float scale2, int8_t *q,
                                        float *scale, int n, int k, cudaStream_t s) {
    const int64_t nb = (int64_t)n * k / 16;
    k_requant_w_nvfp4_int8<<<grid_for(nb, 256), 256, 0, s>>>(reinterpret_cast<const uint2 *>(packed), sf, scale2,
                                                             reinterpret_cast<uint4 *>(q), scale, nb);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_quant_act_int8_per32(const uint16_t *a, int8_t *q, float *scale, int m, int k,
                                        cudaStream_t s) {
    const int64_t ng = (int64_t)m * k / 8;
    k_quant_act_int8_per32<<<grid_for((ng + kQuantUnroll - 1) / kQuantUnroll, 256), 256, 0, s>>>(a, reinterpret_cast<uint2 *>(q), scale, ng);
    note_launch();
    return cudaGetLastError();
}

uint32_t take_timeouts_quant() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_quant_timeouts, sizeof(v)) != cudaSuccess) return 0xFFFFFFFFu;
    cudaMemcpyToSymbol(g_quant_timeouts, &zero, sizeof(zero));
    return v;
}

cudaError_t launch_amax_bf16(const uint16_t *x, size_t count, float *amax, cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(float), s);
    if (e != cudaSuccess) return e;
    if (count == 0) return cudaSuccess;
    k_amax_bf16<<<grid_for((int64_t)(count / 8 + 1), 256), 256, 0, s>>>(x, (int64_t)count,
                                                                        reinterpret_cast<uint32_t *>(amax));
    note_launch();
    return cudaGetLastError();
}

}  // namespace bsq
