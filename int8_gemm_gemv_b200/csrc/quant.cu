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
// compiler cannot contract or reorder it.
#include "bsq_common.cuh"

namespace bsq {

namespace {

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

// Eight x / d quotients -> eight E2M1 nibbles in one 32-bit word, element 0
// in the lowest nibble.
__device__ __forceinline__ uint32_t nvfp4_codes_8(const uint4 &v, float d) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t out = 0;
#pragma unroll
    for (int j = 0; j < 4; j++) {
        float lo = __fdiv_rn(lo_bf16(w[j]), d);
        float hi = __fdiv_rn(hi_bf16(w[j]), d);
        out |= f32x2_to_e2m1x2(lo, hi) << (8 * j);
    }
    return out;
}

// Two threads per 16-element block, eight elements (16 bytes) each.
__global__ void __launch_bounds__(256) k_quant_nvfp4(const uint16_t *__restrict__ in, uint32_t *__restrict__ packed,
                                                     uint8_t *__restrict__ sf, float scale2, float t6,
                                                     int64_t nhalf) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t h = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; h < nhalf; h += stride) {
        const uint4 v = ld_nc_v4(in + h * 8);
        uint32_t mx = amax_bits_8(v);
        mx = max(mx, __shfl_xor_sync(__activemask(), mx, 1));
        const float amax = __uint_as_float(mx << 16);
        const uint8_t sc = f32_to_e4m3(__fdiv_rn(amax, t6));
        const float sfv = e4m3_to_f32(sc);
        uint32_t codes = 0;
        if (sfv != 0.0f) codes = nvfp4_codes_8(v, __fmul_rn(sfv, scale2));
        packed[h] = codes;
        if ((h & 1) == 0) sf[h >> 1] = sc;
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

// Eight E4M3 codes of x / s (RNE, satfinite) packed little-endian.
__device__ __forceinline__ uint2 e4m3_codes_8(const float (&x)[8], float s) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; j++) w[j] = f32x2_to_e4m3x2(__fdiv_rn(x[2 * j], s), __fdiv_rn(x[2 * j + 1], s));
    return make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
}

__device__ __forceinline__ void unpack_bf16_8(const uint4 &v, float (&x)[8]) {
    x[0] = lo_bf16(v.x); x[1] = hi_bf16(v.x); x[2] = lo_bf16(v.y); x[3] = hi_bf16(v.y);
    x[4] = lo_bf16(v.z); x[5] = hi_bf16(v.z); x[6] = lo_bf16(v.w); x[7] = hi_bf16(v.w);
}

__device__ __forceinline__ uint2 row_codes_8(const uint4 &v, float s) {
    if (s == 0.0f) return make_uint2(0, 0);
    float f[8];
    unpack_bf16_8(v, f);
    return e4m3_codes_8(f, s);
}

// One CTA per row: pass 1 finds the row amax (values kept in registers for
// rows of up to NT*8*CH elements, re-read from cache beyond), pass 2 writes
// the codes.
constexpr int kRowThreads = 256;
constexpr int kRowCh = 4;

__global__ void __launch_bounds__(kRowThreads) k_quant_rowwise_fp8(const uint16_t *__restrict__ in,
                                                                   uint8_t *__restrict__ q,
                                                                   float *__restrict__ scale, int k) {
    __shared__ uint32_t red[32];
    const int64_t row = blockIdx.x;
    const uint16_t *x = in + row * k;
    const int nch = k >> 3;
    uint4 keep[kRowCh];
    uint32_t mx = 0;
#pragma unroll
    for (int i = 0; i < kRowCh; i++) {
        const int c = threadIdx.x + i * kRowThreads;
        keep[i] = make_uint4(0, 0, 0, 0);
        if (c < nch) keep[i] = ld_nc_v4(x + c * 8);
        mx = max(mx, amax_bits_8(keep[i]));
    }
    for (int c = threadIdx.x + kRowCh * kRowThreads; c < nch; c += kRowThreads) mx = max(mx, amax_bits_8(ld_nc_v4(x + c * 8)));
    mx = block_max_u32<kRowThreads>(mx, red);
    const float amax = __uint_as_float(mx << 16);
    const float s = __fdiv_rn(amax, 448.0f);
    if (threadIdx.x == 0) scale[row] = s;
    uint8_t *qr = q + row * k;
#pragma unroll
    for (int i = 0; i < kRowCh; i++) {
        const int c = threadIdx.x + i * kRowThreads;
        if (c < nch) *reinterpret_cast<uint2 *>(qr + c * 8) = row_codes_8(keep[i], s);
    }
    for (int c = threadIdx.x + kRowCh * kRowThreads; c < nch; c += kRowThreads)
        *reinterpret_cast<uint2 *>(qr + c * 8) = row_codes_8(ld_nc_v4(x + c * 8), s);
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
    uint8_t *qo = q + ((int64_t)bi * 128 + r) * k + (int64_t)bj * 128 + c0;
#pragma unroll
    for (int i = 0; i < 8; i++) {
        uint2 out = make_uint2(0, 0);
        if (s != 0.0f) {
            float f[8];
            unpack_bf16_8(v[i], f);
            out = e4m3_codes_8(f, s);
        }
        *reinterpret_cast<uint2 *>(qo + i * 8) = out;
    }
}

// Block-scaled FP8 -> BF16 transient -> row-wise FP8, one CTA per row.  The
// transient b = BF16(e4m3(w) * S) is recomputed in pass 2 instead of stored.
__device__ __forceinline__ void dequant_16(const uint4 &w, float S, float (&b)[16]) {
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 16; j++) {
        const uint8_t code = (ws[j >> 2] >> (8 * (j & 3))) & 0xFF;
        const float p = __fmul_rn(e4m3_to_f32(code), S);
        b[j] = __bfloat162float(__float2bfloat16_rn(p));
    }
}

__global__ void __launch_bounds__(kRowThreads) k_requant_blockfp8_to_rowwise(const uint8_t *__restrict__ w,
                                                                             const float *__restrict__ bscale,
                                                                             uint8_t *__restrict__ q,
                                                                             float *__restrict__ scale, int k) {
    __shared__ uint32_t red[32];
    const int64_t row = blockIdx.x;
    const int kb = k >> 7;
    const float *srow = bscale + (row >> 7) * kb;
    const uint8_t *wr = w + row * k;
    const int nch = k >> 4;  // 16 codes per chunk
    uint32_t mx = 0;
    for (int c = threadIdx.x; c < nch; c += kRowThreads) {
        float b[16];
        dequant_16(ld_nc_v4(wr + c * 16), __ldg(srow + (c >> 3)), b);
#pragma unroll
        for (int j = 0; j < 16; j++) mx = max(mx, __float_as_uint(fabsf(b[j])));
    }
    mx = block_max_u32<kRowThreads>(mx, red);
    const float s = __fdiv_rn(__uint_as_float(mx), 448.0f);
    if (threadIdx.x == 0) scale[row] = s;
    uint8_t *qr = q + row * k;
    for (int c = threadIdx.x; c < nch; c += kRowThreads) {
        uint4 out = make_uint4(0, 0, 0, 0);
        if (s != 0.0f) {
            float b[16];
            dequant_16(ld_nc_v4(wr + c * 16), __ldg(srow + (c >> 3)), b);
            float lo[8], hi[8];
#pragma unroll
            for (int j = 0; j < 8; j++) { lo[j] = b[j]; hi[j] = b[8 + j]; }
            const uint2 a = e4m3_codes_8(lo, s), bb = e4m3_codes_8(hi, s);
            out = make_uint4(a.x, a.y, bb.x, bb.y);
        }
        *reinterpret_cast<uint4 *>(qr + c * 16) = out;
    }
}

// ---------------------------------------------------------------------------
// int8 per-32 blocks, one thread per block.

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

__device__ __forceinline__ void int8_block_store(const float (&v)[32], int8_t *q, float *s_out) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; i++) amax = fmaxf(amax, fabsf(v[i]));
    const float s = __fdiv_rn(amax, 127.0f);
    *s_out = s;
    uint32_t w[8];
#pragma unroll
    for (int j = 0; j < 8; j++) {
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 4; b++) {
            int iv = 0;
            if (s != 0.0f) {
                const float r = fminf(fmaxf(rintf(__fdiv_rn(v[4 * j + b], s)), -127.0f), 127.0f);
                iv = __float2int_rn(r);
            }
            word |= (static_cast<uint32_t>(iv) & 0xFFu) << (8 * b);
        }
        w[j] = word;
    }
    uint4 *dst = reinterpret_cast<uint4 *>(q);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
}

__global__ void __launch_bounds__(128) k_requant_w_nvfp4_int8(const uint8_t *__restrict__ packed,
                                                              const uint8_t *__restrict__ sf, float scale2,
                                                              int8_t *__restrict__ q, float *__restrict__ scale,
                                                              int64_t nblocks) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblocks; b += stride) {
        // block b covers elements [32b, 32b+32) of the flattened [n, k] tensor
        const uint4 p = ld_nc_v4(packed + b * 16);
        const float s0 = e4m3_to_f32(sf[b * 2]), s1 = e4m3_to_f32(sf[b * 2 + 1]);
        const uint32_t pw[4] = {p.x, p.y, p.z, p.w};
        float v[32];
#pragma unroll
        for (int j = 0; j < 16; j++) {
            const float2 e = e2m1x2_to_f32x2((pw[j >> 2] >> (8 * (j & 3))) & 0xFF);
            const float sfv = j < 8 ? s0 : s1;
            v[2 * j] = __fmul_rn(__fmul_rn(e.x, sfv), scale2);
            v[2 * j + 1] = __fmul_rn(__fmul_rn(e.y, sfv), scale2);
        }
        int8_block_store(v, q + b * 32, scale + b);
    }
}

__global__ void __launch_bounds__(128) k_quant_act_int8_per32(const uint16_t *__restrict__ a,
                                                              int8_t *__restrict__ q, float *__restrict__ scale,
                                                              int64_t nblocks) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblocks; b += stride) {
        float v[32];
#pragma unroll
        for (int c = 0; c < 4; c++) {
            float f[8];
            unpack_bf16_8(ld_nc_v4(a + b * 32 + c * 8), f);
#pragma unroll
            for (int i = 0; i < 8; i++) v[c * 8 + i] = f[i];
        }
        int8_block_store(v, q + b * 32, scale + b);
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

cudaError_t launch_quant_nvfp4(const uint16_t *in, uint8_t *packed, uint8_t *scale, float scale2, int m, int k,
                               cudaStream_t s) {
    const int64_t nhalf = (int64_t)m * k / 8;
    const float t6 = 6.0f * scale2;
    k_quant_nvfp4<<<grid_for(nhalf, 256), 256, 0, s>>>(in, reinterpret_cast<uint32_t *>(packed), scale, scale2, t6,
                                                       nhalf);
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
    k_requant_blockfp8_to_rowwise<<<n, kRowThreads, 0, s>>>(w, bscale, q, scale, k);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_requant_w_nvfp4_int8(const uint8_t *packed, const uint8_t *sf, float scale2, int8_t *q,
                                        float *scale, int n, int k, cudaStream_t s) {
    const int64_t nb = (int64_t)n * k / 32;
    k_requant_w_nvfp4_int8<<<grid_for(nb, 128), 128, 0, s>>>(packed, sf, scale2, q, scale, nb);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_quant_act_int8_per32(const uint16_t *a, int8_t *q, float *scale, int m, int k,
                                        cudaStream_t s) {
    const int64_t nb = (int64_t)m * k / 32;
    k_quant_act_int8_per32<<<grid_for(nb, 128), 128, 0, s>>>(a, q, scale, nb);
    note_launch();
    return cudaGetLastError();
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
