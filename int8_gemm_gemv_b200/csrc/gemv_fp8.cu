// Row-scaled FP8 GEMV for 1 <= M <= 16 (fp8_gemv_batch.rs,
// `fp8_gemv_rowscale_batch8_rt2`, `fp8_gemv_rowscale_batch16_rt2`,
// `dense_gemv_fp8w_batch2`):
//   out[m, n] = row_scale[n] * sum_k bf16(in[m, k]) * e4m3(W[n, k])
//
// The weight stream (N*K bytes) is the whole cost, so the kernel reads each
// weight byte once with 16-byte loads and does the arithmetic on the tensor
// cores: E4M3 -> BF16 is exact, so each warp converts its weight bytes in
// registers and issues BF16 m16n8k16 MMAs with W as the 16-row A operand and
// the (at most 16) activation rows as the B operand.  Products are exact in
// FP32; accumulation is FP32; the row scale is applied once at write-out.
//
// Inside a 64-wide K chunk, lane (g = lane/4, t = lane%4) loads bytes
// [16t, 16t+16) of weight rows g and g+8, and the same K range of activation
// rows g and g+8.  The MMA's K positions are permuted accordingly (the sum
// does not depend on the order of its K positions, only on matching A and B).
//
// A CTA of 8 warps covers 16*WR weight rows; its warps split K into WK = 8/WR
// interleaved slices and the slices are summed in a fixed order, so the
// result of one output never depends on M.
#include "bsq_common.cuh"

namespace bsq {

namespace {

__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ uint4 ld_keep_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Two E4M3 bytes (low byte = lower K index) -> BF16x2, exact.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t two) {
    uint32_t h2;
    asm("{\n\t.reg .b16 t;\n\t"
        "cvt.u16.u32 t, %1;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
        : "=r"(h2)
        : "r"(two));
    const __half2 h = *reinterpret_cast<const __half2 *>(&h2);
    const float2 f = __half22float2(h);
    return pack_bf16x2(f.x, f.y);
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

constexpr int kThreads = 256;

template <int MT, int WR>
__global__ void __launch_bounds__(kThreads) k_fp8_gemv(const uint16_t *__restrict__ X, const uint8_t *__restrict__ W,
                                                       const float *__restrict__ row_scale,
                                                       uint16_t *__restrict__ out, int M, int N, int K) {
    constexpr int WK = 8 / WR;
    __shared__ float red[(WK > 1 ? WK - 1 : 1) * WR][MT][4][32];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int rt = warp % WR, ks = warp / WR;
    const int n0 = blockIdx.x * (16 * WR) + rt * 16;
    const int nchunks = (K + 63) >> 6;

    const int rowA = n0 + g, rowB = n0 + g + 8;
    const bool okA = rowA < N, okB = rowB < N;
    const uint8_t *wA = W + (int64_t)(okA ? rowA : 0) * K + 16 * t;
    const uint8_t *wB = W + (int64_t)(okB ? rowB : 0) * K + 16 * t;
    const bool okX0 = g < M, okX1 = (8 + g) < M;
    const uint16_t *x0 = X + (int64_t)(okX0 ? g : 0) * K + 16 * t;
    const uint16_t *x1 = X + (int64_t)(okX1 ? 8 + g : 0) * K + 16 * t;

    float acc[MT][4];
#pragma unroll
    for (int i = 0; i < MT; i++) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;

    const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll 2
    for (int c = ks; c < nchunks; c += WK) {
        const int kk = c * 64;
        const bool kok = kk + 16 * t < K;
        const uint4 wa = (okA && kok) ? ld_stream_v4(wA + kk) : z;
        const uint4 wb = (okB && kok) ? ld_stream_v4(wB + kk) : z;
        uint4 xa[2], xb[2];
        xa[0] = (okX0 && kok) ? ld_keep_v4(x0 + kk) : z;
        xa[1] = (okX0 && kok) ? ld_keep_v4(x0 + kk + 8) : z;
        if (MT == 2) {
            xb[0] = (okX1 && kok) ? ld_keep_v4(x1 + kk) : z;
            xb[1] = (okX1 && kok) ? ld_keep_v4(x1 + kk + 8) : z;
        }
        const uint32_t wa_w[4] = {wa.x, wa.y, wa.z, wa.w};
        const uint32_t wb_w[4] = {wb.x, wb.y, wb.z, wb.w};
        const uint32_t xa_w[8] = {xa[0].x, xa[0].y, xa[0].z, xa[0].w, xa[1].x, xa[1].y, xa[1].z, xa[1].w};
#pragma unroll
        for (int j = 0; j < 4; j++) {
            // MMA j covers bytes [4j, 4j+4) of this lane's 16-byte slice
            uint32_t a[4];
            a[0] = e4m3x2_to_bf16x2(wa_w[j] & 0xFFFF);  // row g,   k 4j, 4j+1
            a[1] = e4m3x2_to_bf16x2(wb_w[j] & 0xFFFF);  // row g+8, k 4j, 4j+1
            a[2] = e4m3x2_to_bf16x2(wa_w[j] >> 16);     // row g,   k 4j+2, 4j+3
            a[3] = e4m3x2_to_bf16x2(wb_w[j] >> 16);     // row g+8, k 4j+2, 4j+3
            mma_bf16_16816(acc[0], a, xa_w[2 * j], xa_w[2 * j + 1]);
            if (MT == 2) {
                const uint32_t xb_w[8] = {xb[0].x, xb[0].y, xb[0].z, xb[0].w, xb[1].x, xb[1].y, xb[1].z, xb[1].w};
                mma_bf16_16816(acc[MT - 1], a, xb_w[2 * j], xb_w[2 * j + 1]);
            }
        }
    }

    // Sum the K slices in a fixed order: slice 0 + slice 1 + ... .
    if (WK > 1) {
        if (ks > 0) {
#pragma unroll
            for (int i = 0; i < MT; i++)
#pragma unroll
                for (int r = 0; r < 4; r++) red[(ks - 1) * WR + rt][i][r][lane] = acc[i][r];
        }
        __syncthreads();
        if (ks != 0) return;
#pragma unroll
        for (int s = 1; s < WK; s++)
#pragma unroll
            for (int i = 0; i < MT; i++)
#pragma unroll
                for (int r = 0; r < 4; r++) acc[i][r] += red[(s - 1) * WR + rt][i][r][lane];
    }

    // acc[i][r]: n = n0 + g + 8*(r >> 1), m = 8*i + 2t + (r & 1)
#pragma unroll
    for (int r = 0; r < 4; r++) {
        const int n = n0 + g + 8 * (r >> 1);
        if (n >= N) continue;
        const float s = __ldg(row_scale + n);
#pragma unroll
        for (int i = 0; i < MT; i++) {
            const int m = 8 * i + 2 * t + (r & 1);
            if (m < M) out[(int64_t)m * N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[i][r] * s));
        }
    }
}

}  // namespace

constexpr int kGemvRowTiles = 2;  // 32 weight rows per CTA, 4 K slices

cudaError_t launch_fp8_gemv_rowscale(const uint16_t *in, const uint8_t *w, const float *row_scale, uint16_t *out,
                                     int m, int n, int k, cudaStream_t s) {
    const int rows_per_cta = 16 * kGemvRowTiles;
    const int grid = (n + rows_per_cta - 1) / rows_per_cta;
    if (m <= 8)
        k_fp8_gemv<1, kGemvRowTiles><<<grid, kThreads, 0, s>>>(in, w, row_scale, out, m, n, k);
    else
        k_fp8_gemv<2, kGemvRowTiles><<<grid, kThreads, 0, s>>>(in, w, row_scale, out, m, n, k);
    note_launch();
    return cudaGetLastError();
}

}  // namespace bsq
