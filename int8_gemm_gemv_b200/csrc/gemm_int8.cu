// int8 x int8 GEMM with per-32 FP32 block scales on both operands
// (gemm_dense_int8.rs, `int8_gemm_faith2_prefill` step (b)):
//   C[m, n] = sum_b (exact int32 sum_{k in b} a*w) * a_scale[m, b] * w_scale[n, b]
//
// The scales change every 32 K, which is exactly one int8 MMA K step, so the
// tensor cores cannot accumulate across blocks.  Each 128x128x32 MMA writes a
// fresh int32 partial into one of four tensor-memory buffers (4 x 128
// columns); eight "fold" warps read each partial back and fold it into FP32
// registers with its two scales while the tensor cores already compute the
// next ones.  The fold (one convert, one multiply, one FMA per output and
// block) on the CUDA cores is the bound of this kernel, not the int8 MMA.
//
//   warp 0       TMA producer: A, W tiles (128 x 128 B) and their scale tiles
//                (128 rows x 4 FP32) into a 6-stage ring
//   warp 1       MMA issuer
//   warp 2       rewrites each stage's W-scale tile from [n][4] to [4][n] so
//                the fold warps read 4 columns per shared-memory load
//   warps 4..11  fold + epilogue; warp w owns tensor-memory lane quarter
//                w % 4 (rows) and column half (w - 4) / 4
#include "bsq_common.cuh"

namespace bsq {

namespace {

constexpr int BM = 128, BN = 128, BK = 128;  // BK bytes = elements = 4 blocks of 32
constexpr int STAGES = 6;
constexpr int A_BYTES = BM * BK, B_BYTES = BN * BK;
constexpr int SA_BYTES = BM * 16, SW_BYTES = BN * 16;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SA_BYTES + SW_BYTES;
constexpr int NACC = 4;  // tensor-memory partial buffers of 128 columns
constexpr int TMEM_COLS = 512;
constexpr int NFOLD = 8;
constexpr int kThreads = 32 * (4 + NFOLD);

static __device__ unsigned int g_timeouts;

struct Smem {
    uint64_t full[STAGES];
    uint64_t swready[STAGES];
    uint64_t empty[STAGES];
    uint64_t acc_full[NACC], acc_empty[NACC];
    uint64_t drain;
    uint32_t tmem_base;
    uint32_t abort;
};

constexpr size_t kSmemBytes = 1024 + (size_t)STAGES * STAGE_BYTES + sizeof(Smem);

__device__ __forceinline__ bool aborted(volatile Smem *s) { return s->abort != 0; }

__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;"
        : "=l"(*reinterpret_cast<uint64_t *>(&d))
        : "l"(*reinterpret_cast<uint64_t *>(&a)), "l"(*reinterpret_cast<uint64_t *>(&b)),
          "l"(*reinterpret_cast<uint64_t *>(&c)));
    return d;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    float2 d;
    asm("mul.rn.f32x2 %0, %1, %2;"
        : "=l"(*reinterpret_cast<uint64_t *>(&d))
        : "l"(*reinterpret_cast<uint64_t *>(&a)), "l"(*reinterpret_cast<uint64_t *>(&b)));
    return d;
}

__global__ void __launch_bounds__(kThreads, 1)
    k_int8_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSW,
                uint16_t *__restrict__ out, int M, int N, int K) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Smem *S = reinterpret_cast<Smem *>(base + (size_t)STAGES * STAGE_BYTES);
    auto a_tile = [&](int s) { return base + (size_t)s * STAGE_BYTES; };
    auto b_tile = [&](int s) { return base + (size_t)s * STAGE_BYTES + A_BYTES; };
    auto sa_tile = [&](int s) { return reinterpret_cast<float *>(base + (size_t)s * STAGE_BYTES + A_BYTES + B_BYTES); };
    auto sw_tile = [&](int s) {
        return reinterpret_cast<float *>(base + (size_t)s * STAGE_BYTES + A_BYTES + B_BYTES + SA_BYTES);
    };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles_m = (M + BM - 1) / BM, tiles_n = (N + BN - 1) / BN;
    const int num_tiles = tiles_m * tiles_n;
    const int nkb = K / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; s++) {
            mbar_init(&S->full[s], 1);
            mbar_init(&S->swready[s], 1);
            mbar_init(&S->empty[s], 1 + NFOLD);
        }
        for (int b = 0; b < NACC; b++) {
            mbar_init(&S->acc_full[b], 1);
            mbar_init(&S->acc_empty[b], NFOLD);
        }
        mbar_init(&S->drain, 1);
        S->abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&S->tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S->tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tensormap(&tmA);
            prefetch_tensormap(&tmB);
            prefetch_tensormap(&tmSA);
            prefetch_tensormap(&tmSW);
            uint32_t it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                const int mt = t % tiles_m, nt = t / tiles_m;
                for (int kb = 0; kb < nkb; kb++, it++) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait(&S->empty[s], ph ^ 1, &g_timeouts) || aborted(S)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&S->full[s], STAGE_BYTES);
                    tma_load_2d(a_tile(s), &tmA, &S->full[s], kb * BK, mt * BM);
                    tma_load_2d(b_tile(s), &tmB, &S->full[s], kb * BK, nt * BN);
                    tma_load_2d(sa_tile(s), &tmSA, &S->full[s], kb * 4, mt * BM);
                    tma_load_2d(sw_tile(s), &tmSW, &S->full[s], kb * 4, nt * BN);
                }
            }
            if (!ok) {
                S->abort = 1;
                const uint32_t first = it > STAGES ? it - STAGES : 0;
                for (uint32_t i = first; i < it; i++) mbar_wait(&S->full[i % STAGES], (i / STAGES) & 1, &g_timeouts);
            }
        }
    } else if (warp == 2) {
        // W scales: [n][4] -> [4][n], in place
        uint32_t it = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
            for (int kb = 0; kb < nkb; kb++, it++) {
                const int s = it % STAGES;
                if (!mbar_wait(&S->full[s], (it / STAGES) & 1, &g_timeouts) || aborted(S)) {
                    ok = false;
                    break;
                }
                float *sw = sw_tile(s);
                float4 v[4];
#pragma unroll
                for (int q = 0; q < 4; q++) v[q] = reinterpret_cast<float4 *>(sw)[32 * q + lane];
                __syncwarp();
#pragma unroll
                for (int q = 0; q < 4; q++) {
                    sw[0 * BN + 32 * q + lane] = v[q].x;
                    sw[1 * BN + 32 * q + lane] = v[q].y;
                    sw[2 * BN + 32 * q + lane] = v[q].z;
                    sw[3 * BN + 32 * q + lane] = v[q].w;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&S->swready[s]);
            }
        }
        if (!ok && lane == 0) S->abort = 1;
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_s8(BM, BN);
            uint32_t it = 0, gs = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                for (int kb = 0; kb < nkb && ok; kb++, it++) {
                    const int s = it % STAGES;
                    if (!mbar_wait(&S->full[s], (it / STAGES) & 1, &g_timeouts) || aborted(S)) {
                        ok = false;
                        break;
                    }
                    const uint32_t a0 = smem_u32(a_tile(s)), b0 = smem_u32(b_tile(s));
                    for (int j = 0; j < 4; j++, gs++) {
                        const int b = gs % NACC;
                        if (!mbar_wait(&S->acc_empty[b], ((gs / NACC) & 1) ^ 1, &g_timeouts) || aborted(S)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        mma_i8(tmem + b * BN, sdesc_k_sw128(a0 + 32 * j), sdesc_k_sw128(b0 + 32 * j), idesc, 0);
                        tc_commit(&S->acc_full[b]);
                    }
                    tc_commit(&S->empty[s]);
                }
            }
            if (!ok) S->abort = 1;
            tc_commit(&S->drain);
            mbar_wait(&S->drain, 0, &g_timeouts);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------ fold + epilogue
        const int q = warp & 3, h = (warp - 4) >> 2;
        const uint32_t lane_off = (uint32_t)(32 * q) << 16;
        uint32_t it = 0, gs = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
            const int mt = t % tiles_m, nt = t / tiles_m;
            float2 acc[32];
#pragma unroll
            for (int i = 0; i < 32; i++) acc[i] = make_float2(0.0f, 0.0f);
            for (int kb = 0; kb < nkb && ok; kb++, it++) {
                const int s = it % STAGES;
                if (!mbar_wait(&S->swready[s], (it / STAGES) & 1, &g_timeouts) || aborted(S)) {
                    ok = false;
                    break;
                }
                const float4 sa4 = reinterpret_cast<const float4 *>(sa_tile(s))[32 * q + lane];
                const float *sw = sw_tile(s) + 64 * h;
#pragma unroll 1
                for (int j = 0; j < 4; j++, gs++) {
                    const int b = gs % NACC;
                    if (!mbar_wait(&S->acc_full[b], (gs / NACC) & 1, &g_timeouts) || aborted(S)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    uint32_t r0[32], r1[32];
                    tmem_ld_32x32b_x32(tmem + b * BN + lane_off + 64 * h, r0);
                    tmem_ld_32x32b_x32(tmem + b * BN + lane_off + 64 * h + 32, r1);
                    tmem_ld_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&S->acc_empty[b]);
                    const float saj = j == 0 ? sa4.x : j == 1 ? sa4.y : j == 2 ? sa4.z : sa4.w;
                    const float2 sa2 = make_float2(saj, saj);
                    const float4 *swj = reinterpret_cast<const float4 *>(sw + j * BN);
#pragma unroll
                    for (int i = 0; i < 8; i++) {
                        const float4 w4 = swj[i];
                        const float2 s01 = mul2(sa2, make_float2(w4.x, w4.y));
                        const float2 s23 = mul2(sa2, make_float2(w4.z, w4.w));
                        acc[2 * i] = fma2(make_float2((float)(int)r0[4 * i], (float)(int)r0[4 * i + 1]), s01, acc[2 * i]);
                        acc[2 * i + 1] =
                            fma2(make_float2((float)(int)r0[4 * i + 2], (float)(int)r0[4 * i + 3]), s23, acc[2 * i + 1]);
                    }
#pragma unroll
                    for (int i = 0; i < 8; i++) {
                        const float4 w4 = swj[8 + i];
                        const float2 s01 = mul2(sa2, make_float2(w4.x, w4.y));
                        const float2 s23 = mul2(sa2, make_float2(w4.z, w4.w));
                        acc[16 + 2 * i] =
                            fma2(make_float2((float)(int)r1[4 * i], (float)(int)r1[4 * i + 1]), s01, acc[16 + 2 * i]);
                        acc[16 + 2 * i + 1] = fma2(make_float2((float)(int)r1[4 * i + 2], (float)(int)r1[4 * i + 3]),
                                                   s23, acc[16 + 2 * i + 1]);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&S->empty[s]);
            }
            if (!ok) {
                if (lane == 0) S->abort = 1;
                break;
            }
            const int row = mt * BM + 32 * q + lane;
            const int n0 = nt * BN + 64 * h;
            if (row < M) {
                uint16_t *orow = out + (int64_t)row * N;
                if ((N % 8) == 0 && n0 + 64 <= N) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + n0);
#pragma unroll
                    for (int i = 0; i < 8; i++)
                        dst[i] = make_uint4(pack_bf16x2(acc[4 * i].x, acc[4 * i].y),
                                            pack_bf16x2(acc[4 * i + 1].x, acc[4 * i + 1].y),
                                            pack_bf16x2(acc[4 * i + 2].x, acc[4 * i + 2].y),
                                            pack_bf16x2(acc[4 * i + 3].x, acc[4 * i + 3].y));
                } else {
#pragma unroll
                    for (int i = 0; i < 32; i++) {
                        if (n0 + 2 * i < N) orow[n0 + 2 * i] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[i].x));
                        if (n0 + 2 * i + 1 < N)
                            orow[n0 + 2 * i + 1] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[i].y));
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace

uint32_t take_timeouts_gemm_int8() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_timeouts, sizeof(v)) != cudaSuccess) return 0xFFFFFFFFu;
    cudaMemcpyToSymbol(g_timeouts, &zero, sizeof(zero));
    return v;
}

cudaError_t launch_int8_blockscaled_gemm(const int8_t *a, const int8_t *w, const float *a_scale,
                                         const float *w_scale, uint16_t *out, int m, int n, int k,
                                         cudaStream_t s) {
    alignas(64) CUtensorMap tA, tB, tSA, tSW;
    const uint64_t kblk = (uint64_t)k / 32;
    if (!make_tmap_2d(&tA, a, 1, k, m, k, BK, BM, true, false) ||
        !make_tmap_2d(&tB, w, 1, k, n, k, BK, BN, true, false) ||
        !make_tmap_2d(&tSA, a_scale, 4, kblk, m, kblk * 4, 4, BM, false, true) ||
        !make_tmap_2d(&tSW, w_scale, 4, kblk, n, kblk * 4, 4, BN, false, true))
        return cudaErrorInvalidValue;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(k_int8_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_done[dev] = true;
    }
    const int tiles = ((m + BM - 1) / BM) * ((n + BN - 1) / BN);
    const int grid = tiles < sm_count() ? tiles : sm_count();
    k_int8_gemm<<<grid, kThreads, kSmemBytes, s>>>(tA, tB, tSA, tSW, out, m, n, k);
    note_launch();
    return cudaGetLastError();
}

}  // namespace bsq
