// Row-scaled FP8 GEMM on the sm_100a tensor cores (dispatch_proj_rowwise.rs,
// `cublas_fp8_rowwise_proj`: per-token activation scales x per-row weight
// scales, "outer-vector" FP32 scales):
//   C[m, n] = a_scale[m] * w_scale[n] * sum_k e4m3(A[m,k]) e4m3(W[n,k])
//
// Persistent warp-specialised kernel, one CTA per SM, 128 x 256 tiles:
//   warp 0      TMA producer, 4-stage ring (A 128x128 B, W 256x128 B per
//               stage, 128-byte swizzle)
//   warp 1      MMA issuer: four 128x256x32 E4M3 MMAs per stage into one of
//               two FP32 accumulators in tensor memory (2 x 256 columns), so
//               the epilogue of tile i overlaps the main loop of tile i+1
//   warps 4..7  epilogue: tensor memory -> registers, both scales, BF16,
//               global stores
// Rows beyond M are zero-filled by the TMA and never stored, so the caller
// pads nothing (the page pads M to 16 with zeroed rows and scales).
#include "bsq_common.cuh"

namespace bsq {

namespace {

constexpr int BM = 128, BN = 256, BK = 128;  // BK in bytes = elements
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK, B_BYTES = BN * BK;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 512;
constexpr int kThreads = 256;

static __device__ unsigned int g_timeouts;

struct Smem {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tfull[2], tempty[2], drain;
    uint32_t tmem_base;
    uint32_t abort;
};

constexpr size_t kSmemBytes = 1024 + (size_t)STAGES * STAGE_BYTES + sizeof(Smem);

__device__ __forceinline__ bool aborted(volatile Smem *s) { return s->abort != 0; }

__global__ void __launch_bounds__(kThreads, 1)
    k_fp8_gemm_rowscale(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const float *__restrict__ a_scale, const float *__restrict__ w_scale,
                        uint16_t *__restrict__ out, int M, int N, int K) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Smem *S = reinterpret_cast<Smem *>(base + (size_t)STAGES * STAGE_BYTES);
    auto a_tile = [&](int s) { return base + (size_t)s * STAGE_BYTES; };
    auto b_tile = [&](int s) { return base + (size_t)s * STAGE_BYTES + A_BYTES; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles_m = (M + BM - 1) / BM, tiles_n = (N + BN - 1) / BN;
    const int num_tiles = tiles_m * tiles_n;
    const int nkb = (K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; s++) {
            mbar_init(&S->full[s], 1);
            mbar_init(&S->empty[s], 1);
        }
        for (int b = 0; b < 2; b++) {
            mbar_init(&S->tfull[b], 1);
            mbar_init(&S->tempty[b], 4);
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
                }
            }
            if (!ok) {
                S->abort = 1;
                const uint32_t first = it > STAGES ? it - STAGES : 0;
                for (uint32_t i = first; i < it; i++) mbar_wait(&S->full[i % STAGES], (i / STAGES) & 1, &g_timeouts);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_e4m3(BM, BN);
            uint32_t it = 0, tc = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, tc++) {
                const int buf = tc & 1;
                if (!mbar_wait(&S->tempty[buf], ((tc >> 1) & 1) ^ 1, &g_timeouts) || aborted(S)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t acc = tmem + buf * BN;
                for (int kb = 0; kb < nkb; kb++, it++) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait(&S->full[s], ph, &g_timeouts) || aborted(S)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(a_tile(s)), b0 = smem_u32(b_tile(s));
#pragma unroll
                    for (int j = 0; j < 4; j++)
                        mma_f8f6f4(acc, sdesc_k_sw128(a0 + 32 * j), sdesc_k_sw128(b0 + 32 * j), idesc, (kb | j) != 0);
                    tc_commit(&S->empty[s]);
                }
                if (!ok) break;
                tc_commit(&S->tfull[buf]);
            }
            if (!ok) S->abort = 1;
            tc_commit(&S->drain);
            mbar_wait(&S->drain, 0, &g_timeouts);
        }
    } else if (warp >= 4) {
        const int q = warp - 4;
        uint32_t tc = 0;
        const bool vec_ok = (N % 8) == 0;
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, tc++) {
            const int mt = t % tiles_m, nt = t / tiles_m;
            const int buf = tc & 1;
            if (!mbar_wait(&S->tfull[buf], (tc >> 1) & 1, &g_timeouts) || aborted(S)) {
                if (lane == 0) S->abort = 1;
                break;
            }
            tc_fence_after();
            const int row = mt * BM + 32 * q + lane;
            const float sa = row < M ? __ldg(a_scale + row) : 0.0f;
            uint16_t *orow = out + (int64_t)row * N;
#pragma unroll 1
            for (int c = 0; c < BN / 32; c++) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem + buf * BN + ((uint32_t)(32 * q) << 16) + c * 32, r);
                const int n0 = nt * BN + c * 32;
                const float sw_lane = (n0 + lane < N) ? __ldg(w_scale + n0 + lane) : 0.0f;
                tmem_ld_wait();
                if (c == BN / 32 - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&S->tempty[buf]);
                }
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; i++) v[i] = (__uint_as_float(r[i]) * sa) * __shfl_sync(0xFFFFFFFFu, sw_lane, i);
                if (row >= M) continue;
                if (vec_ok && n0 + 32 <= N) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + n0);
#pragma unroll
                    for (int i = 0; i < 4; i++)
                        dst[i] = make_uint4(pack_bf16x2(v[8 * i], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                                            pack_bf16x2(v[8 * i + 4], v[8 * i + 5]),
                                            pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
                } else {
#pragma unroll
                    for (int i = 0; i < 32; i++)
                        if (n0 + i < N) orow[n0 + i] = __bfloat16_as_ushort(__float2bfloat16_rn(v[i]));
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

uint32_t take_timeouts_gemm_fp8() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_timeouts, sizeof(v)) != cudaSuccess) return 0xFFFFFFFFu;
    cudaMemcpyToSymbol(g_timeouts, &zero, sizeof(zero));
    return v;
}

cudaError_t launch_fp8_gemm_rowscale(const uint8_t *a, const float *a_scale, const uint8_t *w,
                                     const float *w_scale, uint16_t *out, int m, int n, int k, cudaStream_t s) {
    alignas(64) CUtensorMap tA, tB;
    if (!make_tmap_2d(&tA, a, 1, k, m, k, BK, BM, true, false) ||
        !make_tmap_2d(&tB, w, 1, k, n, k, BK, BN, true, false))
        return cudaErrorInvalidValue;
    static DeviceOnce attrs;
    cudaError_t e = attrs.run([] {
        return cudaFuncSetAttribute(k_fp8_gemm_rowscale, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    });
    if (e != cudaSuccess) return e;
    const int tiles = ((m + BM - 1) / BM) * ((n + BN - 1) / BN);
    const int grid = tiles < sm_count() ? tiles : sm_count();
    k_fp8_gemm_rowscale<<<grid, kThreads, kSmemBytes, s>>>(tA, tB, a_scale, w_scale, out, m, n, k);
    note_launch();
    return cudaGetLastError();
}

}  // namespace bsq
