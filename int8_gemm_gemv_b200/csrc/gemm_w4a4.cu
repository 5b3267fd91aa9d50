// NVFP4 x NVFP4 GEMM on the sm_100a block-scaled tensor cores
// (gemm_fp4.rs, `w4a4_gemm` and `w4a4_gemm_mfast`):
//   C[m, n] = scaleA2 * scaleB2 * sum_k e2m1(A) e4m3(sfA) e2m1(W) e4m3(sfW)
//
// Design (one CTA per SM, persistent over 128 x 256 output tiles):
//   warp 0       TMA producer: A [128 x 256 elem], W [256 x 256 elem] (packed,
//                128-byte swizzle) and the two raw scale tiles per K block,
//                into a 4-stage ring guarded by mbarriers.
//   warps 12..15 scale-factor writers: the scale tiles arrive row-major
//                ([rows, 16 bytes] per 256-wide K block); the MMA reads its
//                scales from tensor memory where, in every 32-lane group,
//                lane i of column j holds row 32j+i.  Each writer warp reads
//                the stage's scales from shared memory and stores them with
//                tcgen05.st into its own lane group (the layout is replicated
//                in all four groups).  Doing this with plain tensor-memory
//                stores keeps it off the tensor core's instruction queue, so
//                it overlaps the MMAs.
//   warp 1       MMA issuer (one thread): four 128x256x64 block-scaled MMAs
//                per K block into one FP32 accumulator in tensor memory.
//   warps 4..11  epilogue: tensor memory -> registers -> scale -> BF16 ->
//                global; warp w owns lane group w % 4 and column half
//                (w - 4) / 4 of the tile.
// Tiles go M-fastest, so consecutive CTAs share the same weight panel (the
// `w4a4_gemm_mfast` raster) and the whole working set stays in L2.
//
// Every mbarrier wait is bounded; on a timeout the kernel records it, stops
// issuing work, drains what it issued, frees tensor memory and exits.
#include "bsq_common.cuh"

namespace bsq {

namespace {

constexpr int BM = 128, BN = 256;
constexpr int BK_BYTES = 128;  // 256 FP4 elements
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK_BYTES;      // 16 KB
constexpr int B_BYTES = BN * BK_BYTES;      // 32 KB
constexpr int SFA_BYTES = BM * 16;          // 2 KB
constexpr int SFB_BYTES = BN * 16;          // 4 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr int TMEM_COLS = 512;
constexpr int ACC_COL = 0;                  // 256 FP32 columns
constexpr int SF_COL = 256;                 // per stage: 16 (A) + 32 (B)
constexpr int SF_STAGE_COLS = 48;
constexpr int kThreads = 512;

static __device__ unsigned int g_timeouts;

struct Smem {
    uint64_t full[STAGES];
    uint64_t sfready[STAGES];
    uint64_t empty[STAGES];
    uint64_t tfull, tempty, drain;
    uint32_t tmem_base;
    uint32_t abort;
};

constexpr size_t kSmemBytes = 1024 /* alignment slack */ + (size_t)STAGES * STAGE_BYTES + sizeof(Smem);

__device__ __forceinline__ bool aborted(volatile Smem *s) { return s->abort != 0; }

__global__ void __launch_bounds__(kThreads, 1)
    k_w4a4_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                uint16_t *__restrict__ out, float scale_ab, int M, int N, int K) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Smem *S = reinterpret_cast<Smem *>(base + (size_t)STAGES * STAGE_BYTES);
    auto a_tile = [&](int s) { return base + (size_t)s * STAGE_BYTES; };
    auto b_tile = [&](int s) { return base + (size_t)s * STAGE_BYTES + A_BYTES; };
    auto sfa_tile = [&](int s) { return base + (size_t)s * STAGE_BYTES + A_BYTES + B_BYTES; };
    auto sfb_tile = [&](int s) { return base + (size_t)s * STAGE_BYTES + A_BYTES + B_BYTES + SFA_BYTES; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles_m = (M + BM - 1) / BM, tiles_n = (N + BN - 1) / BN;
    const int num_tiles = tiles_m * tiles_n;
    const int nkb = K / 256;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; s++) {
            mbar_init(&S->full[s], 1);
            mbar_init(&S->sfready[s], 4);
            mbar_init(&S->empty[s], 1);
        }
        mbar_init(&S->tfull, 1);
        mbar_init(&S->tempty, 8);
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
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tensormap(&tmA);
            prefetch_tensormap(&tmB);
            prefetch_tensormap(&tmSFA);
            prefetch_tensormap(&tmSFB);
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
                    tma_load_2d(a_tile(s), &tmA, &S->full[s], kb * BK_BYTES, mt * BM);
                    tma_load_2d(b_tile(s), &tmB, &S->full[s], kb * BK_BYTES, nt * BN);
                    tma_load_2d(sfa_tile(s), &tmSFA, &S->full[s], kb * 16, mt * BM);
                    tma_load_2d(sfb_tile(s), &tmSFB, &S->full[s], kb * 16, nt * BN);
                }
            }
            if (!ok) {
                S->abort = 1;
                // let the copies already issued land before the CTA can exit
                const uint32_t first = it > STAGES ? it - STAGES : 0;
                for (uint32_t i = first; i < it; i++) mbar_wait(&S->full[i % STAGES], (i / STAGES) & 1, &g_timeouts);
            }
        }
    } else if (warp >= 12) {
        // ------------------------------------------ scale-factor writers
        const int q = warp & 3;
        const uint32_t lane_off = (uint32_t)(32 * q) << 16;
        uint32_t it = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
            for (int kb = 0; kb < nkb; kb++, it++) {
                const int s = it % STAGES;
                const uint32_t ph = (it / STAGES) & 1;
                if (!mbar_wait(&S->full[s], ph, &g_timeouts) || aborted(S)) {
                    ok = false;
                    break;
                }
                // raw tile: row r at r*16 bytes, word j = the 4 scales of MMA step j
                const uint4 *sa = reinterpret_cast<const uint4 *>(sfa_tile(s));
                const uint4 *sb = reinterpret_cast<const uint4 *>(sfb_tile(s));
                uint4 va[4], vb[8];
#pragma unroll
                for (int j = 0; j < 4; j++) va[j] = sa[32 * j + lane];
#pragma unroll
                for (int j = 0; j < 8; j++) vb[j] = sb[32 * j + lane];
                // column (step * groups + j) of this lane = row 32j + lane, step
                uint32_t ra[16], rb[32];
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    ra[0 + j] = va[j].x;
                    ra[4 + j] = va[j].y;
                    ra[8 + j] = va[j].z;
                    ra[12 + j] = va[j].w;
                }
#pragma unroll
                for (int j = 0; j < 8; j++) {
                    rb[0 + j] = vb[j].x;
                    rb[8 + j] = vb[j].y;
                    rb[16 + j] = vb[j].z;
                    rb[24 + j] = vb[j].w;
                }
                const uint32_t col = tmem + lane_off + SF_COL + s * SF_STAGE_COLS;
                tmem_st_32x32b_x16(col, ra);
                tmem_st_32x32b_x32(col + 16, rb);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&S->sfready[s]);
            }
        }
        if (!ok && lane == 0) S->abort = 1;
    } else if (warp == 1) {
        // --------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_nvf4(BM, BN);
            uint32_t it = 0, tc = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, tc++) {
                if (!mbar_wait(&S->tempty, (tc & 1) ^ 1, &g_timeouts) || aborted(S)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kb = 0; kb < nkb; kb++, it++) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait(&S->full[s], ph, &g_timeouts) || !mbar_wait(&S->sfready[s], ph, &g_timeouts) ||
                        aborted(S)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sfa_col = tmem + SF_COL + s * SF_STAGE_COLS;
                    const uint32_t sfb_col = sfa_col + 16;
                    const uint32_t a0 = smem_u32(a_tile(s)), b0 = smem_u32(b_tile(s));
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        mma_nvf4(tmem + ACC_COL, sdesc_k_sw128(a0 + 32 * j), sdesc_k_sw128(b0 + 32 * j), idesc,
                                 sfa_col + 4 * j, sfb_col + 8 * j, (kb | j) != 0);
                    }
                    tc_commit(&S->empty[s]);
                }
                if (!ok) break;
                tc_commit(&S->tfull);
            }
            if (!ok) S->abort = 1;
            // wait for every tensor-core operation this thread issued
            tc_commit(&S->drain);
            mbar_wait(&S->drain, 0, &g_timeouts);
        }
    } else if (warp >= 4) {
        // ----------------------------------------------------- epilogue
        const int q = warp & 3, h = (warp - 4) >> 2;
        uint32_t tc = 0;
        const bool vec_ok = (N % 8) == 0;
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, tc++) {
            const int mt = t % tiles_m, nt = t / tiles_m;
            if (!mbar_wait(&S->tfull, tc & 1, &g_timeouts) || aborted(S)) {
                if (lane == 0) S->abort = 1;
                break;
            }
            tc_fence_after();
            const int row = mt * BM + 32 * q + lane;
            uint16_t *orow = out + (int64_t)row * N;
#pragma unroll 1
            for (int cc = 0; cc < BN / 64; cc++) {
                const int c = h * (BN / 64) + cc;  // 32-column chunk of the tile
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem + ACC_COL + ((uint32_t)(32 * q) << 16) + c * 32, r);
                tmem_ld_wait();
                if (cc == BN / 64 - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&S->tempty);
                }
                if (row >= M) continue;
                const int n0 = nt * BN + c * 32;
                if (vec_ok && n0 + 32 <= N) {
                    uint32_t p[16];
#pragma unroll
                    for (int i = 0; i < 16; i++)
                        p[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * scale_ab, __uint_as_float(r[2 * i + 1]) * scale_ab);
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + n0);
#pragma unroll
                    for (int i = 0; i < 4; i++) dst[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; i++)
                        if (n0 + i < N)
                            orow[n0 + i] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(r[i]) * scale_ab));
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

uint32_t take_timeouts_gemm_w4a4() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_timeouts, sizeof(v)) != cudaSuccess) return 0xFFFFFFFFu;
    cudaMemcpyToSymbol(g_timeouts, &zero, sizeof(zero));
    return v;
}

cudaError_t launch_w4a4_gemm(const uint8_t *a_packed, const uint8_t *a_scale, const uint8_t *w_packed,
                             const uint8_t *w_scale, uint16_t *out, float scale_ab, int m, int n, int k,
                             cudaStream_t s) {
    alignas(64) CUtensorMap tA, tB, tSA, tSB;
    const uint64_t kb = (uint64_t)k / 2, ks = (uint64_t)k / 16;
    if (!make_tmap_2d(&tA, a_packed, 1, kb, m, kb, BK_BYTES, BM, true, false) ||
        !make_tmap_2d(&tB, w_packed, 1, kb, n, kb, BK_BYTES, BN, true, false) ||
        !make_tmap_2d(&tSA, a_scale, 1, ks, m, ks, 16, BM, false, false) ||
        !make_tmap_2d(&tSB, w_scale, 1, ks, n, ks, 16, BN, false, false))
        return cudaErrorInvalidValue;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(k_w4a4_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_done[dev] = true;
    }
    const int tiles = ((m + BM - 1) / BM) * ((n + BN - 1) / BN);
    const int grid = tiles < sm_count() ? tiles : sm_count();
    k_w4a4_gemm<<<grid, kThreads, kSmemBytes, s>>>(tA, tB, tSA, tSB, out, scale_ab, m, n, k);
    note_launch();
    return cudaGetLastError();
}

}  // namespace bsq
