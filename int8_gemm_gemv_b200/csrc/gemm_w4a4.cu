// NVFP4 x NVFP4 GEMM on the sm_100a block-scaled tensor cores
// (gemm_fp4.rs, `w4a4_gemm` and `w4a4_gemm_mfast`):
//   C[m, n] = scaleA2 * scaleB2 * sum_k e2m1(A) e4m3(sfA) e2m1(W) e4m3(sfW)
//
// Design: CTA pairs (clusters of two SMs), persistent over 256 x 256 output
// tiles.  One pair MMA (tcgen05.mma.cta_group::2, 256 x 256 x 64) runs on
// both SMs' tensor cores: each CTA holds 128 rows of A and 128 of the 256
// weight rows in its shared memory and receives 128 x 256 of the output in
// its tensor memory.  Each SM therefore loads half the weight tile a 1-SM
// 128 x 256 tile would need, which is what lets the FP4 tensor cores be
// fed from L2.
//
// Per CTA (512 threads):
//   warp 0        TMA producer of A and the weight halves: a 5-stage ring;
//                 their arrival is counted on the even CTA's barrier (the
//                 MMA issuer's).
//   warp 2        TMA producer of the raw scale tiles (A: own 128 rows, W:
//                 all 256 rows), into a ring of their own that refills as
//                 soon as the writers have moved a slot into tensor memory,
//                 so a stage's scales land well before its A and W tiles.
//   warps 12..15  scale-factor writers: the scale tiles arrive row-major
//                 ([rows, 16 bytes] per 256-wide K block); the MMA reads its
//                 scales from tensor memory where, in every 32-lane group,
//                 lane i of column j holds row 32j+i.  Once the stage's
//                 tensor-memory slot is free they write that layout with
//                 tcgen05.st (off the tensor core's queue) and tell the even
//                 CTA.
//   warp 1        tensor-memory allocation for the pair; in the even CTA,
//                 lane 0 issues the pair MMAs and commits them to both CTAs.
//   warps 4..11   epilogue: tensor memory -> registers -> scale -> BF16 ->
//                 swizzled shared-memory staging -> TMA store; warp w owns
//                 lane group w % 4 and column half (w - 4) / 4 of the CTA's
//                 128 x 256 block, and releases tensor memory as soon as its
//                 part is in registers.
// Tiles go M-fastest, so consecutive pairs share the same weight panel (the
// `w4a4_gemm_mfast` raster) and the working set stays in L2.  No load uses
// cluster multicast.
//
// Launched with programmatic stream serialization: the set-up overlaps the
// previous kernel of the stream, and the producer waits for it
// (griddepcontrol.wait) before the first global load.
//
// Every mbarrier wait is bounded; on a timeout the kernel records it, stops
// issuing work, drains what it issued, frees tensor memory and exits.
#include <cstring>

#include "bsq_common.cuh"

namespace bsq {

namespace {

constexpr int BM = 128;                  // rows of A per CTA (256 per pair)
constexpr int BN = 256;                  // output columns per tile
constexpr int BNH = BN / 2;              // weight rows per CTA
constexpr int BK_BYTES = 128;            // 256 FP4 elements
constexpr int STAGES = 5;
constexpr int A_BYTES = BM * BK_BYTES;   // 16 KB
constexpr int B_BYTES = BNH * BK_BYTES;  // 16 KB
constexpr int SFA_BYTES = BM * 16;       // 2 KB
constexpr int SFB_BYTES = BN * 16;       // 4 KB (all 256 weight rows)
constexpr int AB_STAGE_BYTES = A_BYTES + B_BYTES;      // 32 KB
constexpr int SF_STAGE_BYTES = SFA_BYTES + SFB_BYTES;  // 6 KB
constexpr int TMEM_COLS = 512;
constexpr int ACC_COL = 0;               // 256 FP32 columns
constexpr int SF_COL = 256;              // per stage: 16 (A) + 32 (W)
constexpr int SF_STAGE_COLS = 48;
constexpr int kThreads = 512;
constexpr int kEpiWarps = 8, kSfWarps = 4;
// output staging: per epilogue warp one TMA store box of 32 rows x 64
// columns of BF16 (128-byte rows, 128-byte swizzle), used twice per tile
constexpr int OUT_BOX_COLS = 64, OUT_BOX_ROWS = 32;
constexpr int OUT_BOX_BYTES = OUT_BOX_COLS * 2 * OUT_BOX_ROWS;  // 4 KB
constexpr int OUT_WARP_BYTES = OUT_BOX_BYTES;
constexpr int OUT_BYTES = kEpiWarps * OUT_WARP_BYTES;             // 32 KB

static_assert(AB_STAGE_BYTES % 1024 == 0 && SF_STAGE_BYTES % 128 == 0, "stage alignment");
static_assert(SF_COL + STAGES * SF_STAGE_COLS <= TMEM_COLS, "tensor memory budget");

static __device__ unsigned int g_timeouts;

struct Smem {
    uint64_t ab_full[STAGES];  // even CTA: A + W halves of both CTAs landed
    uint64_t sf_full[STAGES];  // local: raw scale tiles landed
    uint64_t sfready[STAGES];  // even CTA: both CTAs' scales are in tensor memory
    uint64_t empty[STAGES];    // local: the pair MMAs of this stage are done
    uint64_t sf_empty[STAGES]; // local: the scale slot's tiles are in tensor memory
    uint64_t tfull, tempty, drain;
    uint32_t tmem_base;
    uint32_t abort;
};

constexpr size_t kSmemBytes = 1024 + (size_t)STAGES * (AB_STAGE_BYTES + SF_STAGE_BYTES) + OUT_BYTES + sizeof(Smem);

__device__ __forceinline__ bool aborted(volatile Smem *s) { return s->abort != 0; }

__global__ void __launch_bounds__(kThreads, 1)
    k_w4a4_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                const __grid_constant__ CUtensorMap tmOut, int use_tma_store, uint16_t *__restrict__ out,
                float scale_ab, const float *__restrict__ scale_b_dev, int M, int N, int K) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sf_base = base + (size_t)STAGES * AB_STAGE_BYTES;
    uint8_t *out_stage = sf_base + (size_t)STAGES * SF_STAGE_BYTES;
    Smem *S = reinterpret_cast<Smem *>(out_stage + OUT_BYTES);
    auto a_tile = [&](int s) { return base + (size_t)s * AB_STAGE_BYTES; };
    auto b_tile = [&](int s) { return base + (size_t)s * AB_STAGE_BYTES + A_BYTES; };
    auto sfa_tile = [&](int s) { return sf_base + (size_t)s * SF_STAGE_BYTES; };
    auto sfb_tile = [&](int s) { return sf_base + (size_t)s * SF_STAGE_BYTES + SFA_BYTES; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0: issues the pair MMAs
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int tiles_m = (M + 2 * BM - 1) / (2 * BM), tiles_n = (N + BN - 1) / BN;
    const int num_tiles = tiles_m * tiles_n;
    const int nkb = K / 256;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; s++) {
            mbar_init(&S->ab_full[s], 1);
            mbar_init(&S->sf_full[s], 1);
            mbar_init(&S->sfready[s], 2 * kSfWarps);
            mbar_init(&S->empty[s], 1);
            mbar_init(&S->sf_empty[s], kSfWarps);
        }
        mbar_init(&S->tfull, 1);
        mbar_init(&S->tempty, 2 * kEpiWarps);
        mbar_init(&S->drain, 1);
        S->abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(&S->tmem_base, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers exist before any cross-CTA signal
    tc_fence_after();
    const uint32_t tmem = S->tmem_base;
    // cluster addresses of the even CTA's barriers
    auto leader = [&](uint64_t *bar) { return mapa_shared(smem_u32(bar), 0); };

    if (warp == 0) {
        // ------------------------------------------- TMA producer: A, W
        if (lane == 0) {
            prefetch_tensormap(&tmA);
            prefetch_tensormap(&tmB);
            // everything above overlapped the previous kernel of the stream
            // (programmatic stream serialization); global memory is read
            // from here on, after it has completed.  Every other role's
            // global access depends on these loads.
            asm volatile("griddepcontrol.wait;" ::: "memory");
            uint32_t it = 0;
            bool ok = true;
            for (int t = pair; t < num_tiles && ok; t += npairs) {
                const int mt = t % tiles_m, nt = t / tiles_m;
                const int arow = mt * 2 * BM + (int)rank * BM, brow = nt * BN + (int)rank * BNH;
                for (int kb = 0; kb < nkb; kb++, it++) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait(&S->empty[s], ph ^ 1, &g_timeouts) || aborted(S)) {
                        ok = false;
                        break;
                    }
                    if (rank == 0) mbar_arrive_expect_tx(&S->ab_full[s], 2 * (A_BYTES + B_BYTES));
                    const uint32_t abar = leader(&S->ab_full[s]);
                    tma_load_2d_pair(a_tile(s), &tmA, abar, kb * BK_BYTES, arow);
                    tma_load_2d_pair(b_tile(s), &tmB, abar, kb * BK_BYTES, brow);
                }
            }
            if (!ok) S->abort = 1;
        }
    } else if (warp == 2) {
        // -------------------------------------- TMA producer: scale tiles
        // Its own ring: a slot is refilled as soon as the writers have moved
        // its tiles into tensor memory, so the scales of a stage arrive
        // several stages before its A and W tiles.
        if (lane == 0) {
            prefetch_tensormap(&tmSFA);
            prefetch_tensormap(&tmSFB);
            asm volatile("griddepcontrol.wait;" ::: "memory");
            uint32_t it = 0;
            bool ok = true;
            for (int t = pair; t < num_tiles && ok; t += npairs) {
                const int mt = t % tiles_m, nt = t / tiles_m;
                const int arow = mt * 2 * BM + (int)rank * BM;
                for (int kb = 0; kb < nkb; kb++, it++) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait(&S->sf_empty[s], ph ^ 1, &g_timeouts) || aborted(S)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&S->sf_full[s], SFA_BYTES + SFB_BYTES);
                    tma_load_2d(sfa_tile(s), &tmSFA, &S->sf_full[s], kb * 16, arow);
                    tma_load_2d(sfb_tile(s), &tmSFB, &S->sf_full[s], kb * 16, nt * BN);
                }
            }
            if (!ok) {
                S->abort = 1;
                // let this CTA's scale copies land before it can exit
                const uint32_t first = it > STAGES ? it - STAGES : 0;
                for (uint32_t i = first; i < it; i++)
                    mbar_wait(&S->sf_full[i % STAGES], (i / STAGES) & 1, &g_timeouts);
            }
        }
    } else if (warp >= 4 + kEpiWarps) {
        // ------------------------------------------ scale-factor writers
        const int q = warp & 3;
        const uint32_t lane_off = (uint32_t)(32 * q) << 16;
        uint32_t it = 0;
        bool ok = true;
        for (int t = pair; t < num_tiles && ok; t += npairs) {
            for (int kb = 0; kb < nkb; kb++, it++) {
                const int s = it % STAGES;
                const uint32_t ph = (it / STAGES) & 1;
                // the stage's tiles, and its tensor-memory slot: free once the
                // pair MMAs of the stage STAGES earlier are done
                if (!mbar_wait(&S->sf_full[s], ph, &g_timeouts) || !mbar_wait(&S->empty[s], ph ^ 1, &g_timeouts) ||
                    aborted(S)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
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
                if (lane == 0) {
                    mbar_arrive(&S->sf_empty[s]);
                    mbar_arrive_cluster(leader(&S->sfready[s]));
                }
            }
        }
        if (!ok && lane == 0) S->abort = 1;
    } else if (warp == 1) {
        // ---------------------------------------- pair MMA issuer (even CTA)
        if (lane == 0 && rank == 0) {
            const uint32_t idesc = idesc_nvf4(2 * BM, BN);
            uint32_t it = 0, tc = 0;
            bool ok = true;
            for (int t = pair; t < num_tiles && ok; t += npairs, tc++) {
                if (!mbar_wait_cluster(&S->tempty, (tc & 1) ^ 1, &g_timeouts) || aborted(S)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kb = 0; kb < nkb; kb++, it++) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait(&S->ab_full[s], ph, &g_timeouts) ||
                        !mbar_wait_cluster(&S->sfready[s], ph, &g_timeouts) || aborted(S)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sfa_col = tmem + SF_COL + s * SF_STAGE_COLS;
                    const uint32_t sfb_col = sfa_col + 16;
                    const uint32_t a0 = smem_u32(a_tile(s)), b0 = smem_u32(b_tile(s));
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        mma_nvf4_pair(tmem + ACC_COL, sdesc_k_sw128(a0 + 32 * j), sdesc_k_sw128(b0 + 32 * j), idesc,
                                      sfa_col + 4 * j, sfb_col + 8 * j, (kb | j) != 0);
                    }
                    tc_commit_pair_multicast(&S->empty[s], 0x3);
                }
                if (!ok) break;
                tc_commit_pair_multicast(&S->tfull, 0x3);
            }
            if (!ok) S->abort = 1;
            // wait for every tensor-core operation this thread issued
            tc_commit_pair_multicast(&S->drain, 0x1);
            mbar_wait(&S->drain, 0, &g_timeouts);
        }
    } else if (warp >= 4) {
        // ----------------------------------------------------- epilogue
        // Drain the whole accumulator block into registers (packed BF16)
        // before releasing tensor memory, so the next tile's MMAs never wait
        // behind this tile's global stores; then write through shared memory
        // with TMA stores (coalesced, asynchronous).
        const int q = warp & 3, h = (warp - 4) >> 2;
        uint8_t *stage = out_stage + (warp - 4) * OUT_WARP_BYTES;
        bool scale_read = scale_b_dev == nullptr;
        uint32_t tc = 0;
        const uint32_t tempty_leader = leader(&S->tempty);
        if (lane == 0) prefetch_tensormap(&tmOut);
        for (int t = pair; t < num_tiles; t += npairs, tc++) {
            const int mt = t % tiles_m, nt = t / tiles_m;
            if (!mbar_wait(&S->tfull, tc & 1, &g_timeouts) || aborted(S)) {
                if (lane == 0) S->abort = 1;
                break;
            }
            tc_fence_after();
            if (!scale_read) {  // the weight scale2 from device memory, after the producer's dependency wait
                scale_ab = __fmul_rn(scale_ab, __ldg(scale_b_dev));
                scale_read = true;
            }
            const uint32_t tbase = tmem + ACC_COL + ((uint32_t)(32 * q) << 16) + h * 128;
            uint32_t pk[64];  // 128 columns of this lane's row as BF16 pairs
#pragma unroll
            for (int half = 0; half < 2; half++) {
                uint32_t r0[32], r1[32];
                tmem_ld_32x32b_x32(tbase + half * 64, r0);
                tmem_ld_32x32b_x32(tbase + half * 64 + 32, r1);
                tmem_ld_wait();
                if (half == 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(tempty_leader);
                }
#pragma unroll
                for (int i = 0; i < 16; i++) {
                    pk[half * 32 + i] = pack_bf16x2(__uint_as_float(r0[2 * i]) * scale_ab,
                                                    __uint_as_float(r0[2 * i + 1]) * scale_ab);
                    pk[half * 32 + 16 + i] = pack_bf16x2(__uint_as_float(r1[2 * i]) * scale_ab,
                                                         __uint_as_float(r1[2 * i + 1]) * scale_ab);
                }
            }
            const int row0 = mt * 2 * BM + (int)rank * BM + 32 * q;  // first row of this warp
            const int col0 = nt * BN + h * 128;
            if (use_tma_store) {
                // box bx holds columns [64bx, 64bx+64) of the warp's 32 x 128
                // block; lane = row; 16-byte unit u of a row sits at u ^ (row & 7)
#pragma unroll
                for (int bx = 0; bx < 2; bx++) {
                    // the previous store must have finished reading the box
                    if (lane == 0) bulk_wait_group_read0();
                    __syncwarp();
#pragma unroll
                    for (int u = 0; u < 8; u++) {
                        const uint32_t off = lane * 128 + ((u ^ (lane & 7)) << 4);
                        *reinterpret_cast<uint4 *>(stage + off) =
                            make_uint4(pk[bx * 32 + 4 * u], pk[bx * 32 + 4 * u + 1], pk[bx * 32 + 4 * u + 2],
                                       pk[bx * 32 + 4 * u + 3]);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    // boxes past the last row or column are skipped
                    if (lane == 0 && row0 < M && col0 + bx * OUT_BOX_COLS < N) {
                        tma_store_2d(&tmOut, stage, col0 + bx * OUT_BOX_COLS, row0);
                        bulk_commit_group();
                    }
                }
            } else {
                const int row = row0 + lane;
                if (row < M) {
                    uint16_t *orow = out + (int64_t)row * N;
#pragma unroll
                    for (int i = 0; i < 64; i++) {
                        const int n = col0 + 2 * i;
                        if (n < N) orow[n] = (uint16_t)(pk[i] & 0xFFFF);
                        if (n + 1 < N) orow[n + 1] = (uint16_t)(pk[i] >> 16);
                    }
                }
            }
        }
        if (lane == 0) bulk_wait_group0();  // stores complete before the CTA exits
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // no pair MMA or cross-CTA signal is in flight after this
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, TMEM_COLS);
    }
}

}  // namespace

uint32_t take_timeouts_gemm_w4a4() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_timeouts, sizeof(v)) != cudaSuccess) return 0xFFFFFFFFu;
    cudaMemcpyToSymbol(g_timeouts, &zero, sizeof(zero));
    return v;
}

// CTA pairs that can be resident at once (cached per device).
static int w4a4_max_pairs(cudaLaunchConfig_t cfg) {
    // a racing first call computes the same value twice; the store is atomic
    static std::atomic<int> cached[kMaxDevices];
    int dev = 0;
    cudaGetDevice(&dev);
    const bool cacheable = dev >= 0 && dev < kMaxDevices;
    if (cacheable) {
        const int c = cached[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int n = 0;
    cfg.gridDim = dim3(sm_count());
    if (cudaOccupancyMaxActiveClusters(&n, k_w4a4_gemm, &cfg) != cudaSuccess || n <= 0) n = sm_count() / 2;
    if (cacheable) cached[dev].store(n, std::memory_order_relaxed);
    return n;
}

cudaError_t launch_w4a4_gemm(const uint8_t *a_packed, const uint8_t *a_scale, const uint8_t *w_packed,
                             const uint8_t *w_scale, uint16_t *out, float scale_ab, const float *scale_b_dev,
                             int m, int n, int k, cudaStream_t s) {
    alignas(64) CUtensorMap tA, tB, tSA, tSB;
    const uint64_t kb = (uint64_t)k / 2, ks = (uint64_t)k / 16;
    // TMA stores need 16-byte output rows (n % 8 == 0); otherwise plain stores
    alignas(64) CUtensorMap tO;
    const int use_tma_store = (n % 8) == 0;
    if (use_tma_store && !make_tmap_2d(&tO, out, 2, n, m, (uint64_t)n * 2, OUT_BOX_COLS, OUT_BOX_ROWS, true, false))
        return cudaErrorInvalidValue;
    if (!use_tma_store) memset(&tO, 0, sizeof(tO));
    if (!make_tmap_2d(&tA, a_packed, 1, kb, m, kb, BK_BYTES, BM, true, false) ||
        !make_tmap_2d(&tB, w_packed, 1, kb, n, kb, BK_BYTES, BNH, true, false) ||
        !make_tmap_2d(&tSA, a_scale, 1, ks, m, ks, 16, BM, false, false) ||
        !make_tmap_2d(&tSB, w_scale, 1, ks, n, ks, 16, BN, false, false))
        return cudaErrorInvalidValue;
    static DeviceOnce attrs;
    cudaError_t e = attrs.run([] {
        return cudaFuncSetAttribute(k_w4a4_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    });
    if (e != cudaSuccess) return e;
    const int tiles = ((m + 2 * BM - 1) / (2 * BM)) * ((n + BN - 1) / BN);
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const int max_pairs = w4a4_max_pairs(cfg);
    // the prologue (barriers, tensor memory, descriptor prefetch) may
    // overlap the previous kernel, e.g. the activation quantiser's tail
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.numAttrs = 2;
    const int pairs = tiles < max_pairs ? tiles : max_pairs;
    cfg.gridDim = dim3(2 * pairs);
    e = cudaLaunchKernelEx(&cfg, k_w4a4_gemm, tA, tB, tSA, tSB, tO, use_tma_store, out, scale_ab,
                                       scale_b_dev, m, n, k);
    note_launch();
    return e;
}

}  // namespace bsq
