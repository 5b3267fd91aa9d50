// NVFP4 x NVFP4 GEMM for few activation rows (M <= 128), the decode and
// small-batch regime of gemm_fp4.rs `w4a4_gemm`:
//   C[m, n] = scaleA2 * scaleB2 * sum_k e2m1(A) e4m3(sfA) e2m1(W) e4m3(sfW)
//
// With M this small the weight stream (N*K/2 bytes plus scales) is the cost
// and a 256-row A tile would waste most of every MMA.  So the operands are
// swapped: each CTA computes D = W_tile . A^T for 128 weight rows, with the
// weight tile as the MMA's M operand (128 rows) and all M activation rows,
// padded to NA = 32, 64 or 128, as its N operand.  D sits in tensor memory
// as 128 lanes (weight rows n) x NA columns (activation rows m) and is
// written out transposed.  One CTA per 128 weight rows: a 17408-row weight
// occupies 136 SMs, each streaming its rows through a deep TMA ring while
// the activation tile (identical for every CTA) comes from L2.
//
// Per CTA (512 threads):
//   warp 0        TMA producer: weight tile 128 x 128 B, activation tile
//                 NA x 128 B and both raw scale tiles per 256-wide K block.
//   warp 1        tensor-memory allocation and the MMA issuer (one thread).
//   warps 4..7    scale-factor writers: rewrite the row-major scale tiles
//                 into the tensor-memory layout (in every 32-lane group, lane
//                 i of column j holds row 32j+i, replicated in all four
//                 groups) with tcgen05.st.
//   warps 8..15   epilogue: warp w reads lane group w % 4 (32 weight rows)
//                 and half (w - 8) / 4 of the NA columns, scales, rounds to
//                 BF16 and stores out[m, n] (lanes = consecutive n).
// Launched with programmatic stream serialization, like the large kernel.
// Every mbarrier wait is bounded; on a timeout the kernel records it, stops
// issuing work, drains what it issued, frees tensor memory and exits.
#include "bsq_common.cuh"

namespace bsq {

namespace {

constexpr int BW = 128;                  // weight rows per CTA tile (MMA M)
constexpr int BK_BYTES = 128;            // 256 FP4 elements per K block
constexpr int W_BYTES = BW * BK_BYTES;   // 16 KB
constexpr int SFW_BYTES = BW * 16;       // 2 KB
constexpr int TMEM_COLS = 512;
constexpr int SF_COL = 128;              // scale columns start after the accumulator
constexpr int kThreads = 512;
constexpr int kEpiWarps = 8;

static __device__ unsigned int g_timeouts;

template <int NA>
struct Cfg {
    static constexpr int A_BYTES = NA * BK_BYTES;
    static constexpr int SFA_BYTES = NA * 16;
    static constexpr int DATA_BYTES = W_BYTES + A_BYTES + SFW_BYTES + SFA_BYTES;
    static constexpr int STAGE_BYTES = (DATA_BYTES + 1023) / 1024 * 1024;
    static constexpr int STAGES = (227 * 1024 - 2048) / STAGE_BYTES < 8 ? (227 * 1024 - 2048) / STAGE_BYTES : 8;
    static constexpr int GA = NA / 32;                   // scale columns of A per MMA step (1, 2 or 4)
    // per stage: W scales 4 steps x 4 columns, A scales 4 steps x GA
    // columns at a stride of 4, so every scale address is 4-column aligned
    static constexpr int SF_STAGE_COLS = 32;
    static_assert(SF_COL + STAGES * SF_STAGE_COLS <= TMEM_COLS, "tensor memory budget");
    static_assert(NA <= SF_COL, "accumulator columns");
};

// Rows of the activation boxes: NA, or 1 for a one-row activation.
template <int NA>
__host__ __device__ constexpr int act_box_rows(int m) {
    return m == 1 ? 1 : NA;
}

struct Smem {
    uint64_t full[8], sf_full[8], sfready[8], empty[8];
    uint64_t tfull, tempty, drain;
    uint32_t tmem_base;
    uint32_t abort;
};

template <int NA>
constexpr size_t smem_bytes() {
    return 1024 + (size_t)Cfg<NA>::STAGES * Cfg<NA>::STAGE_BYTES + sizeof(Smem);
}

__device__ __forceinline__ bool aborted(volatile Smem *s) { return s->abort != 0; }

template <int N>
__device__ __forceinline__ void ld_cols(uint32_t taddr, uint32_t (&r)[N]);
template <>
__device__ __forceinline__ void ld_cols<16>(uint32_t taddr, uint32_t (&r)[16]) {
    tmem_ld_32x32b_x16(taddr, r);
}
template <>
__device__ __forceinline__ void ld_cols<32>(uint32_t taddr, uint32_t (&r)[32]) {
    tmem_ld_32x32b_x32(taddr, r);
}
template <>
__device__ __forceinline__ void ld_cols<64>(uint32_t taddr, uint32_t (&r)[64]) {
    tmem_ld_32x32b_x64(taddr, r);
}

template <int NA>
__global__ void __launch_bounds__(kThreads, 1)
    k_w4a4_small(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW,
                 const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFW,
                 uint16_t *__restrict__ out, float scale_ab, const float *__restrict__ scale_b_dev, int M, int N,
                 int K) {
    using C = Cfg<NA>;
    constexpr int STAGES = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Smem *S = reinterpret_cast<Smem *>(base + (size_t)STAGES * C::STAGE_BYTES);
    auto w_tile = [&](int s) { return base + (size_t)s * C::STAGE_BYTES; };
    auto a_tile = [&](int s) { return base + (size_t)s * C::STAGE_BYTES + W_BYTES; };
    auto sfw_tile = [&](int s) { return base + (size_t)s * C::STAGE_BYTES + W_BYTES + C::A_BYTES; };
    auto sfa_tile = [&](int s) { return base + (size_t)s * C::STAGE_BYTES + W_BYTES + C::A_BYTES + SFW_BYTES; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_tiles = (N + BW - 1) / BW;
    const int nkb = K / 256;
    // Activation boxes have NA rows, the rows past M zero-filled by the
    // copy -- except for a single row (M = 1), where a one-row box is much
    // faster: its padding rows are zeroed here once and never copied.
    const int ma = act_box_rows<NA>(M);
    if (ma < NA) {
        for (int s = 0; s < STAGES; s++) {
            for (int i = ma * (BK_BYTES / 16) + threadIdx.x; i < NA * (BK_BYTES / 16); i += kThreads)
                reinterpret_cast<uint4 *>(a_tile(s))[i] = make_uint4(0u, 0u, 0u, 0u);
            for (int i = ma + threadIdx.x; i < NA; i += kThreads)
                reinterpret_cast<uint4 *>(sfa_tile(s))[i] = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
    }
    // per stage: the scale tiles on their own barrier, requested first, so the
    // writers move them into tensor memory while the operand tiles land
    const uint32_t sf_bytes = SFW_BYTES + (uint32_t)ma * 16, ab_bytes = W_BYTES + (uint32_t)ma * BK_BYTES;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; s++) {
            mbar_init(&S->full[s], 1);
            mbar_init(&S->sf_full[s], 1);
            mbar_init(&S->sfready[s], 4);
            mbar_init(&S->empty[s], 1);
        }
        mbar_init(&S->tfull, 1);
        mbar_init(&S->tempty, kEpiWarps);
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
            prefetch_tensormap(&tmW);
            prefetch_tensormap(&tmSFA);
            prefetch_tensormap(&tmSFW);
            // global memory is read only after the previous kernel of the
            // stream has completed (programmatic stream serialization)
            asm volatile("griddepcontrol.wait;" ::: "memory");
            uint32_t it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                for (int kb = 0; kb < nkb; kb++, it++) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait(&S->empty[s], ph ^ 1, &g_timeouts) || aborted(S)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&S->sf_full[s], sf_bytes);
                    tma_load_2d(sfw_tile(s), &tmSFW, &S->sf_full[s], kb * 16, t * BW);
                    tma_load_2d(sfa_tile(s), &tmSFA, &S->sf_full[s], kb * 16, 0);
                    mbar_arrive_expect_tx(&S->full[s], ab_bytes);
                    tma_load_2d(w_tile(s), &tmW, &S->full[s], kb * BK_BYTES, t * BW);
                    tma_load_2d(a_tile(s), &tmA, &S->full[s], kb * BK_BYTES, 0);
                }
            }
            if (!ok) {
                S->abort = 1;
                // let the copies already issued land before the CTA can exit
                const uint32_t first = it > STAGES ? it - STAGES : 0;
                for (uint32_t i = first; i < it; i++) {
                    mbar_wait(&S->sf_full[i % STAGES], (i / STAGES) & 1, &g_timeouts);
                    mbar_wait(&S->full[i % STAGES], (i / STAGES) & 1, &g_timeouts);
                }
            }
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------ scale-factor writers
        const int q = warp & 3;
        const uint32_t lane_off = (uint32_t)(32 * q) << 16;
        uint32_t it = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
            for (int kb = 0; kb < nkb; kb++, it++) {
                const int s = it % STAGES;
                if (!mbar_wait(&S->sf_full[s], (it / STAGES) & 1, &g_timeouts) || aborted(S)) {
                    ok = false;
                    break;
                }
                // raw tiles: row r at r*16 bytes, word j = the 4 scales of MMA step j
                const uint4 *sw = reinterpret_cast<const uint4 *>(sfw_tile(s));
                const uint4 *sa = reinterpret_cast<const uint4 *>(sfa_tile(s));
                uint4 vw[4], va[C::GA];
#pragma unroll
                for (int j = 0; j < 4; j++) vw[j] = sw[32 * j + lane];
#pragma unroll
                for (int j = 0; j < C::GA; j++) va[j] = sa[32 * j + lane];
                // column (step * groups + j) of this lane = row 32j + lane, step
                uint32_t rw[16], ra[16];
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    rw[0 + j] = vw[j].x;
                    rw[4 + j] = vw[j].y;
                    rw[8 + j] = vw[j].z;
                    rw[12 + j] = vw[j].w;
                    const bool used = j < C::GA;
                    ra[0 + j] = used ? va[used ? j : 0].x : 0u;
                    ra[4 + j] = used ? va[used ? j : 0].y : 0u;
                    ra[8 + j] = used ? va[used ? j : 0].z : 0u;
                    ra[12 + j] = used ? va[used ? j : 0].w : 0u;
                }
                const uint32_t col = tmem + lane_off + SF_COL + s * C::SF_STAGE_COLS;
                tmem_st_32x32b_x16(col, rw);
                tmem_st_32x32b_x16(col + 16, ra);
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
            const uint32_t idesc = idesc_nvf4(BW, NA);
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
                    // the MMA's A operand is the weight tile, B the activations
                    const uint32_t sfw_col = tmem + SF_COL + s * C::SF_STAGE_COLS;
                    const uint32_t sfa_col = sfw_col + 16;
                    const uint32_t w0 = smem_u32(w_tile(s)), a0 = smem_u32(a_tile(s));
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        mma_nvf4(tmem, sdesc_k_sw128(w0 + 32 * j), sdesc_k_sw128(a0 + 32 * j), idesc, sfw_col + 4 * j,
                                 sfa_col + 4 * j, (kb | j) != 0);
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
    } else if (warp >= 8) {
        // ----------------------------------------------------- epilogue
        constexpr int HALF = NA / 2;
        const int q = warp & 3, h = (warp - 8) >> 2;
        uint32_t tc = 0;
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, tc++) {
            if (!mbar_wait(&S->tfull, tc & 1, &g_timeouts) || aborted(S)) {
                if (lane == 0) S->abort = 1;
                break;
            }
            tc_fence_after();
            // the weight scale2 from device memory, after the producer's dependency wait
            if (scale_b_dev != nullptr && tc == 0) scale_ab = __fmul_rn(scale_ab, __ldg(scale_b_dev));
            uint32_t r[HALF];
            ld_cols<HALF>(tmem + ((uint32_t)(32 * q) << 16) + h * HALF, r);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S->tempty);
            // lane = weight row n, column c = activation row m
            const int n = t * BW + 32 * q + lane;
            if (n < N) {
#pragma unroll
                for (int c = 0; c < HALF; c++) {
                    const int m = h * HALF + c;
                    if (m < M)
                        out[(int64_t)m * N + n] =
                            __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(r[c]) * scale_ab));
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

template <int NA>
cudaError_t launch_na(const uint8_t *a_packed, const uint8_t *a_scale, const uint8_t *w_packed,
                      const uint8_t *w_scale, uint16_t *out, float scale_ab, const float *scale_b_dev, int m, int n,
                      int k, cudaStream_t s) {
    alignas(64) CUtensorMap tA, tW, tSA, tSW;
    const uint64_t kb = (uint64_t)k / 2, ks = (uint64_t)k / 16;
    const uint32_t ma = (uint32_t)act_box_rows<NA>(m);
    if (!make_tmap_2d(&tA, a_packed, 1, kb, m, kb, BK_BYTES, ma, true, false) ||
        !make_tmap_2d(&tW, w_packed, 1, kb, n, kb, BK_BYTES, BW, true, false) ||
        !make_tmap_2d(&tSA, a_scale, 1, ks, m, ks, 16, ma, false, false) ||
        !make_tmap_2d(&tSW, w_scale, 1, ks, n, ks, 16, BW, false, false))
        return cudaErrorInvalidValue;
    static DeviceOnce attrs;
    cudaError_t e = attrs.run([] {
        return cudaFuncSetAttribute(k_w4a4_small<NA>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)smem_bytes<NA>());
    });
    if (e != cudaSuccess) return e;
    const int tiles = (n + BW - 1) / BW;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(tiles < sm_count() ? tiles : sm_count());
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem_bytes<NA>();
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_w4a4_small<NA>, tA, tW, tSA, tSW, out, scale_ab, scale_b_dev, m, n, k);
}

}  // namespace

uint32_t take_timeouts_gemm_w4a4_small() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_timeouts, sizeof(v)) != cudaSuccess) return 0xFFFFFFFFu;
    cudaMemcpyToSymbol(g_timeouts, &zero, sizeof(zero));
    return v;
}

cudaError_t launch_w4a4_gemm_small(const uint8_t *a_packed, const uint8_t *a_scale, const uint8_t *w_packed,
                                   const uint8_t *w_scale, uint16_t *out, float scale_ab, const float *scale_b_dev,
                                   int m, int n, int k, cudaStream_t s) {
    cudaError_t e;
    if (m <= 32)
        e = launch_na<32>(a_packed, a_scale, w_packed, w_scale, out, scale_ab, scale_b_dev, m, n, k, s);
    else if (m <= 64)
        e = launch_na<64>(a_packed, a_scale, w_packed, w_scale, out, scale_ab, scale_b_dev, m, n, k, s);
    else
        e = launch_na<128>(a_packed, a_scale, w_packed, w_scale, out, scale_ab, scale_b_dev, m, n, k, s);
    note_launch();
    return e;
}

}  // namespace bsq
