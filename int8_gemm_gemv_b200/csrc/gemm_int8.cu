// int8 x int8 GEMM with per-32 FP32 block scales on both operands
// (gemm_dense_int8.rs, `int8_gemm_faith2_prefill` step (b)):
//   C[m, n] = sum_b (exact int32 sum_{k in b} a*w) * a_scale[m, b] * w_scale[n, b]
//
// The scales change every 32 K, which is exactly one int8 MMA K step, so the
// tensor cores cannot accumulate across blocks.  Each 128x128x32 MMA writes a
// fresh int32 partial into one of four tensor-memory buffers (4 x 128
// columns); sixteen "fold" warps read each partial back and fold it into FP32
// registers with its two scales while the tensor cores already compute the
// next ones.  The fold on the CUDA cores is the bound of this kernel, not the
// int8 MMA.
//
// No int32 -> FP32 convert in the fold.  Before each block's int8 MMA, an
// FP16 MMA over a constant tile (every element 768, K = 16) writes the FP32
// value C = 16 * 768^2 = 9 * 2^20 into every word of the buffer, and the
// int8 MMA accumulates onto those bits as an int32.  A block's partial p has
// |p| <= 32 * 128 * 128 = 2^19, and C +- 2^19 stays inside [2^23, 2^24),
// where consecutive FP32 encodings are consecutive integers: the buffer then
// holds the FP32 encoding of exactly C + p, and one FP32 subtraction gives p
// back exactly.  The fold is one subtraction, one scale product and one FMA
// per output and block, all packed two-wide on the FMA pipe.
//
//   warp 0       TMA producer: A, W tiles (128 x 128 B) and their scale tiles
//                (128 rows x 4 FP32) into a 6-stage ring
//   warp 1       MMA issuer
//   warp 2       rewrites each stage's W-scale tile from [n][4] to [4][n]
//   warps 4..19  fold + epilogue; warp w owns tensor-memory lane quarter
//                w % 4 (rows) and column quarter (w - 4) / 4: a 32 x 32
//                sub-tile of every partial
//
// The fold reads partials with the 16-lane x 256-bit tensor-memory shape: a
// thread holds 4 rows x 8 columns of its warp's sub-tile, so it needs 4 row
// scales and 4 column-scale pairs per block (each pair shared by 8 lanes).
// The two 16-row halves of a partial are loaded one ahead of the other, so
// each half is folded while the next is in flight.  Four fold warps per
// SM sub-partition hide the remaining latency; to fit them, warps 0-3 give
// up registers (setmaxnreg).
//
// Tiles go round-robin over one CTA per SM.  With a caller workspace, a last
// round that would leave most SMs idle is split along K: each of its tiles
// becomes S pieces on S CTAs.  A piece stores its FP32 sums in the
// workspace and counts itself in the tile's counter; the piece that counts
// last adds all S in piece order (so the result never depends on which
// finished last), stores the tile and puts the counter back to zero.
#include "bsq_common.cuh"

namespace bsq {

namespace {

constexpr int BM = 128, BN = 128, BK = 128;  // BK bytes = elements = 4 blocks of 32
constexpr int STAGES = 6;
constexpr int A_BYTES = BM * BK, B_BYTES = BN * BK;
constexpr int SA_BYTES = BM * 16, SW_BYTES = BN * 16;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SA_BYTES + SW_BYTES;
constexpr int OFS_BYTES = 4096;  // constant tile: 128 x 16 FP16, both operands of the offset MMA
constexpr int NACC = 4;  // tensor-memory partial buffers of 128 columns
constexpr int TMEM_COLS = 512;
constexpr int NFOLD = 16;
constexpr int kThreads = 32 * (4 + NFOLD);
// Register split: the block is launched with kLaunchRegs per thread; warps
// 0-3 (one warpgroup) drop to kCtlRegs and the two fold warpgroups take the
// rest.  The launcher checks the compiled count before the first launch.
constexpr int kLaunchRegs = 96, kCtlRegs = 48, kFoldRegs = 104;
static_assert(128 * kCtlRegs + 32 * NFOLD * kFoldRegs <= kThreads * kLaunchRegs, "register split");

static __device__ unsigned int g_timeouts;

struct Smem {
    uint64_t full[STAGES];
    uint64_t swready[STAGES];
    uint64_t empty[STAGES];
    uint64_t acc_full[NACC], acc_empty[NACC];
    uint64_t drain;
    uint32_t tmem_base;
    uint32_t abort;
    uint32_t last_piece;  // this CTA's piece was the last of its tile
    uint64_t fold_bar;    // the 16 fold warps of a split-tile hand-off (two phases)
};

constexpr size_t kSmemBytes = 1024 + (size_t)STAGES * STAGE_BYTES + OFS_BYTES + sizeof(Smem);
static_assert(kSmemBytes <= 232448, "shared memory per block");

__device__ __forceinline__ bool aborted(volatile Smem *s) { return s->abort != 0; }

template <int R> __device__ __forceinline__ void setmaxnreg_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R));
}
template <int R> __device__ __forceinline__ void setmaxnreg_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R));
}

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
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    float2 d;
    asm("add.rn.f32x2 %0, %1, %2;"
        : "=l"(*reinterpret_cast<uint64_t *>(&d))
        : "l"(*reinterpret_cast<uint64_t *>(&a)), "l"(*reinterpret_cast<uint64_t *>(&b)));
    return d;
}

// Offset under every int32 partial: the FP16 MMA over the constant tile sums
// 16 products 768 * 768 (all exact in FP32).
constexpr uint16_t kOffsetHalfBits = 0x6200u;  // FP16 768 = 1.5 * 2^9
constexpr float kOffset = 9437184.0f;         // 16 * 768^2 = 9 * 2^20
static_assert(kOffset - 524288.0f >= 8388608.0f && kOffset + 524288.0f < 16777216.0f,
              "offset +- 2^19 must stay in the FP32 binade of spacing 1");

// The i-th tile of this CTA: tile t over K blocks [kb0, kb1) (blocks of BK),
// piece `piece` of `split` pieces when split > 1.  False past the CTA's last
// tile.  Every role walks the same list.
struct ITile {
    int t, kb0, kb1, piece;
};
__device__ __forceinline__ bool int8_tile(int i, int num_tiles, int nkb, int split, ITile &o) {
    const int G = gridDim.x, b = blockIdx.x;
    const int full = num_tiles / G, rem = num_tiles % G;
    if (i < full) {
        o = {b + i * G, 0, nkb, 0};
        return true;
    }
    if (i != full || rem == 0) return false;
    if (split > 1) {
        if (b >= rem * split) return false;
        const int r = b / split, p = b % split;
        o = {full * G + r, p * nkb / split, (p + 1) * nkb / split, p};
        return true;
    }
    if (b >= rem) return false;
    o = {full * G + b, 0, nkb, 0};
    return true;
}

// Pieces per tile of the last round: up to four, as many as the idle CTAs
// allow, 1 when that round is full or K has a single block.
__host__ __device__ __forceinline__ int int8_split(int num_tiles, int grid, int nkb) {
    const int rem = num_tiles % grid;
    if (rem == 0) return 1;
    int sp = grid / rem;
    sp = sp < 4 ? sp : 4;
    sp = sp < nkb ? sp : nkb;
    return sp > 1 ? sp : 1;
}

__global__ void __launch_bounds__(kThreads, 1)
    k_int8_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSW,
                uint16_t *__restrict__ out, int M, int N, int K, float *__restrict__ ws_part,
                uint32_t *__restrict__ ws_cnt, int split) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ofs_tile = base + (size_t)STAGES * STAGE_BYTES;  // 1024-aligned
    Smem *S = reinterpret_cast<Smem *>(ofs_tile + OFS_BYTES);
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
        mbar_init(&S->fold_bar, NFOLD);
        S->abort = 0;
        fence_mbar_init();
    }
    if (threadIdx.x < OFS_BYTES / 16) {
        const uint32_t h2 = (uint32_t)kOffsetHalfBits * 0x10001u;
        reinterpret_cast<uint4 *>(ofs_tile)[threadIdx.x] = make_uint4(h2, h2, h2, h2);
        fence_proxy_async_smem();  // visible to the tensor cores
    }
    if (warp == 1) {
        tmem_alloc(&S->tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S->tmem_base;
    if (warp < 4) setmaxnreg_dec<kCtlRegs>();

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tensormap(&tmA);
            prefetch_tensormap(&tmB);
            prefetch_tensormap(&tmSA);
            prefetch_tensormap(&tmSW);
            uint32_t it = 0;
            bool ok = true;
            ITile tl;
            for (int ti = 0; ok && int8_tile(ti, num_tiles, nkb, split, tl); ti++) {
                const int mt = tl.t % tiles_m, nt = tl.t / tiles_m;
                for (int kb = tl.kb0; kb < tl.kb1; kb++, it++) {
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
        ITile tl;
        for (int ti = 0; ok && int8_tile(ti, num_tiles, nkb, split, tl); ti++) {
            for (int kb = tl.kb0; kb < tl.kb1; kb++, it++) {
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
            const uint32_t idesc_ofs = idesc_f16(BM, BN);
            const uint64_t dofs = sdesc_k_none_128x32(smem_u32(ofs_tile));
            uint32_t it = 0, gs = 0;
            bool ok = true;
            ITile tl;
            for (int ti = 0; ok && int8_tile(ti, num_tiles, nkb, split, tl); ti++) {
                for (int kb = tl.kb0; kb < tl.kb1 && ok; kb++, it++) {
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
                        // offset C into the buffer, then the block's int8
                        // partial on top of it (MMAs of one thread run in order)
                        mma_f16(tmem + b * BN, dofs, dofs, idesc_ofs, 0);
                        mma_i8(tmem + b * BN, sdesc_k_sw128(a0 + 32 * j), sdesc_k_sw128(b0 + 32 * j), idesc, 1);
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
        setmaxnreg_inc<kFoldRegs>();
        const int q = warp & 3, h = (warp - 4) >> 2;
        // this warp's 32 x 32 sub-tile: lanes 32q.., columns 32h..
        const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16) + 32 * h;
        const int r0 = 32 * q + (lane >> 2);  // rows r0, r0 + 8 (upper half), r0 + 16, r0 + 24 (lower half)
        const int c0 = 32 * h + 2 * (lane & 3);  // columns c0 + 8g, c0 + 8g + 1
        uint32_t it = 0, gs = 0;
        bool ok = true;
        uint32_t RA[16], RB[16];  // upper / lower 16 rows of the sub-tile
        float2 acc[16];           // [row 0..3][group 0..3], a column pair each
        // (no abort-flag read per block: if another role gives up, no more
        // partials are committed and this bounded wait ends the fold)
        auto wait_full = [&](uint32_t g) -> bool {
            if (!mbar_wait(&S->acc_full[g % NACC], (g / NACC) & 1, &g_timeouts)) return false;
            tc_fence_after();
            return true;
        };
        // rows u0, u0 + 1 of the accumulator from one 16-row half
        auto fold_half = [&](const uint32_t (&R)[16], int u0, float s0, float s1, const float2 (&w2)[4]) {
            const float2 off = make_float2(-kOffset, -kOffset);
#pragma unroll
            for (int g = 0; g < 4; g++) {
                const float2 c0v = mul2(make_float2(s0, s0), w2[g]);
                const float2 c1v = mul2(make_float2(s1, s1), w2[g]);
                const float2 p0 = add2(make_float2(__uint_as_float(R[4 * g]), __uint_as_float(R[4 * g + 1])), off);
                const float2 p1 = add2(make_float2(__uint_as_float(R[4 * g + 2]), __uint_as_float(R[4 * g + 3])), off);
                acc[4 * u0 + g] = fma2(p0, c0v, acc[4 * u0 + g]);
                acc[4 * u0 + 4 + g] = fma2(p1, c1v, acc[4 * u0 + 4 + g]);
            }
        };
        auto store_tile = [&](int mt, int nt) {
            // rows r0 + 8u, column pairs c0 + 8g
#pragma unroll
            for (int u = 0; u < 4; u++) {
                const int row = mt * BM + r0 + 8 * u;
                if (row >= M) continue;
                uint16_t *orow = out + (int64_t)row * N;
#pragma unroll
                for (int g = 0; g < 4; g++) {
                    const int col = nt * BN + c0 + 8 * g;
                    const float2 v = acc[4 * u + g];
                    if ((N & 1) == 0 && col + 1 < N) {
                        *reinterpret_cast<uint32_t *>(orow + col) = pack_bf16x2(v.x, v.y);
                    } else {
                        if (col < N) orow[col] = __bfloat16_as_ushort(__float2bfloat16_rn(v.x));
                        if (col + 1 < N) orow[col + 1] = __bfloat16_as_ushort(__float2bfloat16_rn(v.y));
                    }
                }
            }
        };
        ITile tl;
        for (int ti = 0; ok && int8_tile(ti, num_tiles, nkb, split, tl); ti++) {
            const int mt = tl.t % tiles_m, nt = tl.t / tiles_m;
#pragma unroll
            for (int i = 0; i < 16; i++) acc[i] = make_float2(0.0f, 0.0f);
            if (!wait_full(gs)) {
                ok = false;
                break;
            }
            tmem_ld_16x256b_x4(tq + (gs % NACC) * BN, RA);
            tmem_ld_wait();
            for (int kb = tl.kb0; kb < tl.kb1 && ok; kb++, it++) {
                const int s = it % STAGES;
                if (!mbar_wait(&S->swready[s], (it / STAGES) & 1, &g_timeouts) || aborted(S)) {
                    ok = false;
                    break;
                }
                const float *sat = sa_tile(s);
                const bool last = kb == tl.kb1 - 1;
#pragma unroll
                for (int j = 0; j < 4; j++, gs++) {
                    // Upper half of block gs is in RA.  Load the lower half,
                    // fold the upper; then load the upper half of the next
                    // block while the lower one is folded.
                    const uint32_t b = gs % NACC;
                    tmem_ld_16x256b_x4(tq + (16u << 16) + b * BN, RB);
                    float sr[4];
#pragma unroll
                    for (int u = 0; u < 4; u++) sr[u] = sat[(r0 + 8 * u) * 4 + j];
                    float2 w2[4];
                    const float *swt = sw_tile(s) + j * BN + c0;
#pragma unroll
                    for (int g = 0; g < 4; g++) w2[g] = *reinterpret_cast<const float2 *>(swt + 8 * g);
                    fold_half(RA, 0, sr[0], sr[1], w2);
                    tmem_ld_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&S->acc_empty[b]);
                    const bool nxt = !(last && j == 3);
                    if (nxt) {
                        if (!wait_full(gs + 1)) {
                            ok = false;
                            break;
                        }
                        tmem_ld_16x256b_x4(tq + ((gs + 1) % NACC) * BN, RA);
                    }
                    fold_half(RB, 2, sr[2], sr[3], w2);
                    if (nxt) tmem_ld_wait();
                }
                if (!ok) break;
                __syncwarp();
                if (lane == 0) mbar_arrive(&S->empty[s]);
            }
            if (!ok) {
                tmem_ld_wait();
                if (lane == 0) S->abort = 1;
                break;
            }
            const int tail0 = num_tiles - num_tiles % (int)gridDim.x;  // first tile of the last round
            if (split > 1 && tl.t >= tail0) {
                // a piece of a split tile (the CTA's last tile): FP32 sums to
                // the workspace, 128 bytes per fold thread; the last piece to
                // count adds them.  The fold warps meet on an mbarrier with
                // the usual bounded waits (a warp that timed out earlier never
                // arrives, and the others give up after the limit).
                const int ft = threadIdx.x - 4 * 32;  // 0 .. 511
                const int r = tl.t - tail0;
                float4 *mine = reinterpret_cast<float4 *>(ws_part + ((size_t)(r * split + tl.piece) * 512 + ft) * 32);
#pragma unroll
                for (int i = 0; i < 8; i++)
                    mine[i] = make_float4(acc[2 * i].x, acc[2 * i].y, acc[2 * i + 1].x, acc[2 * i + 1].y);
                __syncwarp();
                if (lane == 0) mbar_arrive(&S->fold_bar);
                if (!mbar_wait(&S->fold_bar, 0, &g_timeouts)) {  // every fold thread's sums are stored
                    if (lane == 0) S->abort = 1;
                    break;
                }
                if (ft == 0) {
                    __threadfence();
                    S->last_piece = atomicAdd(&ws_cnt[r], 1u) == (uint32_t)(split - 1);
                    __threadfence();
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&S->fold_bar);
                if (!mbar_wait(&S->fold_bar, 1, &g_timeouts)) {
                    if (lane == 0) S->abort = 1;
                    break;
                }
                if (S->last_piece) {
#pragma unroll
                    for (int i = 0; i < 16; i++) acc[i] = make_float2(0.0f, 0.0f);
                    for (int p = 0; p < split; p++) {  // piece order, whichever came last
                        const float4 *src =
                            reinterpret_cast<const float4 *>(ws_part + ((size_t)(r * split + p) * 512 + ft) * 32);
#pragma unroll
                        for (int i = 0; i < 8; i++) {
                            const float4 v = __ldcg(src + i);
                            acc[2 * i].x += v.x;
                            acc[2 * i].y += v.y;
                            acc[2 * i + 1].x += v.z;
                            acc[2 * i + 1].y += v.w;
                        }
                    }
                    store_tile(mt, nt);
                    if (ft == 0) ws_cnt[r] = 0;  // ready for the next call on this workspace
                }
                continue;
            }
            store_tile(mt, nt);
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

// Workspace of the tail split: one 64 KB piece of FP32 sums and one
// counter per SM (a split never has more pieces or tiles than CTAs).
static size_t ws_part_bytes() { return (size_t)sm_count() * 512 * 32 * 4; }
size_t int8_gemm_workspace_bytes() {
    const int sms = sm_count();
    return sms > 0 ? ws_part_bytes() + (size_t)sms * 4 : 0;
}

static cudaError_t launch_int8(const int8_t *a, const int8_t *w, const float *a_scale, const float *w_scale,
                               uint16_t *out, void *ws, int m, int n, int k, cudaStream_t s) {
    alignas(64) CUtensorMap tA, tB, tSA, tSW;
    const uint64_t kblk = (uint64_t)k / 32;
    if (!make_tmap_2d(&tA, a, 1, k, m, k, BK, BM, true, false) ||
        !make_tmap_2d(&tB, w, 1, k, n, k, BK, BN, true, false) ||
        !make_tmap_2d(&tSA, a_scale, 4, kblk, m, kblk * 4, 4, BM, false, true) ||
        !make_tmap_2d(&tSW, w_scale, 4, kblk, n, kblk * 4, 4, BN, false, true))
        return cudaErrorInvalidValue;
    static DeviceOnce attrs;
    cudaError_t e = attrs.run([] {
        // The register split is only valid for a block launched with exactly
        // kLaunchRegs registers per thread.
        cudaFuncAttributes fa;
        cudaError_t r = cudaFuncGetAttributes(&fa, k_int8_gemm);
        if (r != cudaSuccess) return r;
        if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
        return cudaFuncSetAttribute(k_int8_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    });
    if (e != cudaSuccess) return e;
    const int tiles = ((m + BM - 1) / BM) * ((n + BN - 1) / BN);
    const int grid = tiles < sm_count() ? tiles : sm_count();
    const int split = ws ? int8_split(tiles, grid, k / BK) : 1;
    float *ws_part = ws ? static_cast<float *>(ws) : nullptr;
    uint32_t *ws_cnt = ws ? reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(ws) + ws_part_bytes()) : nullptr;
    k_int8_gemm<<<grid, kThreads, kSmemBytes, s>>>(tA, tB, tSA, tSW, out, m, n, k, ws_part, ws_cnt, split);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_int8_blockscaled_gemm(const int8_t *a, const int8_t *w, const float *a_scale,
                                         const float *w_scale, uint16_t *out, int m, int n, int k,
                                         cudaStream_t s) {
    return launch_int8(a, w, a_scale, w_scale, out, nullptr, m, n, k, s);
}

cudaError_t launch_int8_blockscaled_gemm_ws(const int8_t *a, const int8_t *w, const float *a_scale,
                                            const float *w_scale, uint16_t *out, void *workspace, int m, int n,
                                            int k, cudaStream_t s) {
    return launch_int8(a, w, a_scale, w_scale, out, workspace, m, n, k, s);
}

}  // namespace bsq
