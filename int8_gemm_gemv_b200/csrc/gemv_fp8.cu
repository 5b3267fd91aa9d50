// Row-scaled FP8 GEMV for 1 <= M <= 16 (fp8_gemv_batch.rs,
// `fp8_gemv_rowscale_batch8_rt2`, `fp8_gemv_rowscale_batch16_rt2`,
// `dense_gemv_fp8w_batch2`):
//   out[m, n] = row_scale[n] * sum_k bf16(in[m, k]) * e4m3(W[n, k])
// and its block-scaled sibling (`w8a16_gemv_batch4`, `w8a16_gemv_batch2`):
//   out[m, n] = sum_k bf16(in[m, k]) * e4m3(W[n, k]) * S[n / 128, k / 128]
// where each warp's 64-byte K chunk of a stage lies in one 128-wide scale
// block, so its MMAs for the stage go into a zeroed accumulator that is
// then added to the running sum times the scale of the row's block.
//
// The weight stream (N*K bytes, read once) is the whole cost.  Design:
//   * persistent: one CTA per SM, each owning a contiguous range of 8-row
//     weight units (balanced to within 8 rows), streamed as 16-row tiles
//     with a final 8-row tile where the count is odd;
//   * warp 16 streams the CTA's weight rows with TMA into a 192 KB ring of
//     stages (two 16-row tiles x 1024 K bytes each, 128-byte swizzle), so
//     up to 192 KB of loads are in flight per SM: for a 5120 x 5120 weight
//     that is an SM's whole share in one round trip;
//   * warps 0..15 each take one 64-byte K chunk of every stage: they convert
//     E4M3 -> BF16 in registers (exact) and run BF16 m16n8k16 MMAs with the
//     16 weight rows as A and the (at most 16) activation rows as B.  The
//     two tiles of a stage share the activation fragments.  Products are
//     exact in FP32; accumulation is FP32;
//   * at the end of a tile pair the sixteen K slices are summed in a fixed
//     order through shared memory and the row scale is applied at write-out.
// The summation order of one output never depends on M.
//
// Launched with programmatic stream serialization: the prologue overlaps the
// previous kernel on the stream -- including an L2 prefetch of the CTA's
// first 256 KB of weight rows, which is safe before the dependency because
// L2 is the GPU's point of coherence -- and every load and store waits for
// it (griddepcontrol.wait), so the ordering of the stream is unchanged.
//
// Inside a 64-byte K chunk, lane (g = lane/4, t = lane%4) reads bytes
// [16t, 16t+16) of tile rows g and g+8 and the same K range of activation
// rows g and g+8; the MMA's K positions are permuted to match (the sum does
// not depend on the order of its K positions, only on matching A and B).
#include "bsq_common.cuh"

namespace bsq {

namespace {

constexpr int kConsumers = 16;
constexpr int kThreads = 32 * (kConsumers + 1);
constexpr int KS = 1024;                     // K bytes per stage (64 per consumer warp)
constexpr int TILE_BYTES = 16 * KS;          // 16 KB: 16 rows x 1024 B
constexpr int STAGE_BYTES = 2 * TILE_BYTES;  // two tiles
constexpr int STAGES = 6;                    // ring of STAGES x 2 tiles
constexpr int BOX = 128;                     // TMA box: 128 B x 16 rows
constexpr uint64_t kPrefetchBytes = 256 << 10;  // per CTA, before the stream dependency

static __device__ unsigned int g_timeouts;

struct Smem {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint32_t abort;
};

template <int MT>
constexpr size_t smem_bytes() {
    return 1024 + (size_t)STAGES * STAGE_BYTES + (size_t)kConsumers * 2 * MT * 4 * 32 * sizeof(float) + sizeof(Smem);
}

__device__ __forceinline__ uint4 ld_x_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr));
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

__device__ __forceinline__ void consumers_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kConsumers) : "memory");
}

// Byte offset, inside one stage, of the 16 bytes that lane (g, t) of
// consumer warp w reads from row r of tile u (128-byte swizzle of the TMA
// box: 16-byte unit c of box row r sits at unit c ^ (r & 7)).
__device__ __forceinline__ uint32_t stage_offset(int u, int w, int r, int t) {
    const int box = w >> 1;                  // 128-byte column box of this chunk
    const int unit = 4 * (w & 1) + t;        // 16-byte unit inside the box row
    return (uint32_t)(u * TILE_BYTES + box * (16 * BOX) + r * BOX + ((unit ^ (r & 7)) << 4));
}

template <int MT, bool BS>
__global__ void __launch_bounds__(kThreads, 1)
    k_fp8_gemv(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmW8,
               const uint8_t *__restrict__ wptr, const uint16_t *__restrict__ X, const float *__restrict__ row_scale,
               uint16_t *__restrict__ out, int M, int N, int K, int tm3d) {
    extern __shared__ uint8_t smem_raw[];
    // the next kernel of the stream may start its own prologue now
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *red = reinterpret_cast<float *>(base + (size_t)STAGES * STAGE_BYTES);  // [w][u][MT][4][32]
    Smem *S = reinterpret_cast<Smem *>(red + kConsumers * 2 * MT * 4 * 32);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // this CTA's rows [row_begin, row_end): a range of 8-row units, taken as
    // 16-row tiles, the last one 8 rows (its other 8 rows are neither loaded
    // nor stored) when the unit count is odd
    const int units = (N + 7) >> 3;
    const int u_begin = (int)((int64_t)units * blockIdx.x / gridDim.x);
    const int u_end = (int)((int64_t)units * (blockIdx.x + 1) / gridDim.x);
    const int row_begin = 8 * u_begin, row_end = min(8 * u_end, N);
    const int t_end = (u_end - u_begin + 1) >> 1;  // tiles, counted from 0
    const bool half_last = ((u_end - u_begin) & 1) != 0;
    const int nst = (K + KS - 1) / KS;  // stages per tile pair

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; s++) {
            mbar_init(&S->full[s], 1);
            mbar_init(&S->empty[s], kConsumers);
        }
        S->abort = 0;
        fence_mbar_init();
    }
    // Start pulling this CTA's first weight rows into L2 while the previous
    // kernel of the stream may still be running (up to kPrefetchBytes; a
    // tile of 16 rows is one contiguous block of 16*K bytes).
    if (threadIdx.x == 0) {
        const uint8_t *wbase = reinterpret_cast<const uint8_t *>(wptr);
        uint64_t done = 0;
        for (int r = row_begin; r < row_end && done < kPrefetchBytes; r += 16) {
            const int rows = min(16, row_end - r);
            const uint64_t bytes = (uint64_t)rows * K;
            prefetch_l2_bulk(wbase + (uint64_t)r * K, (uint32_t)bytes);
            done += bytes;
        }
    }
    __syncthreads();
    // everything above touched shared memory or only prefetched into L2;
    // global memory is read and written after the previous kernel of the
    // stream has completed
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == kConsumers) {
        // ------------------------------------------------- TMA producer
        if (lane == 0) {
            prefetch_tensormap(&tmW);
            uint32_t it = 0;
            bool ok = true;
            for (int t0 = 0; t0 < t_end && ok; t0 += 2) {
                const int nt = min(2, t_end - t0);
                const bool half = half_last && t0 + nt == t_end;  // the pair's last tile has 8 rows
                for (int q = 0; q < nst; q++, it++) {
                    const int s = it % STAGES;
                    if (!mbar_wait(&S->empty[s], ((it / STAGES) & 1) ^ 1, &g_timeouts) || S->abort) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = base + (size_t)s * STAGE_BYTES;
                    mbar_arrive_expect_tx(&S->full[s], nt * TILE_BYTES - (half ? TILE_BYTES / 2 : 0));
                    for (int u = 0; u < nt; u++) {
                        const int row0 = row_begin + 16 * (t0 + u);
                        if (half && u == nt - 1) {  // 8 rows: eight 1 KB copies into the tile's first halves
#pragma unroll
                            for (int j = 0; j < KS / BOX; j++)
                                tma_load_2d(st + u * TILE_BYTES + j * 16 * BOX, &tmW8, &S->full[s], q * KS + j * BOX,
                                            row0);
                        } else if (tm3d) {  // one copy: 16 rows x 8 chunks of 128 B
                            tma_load_3d(st + u * TILE_BYTES, &tmW, &S->full[s], 0, row0, q * (KS / BOX));
                        } else {
#pragma unroll
                            for (int j = 0; j < KS / BOX; j++)
                                tma_load_2d(st + u * TILE_BYTES + j * 16 * BOX, &tmW, &S->full[s], q * KS + j * BOX,
                                            row0);
                        }
                    }
                }
            }
            if (!ok) {
                S->abort = 1;
                const uint32_t first = it > STAGES ? it - STAGES : 0;
                for (uint32_t i = first; i < it; i++) mbar_wait(&S->full[i % STAGES], (i / STAGES) & 1, &g_timeouts);
            }
        }
        return;
    }

    // ----------------------------------------------------- consumers
    const int g = lane >> 2, t = lane & 3;
    const bool okX0 = g < M, okX1 = (8 + g) < M;
    const uint16_t *x0 = X + (int64_t)(okX0 ? g : 0) * K + 16 * t + 64 * warp;
    const uint16_t *x1 = X + (int64_t)(okX1 ? 8 + g : 0) * K + 16 * t + 64 * warp;
    const uint32_t sbase = smem_u32(base);
    const uint32_t offA0 = stage_offset(0, warp, g, t), offB0 = stage_offset(0, warp, g + 8, t);
    const uint32_t offA1 = stage_offset(1, warp, g, t), offB1 = stage_offset(1, warp, g + 8, t);
    const uint4 z = make_uint4(0, 0, 0, 0);

    uint32_t it = 0;
    bool ok = true;
    for (int t0 = 0; t0 < t_end; t0 += 2) {
        const int nt = min(2, t_end - t0);
        float acc[2][MT][4];
#pragma unroll
        for (int u = 0; u < 2; u++)
#pragma unroll
            for (int i = 0; i < MT; i++) acc[u][i][0] = acc[u][i][1] = acc[u][i][2] = acc[u][i][3] = 0.0f;

        for (int q = 0; q < nst; q++, it++) {
            const int s = it % STAGES;
            const int kk = q * KS;  // + 64 * warp + 16 * t, folded into x0/x1
            const bool kok = kk + 64 * warp + 16 * t < K;
            // block scales of this warp's chunk for rows g and g + 8 of each
            // tile (row_scale is the [N/128, K/128] grid here)
            float bs[2][2];
            if (BS) {
                const int kbn = K >> 7;
                const int kbi = min((kk + 64 * warp) >> 7, kbn - 1);
#pragma unroll
                for (int u = 0; u < 2; u++) {
                    const int r0 = min(row_begin + (t0 + u) * 16 + g, N - 1);
                    const int r1 = min(r0 + 8, N - 1);
                    bs[u][0] = __ldg(row_scale + (int64_t)(r0 >> 7) * kbn + kbi);
                    bs[u][1] = __ldg(row_scale + (int64_t)(r1 >> 7) * kbn + kbi);
                }
            }
            // activation fragments for this chunk (shared by both tiles)
            uint4 xa[2], xb[2];
            xa[0] = (okX0 && kok) ? ld_x_v4(x0 + kk) : z;
            xa[1] = (okX0 && kok) ? ld_x_v4(x0 + kk + 8) : z;
            if (MT == 2) {
                xb[0] = (okX1 && kok) ? ld_x_v4(x1 + kk) : z;
                xb[1] = (okX1 && kok) ? ld_x_v4(x1 + kk + 8) : z;
            }
            // after a timeout the warp keeps its loop and barrier sequence
            // (so no other warp waits on it) but touches no stage
            if (ok && !mbar_wait(&S->full[s], (it / STAGES) & 1, &g_timeouts)) ok = false;
            if (!ok) continue;
            const uint32_t st = sbase + (uint32_t)s * STAGE_BYTES;
            uint4 wa[2], wb[2];
            wa[0] = lds_v4(st + offA0);
            wb[0] = lds_v4(st + offB0);
            if (nt == 2) {
                wa[1] = lds_v4(st + offA1);
                wb[1] = lds_v4(st + offB1);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&S->empty[s]);
            const uint32_t xa_w[8] = {xa[0].x, xa[0].y, xa[0].z, xa[0].w, xa[1].x, xa[1].y, xa[1].z, xa[1].w};
            uint32_t xb_w[8];
            if (MT == 2) {
                xb_w[0] = xb[0].x; xb_w[1] = xb[0].y; xb_w[2] = xb[0].z; xb_w[3] = xb[0].w;
                xb_w[4] = xb[1].x; xb_w[5] = xb[1].y; xb_w[6] = xb[1].z; xb_w[7] = xb[1].w;
            }
#pragma unroll
            for (int u = 0; u < 2; u++) {
                if (u == 1 && nt < 2) break;
                const uint32_t a_w[4] = {wa[u].x, wa[u].y, wa[u].z, wa[u].w};
                const uint32_t b_w[4] = {wb[u].x, wb[u].y, wb[u].z, wb[u].w};
                // block-scaled: this chunk's sums first, then scaled into acc
                float d[MT][4];
#pragma unroll
                for (int i = 0; i < MT; i++) d[i][0] = d[i][1] = d[i][2] = d[i][3] = 0.0f;
                float(&dst)[MT][4] = BS ? d : acc[u];
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    uint32_t a[4];
                    a[0] = e4m3x2_to_bf16x2(a_w[j] & 0xFFFF);  // row g,   k 4j, 4j+1
                    a[1] = e4m3x2_to_bf16x2(b_w[j] & 0xFFFF);  // row g+8, k 4j, 4j+1
                    a[2] = e4m3x2_to_bf16x2(a_w[j] >> 16);     // row g,   k 4j+2, 4j+3
                    a[3] = e4m3x2_to_bf16x2(b_w[j] >> 16);     // row g+8, k 4j+2, 4j+3
                    mma_bf16_16816(dst[0], a, xa_w[2 * j], xa_w[2 * j + 1]);
                    if (MT == 2) mma_bf16_16816(dst[MT - 1], a, xb_w[2 * j], xb_w[2 * j + 1]);
                }
                if (BS) {
                    // d[i][0..1]: row g; d[i][2..3]: row g + 8
#pragma unroll
                    for (int i = 0; i < MT; i++) {
                        acc[u][i][0] = __fmaf_rn(d[i][0], bs[u][0], acc[u][i][0]);
                        acc[u][i][1] = __fmaf_rn(d[i][1], bs[u][0], acc[u][i][1]);
                        acc[u][i][2] = __fmaf_rn(d[i][2], bs[u][1], acc[u][i][2]);
                        acc[u][i][3] = __fmaf_rn(d[i][3], bs[u][1], acc[u][i][3]);
                    }
                }
            }
        }

        // ---- sum the eight K slices in warp order, then scale and store
#pragma unroll
        for (int u = 0; u < 2; u++)
#pragma unroll
            for (int i = 0; i < MT; i++)
#pragma unroll
                for (int r = 0; r < 4; r++) red[(((warp * 2 + u) * MT + i) * 4 + r) * 32 + lane] = acc[u][i][r];
        consumers_sync();
        if (warp < 2 * MT && (warp >> (MT - 1)) < nt) {
            // warp -> (tile u, m-tile i): one 16 x 8 output block each
            const int u = MT == 2 ? warp >> 1 : warp, i = MT == 2 ? warp & 1 : 0;
            float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            for (int w = 0; w < kConsumers; w++)
#pragma unroll
                for (int r = 0; r < 4; r++) v[r] += red[(((w * 2 + u) * MT + i) * 4 + r) * 32 + lane];
#pragma unroll
            for (int r = 0; r < 4; r++) {
                const int n = row_begin + (t0 + u) * 16 + g + 8 * (r >> 1);
                const int m = 8 * i + 2 * t + (r & 1);
                if (n < row_end && m < M)
                    out[(int64_t)m * N + n] =
                        __bfloat16_as_ushort(__float2bfloat16_rn(BS ? v[r] : v[r] * __ldg(row_scale + n)));
            }
        }
        consumers_sync();
    }
    if (!ok && lane == 0) S->abort = 1;
}

}  // namespace

uint32_t take_timeouts_gemv() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_timeouts, sizeof(v)) != cudaSuccess) return 0xFFFFFFFFu;
    cudaMemcpyToSymbol(g_timeouts, &zero, sizeof(zero));
    return v;
}

template <int MT, bool BS>
static cudaError_t launch_mt(const CUtensorMap &tm, const CUtensorMap &tm8, int tm3d, const uint8_t *w,
                             const uint16_t *in, const float *row_scale, uint16_t *out, int m, int n, int k,
                             cudaStream_t s) {
    static DeviceOnce attrs;
    cudaError_t e = attrs.run([] {
        return cudaFuncSetAttribute(k_fp8_gemv<MT, BS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)smem_bytes<MT>());
    });
    if (e != cudaSuccess) return e;
    const int units = (n + 7) / 8;
    const int grid = units < sm_count() ? units : sm_count();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem_bytes<MT>();
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_fp8_gemv<MT, BS>, tm, tm8, w, in, row_scale, out, m, n, k, tm3d);
}

template <bool BS>
static cudaError_t launch_gemv(const uint16_t *in, const uint8_t *w, const float *scale, uint16_t *out, int m, int n,
                               int k, cudaStream_t s) {
    alignas(64) CUtensorMap tm, tm8;
    // K a multiple of 128: one 16 KB copy per tile and stage; otherwise eight
    // 2 KB copies (the last chunk of a row may be partial).  8-row tiles:
    // eight 1 KB copies.
    const int tm3d = (k % BOX) == 0;
    const bool ok = (tm3d ? make_tmap_rows_chunks(&tm, w, k, n, 16, KS / BOX)
                          : make_tmap_2d(&tm, w, 1, k, n, k, BOX, 16, true, false)) &&
                    make_tmap_2d(&tm8, w, 1, k, n, k, BOX, 8, true, false);
    if (!ok) return cudaErrorInvalidValue;
    cudaError_t e = m <= 8 ? launch_mt<1, BS>(tm, tm8, tm3d, w, in, scale, out, m, n, k, s)
                           : launch_mt<2, BS>(tm, tm8, tm3d, w, in, scale, out, m, n, k, s);
    note_launch();
    return e;
}

cudaError_t launch_fp8_gemv_rowscale(const uint16_t *in, const uint8_t *w, const float *row_scale, uint16_t *out,
                                     int m, int n, int k, cudaStream_t s) {
    return launch_gemv<false>(in, w, row_scale, out, m, n, k, s);
}

cudaError_t launch_fp8_gemv_blockscaled(const uint16_t *in, const uint8_t *w, const float *block_scale,
                                        uint16_t *out, int m, int n, int k, cudaStream_t s) {
    return launch_gemv<true>(in, w, block_scale, out, m, n, k, s);
}

}  // namespace bsq
