// Row-scaled FP8 GEMV for 1 <= M <= 16 (fp8_gemv_batch.rs,
// `fp8_gemv_rowscale_batch8_rt2`, `fp8_gemv_rowscale_batch16_rt2`,
// `dense_gemv_fp8w_batch2`):
//   out[m, n] = row_scale[n] * sum_k bf16(in[m, k]) * e4m3(W[n, k])
// and its block-scaled sibling (`w8a16_gemv_batch4`, `w8a16_gemv_batch2`):
//   out[m, n] = sum_k bf16(in[m, k]) * e4m3(W[n, k]) * S[n / 128, k / 128]
// where every warp's 64-wide K chunk lies in one 128-wide scale block, so its
// MMAs for a chunk go into a zeroed accumulator that is then added to the
// running sum times the scale of the row's block.
//
// The weight stream (N*K bytes, read once) is the whole cost, so the kernel
// is built like a plain streaming read: one CTA per SM owns a contiguous
// range of 16-row tiles (balanced to within one tile) and warp 16 streams it
// with TMA into a ring of 16 KB slots, each one tile x 1 KB of K (one box;
// 64-byte swizzle, so a warp's 16-byte reads hit distinct banks).  Splitting
// finer, into 8- or 4-row boxes, balances the SMs better but streams slower
// on this part, and loses more than it gains.  Warps
// 0..15 split every slot's K: warp w takes the 64-byte chunk w, and lane
// (g, t) bytes [16t, 16t+16) of rows g and g+8.
//
// Arithmetic: FP16 m16n8k16 MMAs with FP32 accumulation.  Every E4M3 value
// is an FP16 normal or zero, so one conversion instruction per byte pair
// gives the weight operand exactly (the exact E4M3 -> BF16 route costs four,
// and made the kernel issue-bound).  The activations are BF16; each row m is
// multiplied by a power of two 2^s_m that puts its largest magnitude in
// [2^14, 2^15) and rounded to FP16, which is exact for every element within
// 2^31 of that magnitude (smaller elements are below the FP16 grid and are
// rounded, an error under 2^-39 of the row's largest term).  The sums are
// multiplied by 2^-s_m on the way out, exactly.  So every product of an
// activation within that range is exact in FP32, as with BF16 operands.  The
// row maxima are found at the start by all consumer warps together, while
// the first weight copies and activation fragments are in flight.
//
// The activation fragments (L2-resident) come straight from global memory
// into registers one K stage ahead of their use, are converted once per
// stage, and serve every tile of a group of three: the slots of a group go K
// stage by K stage, tile by tile.  At the end of a group the sixteen K
// partial sums of each output are added in warp order through shared memory,
// every consumer thread summing its share, so the order of one output's sum
// never depends on M (nor does its activation scale, which is per row).
//
// Launched with programmatic stream serialization: the prologue overlaps the
// previous kernel of the stream; every global read waits for it
// (griddepcontrol.wait), so the ordering of the stream is unchanged.
#include "bsq_common.cuh"

namespace bsq {

namespace {

constexpr int kConsumers = 16;
constexpr int kThreads = 32 * (kConsumers + 1);
constexpr int CH = 64;              // weight bytes (= K elements) of one warp chunk
constexpr int KS = kConsumers * CH; // K bytes of one slot
constexpr int SLOT = 16 * KS;       // a 16-row tile x 1 KB of K
// slots: 12 (192 KB) when the reduction buffer is small, 11 for M > 8
template <int MT> constexpr int slots() { return MT == 2 ? 11 : 12; }
constexpr int kSlots = 12;  // the most slots any instance uses

static __device__ unsigned int g_timeouts;

struct Bars {
    uint64_t full[kSlots];
    uint64_t empty[kSlots];
    uint32_t rowmax[16];  // largest |activation| of each row, as BF16 bits
    uint32_t abort;
};

// tiles sharing one pass over K (their accumulators stay in registers)
template <int MT> constexpr int group_tiles() { return 3; }
template <int MT> constexpr int red_floats() { return kConsumers * group_tiles<MT>() * MT * 4 * 32; }
template <int MT> constexpr size_t smem_bytes() {
    return 1024 + (size_t)slots<MT>() * SLOT + (size_t)red_floats<MT>() * 4 + sizeof(Bars);
}
static_assert(smem_bytes<1>() <= 232448 && smem_bytes<2>() <= 232448, "shared memory");

// Byte offset of 16-byte unit t of row r in a chunk [rows][64 B], 64-byte
// swizzle (unit t of row r sits at unit t ^ ((r >> 1) & 3)).
__device__ __forceinline__ uint32_t w_off(int r, int t) { return (uint32_t)(r * CH + ((t ^ ((r >> 1) & 3)) << 4)); }
__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr));
    return r;
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

// Four E4M3 bytes (byte 0 = lowest K index) -> two FP16x2 (bytes 0, 1 in
// lo; bytes 2, 3 in hi), exact: every E4M3 value is an FP16 normal or zero.
__device__ __forceinline__ void e4m3x4_to_f16x2(uint32_t four, uint32_t &lo, uint32_t &hi) {
    asm("{\n\t.reg .b16 a, b;\n\t"
        "mov.b32 {a, b}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, a;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(four));
}

// Two BF16 values times the power of two f, rounded to FP16x2: exact when
// the scaled value is representable, which the caller's choice of f makes
// true for every element within 2^31 of its row's largest magnitude.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_scaled(uint32_t two, float f) {
    const uint64_t v = ((uint64_t)(two & 0xFFFF0000u) << 32) | (uint64_t)(two << 16);  // {lo, hi} as FP32
    uint64_t p;
    const uint64_t ff = ((uint64_t)__float_as_uint(f) << 32) | __float_as_uint(f);
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(p) : "l"(v), "l"(ff));
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(__uint_as_float((uint32_t)(p >> 32))),
        "f"(__uint_as_float((uint32_t)p)));
    return r;
}

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// A lane's share of one chunk: weight rows g and g + 8 (16 E4M3 bytes each)
// and the FP16 activation fragments of rows g (xa) and g + 8 (xb, MT == 2),
// 16 elements each, at the same 16 K positions.
template <int MT>
struct Frag {
    uint4 wa, wb;
    uint32_t xa[8], xb[8];
};

// d[i] (+)= W[16 rows of the chunk] x X[8 rows of n-tile i]^T over the
// chunk's 64 K positions.
template <int MT>
__device__ __forceinline__ void chunk_mma(float (&d)[MT][4], const Frag<MT> &f) {
    const uint32_t a_w[4] = {f.wa.x, f.wa.y, f.wa.z, f.wa.w};
    const uint32_t b_w[4] = {f.wb.x, f.wb.y, f.wb.z, f.wb.w};
#pragma unroll
    for (int j = 0; j < 4; j++) {
        uint32_t a[4];
        e4m3x4_to_f16x2(a_w[j], a[0], a[2]);  // row g:   k 4j, 4j+1 | 4j+2, 4j+3
        e4m3x4_to_f16x2(b_w[j], a[1], a[3]);  // row g+8: the same K
        mma_f16_16816(d[0], a, f.xa[2 * j], f.xa[2 * j + 1]);
        if (MT == 2) mma_f16_16816(d[MT - 1], a, f.xb[2 * j], f.xb[2 * j + 1]);
    }
}

// 2^e for -127 <= e <= 127 (2^-127 is the one subnormal needed).
__device__ __forceinline__ float pow2i(int e) {
    return e >= -126 ? __uint_as_float((uint32_t)(e + 127) << 23) : __uint_as_float(0x00400000u);
}

// The power of two 2^s that puts a row's largest magnitude (given as BF16
// bits) in [2^14, 2^15): the row times 2^s converts to FP16 without overflow,
// and exactly for every element within 2^31 of that magnitude.  Zero rows
// get s = 0.
__device__ __forceinline__ int row_shift(uint32_t amax_bits) {
    const int e = (int)(amax_bits >> 7) - 127;  // floor(log2); BF16 subnormals count as 2^-127
    return amax_bits == 0 ? 0 : min(14 - e, 127);
}

template <int MT>
__device__ __forceinline__ void x_to_f16(const uint4 (&v)[2], float f, uint32_t (&o)[8]) {
    const uint32_t w[8] = {v[0].x, v[0].y, v[0].z, v[0].w, v[1].x, v[1].y, v[1].z, v[1].w};
#pragma unroll
    for (int j = 0; j < 8; j++) o[j] = bf16x2_to_f16x2_scaled(w[j], f);
}

// acc += chunk sum (row scale: applied at write-out), or acc += chunk sum x
// the block scales s0 (weight row g) and s1 (row g + 8) (BS).
template <int MT, bool BS>
__device__ __forceinline__ void chunk_accumulate(float (&acc)[MT][4], const Frag<MT> &f, float s0, float s1) {
    if constexpr (!BS) {
        chunk_mma<MT>(acc, f);
    } else {
        float d[MT][4];
#pragma unroll
        for (int i = 0; i < MT; i++) d[i][0] = d[i][1] = d[i][2] = d[i][3] = 0.0f;
        chunk_mma<MT>(d, f);
        // d[i][0..1]: row g; d[i][2..3]: row g + 8
#pragma unroll
        for (int i = 0; i < MT; i++) {
            acc[i][0] = __fmaf_rn(d[i][0], s0, acc[i][0]);
            acc[i][1] = __fmaf_rn(d[i][1], s0, acc[i][1]);
            acc[i][2] = __fmaf_rn(d[i][2], s1, acc[i][2]);
            acc[i][3] = __fmaf_rn(d[i][3], s1, acc[i][3]);
        }
    }
}

__device__ __forceinline__ void consumers_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kConsumers) : "memory");
}

// ---------------------------------------------------------------------------
//   tmW   weights, wide (K % 64 == 0): 3-D (64 B, N rows, K/64 chunks), box
//         (64, 16, 16): one slot; narrow: 2-D (K, N), box (64, 16): one chunk
template <int MT, bool BS>
__global__ void __launch_bounds__(kThreads, 1)
    k_fp8_gemv(const __grid_constant__ CUtensorMap tmW, int wide,
               const uint16_t *__restrict__ X, const float *__restrict__ scale, uint16_t *__restrict__ out, int M,
               int N, int K) {
    constexpr int TG = group_tiles<MT>(), NS = slots<MT>();
    extern __shared__ uint8_t smem_raw[];
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *red = reinterpret_cast<float *>(base + (size_t)NS * SLOT);  // [w][u][MT][4][32]
    Bars *S = reinterpret_cast<Bars *>(red + red_floats<MT>());

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // this CTA's rows: a range of 16-row tiles (rows past N read as zeros)
    const int tiles = (N + 15) >> 4;
    const int t_begin = (int)((int64_t)tiles * blockIdx.x / gridDim.x);
    const int t_end = (int)((int64_t)tiles * (blockIdx.x + 1) / gridDim.x) - t_begin;
    const int row_begin = 16 * t_begin, row_end = min(16 * (t_begin + t_end), N);
    const int nst = (K + KS - 1) / KS;  // K stages

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; s++) {
            mbar_init(&S->full[s], 1);
            mbar_init(&S->empty[s], kConsumers);
        }
        for (int m = 0; m < 16; m++) S->rowmax[m] = 0;
        S->abort = 0;
        fence_mbar_init();
    }
    __syncthreads();
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == kConsumers) {
        // ------------------------------------------------- TMA producer
        if (lane == 0) {
            prefetch_tensormap(&tmW);
            uint32_t it = 0;
            bool ok = true;
            for (int g0 = 0; g0 < t_end && ok; g0 += TG) {
                const int gt = min(TG, t_end - g0);
                for (int q = 0; q < nst && ok; q++) {
                    const int nch = wide ? 16 : min(16, (K - q * KS + CH - 1) / CH);
                    for (int u = 0; u < gt; u++, it++) {
                        const int s = it % NS;
                        if (!mbar_wait(&S->empty[s], ((it / NS) & 1) ^ 1, &g_timeouts) || S->abort) {
                            ok = false;
                            break;
                        }
                        uint8_t *dst = base + (size_t)s * SLOT;
                        const int row0 = row_begin + 16 * (g0 + u);
                        mbar_arrive_expect_tx(&S->full[s], (uint32_t)(nch * 16 * CH));
                        if (wide) {
                            tma_load_3d(dst, &tmW, &S->full[s], 0, row0, q * 16);
                        } else {
                            for (int c = 0; c < nch; c++)
                                tma_load_2d(dst + c * 16 * CH, &tmW, &S->full[s], q * KS + c * CH, row0);
                        }
                    }
                }
            }
            if (!ok) {
                // wait out the copies still in flight so none lands after exit
                S->abort = 1;
                const uint32_t first = it > (uint32_t)NS ? it - NS : 0;
                for (uint32_t i = first; i < it; i++)
                    mbar_wait(&S->full[i % NS], (i / NS) & 1, &g_timeouts);
            }
        }
        return;
    }

    // ----------------------------------------------------- consumers
    const int g = lane >> 2, t = lane & 3;
    const int tid = threadIdx.x;
    const uint32_t sbase = smem_u32(base);

    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    // this lane's activation rows (g and, for MT == 2, g + 8) at K offset
    // 64 * warp + 16 * t of every stage; rows past M read row 0 and are
    // zeroed.  The first stage's fragments are requested before the row
    // maxima below, so the two round trips overlap.
    const bool xv0 = g < M, xv1 = MT == 2 && g + 8 < M;
    const uint16_t *x0 = X + (int64_t)(xv0 ? g : 0) * K + CH * warp + 16 * t;
    const uint16_t *x1 = X + (int64_t)(xv1 ? g + 8 : 0) * K + CH * warp + 16 * t;
    auto load_x = [&](int q, uint4 (&xa)[2], uint4 (&xb)[2]) {
        const bool in = q * KS + CH * warp + 16 * t < K;
        xa[0] = (in && xv0) ? ldg_nc_v4(x0 + q * KS) : z;
        xa[1] = (in && xv0) ? ldg_nc_v4(x0 + q * KS + 8) : z;
        if (MT == 2) {
            xb[0] = (in && xv1) ? ldg_nc_v4(x1 + q * KS) : z;
            xb[1] = (in && xv1) ? ldg_nc_v4(x1 + q * KS + 8) : z;
        }
    };
    uint4 nxa[2], nxb[2];
    load_x(0, nxa, nxb);

    // ---- each activation row's largest magnitude, found by all consumer
    // warps together: warp w scans part w / M of row w % M (16 / M parts per
    // row), up to twelve 16-byte loads in flight per lane (a 5120-wide row
    // of sixteen takes two round trips); the shuffles come after the loop,
    // so every lane of the warp reaches them
    {
        constexpr int B = 12;
        const int parts = kConsumers / M, m = warp % M, p = warp / M;
        uint32_t mx = 0;
        if (p < parts) {
            const int units = K >> 3;  // 16-byte units of a row
            const int per = (units + parts - 1) / parts;
            const int u0 = p * per, u1 = min(units, u0 + per);
            const uint4 *xr = reinterpret_cast<const uint4 *>(X + (int64_t)m * K);
            for (int u = u0 + lane; u < u1; u += 32 * B) {
                uint4 v[B];
#pragma unroll
                for (int j = 0; j < B; j++) v[j] = u + 32 * j < u1 ? ldg_nc_v4(xr + u + 32 * j) : z;
#pragma unroll
                for (int j = 0; j < B; j++)
                    mx = __vmaxu2(mx, __vmaxu2(__vmaxu2(v[j].x & 0x7FFF7FFFu, v[j].y & 0x7FFF7FFFu),
                                               __vmaxu2(v[j].z & 0x7FFF7FFFu, v[j].w & 0x7FFF7FFFu)));
            }
        }
        mx = max(mx & 0xFFFFu, mx >> 16);
        mx = __reduce_max_sync(0xFFFFFFFFu, mx);
        if (lane == 0 && p < parts) atomicMax(&S->rowmax[m], mx);
    }
    consumers_sync();
    const float xs0 = pow2i(row_shift(S->rowmax[g < M ? g : 0]));
    const float xs1 = pow2i(row_shift(S->rowmax[(MT == 2 && g + 8 < M) ? g + 8 : 0]));

    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int g0 = 0; g0 < t_end; g0 += TG) {
        const int gt = min(TG, t_end - g0);
        float acc[TG][MT][4];
#pragma unroll
        for (int u = 0; u < TG; u++)
#pragma unroll
            for (int i = 0; i < MT; i++) acc[u][i][0] = acc[u][i][1] = acc[u][i][2] = acc[u][i][3] = 0.0f;

        for (int q = 0; q < nst; q++) {
            Frag<MT> f;
            x_to_f16<MT>(nxa, xs0, f.xa);
            if (MT == 2) x_to_f16<MT>(nxb, xs1, f.xb);
            load_x(q + 1 < nst ? q + 1 : 0, nxa, nxb);  // one stage ahead (the next group starts at 0)
            const int kc = q * KS + CH * warp;  // this warp's chunk
            const bool active = kc < K;
#pragma unroll
            for (int u = 0; u < TG; u++) {
                if (u >= gt) break;
                const int cs = s;
                const uint32_t cph = ph;
                if (++s == NS) {
                    s = 0;
                    ph ^= 1;
                }
                // block scales of this chunk for rows g and g + 8 of the tile
                float s0 = 1.0f, s1 = 1.0f;
                if (BS && active) {
                    const int kbn = K >> 7;
                    const int r0 = min(row_begin + (g0 + u) * 16 + g, N - 1);
                    const int r1 = min(r0 + 8, N - 1);
                    s0 = __ldg(scale + (int64_t)(r0 >> 7) * kbn + (kc >> 7));
                    s1 = __ldg(scale + (int64_t)(r1 >> 7) * kbn + (kc >> 7));
                }
                // after a timeout the warp keeps its loop and barrier sequence
                // (so no other warp waits on it) but touches no slot; the vote
                // keeps `ok` the same in every lane, so the __syncwarp below is
                // reached by all lanes or by none
                if (ok) ok = mbar_wait(&S->full[cs], cph, &g_timeouts);
                ok = __all_sync(0xFFFFFFFFu, ok);
                if (!ok) continue;
                if (active) {
                    const uint32_t chunk = sbase + (uint32_t)cs * SLOT + warp * 16 * CH;
                    f.wa = lds_v4(chunk + w_off(g, t));
                    f.wb = lds_v4(chunk + w_off(g + 8, t));
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&S->empty[cs]);
                if (active) chunk_accumulate<MT, BS>(acc[u], f, s0, s1);
            }
        }

        // ---- the group's sixteen K partial sums, added in warp order by all
        // consumer threads, then scaled and stored
        consumers_sync();  // the previous group's sums have been read
#pragma unroll
        for (int u = 0; u < TG; u++)
#pragma unroll
            for (int i = 0; i < MT; i++)
#pragma unroll
                for (int r = 0; r < 4; r++) red[(((warp * TG + u) * MT + i) * 4 + r) * 32 + lane] = acc[u][i][r];
        consumers_sync();
        for (int v = tid; v < gt * MT * 128; v += 32 * kConsumers) {
            const int u = v / (MT * 128), rem = v % (MT * 128);
            const int i = rem >> 7, r = (rem >> 5) & 3, ln = rem & 31;
            float sum = 0.0f;
            for (int w = 0; w < kConsumers; w++) sum += red[(((w * TG + u) * MT + i) * 4 + r) * 32 + ln];
            const int n = row_begin + (g0 + u) * 16 + (ln >> 2) + 8 * (r >> 1);
            const int m = 8 * i + 2 * (ln & 3) + (r & 1);
            if (n < row_end && m < M) {
                sum *= pow2i(-row_shift(S->rowmax[m]));  // undo the activation row's power of two (exact)
                out[(int64_t)m * N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(BS ? sum : sum * __ldg(scale + n)));
            }
        }
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
static cudaError_t launch_mt(const uint16_t *in, const uint8_t *w, const float *scale, uint16_t *out, int m, int n,
                             int k, cudaStream_t s) {
    static DeviceOnce attrs;
    cudaError_t e = attrs.run([] {
        return cudaFuncSetAttribute(k_fp8_gemv<MT, BS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)smem_bytes<MT>());
    });
    if (e != cudaSuccess) return e;
    alignas(64) CUtensorMap tW;
    const int wide = (k % CH) == 0;
    const uint64_t K = (uint64_t)k, N = (uint64_t)n;
    bool ok;
    if (wide) {
        const uint64_t d[3] = {CH, N, K / CH}, st[2] = {K, CH};
        const uint32_t b16[3] = {CH, 16, 16};
        ok = make_tmap(&tW, w, 1, 3, d, st, b16, 64);
    } else {
        const uint64_t d[2] = {K, N}, st[1] = {K};
        const uint32_t b16[2] = {CH, 16};
        ok = make_tmap(&tW, w, 1, 2, d, st, b16, 64);
    }
    if (!ok) return cudaErrorInvalidValue;
    const int tiles = (n + 15) / 16;
    const int grid = tiles < sm_count() ? tiles : sm_count();
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
    return cudaLaunchKernelEx(&cfg, k_fp8_gemv<MT, BS>, tW, wide, in, scale, out, m, n, k);
}

template <bool BS>
static cudaError_t launch_gemv(const uint16_t *in, const uint8_t *w, const float *scale, uint16_t *out, int m, int n,
                               int k, cudaStream_t s) {
    const cudaError_t e = m <= 8 ? launch_mt<1, BS>(in, w, scale, out, m, n, k, s)
                                 : launch_mt<2, BS>(in, w, scale, out, m, n, k, s);
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
