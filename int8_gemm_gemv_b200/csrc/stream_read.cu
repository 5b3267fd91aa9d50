// A kernel that only reads: the streaming floor the HBM-bound kernels (the
// GEMVs, the quantisers) are measured against.  One CTA per SM streams its
// contiguous share of a byte range into a ring of shared-memory slots with
// bulk copies and keeps nothing but one word per CTA (XORed into `sink`, so
// the reads have a consumer).  It is launched exactly like the GEMV: with
// programmatic stream serialization, so its set-up overlaps the previous
// kernel of the stream.  Mode 1 also does what the GEMV does before its
// stream dependency: a bulk L2 prefetch of the CTA's share, and a smaller
// ring, so that two CTAs fit on an SM and consecutive launches overlap.
#include "bsq_common.cuh"

namespace bsq {

namespace {

constexpr uint32_t kSlotBytes = 16 << 10;
constexpr int kMaxSlots = 8;
constexpr uint64_t kPrefetchCap = 1 << 20;  // per CTA, before the dependency

static __device__ unsigned int g_stream_timeouts;

__global__ void __launch_bounds__(32) k_stream_read(const uint8_t *__restrict__ src, uint64_t bytes,
                                                    uint32_t *__restrict__ sink, int slots, int prefetch) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t full[kMaxSlots];
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    const uint64_t units = bytes / 16;
    const uint64_t b0 = 16 * (units * blockIdx.x / gridDim.x);
    const uint64_t b1 = 16 * (units * (blockIdx.x + 1) / gridDim.x);
    if (threadIdx.x != 0) return;
    for (int s = 0; s < slots; s++) mbar_init(&full[s], 1);
    fence_mbar_init();
    if (prefetch) {
        const uint64_t end = b1 - b0 > kPrefetchCap ? b0 + kPrefetchCap : b1;
        for (uint64_t p = b0; p < end; p += 64 << 10) {
            const uint64_t len = end - p < (64u << 10) ? end - p : (64u << 10);
            prefetch_l2_bulk(src + p, (uint32_t)len);
        }
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const uint64_t n = (b1 - b0 + kSlotBytes - 1) / kSlotBytes;
    uint32_t acc = 0;
    bool ok = true;
    uint64_t c = 0;
    for (; c < n; c++) {
        const int s = (int)(c % slots);
        if (c >= (uint64_t)slots && !mbar_wait(&full[s], (uint32_t)((c / slots - 1) & 1), &g_stream_timeouts)) {
            ok = false;
            break;
        }
        const uint64_t off = b0 + c * kSlotBytes;
        const uint32_t len = (uint32_t)(b1 - off < kSlotBytes ? b1 - off : kSlotBytes);
        mbar_arrive_expect_tx(&full[s], len);
        bulk_load_g2s(ring + (size_t)s * kSlotBytes, src + off, len, &full[s]);
    }
    // wait for every copy still in flight (also after a timeout, so none
    // lands after the CTA has exited)
    const uint64_t first = c > (uint64_t)slots ? c - slots : 0;
    for (uint64_t i = first; i < c; i++) {
        const int s = (int)(i % slots);
        if (mbar_wait(&full[s], (uint32_t)((i / slots) & 1), &g_stream_timeouts) && ok)
            acc ^= *reinterpret_cast<const uint32_t *>(ring + (size_t)s * kSlotBytes);
    }
    atomicXor(sink, acc);
}

}  // namespace

uint32_t take_timeouts_stream_read() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_stream_timeouts, sizeof(v)) != cudaSuccess) return 0xFFFFFFFFu;
    cudaMemcpyToSymbol(g_stream_timeouts, &zero, sizeof(zero));
    return v;
}

cudaError_t launch_stream_read(const void *src, uint64_t bytes, uint32_t *sink, int mode, cudaStream_t s) {
    const int slots = mode == 1 ? 4 : kMaxSlots;
    const size_t smem = 128 + (size_t)slots * kSlotBytes;
    static DeviceOnce attrs;
    cudaError_t e = attrs.run([] {
        return cudaFuncSetAttribute(k_stream_read, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)(128 + (size_t)kMaxSlots * kSlotBytes));
    });
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sm_count());
    cfg.blockDim = dim3(32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, k_stream_read, static_cast<const uint8_t *>(src), bytes, sink, slots, mode == 1);
    note_launch();
    return e;
}

}  // namespace bsq
