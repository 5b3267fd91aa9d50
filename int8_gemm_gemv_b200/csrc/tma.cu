// Tensor maps for the TMA copies and small per-device host queries.  The
// driver's encoder is fetched through the runtime, so the library does not
// link libcuda and can be loaded on a machine without a GPU driver.
#include <cudaTypedefs.h>
#include <atomic>
#include <mutex>

#include "bsq_common.cuh"

namespace bsq {

namespace {
// The driver's tensor-map encoder, fetched through the runtime.  Only a
// successful lookup is kept; a failed one is tried again by the next call.
std::mutex g_encode_mutex;
std::atomic<PFN_cuTensorMapEncodeTiled_v12000> g_encode{nullptr};

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    PFN_cuTensorMapEncodeTiled_v12000 fn = g_encode.load(std::memory_order_acquire);
    if (fn) return fn;
    std::lock_guard<std::mutex> lock(g_encode_mutex);
    fn = g_encode.load(std::memory_order_relaxed);
    if (fn) return fn;
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess && p != nullptr) {
        fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        g_encode.store(fn, std::memory_order_release);
    }
    return fn;
}

// The encoder is a driver call and needs a context current on the calling
// thread.  A host thread that has made no CUDA call yet (or only calls
// through another copy of the CUDA runtime) may have none, so the first
// call on each thread makes the current device's primary context current.
bool ensure_context() {
    static thread_local bool ready = false;
    if (ready) return true;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess) return false;
    ready = true;
    return true;
}
}  // namespace

bool make_tmap_2d(void *tmap_out, const void *base, int elem_bytes, uint64_t cols, uint64_t rows,
                  uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows, bool swizzle128,
                  bool elem_is_float) {
    auto fn = encode_fn();
    if (!fn || !ensure_context()) return false;
    CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_UINT8;
    if (elem_bytes == 2) dt = CU_TENSOR_MAP_DATA_TYPE_UINT16;
    if (elem_bytes == 4) dt = elem_is_float ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_UINT32;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {row_stride_bytes};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(reinterpret_cast<CUtensorMap *>(tmap_out), dt, 2, const_cast<void *>(base), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap_rows_chunks(void *tmap_out, const void *base, uint64_t k_bytes, uint64_t rows, uint32_t box_rows,
                           uint32_t box_chunks) {
    // dims (innermost first): 128 bytes of a chunk, rows (stride k_bytes),
    // 128-byte chunks along K (stride 128); one box = box_rows x box_chunks
    // chunks, landing as [chunk][row][128 B] with the 128-byte swizzle.
    auto fn = encode_fn();
    if (!fn || k_bytes % 128 || !ensure_context()) return false;
    const cuuint64_t dims[3] = {128, rows, k_bytes / 128};
    const cuuint64_t strides[2] = {k_bytes, 128};
    const cuuint32_t box[3] = {128, box_rows, box_chunks};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(reinterpret_cast<CUtensorMap *>(tmap_out), CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
                    const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap(void *tmap_out, const void *base, int elem_bytes, int rank, const uint64_t *dims,
               const uint64_t *strides, const uint32_t *box, int swizzle_bytes) {
    auto fn = encode_fn();
    if (!fn || rank < 1 || rank > 5 || !ensure_context()) return false;
    CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_UINT8;
    if (elem_bytes == 2) dt = CU_TENSOR_MAP_DATA_TYPE_UINT16;
    if (elem_bytes == 4) dt = CU_TENSOR_MAP_DATA_TYPE_UINT32;
    CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_NONE;
    if (swizzle_bytes == 32) sw = CU_TENSOR_MAP_SWIZZLE_32B;
    if (swizzle_bytes == 64) sw = CU_TENSOR_MAP_SWIZZLE_64B;
    if (swizzle_bytes == 128) sw = CU_TENSOR_MAP_SWIZZLE_128B;
    cuuint64_t d[5], st[4];
    cuuint32_t b[5], e[5];
    for (int i = 0; i < rank; i++) {
        d[i] = dims[i];
        b[i] = box[i];
        e[i] = 1;
        if (i + 1 < rank) st[i] = strides[i];
    }
    CUresult r = fn(reinterpret_cast<CUtensorMap *>(tmap_out), dt, (cuuint32_t)rank, const_cast<void *>(base), d, st,
                    b, e, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int sm_count() {
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
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
    if (cacheable) cached[dev].store(n, std::memory_order_relaxed);
    return n;
}

}  // namespace bsq
