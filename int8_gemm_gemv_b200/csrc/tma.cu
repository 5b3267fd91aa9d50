// Tensor maps for the TMA copies and small per-device host queries.  The
// driver's encoder is fetched through the runtime, so the library does not
// link libcuda and can be loaded on a machine without a GPU driver.
#include <cudaTypedefs.h>
#include <mutex>

#include "bsq_common.cuh"

namespace bsq {

namespace {
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}
}  // namespace

bool make_tmap_2d(void *tmap_out, const void *base, int elem_bytes, uint64_t cols, uint64_t rows,
                  uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows, bool swizzle128,
                  bool elem_is_float) {
    auto fn = encode_fn();
    if (!fn) return false;
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
    if (!fn || k_bytes % 128) return false;
    const cuuint64_t dims[3] = {128, rows, k_bytes / 128};
    const cuuint64_t strides[2] = {k_bytes, 128};
    const cuuint32_t box[3] = {128, box_rows, box_chunks};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(reinterpret_cast<CUtensorMap *>(tmap_out), CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
                    const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
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
