// The W4A8 prefill (per-32 int8 activation quantisation followed by the int8
// block-scaled GEMM) for callers that cannot allocate device memory and so
// cannot hand over the two scratch buffers int8_w4a8_prefill asks for.
//
// The scratch lives in one file-scope device array of fixed size.  Every GPU
// on which this file's device code is loaded reserves it until the process
// exits.  Host code must not use the array's name as a device address (on
// the host it names a host-side stand-in); its device address is looked up
// with cudaGetSymbolAddress on the first call made on each device and kept.
// A cudaDeviceReset destroys the array with the context and leaves the kept
// address stale, so a process that resets a device must not call this entry
// point on that device afterwards.
#include <mutex>

#include "../../include/bsq.h"
#include "bsq_internal.h"

namespace {

// Largest m * k one call accepts: 40 Mi activation elements.  The array
// holds their int8 codes, then one FP32 scale per 32 of them.
constexpr size_t kMaxElems = size_t(40) << 20;
constexpr size_t kCodeBytes = kMaxElems;  // a multiple of 256: the scales stay aligned
constexpr size_t kScaleBytes = kMaxElems / 32 * sizeof(float);

static __device__ __align__(256) unsigned char g_prefill_scratch[kCodeBytes + kScaleBytes];

constexpr int kMaxDevices = 64;
std::mutex g_lookup_mutex;
void *g_device_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  Only a
// successful lookup is kept, so a lookup that failed (for example one made
// during a stream capture) is simply tried again by the next call.
cudaError_t scratch_on_current_device(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_lookup_mutex);
    if (g_device_ptr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_prefill_scratch);
        if (e != cudaSuccess || p == nullptr) return e != cudaSuccess ? e : cudaErrorInvalidSymbol;
        g_device_ptr[dev] = p;
    }
    *out = g_device_ptr[dev];
    return cudaSuccess;
}

inline bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" bsq_status int8_w4a8_prefill_noalloc(const uint16_t *a_bf16, const int8_t *w_i8, const float *w_scale,
                                                uint16_t *out, int m, int n, int k, bsq_stream_t stream) {
    if (m < 0 || n < 0 || k <= 0 || k % 32) return BSQ_ERR_INVALID_ARG;
    if (k % 128) return BSQ_ERR_UNSUPPORTED;
    if ((size_t)m * (size_t)k > kMaxElems) return BSQ_ERR_UNSUPPORTED;  // beyond the fixed scratch
    if (m == 0 || n == 0) return BSQ_OK;
    if (!a_bf16 || !w_i8 || !w_scale || !out) return BSQ_ERR_INVALID_ARG;
    if (!al16(a_bf16) || !al16(w_i8) || !al16(w_scale) || !al16(out)) return BSQ_ERR_MISALIGNED;
    void *base = nullptr;
    if (scratch_on_current_device(&base) != cudaSuccess) return BSQ_ERR_CUDA;
    int8_t *a_i8 = static_cast<int8_t *>(base);
    float *a_scale = reinterpret_cast<float *>(static_cast<unsigned char *>(base) + kCodeBytes);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // every byte of the scratch this call reads is written by its first
    // launch, so nothing needs clearing between calls
    if (bsq::launch_quant_act_int8_per32(a_bf16, a_i8, a_scale, m, k, s) != cudaSuccess) return BSQ_ERR_CUDA;
    if (bsq::launch_int8_blockscaled_gemm(a_i8, w_i8, a_scale, w_scale, out, m, n, k, s) != cudaSuccess)
        return BSQ_ERR_CUDA;
    return BSQ_OK;
}
