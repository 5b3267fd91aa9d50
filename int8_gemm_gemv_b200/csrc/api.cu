// The C ABI of libbsq (include/bsq.h): argument validation, then one or two
// stream-ordered launches.  Validation never touches the device, so a call
// that fails it launches nothing and needs no GPU.
#include <atomic>
#include <cfloat>
#include <cmath>

#include "../../include/bsq.h"
#include "bsq_internal.h"

namespace bsq {
static std::atomic<uint64_t> g_launches{0};
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
// the CUDA error behind the calling thread's last BSQ_ERR_CUDA
static thread_local cudaError_t t_last_cuda_error = cudaSuccess;
void note_cuda_error(cudaError_t e) {
    if (e != cudaSuccess) t_last_cuda_error = e;
}
}  // namespace bsq

namespace {

inline bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool al4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
inline bsq_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return BSQ_OK;
    bsq::note_cuda_error(e);
    return BSQ_ERR_CUDA;
}
inline cudaStream_t cs(bsq_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }
// scale2 divides and multiplies block scales: a finite, positive, normal float
inline bool valid_scale2(float s) { return std::isfinite(s) && s >= FLT_MIN; }

bsq_status check_int8_gemm(const int8_t *a, const int8_t *w, const float *as, const float *ws, const uint16_t *out,
                           int m, int n, int k) {
    if (m < 0 || n < 0 || k <= 0 || k % 32) return BSQ_ERR_INVALID_ARG;
    if (k % 128) return BSQ_ERR_UNSUPPORTED;
    if (m == 0 || n == 0) return BSQ_OK;
    if (!a || !w || !as || !ws || !out) return BSQ_ERR_INVALID_ARG;
    if (!al16(a) || !al16(w) || !al16(as) || !al16(ws) || !al16(out)) return BSQ_ERR_MISALIGNED;
    return BSQ_OK;
}

bsq_status check_act_int8(const uint16_t *a, const int8_t *q, const float *s, int m, int k) {
    if (m < 0 || k <= 0 || k % 32) return BSQ_ERR_INVALID_ARG;
    if (m == 0) return BSQ_OK;
    if (!a || !q || !s) return BSQ_ERR_INVALID_ARG;
    if (!al16(a) || !al16(q) || !al4(s)) return BSQ_ERR_MISALIGNED;
    return BSQ_OK;
}

}  // namespace

extern "C" {

bsq_status quantize_bf16_to_nvfp4(const uint16_t *in, uint8_t *packed, uint8_t *scale, float scale2, int m, int k,
                                  bsq_stream_t stream) {
    if (m < 0 || k <= 0 || k % 16 || !valid_scale2(scale2)) return BSQ_ERR_INVALID_ARG;
    if (m == 0) return BSQ_OK;
    if (!in || !packed || !scale) return BSQ_ERR_INVALID_ARG;
    if (!al16(in) || !al16(packed)) return BSQ_ERR_MISALIGNED;
    return cuda_status(bsq::launch_quant_nvfp4(in, packed, scale, scale2, nullptr, nullptr, m, k, cs(stream)));
}

bsq_status quantize_bf16_to_nvfp4_devscale(const uint16_t *in, uint8_t *packed, uint8_t *scale, const float *amax,
                                           float *scale2_out, int m, int k, bsq_stream_t stream) {
    if (m < 0 || k <= 0 || k % 16) return BSQ_ERR_INVALID_ARG;
    if (m == 0) return BSQ_OK;
    if (!in || !packed || !scale || !amax) return BSQ_ERR_INVALID_ARG;
    if (!al16(in) || !al16(packed) || !al4(amax) || (scale2_out && !al4(scale2_out))) return BSQ_ERR_MISALIGNED;
    return cuda_status(bsq::launch_quant_nvfp4(in, packed, scale, 0.0f, amax, scale2_out, m, k, cs(stream)));
}

namespace {

bsq_status w4a4_common(const uint8_t *a_packed, const uint8_t *a_scale, const uint8_t *w_packed,
                       const uint8_t *w_scale, uint16_t *out, float scale_ab, const float *scale_b_dev, int m, int n,
                       int k, bsq_stream_t stream) {
    if (k % 256) return BSQ_ERR_UNSUPPORTED;
    if (m == 0 || n == 0) return BSQ_OK;
    if (!a_packed || !a_scale || !w_packed || !w_scale || !out) return BSQ_ERR_INVALID_ARG;
    if (!al16(a_packed) || !al16(a_scale) || !al16(w_packed) || !al16(w_scale) || !al16(out))
        return BSQ_ERR_MISALIGNED;
    // up to 128 activation rows the weight stream dominates: swapped
    // operands, one CTA per 128 weight rows; above, CTA-pair 256 x 256 tiles
    if (m <= 128)
        return cuda_status(bsq::launch_w4a4_gemm_small(a_packed, a_scale, w_packed, w_scale, out, scale_ab,
                                                       scale_b_dev, m, n, k, cs(stream)));
    return cuda_status(bsq::launch_w4a4_gemm(a_packed, a_scale, w_packed, w_scale, out, scale_ab, scale_b_dev, m, n,
                                             k, cs(stream)));
}

}  // namespace

bsq_status w4a4_gemm(const uint8_t *a_packed, const uint8_t *a_scale, const uint8_t *w_packed,
                     const uint8_t *w_scale, uint16_t *out, float scaleA2, float scaleB2, int m, int n, int k,
                     bsq_stream_t stream) {
    if (m < 0 || n < 0 || k <= 0 || k % 16 || !std::isfinite(scaleA2) || !std::isfinite(scaleB2))
        return BSQ_ERR_INVALID_ARG;
    return w4a4_common(a_packed, a_scale, w_packed, w_scale, out, scaleA2 * scaleB2, nullptr, m, n, k, stream);
}

bsq_status w4a4_gemm_devscale(const uint8_t *a_packed, const uint8_t *a_scale, const uint8_t *w_packed,
                              const uint8_t *w_scale, uint16_t *out, float scaleA2, const float *scaleB2, int m,
                              int n, int k, bsq_stream_t stream) {
    if (m < 0 || n < 0 || k <= 0 || k % 16 || !std::isfinite(scaleA2)) return BSQ_ERR_INVALID_ARG;
    if (m > 0 && n > 0 && !scaleB2) return BSQ_ERR_INVALID_ARG;
    if (scaleB2 && !al4(scaleB2)) return BSQ_ERR_MISALIGNED;
    return w4a4_common(a_packed, a_scale, w_packed, w_scale, out, scaleA2, scaleB2, m, n, k, stream);
}

bsq_status fp8_gemv_rowscale(const uint16_t *in, const uint8_t *w, const float *row_scale, uint16_t *out, int m,
                             int n, int k, bsq_stream_t stream) {
    if (m < 1 || m > 16 || n < 0 || k <= 0 || k % 16) return BSQ_ERR_INVALID_ARG;
    if (n == 0) return BSQ_OK;
    if (!in || !w || !row_scale || !out) return BSQ_ERR_INVALID_ARG;
    if (!al16(in) || !al16(w) || !al4(row_scale) || (reinterpret_cast<uintptr_t>(out) & 1u))
        return BSQ_ERR_MISALIGNED;
    return cuda_status(bsq::launch_fp8_gemv_rowscale(in, w, row_scale, out, m, n, k, cs(stream)));
}

bsq_status fp8_gemv_blockscaled(const uint16_t *in, const uint8_t *w, const float *block_scale, uint16_t *out,
                                int m, int n, int k, bsq_stream_t stream) {
    if (m < 1 || m > 16 || n < 0 || k <= 0 || k % 16) return BSQ_ERR_INVALID_ARG;
    if (n % 128 || k % 128) return BSQ_ERR_UNSUPPORTED;
    if (n == 0) return BSQ_OK;
    if (!in || !w || !block_scale || !out) return BSQ_ERR_INVALID_ARG;
    if (!al16(in) || !al16(w) || !al4(block_scale) || (reinterpret_cast<uintptr_t>(out) & 1u))
        return BSQ_ERR_MISALIGNED;
    return cuda_status(bsq::launch_fp8_gemv_blockscaled(in, w, block_scale, out, m, n, k, cs(stream)));
}

bsq_status quant_rowwise_fp8(const uint16_t *in, uint8_t *q, float *scale, int rows, int k, bsq_stream_t stream) {
    if (rows < 0 || k <= 0 || k % 16) return BSQ_ERR_INVALID_ARG;
    if (rows == 0) return BSQ_OK;
    if (!in || !q || !scale) return BSQ_ERR_INVALID_ARG;
    if (!al16(in) || !al16(q) || !al4(scale)) return BSQ_ERR_MISALIGNED;
    return cuda_status(bsq::launch_quant_rowwise_fp8(in, q, scale, rows, k, cs(stream)));
}

bsq_status quant_blockfp8(const uint16_t *in, uint8_t *q, float *scale, int n, int k, bsq_stream_t stream) {
    if (n < 0 || k <= 0 || n % 128 || k % 128) return BSQ_ERR_INVALID_ARG;
    if (n == 0) return BSQ_OK;
    if (!in || !q || !scale) return BSQ_ERR_INVALID_ARG;
    if (!al16(in) || !al16(q) || !al4(scale)) return BSQ_ERR_MISALIGNED;
    return cuda_status(bsq::launch_quant_blockfp8(in, q, scale, n, k, cs(stream)));
}

bsq_status requant_w_nvfp4_int8(const uint8_t *w_packed, const uint8_t *w_e4m3, float scale2, int8_t *w_i8,
                                float *w_scale, int n, int k, bsq_stream_t stream) {
    if (n < 0 || k <= 0 || k % 32 || !valid_scale2(scale2)) return BSQ_ERR_INVALID_ARG;
    if (n == 0) return BSQ_OK;
    if (!w_packed || !w_e4m3 || !w_i8 || !w_scale) return BSQ_ERR_INVALID_ARG;
    if (!al16(w_packed) || !al16(w_i8) || !al4(w_scale) || (reinterpret_cast<uintptr_t>(w_e4m3) & 1u))
        return BSQ_ERR_MISALIGNED;
    return cuda_status(bsq::launch_requant_w_nvfp4_int8(w_packed, w_e4m3, scale2, w_i8, w_scale, n, k, cs(stream)));
}

bsq_status quant_act_int8_per32(const uint16_t *a, int8_t *a_i8, float *a_scale, int m, int k,
                                bsq_stream_t stream) {
    bsq_status st = check_act_int8(a, a_i8, a_scale, m, k);
    if (st != BSQ_OK || m == 0) return st;
    return cuda_status(bsq::launch_quant_act_int8_per32(a, a_i8, a_scale, m, k, cs(stream)));
}

bsq_status int8_blockscaled_gemm(const int8_t *a_i8, const int8_t *w_i8, const float *a_scale,
                                 const float *w_scale, uint16_t *out, int m, int n, int k, bsq_stream_t stream) {
    bsq_status st = check_int8_gemm(a_i8, w_i8, a_scale, w_scale, out, m, n, k);
    if (st != BSQ_OK || m == 0 || n == 0) return st;
    return cuda_status(bsq::launch_int8_blockscaled_gemm(a_i8, w_i8, a_scale, w_scale, out, m, n, k, cs(stream)));
}

size_t int8_gemm_workspace_bytes(void) {
    // ensure a context on the caller's current device, as the launchers do
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    return bsq::int8_gemm_workspace_bytes();
}

bsq_status int8_blockscaled_gemm_ws(const int8_t *a_i8, const int8_t *w_i8, const float *a_scale,
                                    const float *w_scale, uint16_t *out, void *workspace, size_t ws_bytes, int m,
                                    int n, int k, bsq_stream_t stream) {
    bsq_status st = check_int8_gemm(a_i8, w_i8, a_scale, w_scale, out, m, n, k);
    if (st != BSQ_OK || m == 0 || n == 0) return st;
    if (!workspace) return BSQ_ERR_INVALID_ARG;
    if (!al16(workspace)) return BSQ_ERR_MISALIGNED;
    const size_t need = bsq::int8_gemm_workspace_bytes();
    if (need == 0) return BSQ_ERR_CUDA;
    if (ws_bytes < need) return BSQ_ERR_INVALID_ARG;
    return cuda_status(
        bsq::launch_int8_blockscaled_gemm_ws(a_i8, w_i8, a_scale, w_scale, out, workspace, m, n, k, cs(stream)));
}

bsq_status int8_w4a8_prefill(const uint16_t *a_bf16, const int8_t *w_i8, const float *w_scale,
                             int8_t *a_i8_scratch, float *a_scale_scratch, uint16_t *out, int m, int n, int k,
                             bsq_stream_t stream) {
    bsq_status st = check_act_int8(a_bf16, a_i8_scratch, a_scale_scratch, m, k);
    if (st != BSQ_OK) return st;
    st = check_int8_gemm(a_i8_scratch, w_i8, a_scale_scratch, w_scale, out, m, n, k);
    if (st != BSQ_OK || m == 0 || n == 0) return st;
    cudaError_t e = bsq::launch_quant_act_int8_per32(a_bf16, a_i8_scratch, a_scale_scratch, m, k, cs(stream));
    if (e != cudaSuccess) return cuda_status(e);
    return cuda_status(
        bsq::launch_int8_blockscaled_gemm(a_i8_scratch, w_i8, a_scale_scratch, w_scale, out, m, n, k, cs(stream)));
}

bsq_status requant_blockfp8_to_rowwise(bsq_format tag, const uint8_t *w, const float *scale, int n, int k,
                                       uint8_t *w_out, float *scale_out, const uint8_t **w_used,
                                       const float **scale_used, bsq_stream_t stream) {
    if (!w_used || !scale_used) return BSQ_ERR_INVALID_ARG;
    switch (tag) {
        case BSQ_FP8_PER_ROW:
            // Already the row-wise pair: hand back the caller's own pointers,
            // launch nothing, write nothing.
            if (!w || !scale) return BSQ_ERR_INVALID_ARG;
            *w_used = w;
            *scale_used = scale;
            return BSQ_OK;
        case BSQ_FP8_BLOCK_SCALED:
            break;
        case BSQ_FP8_SINGLE_SCALE:
        case BSQ_BF16:
        case BSQ_NVFP4:
            return BSQ_ERR_UNSUPPORTED;
        default:
            return BSQ_ERR_INVALID_ARG;
    }
    if (n < 0 || k <= 0 || n % 128 || k % 128) return BSQ_ERR_INVALID_ARG;
    if (!w || !scale || !w_out || !scale_out) return BSQ_ERR_INVALID_ARG;
    if (!al16(w) || !al16(w_out) || !al4(scale) || !al4(scale_out)) return BSQ_ERR_MISALIGNED;
    if (n > 0) {
        cudaError_t e = bsq::launch_requant_blockfp8_to_rowwise(w, scale, n, k, w_out, scale_out, cs(stream));
        if (e != cudaSuccess) return cuda_status(e);
    }
    *w_used = w_out;
    *scale_used = scale_out;
    return BSQ_OK;
}

bsq_status fp8_gemm_rowscale(const uint8_t *a, const float *a_scale, const uint8_t *w, const float *w_scale,
                             uint16_t *out, int m, int n, int k, bsq_stream_t stream) {
    if (m < 0 || n < 0 || k <= 0 || k % 16) return BSQ_ERR_INVALID_ARG;
    if (m == 0 || n == 0) return BSQ_OK;
    if (!a || !a_scale || !w || !w_scale || !out) return BSQ_ERR_INVALID_ARG;
    if (!al16(a) || !al16(w) || !al16(out) || !al4(a_scale) || !al4(w_scale)) return BSQ_ERR_MISALIGNED;
    return cuda_status(bsq::launch_fp8_gemm_rowscale(a, a_scale, w, w_scale, out, m, n, k, cs(stream)));
}

bsq_status bsq_amax_bf16(const uint16_t *x, size_t count, float *amax_dev, bsq_stream_t stream) {
    if (!amax_dev) return BSQ_ERR_INVALID_ARG;
    if (count > 0 && !x) return BSQ_ERR_INVALID_ARG;
    if (!al16(x) || !al4(amax_dev)) return BSQ_ERR_MISALIGNED;
    return cuda_status(bsq::launch_amax_bf16(x, count, amax_dev, cs(stream)));
}

bsq_status bsq_debug_stream_read(const void *src, size_t bytes, uint32_t *sink, int mode, bsq_stream_t stream) {
    if ((mode != 0 && mode != 1) || bytes % 16) return BSQ_ERR_INVALID_ARG;
    if (bytes == 0) return BSQ_OK;
    if (!src || !sink) return BSQ_ERR_INVALID_ARG;
    if (!al16(src) || !al4(sink)) return BSQ_ERR_MISALIGNED;
    return cuda_status(bsq::launch_stream_read(src, bytes, sink, mode, cs(stream)));
}

const char *bsq_status_string(bsq_status status) {
    switch (status) {
        case BSQ_OK: return "BSQ_OK";
        case BSQ_ERR_INVALID_ARG: return "BSQ_ERR_INVALID_ARG: invalid argument";
        case BSQ_ERR_MISALIGNED: return "BSQ_ERR_MISALIGNED: pointer below its required alignment";
        case BSQ_ERR_UNSUPPORTED: return "BSQ_ERR_UNSUPPORTED: shape or format not supported by this kernel";
        case BSQ_ERR_CUDA: return "BSQ_ERR_CUDA: a CUDA call failed";
    }
    return "unknown bsq_status";
}

uint64_t bsq_debug_launch_count(void) { return bsq::g_launches.load(std::memory_order_relaxed); }

int bsq_debug_take_cuda_error(void) {
    const cudaError_t e = bsq::t_last_cuda_error;
    bsq::t_last_cuda_error = cudaSuccess;
    return (int)e;
}

const char *bsq_debug_cuda_error_string(int code) { return cudaGetErrorString((cudaError_t)code); }

uint32_t bsq_debug_take_timeouts(void) {
    if (cudaDeviceSynchronize() != cudaSuccess) return 0xFFFFFFFFu;
    return bsq::take_timeouts_gemm_w4a4() | bsq::take_timeouts_gemm_w4a4_small() | bsq::take_timeouts_gemm_fp8() |
           bsq::take_timeouts_gemm_int8() | bsq::take_timeouts_gemv() | bsq::take_timeouts_quant() |
           bsq::take_timeouts_stream_read();
}

}  // extern "C"
