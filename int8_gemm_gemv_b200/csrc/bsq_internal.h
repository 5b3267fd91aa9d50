// Internal host-side interface between the C-ABI layer (api.cu) and the
// kernel files.  Launchers assume their arguments were validated by api.cu.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

namespace bsq {

constexpr int kMaxDevices = 64;

// Runs a per-device set-up step (kernel attributes) once per device, with
// that device current, keeping only a success.  Any host thread may call
// it: concurrent first calls serialise on the mutex, later ones read one
// atomic flag.  Devices past kMaxDevices run the step on every call.
class DeviceOnce {
  public:
    template <class F>
    cudaError_t run(F &&init) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= kMaxDevices) return init();
        if (done_[dev].load(std::memory_order_acquire)) return cudaSuccess;
        std::lock_guard<std::mutex> lock(mu_);
        if (done_[dev].load(std::memory_order_relaxed)) return cudaSuccess;
        e = init();
        if (e == cudaSuccess) done_[dev].store(true, std::memory_order_release);
        return e;
    }

  private:
    std::atomic<bool> done_[kMaxDevices] = {};
    std::mutex mu_;
};

// Count of kernels launched by the library (bsq_debug_launch_count).
void note_launch();
// Records the CUDA error behind a BSQ_ERR_CUDA for the calling thread
// (bsq_debug_take_cuda_error).
void note_cuda_error(cudaError_t e);

// Per-file flags of bounded waits that ran out (read and cleared with a
// device synchronisation; used by tests only).
uint32_t take_timeouts_gemm_w4a4();
uint32_t take_timeouts_quant();
uint32_t take_timeouts_gemm_w4a4_small();
uint32_t take_timeouts_gemm_fp8();
uint32_t take_timeouts_gemm_int8();
uint32_t take_timeouts_gemv();
uint32_t take_timeouts_stream_read();

// Number of SMs of the current device (cached per device).
int sm_count();

// ---- launchers (quant.cu) ----
// amax_dev: NULL (scale2 given), or the tensor's device amax, from which the
// kernel derives scale2 (and writes it to scale2_out if that is not NULL)
cudaError_t launch_quant_nvfp4(const uint16_t *in, uint8_t *packed, uint8_t *scale, float scale2,
                               const float *amax_dev, float *scale2_out, int m, int k, cudaStream_t s);
cudaError_t launch_quant_rowwise_fp8(const uint16_t *in, uint8_t *q, float *scale, int rows, int k,
                                     cudaStream_t s);
cudaError_t launch_quant_blockfp8(const uint16_t *in, uint8_t *q, float *scale, int n, int k, cudaStream_t s);
cudaError_t launch_requant_blockfp8_to_rowwise(const uint8_t *w, const float *bscale, int n, int k, uint8_t *q,
                                               float *scale, cudaStream_t s);
cudaError_t launch_requant_w_nvfp4_int8(const uint8_t *packed, const uint8_t *sf, float scale2, int8_t *q,
                                        float *scale, int n, int k, cudaStream_t s);
cudaError_t launch_quant_act_int8_per32(const uint16_t *a, int8_t *q, float *scale, int m, int k,
                                        cudaStream_t s);
cudaError_t launch_amax_bf16(const uint16_t *x, size_t count, float *amax, cudaStream_t s);

// ---- launchers (stream_read.cu) ----
// mode 0: one CTA per SM, 128 KB ring; mode 1: L2 prefetch of each CTA's
// share before the stream dependency and a 64 KB ring (two CTAs per SM)
cudaError_t launch_stream_read(const void *src, uint64_t bytes, uint32_t *sink, int mode, cudaStream_t s);

// ---- launchers (gemv_fp8.cu) ----
cudaError_t launch_fp8_gemv_rowscale(const uint16_t *in, const uint8_t *w, const float *row_scale, uint16_t *out,
                                     int m, int n, int k, cudaStream_t s);
cudaError_t launch_fp8_gemv_blockscaled(const uint16_t *in, const uint8_t *w, const float *block_scale,
                                        uint16_t *out, int m, int n, int k, cudaStream_t s);

// ---- launchers (gemm_*.cu) ----
// scale_b_dev: NULL, or a device float that multiplies scale_ab in the kernel
cudaError_t launch_w4a4_gemm(const uint8_t *a_packed, const uint8_t *a_scale, const uint8_t *w_packed,
                             const uint8_t *w_scale, uint16_t *out, float scale_ab, const float *scale_b_dev,
                             int m, int n, int k, cudaStream_t s);
// M <= 128: swapped operands, one CTA per 128 weight rows (gemm_w4a4_small.cu)
cudaError_t launch_w4a4_gemm_small(const uint8_t *a_packed, const uint8_t *a_scale, const uint8_t *w_packed,
                                   const uint8_t *w_scale, uint16_t *out, float scale_ab, const float *scale_b_dev,
                                   int m, int n, int k, cudaStream_t s);
cudaError_t launch_fp8_gemm_rowscale(const uint8_t *a, const float *a_scale, const uint8_t *w,
                                     const float *w_scale, uint16_t *out, int m, int n, int k, cudaStream_t s);
cudaError_t launch_int8_blockscaled_gemm(const int8_t *a, const int8_t *w, const float *a_scale,
                                         const float *w_scale, uint16_t *out, int m, int n, int k,
                                         cudaStream_t s);
// The same with a workspace of int8_gemm_workspace_bytes() bytes (zeroed once
// before first use; calls sharing it must be stream-ordered): a last round of
// tiles that would leave SMs idle is split along K (gemm_int8.cu).
cudaError_t launch_int8_blockscaled_gemm_ws(const int8_t *a, const int8_t *w, const float *a_scale,
                                            const float *w_scale, uint16_t *out, void *workspace, int m, int n,
                                            int k, cudaStream_t s);
size_t int8_gemm_workspace_bytes();

// ---- tensor maps (tma.cu) ----
// 2-D row-major tensor of `rows` x `cols` elements of `elem_bytes` bytes,
// row stride `row_stride_bytes`; box of box_cols x box_rows.  swizzle128
// selects the 128-byte swizzle (box_cols * elem_bytes must be 128 then).
struct CUtensorMap_st_holder;
bool make_tmap_2d(void *tmap_out, const void *base, int elem_bytes, uint64_t cols, uint64_t rows,
                  uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows, bool swizzle128,
                  bool elem_is_float);

// General tiled tensor map: `rank` dimensions (innermost first) of `dims`
// elements of elem_bytes bytes, `strides` (rank - 1 byte strides of dims 1..),
// box `box`, swizzle of 0, 32, 64 or 128 bytes.  Out-of-range box elements
// are zero-filled on load.
bool make_tmap(void *tmap_out, const void *base, int elem_bytes, int rank, const uint64_t *dims,
               const uint64_t *strides, const uint32_t *box, int swizzle_bytes);

// 3-D view of a row-major [rows, k_bytes] byte matrix as (128 B, rows,
// k_bytes/128 chunks) so one TMA copy moves box_rows x (box_chunks * 128 B)
// with the 128-byte swizzle.  Needs k_bytes % 128 == 0.
bool make_tmap_rows_chunks(void *tmap_out, const void *base, uint64_t k_bytes, uint64_t rows, uint32_t box_rows,
                           uint32_t box_chunks);

}  // namespace bsq
