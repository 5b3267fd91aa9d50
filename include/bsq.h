/*
 * libbsq -- block-scaled low-precision linear layers for NVIDIA B200 (sm_100a).
 *
 * C ABI.  Every entry point returns a bsq_status and never aborts.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensor pointers are DEVICE pointers, allocated and owned by the caller
 *    (the caller-owned-scratch convention of gemm_dense_int8.rs,
 *    `int8_gemm_faith2_prefill` doc comment, and of dispatch_proj_rowwise.rs,
 *    `cublas_fp8_rowwise_proj` doc comment).  The library allocates no device
 *    memory at run time.  Its host state is a launch counter and per-device
 *    caches (SM count, kernel attributes, one device address), each set
 *    under a lock or atomically, so any host thread may call any entry
 *    point.  The one piece of device memory it owns is the fixed scratch
 *    array of int8_w4a8_prefill_noalloc (below), which every GPU that loads
 *    the library's device code holds until the process exits.
 *  - BF16 tensors are passed as uint16_t bit patterns; E4M3 and packed E2M1
 *    as uint8_t.
 *  - Layouts are row-major with K innermost:
 *      NVFP4 packed  [rows, K/2]   element 2j in the LOW nibble of byte j
 *      NVFP4 scales  [rows, K/16]  one E4M3 byte per 16 elements
 *      row FP8       [rows, K] E4M3 + FP32 [rows]
 *      block FP8     [N, K] E4M3 + FP32 [N/128, K/128]
 *      int8 per-32   [rows, K] int8 + FP32 [rows, K/32]
 *      outputs       BF16 [M, N]
 *  - The last argument is the CUDA stream (a cudaStream_t; NULL is the
 *    legacy default stream).  Every call is asynchronous and stream-ordered;
 *    no entry point synchronises the host (gemm_dense_int8.rs,
 *    `int8_gemm_faith2_prefill` doc comment: its launches are ordered on the
 *    caller's stream).
 *  - Scalars (scale2, scaleA2, scaleB2) are host floats passed by value, as
 *    the pages pass them with `arg_f32`.
 *  - All scales are DEQUANT scales: value = code * scale.
 *  - Validation happens before any launch; a call that fails validation
 *    launches nothing and writes nothing.
 *  - Empty work (M == 0 or N == 0 where allowed) returns BSQ_OK and
 *    launches nothing.  Negative sizes are BSQ_ERR_INVALID_ARG.
 *  - Inputs must be finite.
 *  - Concurrent calls on different streams may run concurrently; they share
 *    no device memory, except calls of int8_w4a8_prefill_noalloc, which share
 *    its scratch array and must not overlap on the GPU, and calls of
 *    int8_blockscaled_gemm_ws given the same workspace, which must not
 *    overlap either.
 *
 * Rounding: every quantised code and scale is defined bit-exactly (see each
 * function); GEMM and GEMV outputs are FP32 sums rounded once to BF16 and
 * agree with the exact sum within 1e-2*|out| + 1e-3*sum|a*w|.
 */
#ifndef BSQ_H
#define BSQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define BSQ_API __attribute__((visibility("default")))
#else
#define BSQ_API
#endif

struct CUstream_st;
typedef struct CUstream_st *bsq_stream_t; /* same type as cudaStream_t */

typedef enum bsq_status {
    BSQ_OK = 0,
    BSQ_ERR_INVALID_ARG = 1, /* NULL pointer, negative size, size outside the
                                documented range, block-multiple violated,
                                non-finite or non-positive scale           */
    BSQ_ERR_MISALIGNED = 2,  /* a pointer below its required alignment     */
    BSQ_ERR_UNSUPPORTED = 3, /* valid, but outside this kernel's shape
                                constraints, or a weight format tag this
                                path does not convert                      */
    BSQ_ERR_CUDA = 4         /* a CUDA call failed (see cudaGetLastError)  */
} bsq_status;

/* Weight format tags (dispatch_proj_rowwise.rs, `WeightQuantFormat`). */
typedef enum bsq_format {
    BSQ_FP8_PER_ROW = 0,      /* E4M3 [N,K] + FP32 [N]                      */
    BSQ_FP8_BLOCK_SCALED = 1, /* E4M3 [N,K] + FP32 [N/128, K/128]           */
    BSQ_FP8_SINGLE_SCALE = 2,
    BSQ_BF16 = 3,
    BSQ_NVFP4 = 4
} bsq_format;

/* ------------------------------------------------------------------------
 * quantize_bf16_to_nvfp4 -- gemm_fp4.rs, `quantize_bf16_to_nvfp4`.
 *   in      BF16 [m, k]            (16-byte aligned)
 *   packed  u8   [m, k/2]  out     (16-byte aligned)
 *   scale   u8   [m, k/16] out     E4M3 block scales
 *   scale2  per-tensor FP32 scale: 1.0 for activations (as the page
 *           launches it), amax(W)/(6*448) for weights.  Must be finite, > 0.
 * Per 16-element block: amax = max|x|; sf = E4M3_rne_satfinite(amax /
 * (6*scale2)) (FP32 steps); if sf decodes to 0 all codes are +0; else
 * code_i = E2M1_rne_satfinite(x_i / (e4m3(sf)*scale2)) (FP32 steps), sign
 * kept when the magnitude rounds to 0.
 * Errors: k % 16 != 0 -> INVALID_ARG; m < 0 or k <= 0 -> INVALID_ARG.
 * ---------------------------------------------------------------------- */
BSQ_API bsq_status quantize_bf16_to_nvfp4(const uint16_t *in, uint8_t *packed,
                                  uint8_t *scale, float scale2, int m, int k,
                                  bsq_stream_t stream);

/* ------------------------------------------------------------------------
 * quantize_bf16_to_nvfp4_devscale -- quantize_bf16_to_nvfp4 with the
 * per-tensor scale2 formed on the device from the tensor's amax (the weight
 * rule of gemm_fp4.rs: scale2 = amax / (6 * 448)), so a weight can be
 * quantised without a round trip through the host.
 *   amax       FP32 [1] device, e.g. from bsq_amax_bf16 (4-byte aligned)
 *   scale2_out FP32 [1] device or NULL: receives scale2, for
 *              w4a4_gemm_devscale (4-byte aligned)
 *   The kernel computes scale2 = amax / 2688 and t = 6 * scale2 with the
 *   same FP32 round-to-nearest steps as the host form, so its codes and
 *   scales equal those of quantize_bf16_to_nvfp4 given that scale2.  An
 *   all-zero tensor (amax = 0) gets scale codes 0 and codes +0/-0.
 *   The amax is only known on the device, so the scale2 checks of the host
 *   form (finite, >= FLT_MIN) happen in the kernel: an amax that is NaN,
 *   infinite, or non-zero but below 2688 * FLT_MIN makes the kernel write
 *   scale2 = 0 and all-zero scales and codes (as for an all-zero tensor), so
 *   w4a4_gemm_devscale then yields zeros, and sets bit 1 of the flags that
 *   bsq_debug_take_timeouts returns.  The call itself still returns BSQ_OK.
 * Errors: as quantize_bf16_to_nvfp4; amax NULL -> INVALID_ARG.
 * ---------------------------------------------------------------------- */
BSQ_API bsq_status quantize_bf16_to_nvfp4_devscale(const uint16_t *in, uint8_t *packed,
                                  uint8_t *scale, const float *amax,
                                  float *scale2_out, int m, int k,
                                  bsq_stream_t stream);

/* ------------------------------------------------------------------------
 * w4a4_gemm -- gemm_fp4.rs, `w4a4_gemm` (NVFP4 x NVFP4 on FP4 tensor cores).
 *   a_packed [m, k/2], a_scale [m, k/16]   activations (NVFP4)
 *   w_packed [n, k/2], w_scale [n, k/16]   weight (NVFP4)
 *   out      BF16 [m, n]
 *   C[i,j] = scaleA2 * scaleB2 * sum_k e2m1(A)e4m3(sfA) e2m1(W)e4m3(sfW)
 * FP32 accumulation in tensor memory, one BF16 rounding.  m <= 128 runs a
 * kernel with the operands swapped (weight rows as the MMA's M operand),
 * larger m one with 256 x 256 tiles on CTA pairs; the result is the same
 * sum either way.  The kernel may begin its set-up while the previous kernel
 * of the stream finishes (programmatic stream serialization); it reads its
 * inputs only after that kernel has completed.
 * All pointers 16-byte aligned.
 * Errors: k % 16 != 0 -> INVALID_ARG; k % 256 != 0 -> UNSUPPORTED (the
 * scale rows must be 16-byte strided for the tensor-memory-access copies).
 * ---------------------------------------------------------------------- */
BSQ_API bsq_status w4a4_gemm(const uint8_t *a_packed, const uint8_t *a_scale,
                     const uint8_t *w_packed, const uint8_t *w_scale,
                     uint16_t *out, float scaleA2, float scaleB2,
                     int m, int n, int k, bsq_stream_t stream);

/* ------------------------------------------------------------------------
 * w4a4_gemm_devscale -- w4a4_gemm with the weight's scale2 read from device
 * memory (scaleB2 -> FP32 [1] device, 4-byte aligned, e.g. the scale2_out
 * of quantize_bf16_to_nvfp4_devscale).  The kernel multiplies scaleA2 by
 * it in FP32 (as the host form multiplies the two floats) after the
 * previous kernel of the stream has completed.
 * Errors: as w4a4_gemm; scaleB2 NULL with m, n > 0 -> INVALID_ARG.
 * ---------------------------------------------------------------------- */
BSQ_API bsq_status w4a4_gemm_devscale(const uint8_t *a_packed, const uint8_t *a_scale,
                     const uint8_t *w_packed, const uint8_t *w_scale,
                     uint16_t *out, float scaleA2, const float *scaleB2,
                     int m, int n, int k, bsq_stream_t stream);

/* ------------------------------------------------------------------------
 * fp8_gemv_rowscale -- fp8_gemv_batch.rs, `fp8_gemv_rowscale_batch8_rt2`,
 * `fp8_gemv_rowscale_batch16_rt2` and `dense_gemv_fp8w_batch2` (one kernel
 * for every 1 <= m <= 16).
 *   in        BF16 [m, k]       (16-byte aligned)
 *   w         E4M3 [n, k]       (16-byte aligned)
 *   row_scale FP32 [n]          per-row dequant scale, applied at write-out
 *   out       BF16 [m, n]
 *   out[i,j] = row_scale[j] * sum_k bf16(in[i,k]) * e4m3(w[j,k])
 * FP32 sums, one BF16 rounding.  Inside, each activation row is scaled by a
 * power of two and run through FP16 tensor-core MMAs: products are exact for
 * every activation within 2^31 of its row's largest magnitude; smaller ones
 * are rounded, each by less than 2^-39 of that magnitude.  The sum for one
 * output does not depend on m (a row computed alone or in a batch of 16
 * gives the same bits).
 * Errors: m outside 1..16 -> INVALID_ARG; k % 16 != 0 -> INVALID_ARG
 * (both as the page's launchers reject them).
 * ---------------------------------------------------------------------- */
BSQ_API bsq_status fp8_gemv_rowscale(const uint16_t *in, const uint8_t *w,
                             const float *row_scale, uint16_t *out,
                             int m, int n, int k, bsq_stream_t stream);

/* ------------------------------------------------------------------------
 * fp8_gemv_blockscaled -- fp8_gemv_batch.rs, `w8a16_gemv_batch4` and
 * `w8a16_gemv_batch2` (the pages run them for m <= 4; here any 1 <= m <= 16).
 *   in          BF16 [m, k]               (16-byte aligned)
 *   w           E4M3 [n, k]               (16-byte aligned)
 *   block_scale FP32 [n/128, k/128]       the block FP8 scale grid (4-byte
 *                                          aligned), as quant_blockfp8 writes
 *   out         BF16 [m, n]
 *   out[i,j] = sum_k bf16(in[i,k]) * e4m3(w[j,k]) * block_scale[j/128, k/128]
 * FP32 sums per 64-wide K chunk, scaled by their block and accumulated in
 * FP32; one BF16 rounding.  The same FP16 datapath and exactness condition
 * as fp8_gemv_rowscale; an output does not depend on m.
 * Errors: m outside 1..16 or k % 16 != 0 -> INVALID_ARG; n or k not a
 * multiple of 128 -> UNSUPPORTED (the block grid needs whole blocks).
 * ---------------------------------------------------------------------- */
BSQ_API bsq_status fp8_gemv_blockscaled(const uint16_t *in, const uint8_t *w,
                             const float *block_scale, uint16_t *out,
                             int m, int n, int k, bsq_stream_t stream);

/* ------------------------------------------------------------------------
 * quant_rowwise_fp8 -- quantize_fns.rs, `quantize_to_fp8`, and
 * dispatch_proj_rowwise.rs, `quant_rowwise_fp8` (weights once, activations
 * per token).
 *   in BF16 [rows, k] (16-byte aligned); q E4M3 [rows, k] (16-byte
 *   aligned); scale FP32 [rows].
 *   s = rowamax / 448 (FP32); q = E4M3_rne_satfinite(x / s); rowamax = 0
 *   gives s = 0 and q = 0.
 * Errors: k % 16 != 0 -> INVALID_ARG.
 * ---------------------------------------------------------------------- */
BSQ_API bsq_status quant_rowwise_fp8(const uint16_t *in, uint8_t *q, float *scale,
                             int rows, int k, bsq_stream_t stream);

/* ------------------------------------------------------------------------
 * quant_blockfp8 -- produces the block-scaled FP8 weight format read by
 * dispatch_proj_rowwise.rs, `requant_weight_rowwise_fp8_cached` (E4M3 [n,k]
 * + FP32 grid [n/128, k/128]).  Per 128x128 block: S = amax / 448 (FP32);
 * q = E4M3_rne_satfinite(x / S); amax = 0 gives S = 0, q = 0.
 * Errors: n % 128 or k % 128 != 0 -> INVALID_ARG.
 * ---------------------------------------------------------------------- */
BSQ_API bsq_status quant_blockfp8(const uint16_t *in, uint8_t *q, float *scale,
                          int n, int k, bsq_stream_t stream);

/* ------------------------------------------------------------------------
 * requant_w_nvfp4_int8 -- gemm_dense_int8.rs, `requant_w_nvfp4_int8`.
 * One-time per weight.  Reads w_packed [n, k/2], w_e4m3 [n, k/16] and
 * scale2; writes w_i8 [n, k] and w_scale FP32 [n, k/32].
 * Per 32-element block (two NVFP4 16-blocks): v = (e2m1(c) * e4m3(sf)) *
 * scale2 (FP32); s = amax(v)/127 (FP32); q = clamp(rne(v/s), -127, 127);
 * amax = 0 gives s = 0 and q = 0.
 * Errors: k % 32 != 0 -> INVALID_ARG; scale2 not finite or <= 0 ->
 * INVALID_ARG.  w_packed, w_i8 16-byte aligned.
 * ---------------------------------------------------------------------- */
BSQ_API bsq_status requant_w_nvfp4_int8(const uint8_t *w_packed, const uint8_t *w_e4m3,
                                float scale2, int8_t *w_i8, float *w_scale,
                                int n, int k, bsq_stream_t stream);

/* ------------------------------------------------------------------------
 * quant_act_int8_per32 -- gemm_dense_int8.rs, `int8_gemm_faith2_prefill`
 * step (a) (`requant_a`).  a BF16 [m, k] -> a_i8 int8 [m, k] + a_scale FP32
 * [m, k/32]; the per-32 rule of requant_w_nvfp4_int8 on the BF16 values.
 * Errors: k % 32 != 0 -> INVALID_ARG.  a, a_i8 16-byte aligned.
 * ---------------------------------------------------------------------- */
BSQ_API bsq_status quant_act_int8_per32(const uint16_t *a, int8_t *a_i8, float *a_scale,
                                int m, int k, bsq_stream_t stream);

/* ------------------------------------------------------------------------
 * int8_blockscaled_gemm -- gemm_dense_int8.rs, `int8_gemm_faith2_prefill`
 * step (b) (`int8_gemm_faith2`).
 *   a_i8 [m, k], w_i8 [n, k] int8; a_scale [m, k/32], w_scale [n, k/32]
 *   FP32; out BF16 [m, n].
 *   C[i,j] = sum_b (exact int32 sum_{k in b} a*w) * a_scale[i,b] * w_scale[j,b]
 * Int8 tensor cores give the exact per-block partials; the FP32 fold runs
 * on the CUDA cores.  All pointers 16-byte aligned.
 * Errors: k % 32 != 0 -> INVALID_ARG; k % 128 != 0 -> UNSUPPORTED.  The
 * kernel's register split needs the build's register count; a library
 * built with another count refuses to launch and returns BSQ_ERR_CUDA.
 * ---------------------------------------------------------------------- */
BSQ_API bsq_status int8_blockscaled_gemm(const int8_t *a_i8, const int8_t *w_i8,
                                 const float *a_scale, const float *w_scale,
                                 uint16_t *out, int m, int n, int k,
                                 bsq_stream_t stream);

/* ------------------------------------------------------------------------
 * int8_blockscaled_gemm_ws -- int8_blockscaled_gemm with a caller workspace,
 * in the caller-owned-scratch style of gemm_dense_int8.rs
 * `int8_gemm_faith2_prefill`.  Tiles of 128 x 128 outputs go round-robin over
 * one CTA per SM; when the last round would leave most SMs idle, each of its
 * tiles is split along K into up to four pieces on otherwise idle SMs, and
 * the pieces' FP32 sums are added through the workspace in piece order.
 *   workspace  device memory of int8_gemm_workspace_bytes() bytes, 16-byte
 *              aligned, zeroed once before its first use (every call leaves
 *              its counters at zero again).  Calls that share a workspace
 *              must not overlap on the GPU; stream-ordered calls may share.
 *   ws_bytes   its size.
 * Same result definition and tolerance as int8_blockscaled_gemm; the outputs
 * of a split tile are summed piece by piece, so they may differ from that
 * call in the last bits, but never from run to run.
 * Errors: those of int8_blockscaled_gemm; workspace NULL or ws_bytes too
 * small -> INVALID_ARG; misaligned -> MISALIGNED.
 * ---------------------------------------------------------------------- */
BSQ_API bsq_status int8_blockscaled_gemm_ws(const int8_t *a_i8, const int8_t *w_i8,
                                    const float *a_scale, const float *w_scale,
                                    uint16_t *out, void *workspace, size_t ws_bytes,
                                    int m, int n, int k, bsq_stream_t stream);

/* Workspace bytes int8_blockscaled_gemm_ws needs on the current device (64 KB
 * and 4 bytes per SM, for any shape); 0 if the device cannot be queried. */
BSQ_API size_t int8_gemm_workspace_bytes(void);

/* ------------------------------------------------------------------------
 * int8_w4a8_prefill -- gemm_dense_int8.rs, `int8_gemm_faith2_prefill`:
 * quant_act_int8_per32 into the caller's scratch, then
 * int8_blockscaled_gemm, two launches on `stream`.
 *   a_i8_scratch >= m*k bytes, a_scale_scratch >= m*(k/32)*4 bytes.
 * Errors: those of the two calls.
 * ---------------------------------------------------------------------- */
BSQ_API bsq_status int8_w4a8_prefill(const uint16_t *a_bf16, const int8_t *w_i8,
                             const float *w_scale, int8_t *a_i8_scratch,
                             float *a_scale_scratch, uint16_t *out,
                             int m, int n, int k, bsq_stream_t stream);

/* ------------------------------------------------------------------------
 * int8_w4a8_prefill_noalloc -- the same two launches as int8_w4a8_prefill,
 * for callers that cannot allocate device memory and therefore cannot pass
 * the two scratch buffers: code whose device memory is all owned by another
 * allocator (a framework's caching allocator, a fixed arena handed out by the
 * host application), plug-ins that have no allocation API at hand, and
 * latency-critical paths that must not call cudaMalloc, which may
 * synchronise the device.  No counterpart on the pages: their launcher
 * always takes caller-owned scratch.
 *   a_bf16 BF16 [m, k]; w_i8 int8 [n, k]; w_scale FP32 [n, k/32]; out BF16
 *   [m, n]; all 16-byte aligned.  Result identical to int8_w4a8_prefill.
 * Scratch: one fixed array inside the library, 45 MiB, room for m * k <=
 * 41,943,040 activation elements.  Every GPU on which the library's device
 * code is loaded reserves it until the process exits.  The first call on a
 * device looks up the array's device address (cudaGetSymbolAddress) with
 * that device current; make that first call before any stream capture.  A
 * lookup that fails returns BSQ_ERR_CUDA and is tried again by the next
 * call; a successful one is kept for the life of the process, so do not call
 * this entry point on a device after cudaDeviceReset.
 * This entry point allocates nothing and calls no allocating routine.
 * All calls share the array and it keeps the last call's contents; each
 * call writes every scratch byte it reads, so nothing needs clearing, but
 * two calls whose executions overlap on the GPU (different streams, or
 * different host threads) race on it and must be serialised by the caller.
 * Errors: those of int8_w4a8_prefill; m * k above the limit ->
 * BSQ_ERR_UNSUPPORTED (nothing launched); the address lookup failing ->
 * BSQ_ERR_CUDA.
 * ---------------------------------------------------------------------- */
BSQ_API bsq_status int8_w4a8_prefill_noalloc(const uint16_t *a_bf16, const int8_t *w_i8,
                                             const float *w_scale, uint16_t *out,
                                             int m, int n, int k, bsq_stream_t stream);

/* ------------------------------------------------------------------------
 * requant_blockfp8_to_rowwise -- dispatch_proj_rowwise.rs,
 * `rowwise_pair_passthrough` and `requant_weight_rowwise_fp8_cached`.
 *   tag == BSQ_FP8_PER_ROW: *w_used = w, *scale_used = scale; nothing is
 *     launched and nothing is written (the invariant that page's unit tests
 *     check: a row-wise weight comes back unchanged, with no conversion).
 *     w_out/scale_out may be NULL.
 *   tag == BSQ_FP8_BLOCK_SCALED: w E4M3 [n, k] with scale FP32
 *     [n/128, k/128] -> w_out E4M3 [n, k] + scale_out FP32 [n]; then
 *     *w_used = w_out, *scale_used = scale_out.  Per element the BF16
 *     transient b = BF16_rne(e4m3(w) * S) (FP32 multiply) is kept exactly;
 *     each row is then quantised as quant_rowwise_fp8 does.  One fused
 *     kernel; the transient never reaches memory.
 *   any other tag: BSQ_ERR_UNSUPPORTED (the page asserts on it).
 *   w_used / scale_used are HOST pointers to host variables.
 * Errors: block-scaled with n % 128 or k % 128 != 0 -> INVALID_ARG.
 * ---------------------------------------------------------------------- */
BSQ_API bsq_status requant_blockfp8_to_rowwise(bsq_format tag, const uint8_t *w,
                                       const float *scale, int n, int k,
                                       uint8_t *w_out, float *scale_out,
                                       const uint8_t **w_used,
                                       const float **scale_used,
                                       bsq_stream_t stream);

/* ------------------------------------------------------------------------
 * fp8_gemm_rowscale -- dispatch_proj_rowwise.rs, `cublas_fp8_rowwise_proj`
 * (the row-wise FP8 GEMM with outer-vector FP32 scales; here a tcgen05
 * kernel, no library call).
 *   a E4M3 [m, k] + a_scale FP32 [m] (per token); w E4M3 [n, k] + w_scale
 *   FP32 [n] (per row); out BF16 [m, n].
 *   C[i,j] = a_scale[i] * w_scale[j] * sum_k e4m3(a) e4m3(w)
 * No M padding is asked of the caller (the page pads M to 16 with zeroed
 * rows; here out-of-range rows are zero-filled on load and never stored).
 * a, w, out 16-byte aligned.
 * Errors: k % 16 != 0 -> INVALID_ARG.
 * ---------------------------------------------------------------------- */
BSQ_API bsq_status fp8_gemm_rowscale(const uint8_t *a, const float *a_scale,
                             const uint8_t *w, const float *w_scale,
                             uint16_t *out, int m, int n, int k,
                             bsq_stream_t stream);

/* ------------------------------------------------------------------------
 * bsq_amax_bf16 -- max |x| over `count` BF16 values, written as one FP32 to
 * the device pointer amax_dev.  Lets a caller form the weight scale2 =
 * amax / (6*448) on the device.  The maximum is exact.
 * ---------------------------------------------------------------------- */
BSQ_API bsq_status bsq_amax_bf16(const uint16_t *x, size_t count, float *amax_dev,
                         bsq_stream_t stream);

/* ------------------------------------------------------------------------
 * bsq_debug_stream_read -- a kernel that only reads `bytes` bytes at `src`
 * (16-byte aligned, a multiple of 16 bytes) and XORs one word per CTA into
 * *sink (device, 4-byte aligned): the HBM streaming floor that the
 * bandwidth-bound kernels are measured against.  It is launched like the
 * FP8 GEMV (one CTA per SM, programmatic stream serialization).  mode 0: a
 * 128 KB ring of bulk copies per CTA; mode 1: as the GEMV does for
 * consecutive launches, each CTA prefetches its share into L2 before the
 * stream dependency and uses a 64 KB ring, so two launches can overlap.
 * No counterpart on the pages (a measurement aid).
 * Errors: mode not 0 or 1, bytes % 16 != 0 -> INVALID_ARG.
 * ---------------------------------------------------------------------- */
BSQ_API bsq_status bsq_debug_stream_read(const void *src, size_t bytes, uint32_t *sink, int mode,
                                         bsq_stream_t stream);

/* Text of a status code (static storage). */
BSQ_API const char *bsq_status_string(bsq_status status);

/* Number of kernels this library has launched in this process (all
 * devices, all threads).  Lets a caller or test check that a call launched
 * nothing (the passthrough) or count the launches of a timed region. */
BSQ_API uint64_t bsq_debug_launch_count(void);

/* The CUDA error code (a cudaError_t value) behind the last BSQ_ERR_CUDA
 * that an entry point returned on the calling thread, and clears it (0 when
 * there was none).  bsq_debug_cuda_error_string gives its text (static
 * storage). */
BSQ_API int bsq_debug_take_cuda_error(void);
BSQ_API const char *bsq_debug_cuda_error_string(int code);

/* Synchronises the current device, then returns and clears the flags the
 * kernels set on the device (0 when none was set; 0xFFFFFFFF when the device
 * could not be read).  Bit 0: one of their bounded waits ran out -- every
 * wait inside a libbsq kernel gives up after 2 s instead of hanging, and
 * records it here.  Bit 1: quantize_bf16_to_nvfp4_devscale met an amax whose
 * scale2 the host form rejects.  For tests and debugging. */
BSQ_API uint32_t bsq_debug_take_timeouts(void);

#ifdef __cplusplus
}
#endif
#endif /* BSQ_H */
