/*
 * libbsq oracle -- plain, slow CPU reference of the block-scaled low-precision
 * linear layer.  TEST INFRASTRUCTURE ONLY: it is called by the tests, by the
 * smoke check and by the CPU-baseline leg of the benchmark, never by the
 * library.  It shares no code with the CUDA path.
 *
 * Every FP32 step named below is one IEEE round-to-nearest-even operation on
 * `float` values (the file is compiled with -ffp-contract=off).  Products that
 * the method defines as exact sums are accumulated in `double` and rounded
 * once at the end.
 *
 * Formats (the pages' layouts):
 *   NVFP4   : packed E2M1 codes [rows, K/2] (element 2j in the LOW nibble of
 *             byte j), one E4M3 scale byte per 16 elements [rows, K/16], and a
 *             per-tensor FP32 scale2.  (gemm_fp4.rs, `quantize_bf16_to_nvfp4`
 *             and `w4a4_gemm` doc comments; gemm_dense_int8.rs,
 *             `requant_w_nvfp4_int8` doc comment.)
 *   row FP8 : E4M3 [rows, K] + FP32 per-row dequant scale [rows]
 *             (quantize_fns.rs, `quantize_to_fp8`, `load_fp8_weight`).
 *   block FP8: E4M3 [N, K] + FP32 scale grid [N/128, K/128]
 *             (dispatch_proj_rowwise.rs, `requant_weight_rowwise_fp8_cached`).
 *   int8/32 : int8 [rows, K] + FP32 scale [rows, K/32]
 *             (gemm_dense_int8.rs, both doc comments).
 */
#ifndef BSQ_ORACLE_H
#define BSQ_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- codecs ------------------------------------------------------------ */
double  or_e2m1_value(uint8_t code);      /* 4-bit code -> value             */
double  or_e4m3_value(uint8_t code);      /* OCP E4M3 byte -> value (NaN ok) */
uint8_t or_e2m1_encode(float x);          /* RNE onto E2M1, satfinite +-6    */
uint8_t or_e4m3_encode(float x);          /* RNE onto E4M3, satfinite +-448  */
uint16_t or_bf16_encode(double x);        /* RNE onto BF16                   */
float   or_bf16_value(uint16_t b);

/* ---- quantisers ---------------------------------------------------------- */
void or_quant_nvfp4(const uint16_t *x, int64_t rows, int64_t k, float scale2,
                    uint8_t *packed, uint8_t *sf);
void or_quant_rowwise_fp8(const uint16_t *x, int64_t rows, int64_t k,
                          uint8_t *q, float *scale);
void or_quant_blockfp8(const uint16_t *x, int64_t n, int64_t k,
                       uint8_t *q, float *scale);
void or_requant_w_nvfp4_int8(const uint8_t *packed, const uint8_t *sf,
                             float scale2, int64_t n, int64_t k,
                             int8_t *q, float *scale);
void or_quant_act_int8_per32(const uint16_t *x, int64_t m, int64_t k,
                             int8_t *q, float *scale);
void or_requant_blockfp8_to_rowwise(const uint8_t *w, const float *bscale,
                                    int64_t n, int64_t k,
                                    uint8_t *q, float *scale);
float or_amax_bf16(const uint16_t *x, int64_t count);

/* ---- products ------------------------------------------------------------
 * Each computes the output rows listed in `rows` (nrows entries; rows == NULL
 * means all m rows, in order).  out_bf16 / out_exact / abssum are
 * [nrows, n] (any may be NULL).  out_exact is the double-precision value
 * before the single BF16 rounding; abssum is sum |a*w| over the dequantised
 * products, scales included (the tolerance's reference magnitude).
 * Threads: OpenMP over the listed rows.
 */
void or_w4a4_gemm(const uint8_t *a_packed, const uint8_t *a_sf,
                  const uint8_t *w_packed, const uint8_t *w_sf,
                  float scale_a2, float scale_b2,
                  int64_t m, int64_t n, int64_t k,
                  const int64_t *rows, int64_t nrows,
                  uint16_t *out_bf16, double *out_exact, double *abssum);
void or_fp8_gemv_rowscale(const uint16_t *in, const uint8_t *w,
                          const float *row_scale,
                          int64_t m, int64_t n, int64_t k,
                          const int64_t *rows, int64_t nrows,
                          uint16_t *out_bf16, double *out_exact, double *abssum);
/* Block-scaled FP8 GEMV (fp8_gemv_batch.rs, `w8a16_gemv_batch4` and
 * `w8a16_gemv_batch2` doc comments: BF16 input [M, K], E4M3 weight with the
 * 2-D block scales of the block FP8 format, BF16 output [M, N]):
 *   out[m, n] = sum_k bf16(in[m, k]) * e4m3(W[n, k]) * S[n / 128, k / 128]
 * with S the FP32 grid [N/128, K/128] (N, K multiples of 128).            */
void or_fp8_gemv_blockscaled(const uint16_t *in, const uint8_t *w,
                             const float *block_scale,
                             int64_t m, int64_t n, int64_t k,
                             const int64_t *rows, int64_t nrows,
                             uint16_t *out_bf16, double *out_exact, double *abssum);
void or_int8_blockscaled_gemm(const int8_t *a, const int8_t *w,
                              const float *a_scale, const float *w_scale,
                              int64_t m, int64_t n, int64_t k,
                              const int64_t *rows, int64_t nrows,
                              uint16_t *out_bf16, double *out_exact,
                              double *abssum);
void or_fp8_gemm_rowscale(const uint8_t *a, const float *a_scale,
                          const uint8_t *w, const float *w_scale,
                          int64_t m, int64_t n, int64_t k,
                          const int64_t *rows, int64_t nrows,
                          uint16_t *out_bf16, double *out_exact, double *abssum);

int or_num_threads(void);

#ifdef __cplusplus
}
#endif
#endif
