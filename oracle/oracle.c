/*
 * libbsq oracle -- plain, slow, obviously correct CPU implementation.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this.  It shares no code, table or
 * helper with the CUDA library.
 *
 * Pages followed (titles of the pages, with the doc comment or section):
 *   gemm_fp4.rs          `quantize_bf16_to_nvfp4`, `w4a4_gemm` doc comments
 *   gemm_dense_int8.rs   `requant_w_nvfp4_int8`, `int8_gemm_faith2_prefill`
 *   fp8_gemv_batch.rs    `fp8_gemv_rowscale_batch8_rt2` / `_batch16_rt2`
 *   quantize_fns.rs      `quantize_to_fp8`, `load_fp8_weight`
 *   dispatch_proj_rowwise.rs  `requant_weight_rowwise_fp8_cached`,
 *                        `cublas_fp8_rowwise_proj`
 * The pages print launchers only; the arithmetic below is the plain reading
 * of what those doc comments say each kernel computes, with the rounding
 * rules stated at each function.  Where the pages are silent the reading is
 * stated in the comment of the function that takes it.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* Codecs: decode tables, nearest-value encoders.                            */
/* ------------------------------------------------------------------------ */

/* E2M1: sign bit 3, magnitude index 0..7 onto {0,.5,1,1.5,2,3,4,6}. */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

static double E4M3_TAB[256];
static int e4m3_ready = 0;
static void e4m3_build(void);
/* built once at load time, before any thread can read it */
__attribute__((constructor)) static void oracle_init(void) { e4m3_build(); }

/* OCP OFP8 E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa bits; exponent 0 is
 * subnormal (m/8 * 2^-6); S.1111.111 is NaN; there is no infinity; the
 * largest finite magnitude is 1.75 * 2^8 = 448. */
static void e4m3_build(void) {
    for (int c = 0; c < 256; c++) {
        int s = (c >> 7) & 1, e = (c >> 3) & 15, m = c & 7;
        double v;
        if (e == 15 && m == 7)
            v = NAN;
        else if (e == 0)
            v = ldexp((double)m / 8.0, -6);
        else
            v = ldexp(1.0 + (double)m / 8.0, e - 7);
        E4M3_TAB[c] = s ? -v : v;
    }
    e4m3_ready = 1;
}

double or_e2m1_value(uint8_t code) {
    double v = E2M1_MAG[code & 7];
    return (code & 8) ? -v : v;
}

double or_e4m3_value(uint8_t code) {
    if (!e4m3_ready) e4m3_build();
    return E4M3_TAB[code];
}

/* Nearest entry of a non-negative, increasing magnitude table; a tie goes to
 * the even code (for these formats the code's last bit is the mantissa's).
 * Magnitudes beyond the largest entry saturate to it (satfinite). */
static int nearest_code(const double *mag, int ncodes, double a) {
    if (a >= mag[ncodes - 1]) return ncodes - 1;
    int best = 0;
    double bestd = fabs(mag[0] - a);
    for (int c = 1; c < ncodes; c++) {
        double d = fabs(mag[c] - a);
        if (d < bestd || (d == bestd && (c & 1) == 0)) {
            best = c;
            bestd = d;
        }
    }
    return best;
}

/* Sign is kept even when the magnitude rounds to zero (-0 code). */
uint8_t or_e2m1_encode(float x) {
    uint8_t sign = signbit(x) ? 8 : 0;
    if (isnan(x)) return sign | 7; /* not produced by the method */
    return sign | (uint8_t)nearest_code(E2M1_MAG, 8, fabs((double)x));
}

uint8_t or_e4m3_encode(float x) {
    if (!e4m3_ready) e4m3_build();
    uint8_t sign = signbit(x) ? 0x80 : 0;
    if (isnan(x)) return sign | 0x7F;
    /* finite magnitude codes are 0x00..0x7E */
    return sign | (uint8_t)nearest_code(E4M3_TAB, 0x7F, fabs((double)x));
}

/* BF16: 8 significant bits, exponent range of FP32.  Round-to-nearest-even
 * from an exact double, subnormals included. */
uint16_t or_bf16_encode(double x) {
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (isnan(x)) return 0x7FC0;
    if (a == 0.0) return sign;
    int e;
    double f = frexp(a, &e); /* a = f * 2^e, f in [0.5, 1) */
    /* normal range: value = r * 2^(e-8), r in [128, 256) */
    if (e - 1 >= -126) {
        double r = nearbyint(ldexp(f, 8)); /* default mode: ties to even */
        if (r == 256.0) {
            r = 128.0;
            e += 1;
        }
        int biased = (e - 1) + 127;
        if (biased >= 255) return sign | 0x7F80; /* overflow -> inf */
        return sign | (uint16_t)((biased << 7) | ((int)r - 128));
    }
    /* subnormal: quantum 2^-133 */
    double r = nearbyint(ldexp(a, 133));
    return sign | (uint16_t)r; /* r == 128 is the smallest normal, bits 0x80 */
}

float or_bf16_value(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

int or_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* Quantisers                                                                */
/* ------------------------------------------------------------------------ */

/* NVFP4 quantiser (gemm_fp4.rs, `quantize_bf16_to_nvfp4`: packed E2M1
 * [M,K/2] + one E4M3 scale per 16 elements [M,K/16], per-tensor scale2).
 * Per 16-element block, in this order:
 *   amax = max |x|
 *   t    = 6 * scale2                 (FP32)
 *   sf   = E4M3(amax / t)             (FP32 divide, then RNE satfinite)
 *   if sf decodes to 0: every code is +0 (no division)
 *   d    = e4m3(sf) * scale2          (FP32)
 *   code = E2M1(x / d)                (FP32 divide, then RNE satfinite,
 *                                      sign kept when the magnitude is 0)
 * Packing: element 2j in the low nibble of byte j.                          */
void or_quant_nvfp4(const uint16_t *x, int64_t rows, int64_t k, float scale2,
                    uint8_t *packed, uint8_t *sf) {
    if (!e4m3_ready) e4m3_build();
    const float t = 6.0f * scale2;
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t b = 0; b < k / 16; b++) {
            const uint16_t *xb = x + r * k + b * 16;
            float amax = 0.0f;
            for (int i = 0; i < 16; i++) {
                float v = fabsf(or_bf16_value(xb[i]));
                if (v > amax) amax = v;
            }
            float q = amax / t;
            uint8_t sc = or_e4m3_encode(q);
            sf[r * (k / 16) + b] = sc;
            uint8_t codes[16];
            if (E4M3_TAB[sc] == 0.0) {
                memset(codes, 0, sizeof codes);
            } else {
                float d = (float)E4M3_TAB[sc] * scale2;
                for (int i = 0; i < 16; i++)
                    codes[i] = or_e2m1_encode(or_bf16_value(xb[i]) / d);
            }
            uint8_t *pb = packed + r * (k / 2) + b * 8;
            for (int j = 0; j < 8; j++)
                pb[j] = (uint8_t)(codes[2 * j] | (codes[2 * j + 1] << 4));
        }
    }
}

/* Row-wise FP8 (quantize_fns.rs, `quantize_to_fp8`; dispatch_proj_rowwise.rs,
 * `quant_rowwise_fp8` launches): per row
 *   s = rowamax / 448                 (FP32), s = 0 when rowamax = 0
 *   q = E4M3(x / s)                   (FP32 divide, RNE satfinite); q = 0
 *                                      when s = 0
 * s is the dequant scale: x ~ e4m3(q) * s.                                  */
void or_quant_rowwise_fp8(const uint16_t *x, int64_t rows, int64_t k,
                          uint8_t *q, float *scale) {
    for (int64_t r = 0; r < rows; r++) {
        const uint16_t *xr = x + r * k;
        float amax = 0.0f;
        for (int64_t i = 0; i < k; i++) {
            float v = fabsf(or_bf16_value(xr[i]));
            if (v > amax) amax = v;
        }
        float s = amax / 448.0f;
        scale[r] = s;
        for (int64_t i = 0; i < k; i++)
            q[r * k + i] = (s == 0.0f) ? 0 : or_e4m3_encode(or_bf16_value(xr[i]) / s);
    }
}

/* Block-scaled FP8 weight, one FP32 dequant scale per 128x128 block, grid
 * [N/128, K/128] row-major (dispatch_proj_rowwise.rs, the scale grid read by
 * `dequant_fp8_blockscaled_bf16`).  Same rule as the row-wise quantiser with
 * the block's amax: S = amax/448, q = E4M3(x/S).  Requires N, K % 128 == 0. */
void or_quant_blockfp8(const uint16_t *x, int64_t n, int64_t k,
                       uint8_t *q, float *scale) {
    int64_t nb = n / 128, kb = k / 128;
    for (int64_t bi = 0; bi < nb; bi++)
        for (int64_t bj = 0; bj < kb; bj++) {
            float amax = 0.0f;
            for (int64_t i = 0; i < 128; i++)
                for (int64_t j = 0; j < 128; j++) {
                    float v = fabsf(or_bf16_value(x[(bi * 128 + i) * k + bj * 128 + j]));
                    if (v > amax) amax = v;
                }
            float s = amax / 448.0f;
            scale[bi * kb + bj] = s;
            for (int64_t i = 0; i < 128; i++)
                for (int64_t j = 0; j < 128; j++) {
                    int64_t idx = (bi * 128 + i) * k + bj * 128 + j;
                    q[idx] = (s == 0.0f) ? 0 : or_e4m3_encode(or_bf16_value(x[idx]) / s);
                }
        }
}

/* One symmetric int8 block of 32 values v (gemm_dense_int8.rs: "re-blocked to
 * per-32 int8 scales"):  s = amax/127 (FP32); q = clamp(rne(v/s), -127, 127);
 * amax = 0 gives s = 0 and q = 0. */
static void int8_block32(const float *v, int8_t *q, float *s_out) {
    float amax = 0.0f;
    for (int i = 0; i < 32; i++)
        if (fabsf(v[i]) > amax) amax = fabsf(v[i]);
    float s = amax / 127.0f;
    *s_out = s;
    for (int i = 0; i < 32; i++) {
        if (s == 0.0f) {
            q[i] = 0;
            continue;
        }
        float r = nearbyintf(v[i] / s); /* ties to even */
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        q[i] = (int8_t)r;
    }
}

/* NVFP4 weight -> int8 + per-32 FP32 scale (gemm_dense_int8.rs,
 * `requant_w_nvfp4_int8`).  Each 32-block spans two NVFP4 16-blocks; the
 * value of each element is v = (e2m1(code) * e4m3(sf)) * scale2, two FP32
 * multiplies (the first is exact). */
void or_requant_w_nvfp4_int8(const uint8_t *packed, const uint8_t *sf,
                             float scale2, int64_t n, int64_t k,
                             int8_t *q, float *scale) {
    if (!e4m3_ready) e4m3_build();
    for (int64_t r = 0; r < n; r++)
        for (int64_t b = 0; b < k / 32; b++) {
            float v[32];
            for (int i = 0; i < 32; i++) {
                int64_t e = b * 32 + i;
                uint8_t byte = packed[r * (k / 2) + e / 2];
                uint8_t code = (e & 1) ? (byte >> 4) : (byte & 15);
                float p = (float)or_e2m1_value(code) * (float)E4M3_TAB[sf[r * (k / 16) + e / 16]];
                v[i] = p * scale2;
            }
            int8_block32(v, q + r * k + b * 32, scale + r * (k / 32) + b);
        }
}

/* BF16 activations -> int8 + per-32 FP32 scale (gemm_dense_int8.rs,
 * `int8_gemm_faith2_prefill` step (a) `requant_a`). */
void or_quant_act_int8_per32(const uint16_t *x, int64_t m, int64_t k,
                             int8_t *q, float *scale) {
    for (int64_t r = 0; r < m; r++)
        for (int64_t b = 0; b < k / 32; b++) {
            float v[32];
            for (int i = 0; i < 32; i++) v[i] = or_bf16_value(x[r * k + b * 32 + i]);
            int8_block32(v, q + r * k + b * 32, scale + r * (k / 32) + b);
        }
}

/* Block FP8 -> row-wise FP8 (dispatch_proj_rowwise.rs,
 * `requant_weight_rowwise_fp8_cached` steps 1 and 2): the BF16 transient
 *   b = BF16(e4m3(w) * S[n/128, k/128])   (FP32 multiply, then RNE to BF16)
 * followed by the row-wise FP8 quantiser on b. */
void or_requant_blockfp8_to_rowwise(const uint8_t *w, const float *bscale,
                                    int64_t n, int64_t k,
                                    uint8_t *q, float *scale) {
    if (!e4m3_ready) e4m3_build();
    uint16_t *row = (uint16_t *)malloc((size_t)k * sizeof(uint16_t));
    for (int64_t r = 0; r < n; r++) {
        for (int64_t i = 0; i < k; i++) {
            float p = (float)E4M3_TAB[w[r * k + i]] * bscale[(r / 128) * (k / 128) + i / 128];
            row[i] = or_bf16_encode((double)p);
        }
        or_quant_rowwise_fp8(row, 1, k, q + r * k, scale + r);
    }
    free(row);
}

float or_amax_bf16(const uint16_t *x, int64_t count) {
    float amax = 0.0f;
    for (int64_t i = 0; i < count; i++) {
        float v = fabsf(or_bf16_value(x[i]));
        if (v > amax) amax = v;
    }
    return amax;
}

/* ------------------------------------------------------------------------ */
/* Products: exact terms summed in double, one BF16 rounding at the end.     */
/* ------------------------------------------------------------------------ */

static void store_out(int64_t i, int64_t n, int64_t j, double acc, double abs_acc,
                      uint16_t *out_bf16, double *out_exact, double *abssum) {
    if (out_bf16) out_bf16[i * n + j] = or_bf16_encode(acc);
    if (out_exact) out_exact[i * n + j] = acc;
    if (abssum) abssum[i * n + j] = abs_acc;
}

/* W4A4 (gemm_fp4.rs, `w4a4_gemm`):
 *   C[m,n] = scaleA2 * scaleB2 * sum_k e2m1(A) e4m3(sfA[m,k/16])
 *                                       e2m1(W) e4m3(sfW[n,k/16])          */
void or_w4a4_gemm(const uint8_t *a_packed, const uint8_t *a_sf,
                  const uint8_t *w_packed, const uint8_t *w_sf,
                  float scale_a2, float scale_b2,
                  int64_t m, int64_t n, int64_t k,
                  const int64_t *rows, int64_t nrows,
                  uint16_t *out_bf16, double *out_exact, double *abssum) {
    if (!e4m3_ready) e4m3_build();
    if (!rows) nrows = m;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; i++) {
        int64_t r = rows ? rows[i] : i;
        double *a = (double *)malloc((size_t)k * sizeof(double));
        for (int64_t e = 0; e < k; e++) {
            uint8_t byte = a_packed[r * (k / 2) + e / 2];
            a[e] = or_e2m1_value((e & 1) ? (byte >> 4) : (byte & 15)) *
                   E4M3_TAB[a_sf[r * (k / 16) + e / 16]];
        }
        for (int64_t j = 0; j < n; j++) {
            double acc = 0.0, abs_acc = 0.0;
            for (int64_t e = 0; e < k; e++) {
                uint8_t byte = w_packed[j * (k / 2) + e / 2];
                double w = or_e2m1_value((e & 1) ? (byte >> 4) : (byte & 15)) *
                           E4M3_TAB[w_sf[j * (k / 16) + e / 16]];
                acc += a[e] * w;
                abs_acc += fabs(a[e] * w);
            }
            double g = (double)scale_a2 * (double)scale_b2;
            store_out(i, n, j, acc * g, abs_acc * fabs(g), out_bf16, out_exact, abssum);
        }
        free(a);
    }
}

/* Row-scaled FP8 GEMV (fp8_gemv_batch.rs, `fp8_gemv_rowscale_batch16_rt2`:
 * per-row f32 scale applied at write-out):
 *   out[m,n] = row_scale[n] * sum_k bf16(in[m,k]) e4m3(W[n,k])              */
void or_fp8_gemv_rowscale(const uint16_t *in, const uint8_t *w,
                          const float *row_scale,
                          int64_t m, int64_t n, int64_t k,
                          const int64_t *rows, int64_t nrows,
                          uint16_t *out_bf16, double *out_exact, double *abssum) {
    if (!e4m3_ready) e4m3_build();
    if (!rows) nrows = m;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; i++) {
        int64_t r = rows ? rows[i] : i;
        for (int64_t j = 0; j < n; j++) {
            double acc = 0.0, abs_acc = 0.0;
            for (int64_t e = 0; e < k; e++) {
                double p = (double)or_bf16_value(in[r * k + e]) * E4M3_TAB[w[j * k + e]];
                acc += p;
                abs_acc += fabs(p);
            }
            double s = (double)row_scale[j];
            store_out(i, n, j, acc * s, abs_acc * fabs(s), out_bf16, out_exact, abssum);
        }
    }
}

/* Block-scaled FP8 GEMV (fp8_gemv_batch.rs, `w8a16_gemv_batch4` doc
 * comment): every product carries the scale of the 128 x 128 weight block
 * it falls in; the sum is exact in double, rounded once to BF16.           */
void or_fp8_gemv_blockscaled(const uint16_t *in, const uint8_t *w,
                             const float *block_scale,
                             int64_t m, int64_t n, int64_t k,
                             const int64_t *rows, int64_t nrows,
                             uint16_t *out_bf16, double *out_exact, double *abssum) {
    if (!e4m3_ready) e4m3_build();
    if (!rows) nrows = m;
    const int64_t kb = k / 128;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; i++) {
        int64_t r = rows ? rows[i] : i;
        for (int64_t j = 0; j < n; j++) {
            double acc = 0.0, abs_acc = 0.0;
            for (int64_t e = 0; e < k; e++) {
                double sc = (double)block_scale[(j / 128) * kb + e / 128];
                double p = (double)or_bf16_value(in[r * k + e]) * E4M3_TAB[w[j * k + e]] * sc;
                acc += p;
                abs_acc += fabs(p);
            }
            store_out(i, n, j, acc, abs_acc, out_bf16, out_exact, abssum);
        }
    }
}

/* int8 block-scaled GEMM (gemm_dense_int8.rs, `int8_gemm_faith2_prefill`
 * step (b)): for every 32-block b the int32 partial sum of a*w is exact, then
 *   C[m,n] = sum_b partial_b * sA[m,b] * sW[n,b]                           */
void or_int8_blockscaled_gemm(const int8_t *a, const int8_t *w,
                              const float *a_scale, const float *w_scale,
                              int64_t m, int64_t n, int64_t k,
                              const int64_t *rows, int64_t nrows,
                              uint16_t *out_bf16, double *out_exact,
                              double *abssum) {
    if (!rows) nrows = m;
    int64_t nb = k / 32;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; i++) {
        int64_t r = rows ? rows[i] : i;
        for (int64_t j = 0; j < n; j++) {
            double acc = 0.0, abs_acc = 0.0;
            for (int64_t b = 0; b < nb; b++) {
                int64_t part = 0, abs_part = 0;
                for (int64_t e = b * 32; e < b * 32 + 32; e++) {
                    int64_t p = (int64_t)a[r * k + e] * (int64_t)w[j * k + e];
                    part += p;
                    abs_part += p < 0 ? -p : p;
                }
                double s = (double)a_scale[r * nb + b] * (double)w_scale[j * nb + b];
                acc += (double)part * s;
                abs_acc += (double)abs_part * fabs(s);
            }
            store_out(i, n, j, acc, abs_acc, out_bf16, out_exact, abssum);
        }
    }
}

/* Row-scaled FP8 GEMM with per-token activation scales
 * (dispatch_proj_rowwise.rs, `cublas_fp8_rowwise_proj`: outer-vector FP32
 * scales on both operands):
 *   C[m,n] = sA[m] * sW[n] * sum_k e4m3(A[m,k]) e4m3(W[n,k])                */
void or_fp8_gemm_rowscale(const uint8_t *a, const float *a_scale,
                          const uint8_t *w, const float *w_scale,
                          int64_t m, int64_t n, int64_t k,
                          const int64_t *rows, int64_t nrows,
                          uint16_t *out_bf16, double *out_exact, double *abssum) {
    if (!e4m3_ready) e4m3_build();
    if (!rows) nrows = m;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; i++) {
        int64_t r = rows ? rows[i] : i;
        for (int64_t j = 0; j < n; j++) {
            double acc = 0.0, abs_acc = 0.0;
            for (int64_t e = 0; e < k; e++) {
                double p = E4M3_TAB[a[r * k + e]] * E4M3_TAB[w[j * k + e]];
                acc += p;
                abs_acc += fabs(p);
            }
            double s = (double)a_scale[r] * (double)w_scale[j];
            store_out(i, n, j, acc * s, abs_acc * fabs(s), out_bf16, out_exact, abssum);
        }
    }
}
