/*
 * bnb4_oracle.h -- plain, slow CPU oracle for 4-bit blockwise weight
 * quantization (NF4 / FP4) and the matmuls that consume it, with the
 * double-quantized absmax, 8-bit blockwise quantization and the 4-bit
 * embedding lookup.
 *
 * TEST INFRASTRUCTURE ONLY.  This header and bnb4_oracle.c are used by the
 * test suite, by the smoke check and by the benchmark's CPU-baseline leg.
 * The product library (libbnb4.so) neither includes nor links anything in
 * this directory, and this directory includes nothing from the product.
 *
 * Every function is single-threaded, uses no blocking or reordering, and
 * computes in the precision stated beside it.  Sources (page title, section):
 *   - "mps-bitsandbytes 0.4.7", Features table and Functional API
 *     (quantize_nf4 / dequantize_nf4 / matmul_nf4: per-block absmax scaling
 *     to [-1, 1], nearest code of a 16-entry table, two codes per byte).
 *   - "Feat/mps gemm 4bit bf16", table "What runs natively now" (the op list:
 *     quantize_4bit, dequantize_4bit, gemv_4bit, gemm_4bit,
 *     gemm_4bit_backward = grad_output @ dequantize_4bit(B)) and section
 *     "Correctness" (exact nearest-code search, never through a lookup table).
 *   - "mps-bitsandbytes 0.4.7", Functional API, Double Quantization
 *     (double_quant(absmax, double_quant_block=256) -> (absmax_quant,
 *     absmax_scales); dequant_absmax restores the scales).
 */
#ifndef BNB4_ORACLE_H
#define BNB4_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* quant types and dtypes use the same numeric codes as the product ABI, but
 * are declared here independently. */
#define ORACLE_NF4 0
#define ORACLE_FP4 1
#define ORACLE_F32 0
#define ORACLE_F16 1
#define ORACLE_BF16 2

/* 16 fp32 code values for a quant type (index order = stored nibble). */
int oracle_code_table(int qtype, float out[16]);

/* element conversions (the oracle's own, by arithmetic on the values) */
float oracle_f16_to_f32(uint16_t h);
float oracle_bf16_to_f32(uint16_t h);
uint16_t oracle_f32_to_f16_rne(float f);
uint16_t oracle_f32_to_bf16_rne(float f);

/* array forms of the conversions (dtype codes as above) */
int oracle_to_f32_array(const void *in, int dtype, int64_t n, float *out);
int oracle_from_f32_array(const float *in, int64_t n, int dtype, void *out);

/* Quantize n elements of x (dtype) in blocks of `blocksize` consecutive
 * elements.  packed: ceil(n/2) bytes, absmax: ceil(n/blocksize) floats. */
int oracle_quantize(const void *x, int dtype, int64_t n, int blocksize,
                    int qtype, uint8_t *packed, float *absmax);

/* out[i] = RN_dtype( fp32(code[idx_i] * absmax[i / blocksize]) ) */
int oracle_dequantize(const uint8_t *packed, const float *absmax, int64_t n,
                      int blocksize, int qtype, int out_dtype, void *out);

/* Y[m, j] = sum_k X[m, k] * Wdeq[j, k] (+ bias[j]) in float64, where
 * Wdeq = fp32(code * absmax) is the [N, K] weight quantized row-major as one
 * flat array.  X is [M, K] of x_dtype; bias (nullable) is [N] of x_dtype. */
int oracle_matmul(const void *X, int x_dtype, const uint8_t *packed,
                  const float *absmax, const void *bias, int64_t M, int64_t N,
                  int64_t K, int blocksize, int qtype, double *Y);

/* The same product, only at `count` (m, j) positions: Y[i] = Y(ms[i], js[i]). */
int oracle_matmul_entries(const void *X, int x_dtype, const uint8_t *packed,
                          const float *absmax, const void *bias, int64_t M,
                          int64_t N, int64_t K, int blocksize, int qtype,
                          const int64_t *ms, const int64_t *js, int64_t count,
                          double *Y);

/* dX[m, k] = sum_j dY[m, j] * Wdeq[j, k] in float64. dY is [M, N] of dy_dtype. */
int oracle_matmul_backward(const void *dY, int dy_dtype, const uint8_t *packed,
                           const float *absmax, int64_t M, int64_t N, int64_t K,
                           int blocksize, int qtype, double *dX);

/* The backward product at `count` (m, k) positions. */
int oracle_matmul_backward_entries(const void *dY, int dy_dtype,
                                   const uint8_t *packed, const float *absmax,
                                   int64_t M, int64_t N, int64_t K,
                                   int blocksize, int qtype, const int64_t *ms,
                                   const int64_t *ks, int64_t count, double *dX);

/* R9 -- double quantization of an absmax array (the pages give only the
 * call and the group of 256; this is the plainest reading).  Groups of
 * `group` consecutive values (the last one may be short):
 *   scale[g] = max over the group of absmax[i] (values that are not > the
 *              running maximum, NaN included, are skipped; +0 if none is > 0);
 *   q[i]     = clamp(rint(fp32(fp32(absmax[i] / scale[g]) * 255)), 0, 255),
 *              rint rounding ties to even, NaN -> 0, and 0 when scale[g] == 0;
 * and the inverse
 *   out[i]   = fp32(q[i]) * fp32(scale[g] / 255)   (each step one fp32 rounding).
 * An unsigned linear 8-bit code: absmax values are >= 0.
 * Return 0, or -1 when group < 1 or n < 0. */
int oracle_double_quant(const float *absmax, int64_t n, int group, uint8_t *q,
                        float *scales);
int oracle_dequant_absmax(const uint8_t *q, const float *scales, int64_t n,
                          int group, float *out);

/* R10 -- 8-bit blockwise quantization ("Feat/mps gemm 4bit bf16", What
 * runs natively now: quantize_blockwise / dequantize_blockwise; Correctness:
 * the exact float64 reference, never a lookup table).  The pages print no
 * 8-bit code table, so the table is the caller's: code[256] strictly
 * ascending, finite, in [-1, 1], each entry 0 or at least 2^-24 in magnitude
 * (otherwise -1).  Per block of `blocksize` elements (the last may be short):
 * absmax as R3, v = x / absmax as R4, q[i] = argmin_j |v - code[j]| in
 * float64 with ties to the smallest j (one byte per element).
 *   x [n] of dtype; q [n] uint8 (out); absmax [ceil(n/blocksize)] (out).
 * Return 0, or -1 on a bad argument. */
int oracle_quantize_8bit(const void *x, int dtype, int64_t n, int blocksize,
                         const float *code, uint8_t *q, float *absmax);

/* R10 inverse: out[i] = RN_out_dtype(fp32(code[q[i]] * absmax[i/blocksize])). */
int oracle_dequantize_8bit(const uint8_t *q, const float *absmax, int64_t n,
                           int blocksize, const float *code, int out_dtype,
                           void *out);

/* R11 -- 4-bit embedding lookup ("mps-bitsandbytes 0.4.7", Quantized
 * Embeddings: Embedding4bit.from_embedding quantizes an embedding table, NF4
 * by default).  The [V, D] table was quantized as one flat array of V*D
 * elements (R3-R6); row r of the output is table row idx[r] dequantized as
 * R7: out[r*D + k] = dequantized element idx[r]*D + k.
 *   packed [ceil(V*D/2)], absmax [ceil(V*D/blocksize)], idx [n_idx] int64,
 *   out [n_idx * D] of out_dtype.
 * Every index must lie in [0, V); otherwise -1 and out is untouched. */
int oracle_embedding_4bit(const uint8_t *packed, const float *absmax, int64_t V,
                          int64_t D, int blocksize, int qtype,
                          const int64_t *idx, int64_t n_idx, int out_dtype,
                          void *out);

#ifdef __cplusplus
}
#endif
#endif
