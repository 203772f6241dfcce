/*
 * bnb4.h -- C ABI of libbnb4.so: 4-bit blockwise weight quantization (NF4 /
 * FP4) and the 4-bit matmuls that consume it, on NVIDIA B200 (sm_100a).
 *
 * Operations and where they are defined (page title, section):
 *   bnb4_quantize       "mps-bitsandbytes 0.4.7", Functional API
 *                       (quantize_nf4 / quantize_fp4 -> (packed, absmax)),
 *                       Features table (NF4, FP4); "Feat/mps gemm 4bit bf16",
 *                       What runs natively now (quantize_4bit).
 *   bnb4_dequantize     same pages (dequantize_nf4, dequantize_4bit and its
 *                       .out form: the caller gives the output buffer).
 *   bnb4_gemv           "Feat/mps gemm 4bit bf16", What runs natively now
 *                       (gemv_4bit, M == 1, fused dequant + dot) and
 *                       Correctness (bias epilogue); "mps-bitsandbytes
 *                       0.4.7", Functional API (matmul_nf4(..., bias=None)).
 *   bnb4_gemm           "Feat/mps gemm 4bit bf16", What runs natively now
 *                       (gemm_4bit, general M).
 *   bnb4_gemm_backward  "Feat/mps gemm 4bit bf16", What runs natively now and
 *                       the paragraph on the new op: grad_input =
 *                       grad_output @ dequantize_4bit(B).
 *   bnb4_double_quant,  "mps-bitsandbytes 0.4.7", Functional API, Double
 *   bnb4_dequant_absmax Quantization (double_quant(absmax,
 *                       double_quant_block=256), dequant_absmax).
 *   bnb4_gemv_dq,       gemv_4bit, gemm_4bit and its backward whose weight
 *   bnb4_gemm_dq,       carries the double-quantized absmax of the same
 *   bnb4_gemm_backward_dq section (8-bit statistics).
 *   bnb4_quantize_8bit, "Feat/mps gemm 4bit bf16", What runs natively now
 *   bnb4_dequantize_8bit (quantize_blockwise / dequantize_blockwise) and
 *                       Correctness (exact nearest code, no lookup-table snap).
 *   bnb4_embedding_4bit "mps-bitsandbytes 0.4.7", Quantized Embeddings
 *                       (Embedding4bit: rows of a 4-bit-quantized table).
 *
 * Numeric contract (the readings of the pages that the CPU oracle follows):
 *   - absmax[b] = max |x_i| over block b, in fp32; blocks are `blocksize`
 *     consecutive elements of the flat input; the last block may be short.
 *   - v = x / absmax[b] as an IEEE fp32 quotient (v = 0 when absmax == 0).
 *   - code index = argmin_i |v - code[i]| over the 16-entry table, ties to the
 *     smallest index.  NF4 table: the 16 values listed with the gemv NF4
 *     workload; FP4 table: E2M1 (index = sign<<3 | exp<<1 | mant, bias 1,
 *     subnormals) divided by 6 so that the largest magnitude is 1.
 *   - packing: byte j = idx[2j] << 4 | idx[2j+1] (first element in the high
 *     nibble); an odd last element leaves the low nibble 0.
 *   - dequantized value = RN_dtype(fp32(code[idx] * absmax)): one fp32
 *     product, then one round-to-nearest-even conversion.
 *   - matmuls accumulate in fp32 and round the result once to the compute
 *     dtype (bf16 / fp16); the bias, if given, is added in fp32 before that
 *     rounding.  For M >= 17 and the backward the weight is the dequantized
 *     value above (already in the compute dtype).  For M <= 16 (gemv
 *     included) each code is rounded to the compute dtype and the fp32 sums
 *     are scaled by the block's absmax: the same weight up to one rounding of
 *     the code (2^-8 relative in bf16, 2^-11 in fp16).  Either way the result
 *     stays within 5e-3 relative L2 of the float64 product with the
 *     dequantized weights.
 *   - fp32 compute dtype (bnb4_gemv, bnb4_gemm, bnb4_gemm_backward with dt =
 *     BNB4_F32): x, bias and y in float32; the weight is the exact fp32
 *     dequantized value RN32(code * absmax); products and sums are fp32
 *     FMAs, so the result differs from the float64 product only by fp32
 *     summation rounding.
 *
 * Weight layout for the matmuls: W is [N, K] row-major (out x in, like a
 * Linear layer's weight) and was quantized as one flat array of N*K
 * elements, so that with K % blocksize == 0 every block lies in one row:
 *   packedW  uint8 [N, K/2]           absmax  float32 [N, K/blocksize].
 *
 * Ownership and execution:
 *   - Every pointer is a device pointer owned by the caller, except the
 *     8-bit code table (`code`, a host pointer read during the call).  The
 *     library allocates no memory and holds no per-call state.
 *   - Every call is asynchronous on `stream` (0 = the legacy default stream)
 *     and never synchronises the host, except bnb4_device_status, whose job
 *     that is.  Inputs must stay valid, and outputs must not be read, until
 *     work enqueued on `stream` has completed.
 *   - Calls on different streams may run concurrently on disjoint outputs.
 *
 * Errors: each call returns a bnb4_status.  Argument checks happen on the
 * host before anything is enqueued; on any error nothing is enqueued and no
 * output is touched.  Checks that can only be made on the device (embedding
 * indices, which live on the device; bounded waits; the gemv's shared-memory
 * plan) are reported by bnb4_device_status.  BNB4_ERR_CUDA reports a launch
 * failure (the CUDA error
 * is left for the caller's next cudaGetLastError / synchronisation).  No call
 * ever falls back to another implementation.
 */
#ifndef BNB4_H
#define BNB4_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#ifndef __CUDA_RUNTIME_H__
/* Same underlying type as cuda_runtime_api.h's cudaStream_t. */
typedef struct CUstream_st *cudaStream_t;
#endif

typedef enum { BNB4_NF4 = 0, BNB4_FP4 = 1 } bnb4_quant_type;

typedef enum { BNB4_F32 = 0, BNB4_F16 = 1, BNB4_BF16 = 2 } bnb4_dtype;

typedef enum {
    BNB4_OK = 0,
    BNB4_ERR_NULL = 1,      /* a required pointer is NULL                     */
    BNB4_ERR_ALIGN = 2,     /* a pointer is not 16-byte aligned               */
    BNB4_ERR_BLOCKSIZE = 3, /* blocksize not in {64,128,...,4096}             */
    BNB4_ERR_SHAPE = 4,     /* negative size, K % blocksize, K % 32, too big  */
    BNB4_ERR_DTYPE = 5,     /* dtype not accepted by this call                */
    BNB4_ERR_QTYPE = 6,     /* quant type not NF4 / FP4                       */
    BNB4_ERR_CUDA = 7,      /* a kernel launch failed                         */
    BNB4_ERR_TIMEOUT = 8,   /* a bounded device-side wait gave up             */
    BNB4_ERR_CODE = 9,      /* an 8-bit code table that is not usable         */
    BNB4_ERR_INDEX = 10,    /* a lookup index was out of range (device side)  */
    BNB4_ERR_DEVICE = 11    /* a kernel found its launch unusable (device side) */
} bnb4_status;

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int bnb4_version(void);

/* Static text for a status code (never NULL). */
const char *bnb4_status_string(bnb4_status status);

/*
 * Quantize n elements of x.
 *   x        [n] of x_dtype (f32 / f16 / bf16), 16-byte aligned.
 *   packed   [ceil(n/2)] bytes out, 16-byte aligned.
 *   absmax   [ceil(n/blocksize)] float32 out, 16-byte aligned.
 *   n >= 0 (n == 0 enqueues nothing); blocksize in {64, 128, ..., 4096}.
 */
bnb4_status bnb4_quantize(const void *x, uint8_t *packed, float *absmax,
                          int64_t n, int blocksize, bnb4_quant_type quant_type,
                          bnb4_dtype x_dtype, cudaStream_t stream);

/*
 * Dequantize n elements: out[i] = RN_out_dtype(fp32(code[idx_i] * absmax[i / blocksize])).
 *   packed   [ceil(n/2)] bytes, absmax [ceil(n/blocksize)] float32,
 *   out      [n] of out_dtype (f32 / f16 / bf16); all 16-byte aligned.
 */
bnb4_status bnb4_dequantize(const uint8_t *packed, const float *absmax,
                            void *out, int64_t n, int blocksize,
                            bnb4_quant_type quant_type, bnb4_dtype out_dtype,
                            cudaStream_t stream);

/*
 * Matrix-vector product for decode (M == 1): y = x @ dequant(W)^T (+ bias).
 *   x        [K] of dt;  packedW [N, K/2];  absmax [N, K/blocksize];
 *   bias     [N] of dt or NULL;  y [N] of dt (out).
 *   dt in {f32, f16, bf16}; K % blocksize == 0 and K % 32 == 0; N, K >= 1.
 */
bnb4_status bnb4_gemv(const void *x, const uint8_t *packedW,
                      const float *absmax, const void *bias, void *y,
                      int64_t N, int64_t K, int blocksize,
                      bnb4_quant_type quant_type, bnb4_dtype dt,
                      cudaStream_t stream);

/*
 * bnb4_gemv with a double-quantized absmax (see bnb4_double_quant): the
 * weight's absmax array [N, K/blocksize], flattened, arrives as its 8-bit
 * codes absmax_q [N*K/blocksize] and absmax_scales [ceil(N*K/blocksize /
 * group)].  The result equals bnb4_gemv's with absmax =
 * bnb4_dequant_absmax(absmax_q, absmax_scales) (the kernel rebuilds each
 * block's absmax with the same two fp32 operations), reading 1 + 4/group
 * bytes of absmax per block instead of 4.
 *   Same constraints as bnb4_gemv, plus group in {32, ..., 4096} (a power of
 *   two; 256 is the pages' default) and N <= 148 * 1024 (one row slab per
 *   SM), K <= 32768 (BNB4_ERR_SHAPE otherwise).
 */
bnb4_status bnb4_gemv_dq(const void *x, const uint8_t *packedW,
                         const uint8_t *absmax_q, const float *absmax_scales,
                         int group, const void *bias, void *y, int64_t N,
                         int64_t K, int blocksize, bnb4_quant_type quant_type,
                         bnb4_dtype dt, cudaStream_t stream);

/*
 * General matmul: Y[M, N] = X[M, K] @ dequant(W)^T (+ bias), row-major.
 *   X [M, K] of dt;  bias [N] of dt or NULL;  Y [M, N] of dt (out).
 *   Same constraints as bnb4_gemv; M >= 1.  M == 1 runs the gemv kernel,
 *   small M streams the weight once through a register-decode tensor-core
 *   kernel, large M runs the tcgen05 kernel that dequantizes weight tiles
 *   into shared memory.
 */
bnb4_status bnb4_gemm(const void *X, const uint8_t *packedW,
                      const float *absmax, const void *bias, void *Y,
                      int64_t M, int64_t N, int64_t K, int blocksize,
                      bnb4_quant_type quant_type, bnb4_dtype dt,
                      cudaStream_t stream);

/*
 * Backward of bnb4_gemm with respect to its input:
 *   dX[M, K] = dY[M, N] @ dequant(W)   (reduction over N, no bias term).
 *   dY [M, N] of dt;  dX [M, K] of dt (out); same weight arguments and
 *   constraints as bnb4_gemm, plus N % 8 == 0 (dY rows are read with TMA,
 *   which needs a 16-byte row pitch).
 */
bnb4_status bnb4_gemm_backward(const void *dY, const uint8_t *packedW,
                               const float *absmax, void *dX, int64_t M,
                               int64_t N, int64_t K, int blocksize,
                               bnb4_quant_type quant_type, bnb4_dtype dt,
                               cudaStream_t stream);

/*
 * bnb4_gemm and bnb4_gemm_backward with the weight's absmax given as 8-bit
 * statistics (see bnb4_double_quant / bnb4_gemv_dq): absmax_q
 * [N*K/blocksize] codes and absmax_scales [ceil(N*K/blocksize / group)]
 * fp32, both device pointers, 16-byte aligned.  Each block's absmax is
 * rebuilt inside the kernel as bnb4_dequant_absmax computes it, so the
 * result is bit-identical to bnb4_gemm / bnb4_gemm_backward given the
 * array bnb4_dequant_absmax writes, with no such array in memory.
 *   dt in {f16, bf16}; group a power of two in [32, 4096]
 *   (BNB4_ERR_BLOCKSIZE otherwise); other arguments and constraints as for
 *   bnb4_gemm / bnb4_gemm_backward.
 */
bnb4_status bnb4_gemm_dq(const void *X, const uint8_t *packedW,
                         const uint8_t *absmax_q, const float *absmax_scales,
                         int group, const void *bias, void *Y, int64_t M,
                         int64_t N, int64_t K, int blocksize,
                         bnb4_quant_type quant_type, bnb4_dtype dt,
                         cudaStream_t stream);
bnb4_status bnb4_gemm_backward_dq(const void *dY, const uint8_t *packedW,
                                  const uint8_t *absmax_q,
                                  const float *absmax_scales, int group,
                                  void *dX, int64_t M, int64_t N, int64_t K,
                                  int blocksize, bnb4_quant_type quant_type,
                                  bnb4_dtype dt, cudaStream_t stream);

/*
 * Double quantization of an absmax array (the pages give the call and the
 * group of 256, not the arithmetic; this is the plainest reading).  For each
 * group of `group` consecutive values (the last one may be short):
 *   scales[g] = the group maximum in fp32 (values not above the running
 *               maximum, NaN included, are skipped; +0 if none is > 0);
 *   absmax_q[i] = clamp(rint(RN(RN(absmax[i] / scales[g]) * 255)), 0, 255),
 *               rint ties to even, NaN -> 0, and 0 when scales[g] == 0.
 *   absmax   [n] float32, absmax_q [n] uint8 (out), scales [ceil(n/group)]
 *            float32 (out); all 16-byte aligned.
 *   group in {32, 64, ..., 4096} (256 is the pages' default); n >= 0.
 * 8 + 32/group bits per scale instead of 32.
 */
bnb4_status bnb4_double_quant(const float *absmax, int64_t n, int group,
                              uint8_t *absmax_q, float *scales,
                              cudaStream_t stream);

/*
 * Inverse of bnb4_double_quant:
 *   absmax[i] = RN(float(absmax_q[i]) * RN(scales[i / group] / 255)).
 * Same arguments and constraints (absmax is the [n] float32 output).
 */
bnb4_status bnb4_dequant_absmax(const uint8_t *absmax_q, const float *scales,
                                int64_t n, int group, float *absmax,
                                cudaStream_t stream);

/*
 * 8-bit blockwise quantization against the caller's code table (the pages
 * print no 8-bit table).  Per block of `blocksize` elements (the last may be
 * short): absmax = max |x| (fp32), v = x / absmax (IEEE fp32, 0 for an
 * all-zero block), q[i] = the index of the entry nearest v, ties to the
 * smaller index (exact; NaN gives 0), one byte per element.
 *   x      [n] of x_dtype (f32 / f16 / bf16), 16-byte aligned.
 *   q      [n] bytes out, absmax [ceil(n/blocksize)] float32 out; 16-byte aligned.
 *   code   HOST pointer to 256 float32 entries, read during the call only:
 *          strictly ascending, finite, in [-1, 1], each 0 or at least 2^-24
 *          in magnitude (BNB4_ERR_CODE otherwise).
 *   blocksize in {64, ..., 4096}; n >= 0.
 */
bnb4_status bnb4_quantize_8bit(const void *x, uint8_t *q, float *absmax,
                               int64_t n, int blocksize, const float *code,
                               bnb4_dtype x_dtype, cudaStream_t stream);

/*
 * Inverse: out[i] = RN_out_dtype(fp32(code[q[i]] * absmax[i / blocksize])).
 * Same arguments and constraints (out [n] of out_dtype, 16-byte aligned).
 */
bnb4_status bnb4_dequantize_8bit(const uint8_t *q, const float *absmax,
                                 void *out, int64_t n, int blocksize,
                                 const float *code, bnb4_dtype out_dtype,
                                 cudaStream_t stream);

/*
 * 4-bit embedding lookup.  The [V, D] table was quantized by bnb4_quantize as
 * one flat array of V*D elements; out[r, k] = the dequantized element
 * idx[r] * D + k (as bnb4_dequantize computes it), in out_dtype.
 *   packed [ceil(V*D/2)], absmax [ceil(V*D/blocksize)], idx [n_idx] int64
 *   (device), out [n_idx, D]; all 16-byte aligned.  V >= 0, D >= 1,
 *   n_idx >= 0.  Rows with D % 16 == 0 take the vector path.
 *   The indices are on the device and are not checked before the launch: an
 *   index outside [0, V) gives a row of zeros and is counted, and the next
 *   bnb4_device_status returns BNB4_ERR_INDEX.
 */
bnb4_status bnb4_embedding_4bit(const uint8_t *packed, const float *absmax,
                                int64_t V, int64_t D, int blocksize,
                                bnb4_quant_type quant_type, const int64_t *idx,
                                int64_t n_idx, void *out, bnb4_dtype out_dtype,
                                cudaStream_t stream);

/*
 * Device-side status of the library's kernels (no counterpart on the pages:
 * a diagnostic for checks that can only happen on the device).  Three kinds
 * of device-side error are counted, in device words shared by every stream
 * of the current device:
 *   BNB4_ERR_DEVICE   a gemv launch found that its shared-memory plan does not
 *                     fit the memory it was given (it wrote nothing);
 *   BNB4_ERR_TIMEOUT  a bounded mbarrier wait of a tensor-core kernel gave up
 *                     after about one second (that kernel skipped its
 *                     remaining work, so its outputs are undefined, freed its
 *                     tensor memory and returned);
 *   BNB4_ERR_INDEX    an embedding lookup met an index outside [0, V).
 * Synchronises `stream` (blocking the host), then returns the most severe
 * kind with a nonzero count, in the order above, and clears that count alone
 * (one atomic exchange on the device, so an error raised meanwhile by a
 * kernel on another stream is not lost); the other counts stay for the next
 * call.  BNB4_OK when every count is zero; BNB4_ERR_CUDA if the
 * synchronisation or a read failed (for instance after an earlier launch
 * error).  The counts cover every kernel that finished before the call, on
 * any stream; two host threads calling this at once may each see the other's
 * report.
 */
bnb4_status bnb4_device_status(cudaStream_t stream);

/*
 * Enqueues one small kernel whose mbarrier wait nothing completes; the wait
 * gives up after 1 ms, so the next bnb4_device_status reports
 * BNB4_ERR_TIMEOUT.  For testing the timeout path without faulting or
 * hanging the GPU.
 */
bnb4_status bnb4_selftest_wait_timeout(cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* BNB4_H */
