// kernels.h -- host launchers for the libbnb4 kernels (internal to the library).
// Arguments have been validated by the C ABI layer (api.cu) before these run.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/bnb4.h"

namespace bnb4 {

// number of SMs of the current device (cached per device)
int device_sm_count();

cudaError_t launch_quantize(const void *x, uint8_t *packed, float *absmax, int64_t n,
                            int blocksize, bnb4_quant_type qt, bnb4_dtype dt,
                            cudaStream_t stream);

cudaError_t launch_dequantize(const uint8_t *packed, const float *absmax, void *out, int64_t n,
                              int blocksize, bnb4_quant_type qt, bnb4_dtype dt,
                              cudaStream_t stream);

// M == 1, CUDA cores; handles N <= gemv_max_rows() and K <= gemv_max_k()
int64_t gemv_max_rows();
int64_t gemv_max_k();
// absmax_q == nullptr: fp32 absmax; else 8-bit double-quantized absmax codes
// with one fp32 scale per `group` codes (absmax unused)
cudaError_t launch_gemv(const void *x, const uint8_t *W, const float *absmax, const uint8_t *absmax_q,
                        const float *scales, int group, const void *bias, void *y, int64_t N,
                        int64_t K, int blocksize, bnb4_quant_type qt, bnb4_dtype dt,
                        cudaStream_t stream);

// 1 <= M <= 16: TMA-staged weights decoded in registers, mma.sync with the
// 16-row token tile.  absmax_q == nullptr: fp32 absmax; else 8-bit
// double-quantized absmax codes with one fp32 scale per `group` codes
// (absmax_f32 unused)
cudaError_t launch_gemm_small(const void *X, const uint8_t *W, const float *absmax_f32, const uint8_t *absmax_q,
                              const float *scales, int group, const void *bias, void *Y, int64_t M, int64_t N,
                              int64_t K, int blocksize, bnb4_quant_type qt, bnb4_dtype dt,
                              cudaStream_t stream);

// large M: tcgen05 with weight tiles dequantized into shared memory.
// backward == true computes dX[M, K] = dY[M, N] @ dequant(W) instead.
// (absmax as for launch_gemm_small)
cudaError_t launch_gemm_tc(const void *A, const uint8_t *W, const float *absmax_f32, const uint8_t *absmax_q,
                           const float *scales, int group, const void *bias, void *D, int64_t M, int64_t N,
                           int64_t K, int blocksize, bnb4_quant_type qt, bnb4_dtype dt, bool backward,
                           cudaStream_t stream);

// fp32 compute dtype (x, bias, y in float32; the exact fp32 dequantized
// weight; CUDA-core FMAs): M == 1 up to gemv_f32_max_rows() x gemv_f32_max_k(),
// and a tiled kernel for any M (backward == true computes dX = dY @ dequant(W))
int64_t gemv_f32_max_rows();
int64_t gemv_f32_max_k();
cudaError_t launch_gemv_f32(const float *x, const uint8_t *W, const float *absmax, const float *bias, float *y,
                            int64_t N, int64_t K, int blocksize, bnb4_quant_type qt, cudaStream_t stream);
cudaError_t launch_gemm_f32(const float *A, const uint8_t *W, const float *absmax, const float *bias, float *Y,
                            int64_t M, int64_t N, int64_t K, int blocksize, bnb4_quant_type qt, bool backward,
                            cudaStream_t stream);

// double quantization of an absmax array (groups of `group`, a power of two
// in [32, 4096]) and its inverse
cudaError_t launch_double_quant(const float *absmax, int64_t n, int group, uint8_t *q, float *scales,
                                cudaStream_t stream);
cudaError_t launch_dequant_absmax(const uint8_t *q, const float *scales, int64_t n, int group, float *out,
                                  cudaStream_t stream);

// 8-bit blockwise quantization against a caller's 256-entry table (host
// pointer; code8_table_usable must hold)
bool code8_table_usable(const float *code);
cudaError_t launch_quantize_8bit(const void *x, uint8_t *q, float *absmax, int64_t n, int blocksize,
                                 const float *code, bnb4_dtype dt, cudaStream_t stream);
cudaError_t launch_dequantize_8bit(const uint8_t *q, const float *absmax, void *out, int64_t n, int blocksize,
                                   const float *code, bnb4_dtype dt, cudaStream_t stream);

// rows of a 4-bit-quantized [V, D] table; bad indices give zero rows and are
// counted in a device word (quant_bad_indices_address)
cudaError_t launch_embedding_4bit(const uint8_t *packed, const float *absmax, int64_t V, int64_t D, int blocksize,
                                  bnb4_quant_type qt, const int64_t *idx, int64_t n_idx, void *out,
                                  bnb4_dtype dt, cudaStream_t stream);
cudaError_t quant_bad_indices_address(unsigned int **p);

// Device addresses (current device) of the words that count device-side
// errors: gemv launches that found their shared-memory plan unusable (they
// write nothing), and bounded waits that gave up, per kernel file
cudaError_t gemv_layout_errors_address(unsigned int **p);
cudaError_t gemm_tc_timeouts_address(unsigned int **p);
cudaError_t gemm_small_timeouts_address(unsigned int **p);

// one kernel whose mbarrier wait runs out after 1 ms (tests the timeout path)
cudaError_t launch_selftest_wait_timeout(cudaStream_t stream);

// largest M handled by launch_gemm_small
constexpr int64_t kSmallMMax = 16;

}  // namespace bnb4
