// api.cu -- the C ABI of libbnb4.so (declared in include/bnb4.h).
//
// Each entry point validates its arguments on the host, picks a kernel and
// enqueues it on the caller's stream.  Nothing is allocated, nothing is
// synchronised, and a failed check enqueues nothing.  There is no fallback:
// an input the kernels do not handle is an error.
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace bnb4 {

int device_sm_count() {
    static std::atomic<int> cache[kMaxDevices];
    return cached_per_device(cache, [] {
        int dev = 0, v = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) {
            (void)cudaGetLastError();
            return 148;  // every grid here is correct for any size; this only sizes it
        }
        return v;
    });
}

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_blocksize(int b) {
    return b >= 64 && b <= 4096 && (b & (b - 1)) == 0;
}

bool valid_qtype(bnb4_quant_type q) { return q == BNB4_NF4 || q == BNB4_FP4; }

bool valid_dtype(bnb4_dtype d) { return d == BNB4_F32 || d == BNB4_F16 || d == BNB4_BF16; }

constexpr int64_t kMaxDim = (int64_t)1 << 31;

bnb4_status check_matmul(const void *a, const uint8_t *W, const float *absmax, const void *bias,
                         const void *out, int64_t M, int64_t N, int64_t K, int blocksize,
                         bnb4_quant_type qt, bnb4_dtype dt, bool allow_f32) {
    if (!a || !W || !absmax || !out) return BNB4_ERR_NULL;
    if (!aligned16(a) || !aligned16(W) || !aligned16(absmax) || !aligned16(out) ||
        (bias && !aligned16(bias)))
        return BNB4_ERR_ALIGN;
    if (!valid_blocksize(blocksize)) return BNB4_ERR_BLOCKSIZE;
    if (!valid_qtype(qt)) return BNB4_ERR_QTYPE;
    if (dt != BNB4_F16 && dt != BNB4_BF16 && !(allow_f32 && dt == BNB4_F32)) return BNB4_ERR_DTYPE;
    if (M < 1 || N < 1 || K < 1 || M >= kMaxDim || N >= kMaxDim || K >= kMaxDim)
        return BNB4_ERR_SHAPE;
    if (K % 32 != 0 || K % blocksize != 0) return BNB4_ERR_SHAPE;
    return BNB4_OK;
}

bnb4_status from_cuda(cudaError_t e) { return e == cudaSuccess ? BNB4_OK : BNB4_ERR_CUDA; }

// reads and clears a device error count in one atomic exchange
__global__ void take_counter_kernel(unsigned int *count) { (void)atomicExch(count, 0u); }

}  // namespace
}  // namespace bnb4

using namespace bnb4;

extern "C" {

int bnb4_version(void) { return 1 * 10000 + 0 * 100 + 0; }

const char *bnb4_status_string(bnb4_status s) {
    switch (s) {
    case BNB4_OK: return "ok";
    case BNB4_ERR_NULL: return "a required pointer is NULL";
    case BNB4_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case BNB4_ERR_BLOCKSIZE: return "blocksize must be a power of two in [64, 4096]";
    case BNB4_ERR_SHAPE: return "invalid shape (sizes, K % blocksize, K % 32)";
    case BNB4_ERR_DTYPE: return "dtype not supported by this call";
    case BNB4_ERR_QTYPE: return "quant type must be NF4 or FP4";
    case BNB4_ERR_CUDA: return "CUDA kernel launch failed";
    case BNB4_ERR_TIMEOUT: return "a bounded device-side wait timed out";
    case BNB4_ERR_CODE: return "8-bit code table must be 256 strictly ascending entries in [-1, 1], each 0 or >= 2^-24";
    case BNB4_ERR_INDEX: return "an embedding index was out of range";
    case BNB4_ERR_DEVICE: return "a kernel found its launch configuration unusable and wrote nothing";
    }
    return "unknown status";
}

bnb4_status bnb4_quantize(const void *x, uint8_t *packed, float *absmax, int64_t n, int blocksize,
                          bnb4_quant_type qt, bnb4_dtype dt, cudaStream_t stream) {
    if (n < 0) return BNB4_ERR_SHAPE;
    if (!valid_blocksize(blocksize)) return BNB4_ERR_BLOCKSIZE;
    if (!valid_qtype(qt)) return BNB4_ERR_QTYPE;
    if (!valid_dtype(dt)) return BNB4_ERR_DTYPE;
    if (n == 0) return BNB4_OK;
    if (!x || !packed || !absmax) return BNB4_ERR_NULL;
    if (!aligned16(x) || !aligned16(packed) || !aligned16(absmax)) return BNB4_ERR_ALIGN;
    return from_cuda(launch_quantize(x, packed, absmax, n, blocksize, qt, dt, stream));
}

bnb4_status bnb4_dequantize(const uint8_t *packed, const float *absmax, void *out, int64_t n,
                            int blocksize, bnb4_quant_type qt, bnb4_dtype dt, cudaStream_t stream) {
    if (n < 0) return BNB4_ERR_SHAPE;
    if (!valid_blocksize(blocksize)) return BNB4_ERR_BLOCKSIZE;
    if (!valid_qtype(qt)) return BNB4_ERR_QTYPE;
    if (!valid_dtype(dt)) return BNB4_ERR_DTYPE;
    if (n == 0) return BNB4_OK;
    if (!packed || !absmax || !out) return BNB4_ERR_NULL;
    if (!aligned16(packed) || !aligned16(absmax) || !aligned16(out)) return BNB4_ERR_ALIGN;
    return from_cuda(launch_dequantize(packed, absmax, out, n, blocksize, qt, dt, stream));
}

bnb4_status bnb4_gemv(const void *x, const uint8_t *W, const float *absmax, const void *bias,
                      void *y, int64_t N, int64_t K, int blocksize, bnb4_quant_type qt,
                      bnb4_dtype dt, cudaStream_t stream) {
    bnb4_status s = check_matmul(x, W, absmax, bias, y, 1, N, K, blocksize, qt, dt, true);
    if (s != BNB4_OK) return s;
    if (dt == BNB4_F32) return bnb4_gemm(x, W, absmax, bias, y, 1, N, K, blocksize, qt, dt, stream);
    if (N <= gemv_max_rows() && K <= gemv_max_k())
        return from_cuda(launch_gemv(x, W, absmax, nullptr, nullptr, 0, bias, y, N, K, blocksize, qt, dt,
                                     stream));
    // shapes beyond the CUDA-core kernel's shared-memory plan: the same product
    // through the matrix kernels (x is a 1 x K matrix)
    return bnb4_gemm(x, W, absmax, bias, y, 1, N, K, blocksize, qt, dt, stream);
}

bnb4_status bnb4_gemv_dq(const void *x, const uint8_t *W, const uint8_t *absmax_q,
                         const float *absmax_scales, int group, const void *bias, void *y, int64_t N,
                         int64_t K, int blocksize, bnb4_quant_type qt, bnb4_dtype dt,
                         cudaStream_t stream) {
    if (!absmax_scales) return BNB4_ERR_NULL;
    if (!aligned16(absmax_scales)) return BNB4_ERR_ALIGN;
    // absmax_q stands in the fp32 absmax's place for the common checks
    bnb4_status s = check_matmul(x, W, reinterpret_cast<const float *>(absmax_q), bias, y, 1, N, K,
                                 blocksize, qt, dt, false);
    if (s != BNB4_OK) return s;
    if (group < 32 || group > 4096 || (group & (group - 1)) != 0) return BNB4_ERR_BLOCKSIZE;
    if (N > gemv_max_rows() || K > gemv_max_k()) return BNB4_ERR_SHAPE;
    return from_cuda(launch_gemv(x, W, nullptr, absmax_q, absmax_scales, group, bias, y, N, K, blocksize,
                                 qt, dt, stream));
}

bnb4_status bnb4_gemm(const void *X, const uint8_t *W, const float *absmax, const void *bias,
                      void *Y, int64_t M, int64_t N, int64_t K, int blocksize, bnb4_quant_type qt,
                      bnb4_dtype dt, cudaStream_t stream) {
    bnb4_status s = check_matmul(X, W, absmax, bias, Y, M, N, K, blocksize, qt, dt, true);
    if (s != BNB4_OK) return s;
    if (dt == BNB4_F32) {
        // fp32: CUDA-core kernels with the exact fp32 dequantized weight
        if (M == 1 && N <= gemv_f32_max_rows() && K <= gemv_f32_max_k())
            return from_cuda(launch_gemv_f32(static_cast<const float *>(X), W, absmax,
                                             static_cast<const float *>(bias), static_cast<float *>(Y), N, K,
                                             blocksize, qt, stream));
        return from_cuda(launch_gemm_f32(static_cast<const float *>(X), W, absmax, static_cast<const float *>(bias),
                                         static_cast<float *>(Y), M, N, K, blocksize, qt, false, stream));
    }
    // one token: the gemv kernel (the same product, faster at M == 1)
    if (M == 1 && N <= gemv_max_rows() && K <= gemv_max_k())
        return from_cuda(launch_gemv(X, W, absmax, nullptr, nullptr, 0, bias, Y, N, K, blocksize, qt, dt, stream));
    // small M: one pass over the weight stream, tensor-core tiles fed from registers
    if (M <= kSmallMMax)
        return from_cuda(launch_gemm_small(X, W, absmax, nullptr, nullptr, 0, bias, Y, M, N, K, blocksize, qt, dt,
                                           stream));
    return from_cuda(launch_gemm_tc(X, W, absmax, nullptr, nullptr, 0, bias, Y, M, N, K, blocksize, qt, dt, false,
                                    stream));
}

bnb4_status bnb4_gemm_backward(const void *dY, const uint8_t *W, const float *absmax, void *dX,
                               int64_t M, int64_t N, int64_t K, int blocksize, bnb4_quant_type qt,
                               bnb4_dtype dt, cudaStream_t stream) {
    bnb4_status s = check_matmul(dY, W, absmax, nullptr, dX, M, N, K, blocksize, qt, dt, true);
    if (s != BNB4_OK) return s;
    if (dt == BNB4_F32)
        return from_cuda(launch_gemm_f32(static_cast<const float *>(dY), W, absmax, nullptr, static_cast<float *>(dX),
                                         M, N, K, blocksize, qt, true, stream));
    if (N % 8 != 0) return BNB4_ERR_SHAPE;  // dY rows are TMA-loaded: 16-byte row pitch
    return from_cuda(launch_gemm_tc(dY, W, absmax, nullptr, nullptr, 0, nullptr, dX, M, N, K, blocksize, qt, dt,
                                    true, stream));
}

bnb4_status bnb4_gemm_dq(const void *X, const uint8_t *W, const uint8_t *absmax_q, const float *absmax_scales,
                         int group, const void *bias, void *Y, int64_t M, int64_t N, int64_t K, int blocksize,
                         bnb4_quant_type qt, bnb4_dtype dt, cudaStream_t stream) {
    if (!absmax_scales) return BNB4_ERR_NULL;
    if (!aligned16(absmax_scales)) return BNB4_ERR_ALIGN;
    bnb4_status s = check_matmul(X, W, reinterpret_cast<const float *>(absmax_q), bias, Y, M, N, K, blocksize, qt,
                                 dt, false);
    if (s != BNB4_OK) return s;
    if (group < 32 || group > 4096 || (group & (group - 1)) != 0) return BNB4_ERR_BLOCKSIZE;
    if (M == 1 && N <= gemv_max_rows() && K <= gemv_max_k())
        return from_cuda(launch_gemv(X, W, nullptr, absmax_q, absmax_scales, group, bias, Y, N, K, blocksize, qt,
                                     dt, stream));
    if (M <= kSmallMMax)
        return from_cuda(launch_gemm_small(X, W, nullptr, absmax_q, absmax_scales, group, bias, Y, M, N, K,
                                           blocksize, qt, dt, stream));
    return from_cuda(launch_gemm_tc(X, W, nullptr, absmax_q, absmax_scales, group, bias, Y, M, N, K, blocksize,
                                    qt, dt, false, stream));
}

bnb4_status bnb4_gemm_backward_dq(const void *dY, const uint8_t *W, const uint8_t *absmax_q,
                                  const float *absmax_scales, int group, void *dX, int64_t M, int64_t N, int64_t K,
                                  int blocksize, bnb4_quant_type qt, bnb4_dtype dt, cudaStream_t stream) {
    if (!absmax_scales) return BNB4_ERR_NULL;
    if (!aligned16(absmax_scales)) return BNB4_ERR_ALIGN;
    bnb4_status s = check_matmul(dY, W, reinterpret_cast<const float *>(absmax_q), nullptr, dX, M, N, K, blocksize,
                                 qt, dt, false);
    if (s != BNB4_OK) return s;
    if (group < 32 || group > 4096 || (group & (group - 1)) != 0) return BNB4_ERR_BLOCKSIZE;
    if (N % 8 != 0) return BNB4_ERR_SHAPE;
    return from_cuda(launch_gemm_tc(dY, W, nullptr, absmax_q, absmax_scales, group, nullptr, dX, M, N, K,
                                    blocksize, qt, dt, true, stream));
}

bnb4_status bnb4_double_quant(const float *absmax, int64_t n, int group, uint8_t *absmax_q,
                              float *scales, cudaStream_t stream) {
    if (n < 0) return BNB4_ERR_SHAPE;
    if (group < 32 || group > 4096 || (group & (group - 1)) != 0) return BNB4_ERR_BLOCKSIZE;
    if (n == 0) return BNB4_OK;
    if (!absmax || !absmax_q || !scales) return BNB4_ERR_NULL;
    if (!aligned16(absmax) || !aligned16(absmax_q) || !aligned16(scales)) return BNB4_ERR_ALIGN;
    return from_cuda(launch_double_quant(absmax, n, group, absmax_q, scales, stream));
}

bnb4_status bnb4_dequant_absmax(const uint8_t *absmax_q, const float *scales, int64_t n, int group,
                                float *absmax, cudaStream_t stream) {
    if (n < 0) return BNB4_ERR_SHAPE;
    if (group < 32 || group > 4096 || (group & (group - 1)) != 0) return BNB4_ERR_BLOCKSIZE;
    if (n == 0) return BNB4_OK;
    if (!absmax_q || !scales || !absmax) return BNB4_ERR_NULL;
    if (!aligned16(absmax_q) || !aligned16(scales) || !aligned16(absmax)) return BNB4_ERR_ALIGN;
    return from_cuda(launch_dequant_absmax(absmax_q, scales, n, group, absmax, stream));
}

bnb4_status bnb4_quantize_8bit(const void *x, uint8_t *q, float *absmax, int64_t n, int blocksize,
                               const float *code, bnb4_dtype dt, cudaStream_t stream) {
    if (!valid_blocksize(blocksize)) return BNB4_ERR_BLOCKSIZE;
    if (!valid_dtype(dt)) return BNB4_ERR_DTYPE;
    if (n < 0 || n >= ((int64_t)1 << 40)) return BNB4_ERR_SHAPE;
    if (!code) return BNB4_ERR_NULL;
    if (!code8_table_usable(code)) return BNB4_ERR_CODE;
    if (n == 0) return BNB4_OK;
    if (!x || !q || !absmax) return BNB4_ERR_NULL;
    if (!aligned16(x) || !aligned16(q) || !aligned16(absmax)) return BNB4_ERR_ALIGN;
    return from_cuda(launch_quantize_8bit(x, q, absmax, n, blocksize, code, dt, stream));
}

bnb4_status bnb4_dequantize_8bit(const uint8_t *q, const float *absmax, void *out, int64_t n, int blocksize,
                                 const float *code, bnb4_dtype dt, cudaStream_t stream) {
    if (!valid_blocksize(blocksize)) return BNB4_ERR_BLOCKSIZE;
    if (!valid_dtype(dt)) return BNB4_ERR_DTYPE;
    if (n < 0 || n >= ((int64_t)1 << 40)) return BNB4_ERR_SHAPE;
    if (!code) return BNB4_ERR_NULL;
    if (!code8_table_usable(code)) return BNB4_ERR_CODE;
    if (n == 0) return BNB4_OK;
    if (!q || !absmax || !out) return BNB4_ERR_NULL;
    if (!aligned16(q) || !aligned16(absmax) || !aligned16(out)) return BNB4_ERR_ALIGN;
    return from_cuda(launch_dequantize_8bit(q, absmax, out, n, blocksize, code, dt, stream));
}

bnb4_status bnb4_embedding_4bit(const uint8_t *packed, const float *absmax, int64_t V, int64_t D, int blocksize,
                                bnb4_quant_type qt, const int64_t *idx, int64_t n_idx, void *out,
                                bnb4_dtype dt, cudaStream_t stream) {
    if (!valid_blocksize(blocksize)) return BNB4_ERR_BLOCKSIZE;
    if (!valid_qtype(qt)) return BNB4_ERR_QTYPE;
    if (!valid_dtype(dt)) return BNB4_ERR_DTYPE;
    if (V < 0 || D < 1 || n_idx < 0 || V >= kMaxDim || D >= kMaxDim || n_idx >= kMaxDim ||
        (double)V * (double)D >= 0x1p40 || (double)n_idx * (double)D >= 0x1p40)
        return BNB4_ERR_SHAPE;
    if (n_idx == 0) return BNB4_OK;
    if (!packed || !absmax || !idx || !out) return BNB4_ERR_NULL;
    if (!aligned16(packed) || !aligned16(absmax) || !aligned16(idx) || !aligned16(out)) return BNB4_ERR_ALIGN;
    return from_cuda(launch_embedding_4bit(packed, absmax, V, D, blocksize, qt, idx, n_idx, out, dt, stream));
}

bnb4_status bnb4_device_status(cudaStream_t stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return BNB4_ERR_CUDA;
    // in order of severity: the first nonzero count is the one reported, and
    // only it is cleared; the others stay for the next call
    unsigned int *w[4] = {nullptr, nullptr, nullptr, nullptr};
    if (gemv_layout_errors_address(&w[0]) != cudaSuccess || gemm_tc_timeouts_address(&w[1]) != cudaSuccess ||
        gemm_small_timeouts_address(&w[2]) != cudaSuccess || quant_bad_indices_address(&w[3]) != cudaSuccess)
        return BNB4_ERR_CUDA;
    const bnb4_status code[4] = {BNB4_ERR_DEVICE, BNB4_ERR_TIMEOUT, BNB4_ERR_TIMEOUT, BNB4_ERR_INDEX};
    for (int i = 0; i < 4; ++i) {
        unsigned int v = 0;
        if (cudaMemcpy(&v, w[i], sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return BNB4_ERR_CUDA;
        if (v == 0) continue;
        // one atomic exchange on the device per word: an increment that lands
        // after the read above is taken with it, never lost.  The timeout
        // words (one per kernel file) are one status and are taken together.
        const int last = code[i] == BNB4_ERR_TIMEOUT ? 2 : i;
        for (int j = i; j <= last; ++j) {
            take_counter_kernel<<<1, 1, 0, stream>>>(w[j]);
            if (cudaGetLastError() != cudaSuccess) return BNB4_ERR_CUDA;
        }
        if (cudaStreamSynchronize(stream) != cudaSuccess) return BNB4_ERR_CUDA;
        return code[i];
    }
    return BNB4_OK;
}

bnb4_status bnb4_selftest_wait_timeout(cudaStream_t stream) {
    return from_cuda(launch_selftest_wait_timeout(stream));
}

}  // extern "C"
