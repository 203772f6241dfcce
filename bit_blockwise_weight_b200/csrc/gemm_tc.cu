// gemm_tc.cu -- placeholder, replaced by the tcgen05 kernel.
#include "common.cuh"
#include "kernels.h"

namespace bnb4 {
cudaError_t launch_gemm_tc(const void *, const uint8_t *, const float *, const void *, void *,
                           int64_t, int64_t, int64_t, int, bnb4_quant_type, bnb4_dtype, bool,
                           cudaStream_t) {
    return cudaErrorNotSupported;
}
}  // namespace bnb4
