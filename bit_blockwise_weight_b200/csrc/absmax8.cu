// absmax8.cu -- double quantization of an absmax array and its inverse.
//
// "mps-bitsandbytes 0.4.7", Functional API, Double Quantization:
// double_quant(absmax, double_quant_block=256) -> (absmax_quant,
// absmax_scales) and dequant_absmax(absmax_quant, absmax_scales).  Per group
// of G consecutive absmax values (the last one may be short):
//   scale = the group maximum in fp32 (values not above the running maximum,
//           NaN included, are skipped, so a group without a value > 0 has +0);
//   q     = clamp(rint(RN(RN(a / scale) * 255)), 0, 255), rint ties to even,
//           NaN -> 0, and 0 when scale == 0;
//   inverse: out = RN(float(q) * RN(scale / 255)).
// An unsigned linear 8-bit code (absmax values are >= 0); every step is one
// correctly rounded fp32 operation (RN(scale / 255) by div255_rn), so the
// results are bit-exact.
//
// Both kernels are HBM-bound streams.  double_quant: one warp per group, its
// lanes reading and writing consecutive elements (coalesced), the maximum by
// xor-shuffles; persistent grid.  dequant_absmax: four values per thread.
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace bnb4 {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__global__ void __launch_bounds__(kThreads)
double_quant_kernel(const float *__restrict__ absmax, int64_t n, int log2G, uint8_t *__restrict__ q,
                    float *__restrict__ scales) {
    const int lane = threadIdx.x & 31;
    const int G = 1 << log2G;
    const int64_t ngroups = (n + G - 1) >> log2G;
    const int64_t warps = (int64_t)gridDim.x * kWarps;
    for (int64_t g = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); g < ngroups; g += warps) {
        const int64_t g0 = g << log2G;
        float m = 0.0f;
        // unrolled, so a lane's loads of the group leave together instead of
        // each waiting for the comparison before it
#pragma unroll 8
        for (int j = lane; j < G; j += 32) {
            const int64_t i = g0 + j;
            if (i < n) {
                const float v = absmax[i];  // the second pass reads it again from cache
                if (v > m) m = v;  // NaN and values <= m are skipped
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float v = __shfl_xor_sync(FULL, m, o);
            if (v > m) m = v;
        }
        if (lane == 0) scales[g] = m;
#pragma unroll 8
        for (int j = lane; j < G; j += 32) {
            const int64_t i = g0 + j;
            if (i >= n) break;
            uint32_t code = 0u;
            if (m > 0.0f) {
                const float v = __fdiv_rn(absmax[i], m);
                const float r = rintf(__fmul_rn(v, 255.0f));
                if (r > 0.0f) code = r >= 255.0f ? 255u : (uint32_t)r;  // NaN and r <= 0 give 0
            }
            q[i] = (uint8_t)code;
        }
    }
}

__global__ void __launch_bounds__(kThreads)
dequant_absmax_kernel(const uint8_t *__restrict__ q, const float *__restrict__ scales, int64_t n, int log2G,
                      float *__restrict__ out) {
    const int64_t stride = (int64_t)gridDim.x * kThreads * 4;
    for (int64_t i0 = ((int64_t)blockIdx.x * kThreads + threadIdx.x) * 4; i0 < n; i0 += stride) {
        if (i0 + 4 <= n) {
            const uchar4 c = __ldcs(reinterpret_cast<const uchar4 *>(q + i0));
            // four consecutive values never straddle a group (G >= 32)
            const float step = div255_rn(scales[i0 >> log2G]);
            __stcs(reinterpret_cast<float4 *>(out + i0),
                   make_float4(__fmul_rn((float)c.x, step), __fmul_rn((float)c.y, step),
                               __fmul_rn((float)c.z, step), __fmul_rn((float)c.w, step)));
        } else {
            for (int64_t i = i0; i < n; ++i)
                out[i] = __fmul_rn((float)q[i], div255_rn(scales[i >> log2G]));
        }
    }
}

template <typename Kern>
int persistent_grid(Kern kernel, std::atomic<int> (&cache)[kMaxDevices], int64_t work_ctas) {
    const int per_sm = cached_per_device(cache, [&] {
        int v = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, kernel, kThreads, 0) != cudaSuccess || v <= 0) {
            (void)cudaGetLastError();
            v = 4;
        }
        return v;
    });
    int64_t g = (int64_t)device_sm_count() * per_sm;
    if (work_ctas < g) g = work_ctas;
    return (int)(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_double_quant(const float *absmax, int64_t n, int group, uint8_t *q, float *scales,
                                cudaStream_t stream) {
    static std::atomic<int> cache[kMaxDevices];
    const int log2G = ilog2(group);
    const int64_t ngroups = (n + group - 1) / group;
    const int grid = persistent_grid(double_quant_kernel, cache, (ngroups + kWarps - 1) / kWarps);
    double_quant_kernel<<<grid, kThreads, 0, stream>>>(absmax, n, log2G, q, scales);
    return cudaGetLastError();
}

cudaError_t launch_dequant_absmax(const uint8_t *q, const float *scales, int64_t n, int group, float *out,
                                  cudaStream_t stream) {
    static std::atomic<int> cache[kMaxDevices];
    const int log2G = ilog2(group);
    const int grid = persistent_grid(dequant_absmax_kernel, cache, (n + kThreads * 4 - 1) / (kThreads * 4));
    dequant_absmax_kernel<<<grid, kThreads, 0, stream>>>(q, scales, n, log2G, out);
    return cudaGetLastError();
}

}  // namespace bnb4
