// gemv.cu -- gemv_4bit (M == 1): y = x @ dequant(W)^T (+ bias), CUDA cores.
//
// "Feat/mps gemm 4bit bf16", What runs natively now: gemv_4bit is a fused
// dequant + dot kernel; the bias epilogue is added before the one rounding of
// the output (section Correctness).  The weight stream (0.5 B per weight plus
// 4 B of absmax per block) is the whole cost, so the kernel is built around
// reading it once, coalesced, with enough bytes in flight.
//
// Work split:
//   * a CTA (8 warps) owns 32 rows and a K-range; warp w owns 4 rows;
//   * lane l reads 16 packed bytes (32 weights) of each of its warp's 4 rows
//     per 1024-element segment -- 512 contiguous bytes per row per warp load;
//   * x of the CTA's K-range is converted once to fp32 in shared memory;
//   * each lane decodes nibbles through a 16-entry code table held in the
//     warp's lanes (shfl), accumulates sum_k code * x in fp32 over its 32
//     weights (all inside one quantization block) and scales by the block's
//     absmax once;
//   * rows are reduced across lanes with xor-shuffles;
//   * when K is split over CTAs, the CTAs of one row range form a thread-block
//     cluster and add their partial rows through distributed shared memory,
//     so no global scratch is needed.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace bnb4 {

namespace {

constexpr int kWarps = 8;
constexpr int kRowsPerWarp = 4;
constexpr int kRowsPerCta = kWarps * kRowsPerWarp;  // 32
constexpr int kSeg = 1024;                          // elements per warp-wide load
constexpr int kMaxKc = 8192;                        // fp32 x slice <= 32 KB

__device__ __forceinline__ uint32_t shfl_idx(uint32_t v, uint32_t lane_bits) {
    uint32_t r;
    asm volatile("shfl.sync.idx.b32 %0, %1, %2, 0x1f, 0xffffffff;"
                 : "=r"(r)
                 : "r"(v), "r"(lane_bits));
    return r;
}

__device__ __forceinline__ uint4 ld_stream(const uint8_t *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

template <typename D>
__global__ void __launch_bounds__(kWarps * 32)
gemv_kernel(const uint16_t *__restrict__ x, const uint8_t *__restrict__ W,
            const float *__restrict__ absmax, const uint16_t *__restrict__ bias,
            uint16_t *__restrict__ y, int N, int K, int log2B, int Kc, CodeTable tab) {
    extern __shared__ float xs[];  // [Kc] fp32
    __shared__ float partial[kRowsPerCta];

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int ksplit = gridDim.y, kpart = blockIdx.y;
    const int k0 = kpart * Kc;
    const int k1 = min(K, k0 + Kc);
    const int row0 = blockIdx.x * kRowsPerCta;

    // x slice -> fp32 shared memory
    for (int k = k0 + threadIdx.x; k < k1; k += blockDim.x) xs[k - k0] = Dt<D>::to_f32(x[k]);
    __syncthreads();

    const uint32_t my_code = __float_as_uint(tab.v[lane & 15]);
    const int64_t row_bytes = K >> 1;
    const int nblk = K >> log2B;  // absmax entries per row

    int rows[kRowsPerWarp];
    bool rvalid[kRowsPerWarp];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
        rows[r] = row0 + warp * kRowsPerWarp + r;
        rvalid[r] = rows[r] < N;
    }

    float acc[kRowsPerWarp] = {0.f, 0.f, 0.f, 0.f};
    const int nseg = (k1 - k0 + kSeg - 1) / kSeg;

    // software pipeline: weights of segment s+1 are in flight while s computes
    uint4 wcur[kRowsPerWarp], wnext[kRowsPerWarp];
    auto load_seg = [&](int s, uint4 *dst) {
        const int kk = k0 + s * kSeg + lane * 32;
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
            if (rvalid[r] && kk < k1)
                dst[r] = ld_stream(W + (int64_t)rows[r] * row_bytes + (kk >> 1));
            else
                dst[r] = make_uint4(0, 0, 0, 0);
        }
    };
    if (nseg > 0) load_seg(0, wcur);

    for (int s = 0; s < nseg; ++s) {
        if (s + 1 < nseg) load_seg(s + 1, wnext);
        const int kk = k0 + s * kSeg + lane * 32;
        const bool kvalid = kk < k1;  // K % 32 == 0: a lane's 32 weights are all in or all out
        // every lane runs the decode (its shuffles need the whole warp); lanes
        // past the end multiply zero weights by zero x
        float xv[32];
        if (kvalid) {
            const float4 *xp = reinterpret_cast<const float4 *>(xs + (kk - k0));
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                float4 v = xp[q];
                xv[4 * q] = v.x; xv[4 * q + 1] = v.y; xv[4 * q + 2] = v.z; xv[4 * q + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int q = 0; q < 32; ++q) xv[q] = 0.f;
        }
        const int blk = kk >> log2B;
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
            const float a = (rvalid[r] && kvalid) ? __ldg(absmax + (int64_t)rows[r] * nblk + blk) : 0.f;
            const uint32_t w4[4] = {wcur[r].x, wcur[r].y, wcur[r].z, wcur[r].w};
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float ch = __uint_as_float(shfl_idx(my_code, w4[q] >> (8 * j + 4)));
                    const float cl = __uint_as_float(shfl_idx(my_code, w4[q] >> (8 * j)));
                    s0 = __fmaf_rn(ch, xv[8 * q + 2 * j], s0);
                    s1 = __fmaf_rn(cl, xv[8 * q + 2 * j + 1], s1);
                }
            }
            acc[r] = __fmaf_rn(s0 + s1, a, acc[r]);
        }
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) wcur[r] = wnext[r];
    }

#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
        const float v = warp_sum(acc[r]);
        if (lane == 0) partial[warp * kRowsPerWarp + r] = v;
    }

    if (ksplit == 1) {
        __syncthreads();
        if (threadIdx.x < kRowsPerCta) {
            const int row = row0 + threadIdx.x;
            if (row < N) {
                float v = partial[threadIdx.x];
                if (bias) v += Dt<D>::to_f32(bias[row]);
                y[row] = (uint16_t)(Dt<D>::pack2(v, 0.f) & 0xffffu);
            }
        }
        return;
    }

    // K split over the CTAs of a cluster: rank r finishes rows r, r + ksplit, ...
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    const int rank = (int)cluster.block_rank();
    if (threadIdx.x < kRowsPerCta && (threadIdx.x % ksplit) == rank) {
        const int row = row0 + threadIdx.x;
        float v = 0.f;
        for (int q = 0; q < ksplit; ++q) v += *cluster.map_shared_rank(&partial[threadIdx.x], q);
        if (row < N) {
            if (bias) v += Dt<D>::to_f32(bias[row]);
            y[row] = (uint16_t)(Dt<D>::pack2(v, 0.f) & 0xffffu);
        }
    }
    cluster.sync();  // keep every CTA's shared memory alive until all reads are done
}

}  // namespace

cudaError_t launch_gemv(const void *x, const uint8_t *W, const float *absmax, const void *bias,
                        void *y, int64_t N, int64_t K, int blocksize, bnb4_quant_type qt,
                        bnb4_dtype dt, cudaStream_t stream) {
    static const CodeTable nf4 = host_code_table(BNB4_NF4);
    static const CodeTable fp4 = host_code_table(BNB4_FP4);
    const CodeTable &tab = qt == BNB4_NF4 ? nf4 : fp4;

    const int sms = device_sm_count();
    const int groups = (int)((N + kRowsPerCta - 1) / kRowsPerCta);
    const int segs = (int)((K + kSeg - 1) / kSeg);
    int ksplit = 1;
    // enough CTAs to cover the GPU twice, and an x slice that fits 32 KB
    while (ksplit < 8 && ksplit < segs &&
           ((int64_t)groups * ksplit < 2 * sms || (K + ksplit - 1) / ksplit > kMaxKc))
        ++ksplit;
    // K-range per CTA in whole segments
    const int segs_per = (segs + ksplit - 1) / ksplit;
    ksplit = (segs + segs_per - 1) / segs_per;
    int Kc = segs_per * kSeg;
    if (Kc > K) Kc = (int)K;
    if (Kc > kMaxKc) return cudaErrorInvalidValue;  // K > 8 * 8192: not reached by the API limits below

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(groups, ksplit, 1);
    cfg.blockDim = dim3(kWarps * 32, 1, 1);
    cfg.dynamicSmemBytes = (size_t)Kc * sizeof(float);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = ksplit;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;

    const uint16_t *xp = static_cast<const uint16_t *>(x);
    const uint16_t *bp = static_cast<const uint16_t *>(bias);
    uint16_t *yp = static_cast<uint16_t *>(y);
    const int log2B = ilog2(blocksize);
    if (dt == BNB4_F16)
        return cudaLaunchKernelEx(&cfg, gemv_kernel<F16>, xp, W, absmax, bp, yp, (int)N, (int)K,
                                  log2B, Kc, tab);
    return cudaLaunchKernelEx(&cfg, gemv_kernel<BF16>, xp, W, absmax, bp, yp, (int)N, (int)K,
                              log2B, Kc, tab);
}

}  // namespace bnb4
