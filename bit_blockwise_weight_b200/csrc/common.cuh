// common.cuh -- device-side definitions shared by the libbnb4 kernels.
//
// Code tables, decision tables for the nearest-code search, dtype traits and
// small warp helpers.  Everything here is the library's own; the CPU oracle
// under oracle/ is a separate program that shares none of it.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/bnb4.h"

namespace bnb4 {

constexpr unsigned FULL = 0xffffffffu;

// ---------------------------------------------------------------- dtypes

struct F32 {};
struct F16 {};
struct BF16 {};

template <typename D> struct Dt;
template <> struct Dt<F32> {
    using T = float;
    static constexpr int bytes = 4;
};
template <> struct Dt<F16> {
    using T = __half;
    using T2 = __half2;
    static constexpr int bytes = 2;
    __device__ static __forceinline__ float to_f32(uint16_t b) {
        return __half2float(__ushort_as_half(b));
    }
    // round-to-nearest-even pair conversion; lo lands in the low half
    __device__ static __forceinline__ uint32_t pack2(float lo, float hi) {
        __half2 h = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&h);
    }
};
template <> struct Dt<BF16> {
    using T = __nv_bfloat16;
    using T2 = __nv_bfloat162;
    static constexpr int bytes = 2;
    __device__ static __forceinline__ float to_f32(uint16_t b) {
        return __uint_as_float(uint32_t(b) << 16);
    }
    __device__ static __forceinline__ uint32_t pack2(float lo, float hi) {
        __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&h);
    }
};

// ----------------------------------------------------------- code tables
//
// NF4: the 16 values of the NF4 workload definition ("mps-bitsandbytes 0.4.7",
// Features table, names the format; the values are rounded to fp32 here).
// FP4: E2M1 with bias 1 and subnormals, magnitudes {0,.5,1,1.5,2,3,4,6}/6,
// index = sign<<3 | exp<<1 | mant (the pages name FP4 only).

struct CodeTable {
    float v[16];
};

// Host-side construction (also used to build the decision tables).
CodeTable host_code_table(bnb4_quant_type qt);

// ------------------------------------------------------ decision tables
//
// Nearest-code search without a 16-way compare.  v in [-1, 1] falls into one
// of 27 cells k = rn(13 v + 13) (cell width 1/13 is below the smallest gap
// between two decision thresholds, so a cell holds at most one threshold).
// Lane k of a warp keeps thr[k] and lohi[k]; the code index of v is
//     (v > thr[k]) ? lohi[k] >> 4 : lohi[k] & 15,
// which equals argmin_i |v - code_i| with ties to the smallest index: each
// threshold is the fp32 value that splits its two neighbouring codes exactly
// (the largest fp32 <= midpoint, or < midpoint when the tie goes up).
struct QuantTables {
    float thr[32];
    uint32_t lohi[32];
};

QuantTables host_quant_tables(bnb4_quant_type qt);

// 12582925 = 1.5 * 2^23 + 13: the fma lands in [2^23, 2^24) where the fp32
// spacing is 1, so the low mantissa bits hold rn(13 v + 13).
__device__ __forceinline__ uint32_t cell_of(float v) {
    return __float_as_uint(__fmaf_rn(v, 13.0f, 12582925.0f));
}

__device__ __forceinline__ uint32_t nearest_code(float v, float my_thr, uint32_t my_lohi) {
    uint32_t k = cell_of(v);
    float t = __shfl_sync(FULL, my_thr, k);   // shfl reads lane k & 31
    uint32_t lh = __shfl_sync(FULL, my_lohi, k);
    return (v > t) ? (lh >> 4) : (lh & 15u);
}

// ------------------------------------------------------------- helpers

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(FULL, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
    return v;
}

__host__ __device__ constexpr int ilog2(int v) { return v <= 1 ? 0 : 1 + ilog2(v >> 1); }

}  // namespace bnb4
