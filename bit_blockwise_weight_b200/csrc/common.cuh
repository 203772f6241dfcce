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

#include <atomic>

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

// ------------------------------------------- decode by byte permutation
//
// Dequantizing a run of one block without shuffles or table loads: the 16
// values RN_dtype(fp32(code_i * absmax)) are computed once per block and held
// as two byte planes (lo[q]: low bytes of entries 4q..4q+3; hi[q]: high
// bytes), from which prmt selects four entries at a time.  The values are the
// ones a per-element __fmul_rn followed by the dtype conversion produces.

struct ScaledPlanes {
    uint32_t lo[4], hi[4];
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

template <typename D>
__device__ __forceinline__ ScaledPlanes scaled_planes(const CodeTable &tab, float a) {
    ScaledPlanes s;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t p0 = Dt<D>::pack2(__fmul_rn(tab.v[4 * q], a), __fmul_rn(tab.v[4 * q + 1], a));
        const uint32_t p1 = Dt<D>::pack2(__fmul_rn(tab.v[4 * q + 2], a), __fmul_rn(tab.v[4 * q + 3], a));
        s.lo[q] = prmt(p0, p1, 0x6420u);
        s.hi[q] = prmt(p0, p1, 0x7531u);
    }
    return s;
}

// The four codes in the low 16 bits of x (two packed bytes, the first element
// of each byte in its high nibble) -> o0 = (e0, e1), o1 = (e2, e3), the first
// element of each pair in the low half.
__device__ __forceinline__ void decode4(const ScaledPlanes &s, uint32_t x, uint32_t &o0, uint32_t &o1) {
    const uint32_t sel = x & 0x7777u;                     // byte k <- entry (nibble k) & 7
    const uint32_t f = ((x >> 1) & 0x4444u) | 0x3210u;    // entries 8..15 where bit 3 is set
    const uint32_t rl = prmt(prmt(s.lo[0], s.lo[1], sel), prmt(s.lo[2], s.lo[3], sel), f);
    const uint32_t rh = prmt(prmt(s.hi[0], s.hi[1], sel), prmt(s.hi[2], s.hi[3], sel), f);
    // rl, rh list the nibbles in register order: e1, e0, e3, e2
    o0 = prmt(rl, rh, 0x4051u);
    o1 = prmt(rl, rh, 0x6273u);
}

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
    // One-shuffle screen.  key[k]: the threshold of cell k with its low four
    // mantissa bits replaced by the rank (position in ascending value order)
    // just above it, or -2^100 with the low bits holding the cell's only
    // rank.  The replacement moves a threshold by less than 2^-20, so an
    // element whose approximate quotient lies further than kNear from the key
    // decides exactly as its exact quotient would (rank = key & 15, less one
    // below the key); the others are redone exactly, with rank_lohi[k] = rank
    // below | rank above << 4.  fast: 0 = exact search only, 1 = ranks are
    // code indices, 2 = ranks map to code indices by the E2M1 fold
    // (r >= 7 ? r - 7 : 15 - r).
    uint32_t key[32];
    uint32_t rank_lohi[32];
    int fast;
    int valid;  // 0: a cell held two thresholds (the tables are unusable)
};
constexpr float kNear = 0x1p-19f;

QuantTables host_quant_tables(bnb4_quant_type qt);

// FP4 screen tables for inputs whose significands have p bits (bf16: 8,
// fp16: 11), with which the one-shuffle screen decides every element exactly
// (no element is near a threshold; see tables.cu).  Returns false, leaving
// q unusable, if a key cannot be placed.
bool host_fp4_exact_tables(int p, QuantTables &q);

// Screen tables for a code table whose thresholds every ratio of two p-bit
// values stays clear of (NF4 with bf16 inputs), likewise exact (tables.cu).
bool host_ratio_exact_tables(bnb4_quant_type qt, int p, QuantTables &q);

// 12582925 = 1.5 * 2^23 + 13: the fma lands in [2^23, 2^24) where the fp32
// spacing is 1, so the low mantissa bits hold rn(13 v + 13).
__device__ __forceinline__ uint32_t cell_of(float v) {
    return __float_as_uint(__fmaf_rn(v, 13.0f, 12582925.0f));
}

// NaN gives index 0, as a search for the smallest distance that never
// improves on entry 0
__device__ __forceinline__ uint32_t nearest_code(float v, float my_thr, uint32_t my_lohi) {
    uint32_t k = cell_of(v);
    float t = __shfl_sync(FULL, my_thr, k);   // shfl reads lane k & 31
    uint32_t lh = __shfl_sync(FULL, my_lohi, k);
    return v != v ? 0u : (v > t) ? (lh >> 4) : (lh & 15u);
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

// Per-device host caches (occupancy, SM counts, shared-memory attributes:
// function attributes belong to a device's context) hold kMaxDevices slots.
// cache_device() is the current device's slot, or -1 when the device cannot be
// read or its index is kMaxDevices or above; callers then do the work the
// cache would have saved on every call.
constexpr int kMaxDevices = 64;

inline int cache_device() {
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) return -1;
    return d;
}

// cache[device] if set (nonzero), else compute() (stored when nonzero)
template <typename F>
int cached_per_device(std::atomic<int> (&cache)[kMaxDevices], F compute) {
    const int d = cache_device();
    if (d >= 0) {
        const int v = cache[d].load(std::memory_order_relaxed);
        if (v != 0) return v;
    }
    const int v = compute();
    if (d >= 0 && v != 0) cache[d].store(v, std::memory_order_relaxed);
    return v;
}

// calls set() once per device (every time when the device has no cache slot)
template <typename F>
cudaError_t once_per_device(std::atomic<bool> (&done)[kMaxDevices], F set) {
    const int d = cache_device();
    if (d >= 0 && done[d].load(std::memory_order_relaxed)) return cudaSuccess;
    const cudaError_t e = set();
    if (e == cudaSuccess && d >= 0) done[d].store(true, std::memory_order_relaxed);
    return e;
}

// RN(s / 255) in fp32 (the step of a double-quantized absmax) without a
// divide: Markstein's correction (P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", 1990): with y = RN(1/255)
// and q0 = RN(s y), the residual s - 255 q0 is exact in one fma and
// RN(q0 + residual * y) is the correctly rounded quotient.  Used for s == 0
// and 2^-100 <= s <= 2^100, where no step underflows (checked against IEEE
// division over every fp32 significand); other values (negative, tiny,
// huge, inf, NaN) take the IEEE divide.
__device__ __forceinline__ float div255_rn(float s) {
    if (s == 0.0f || (s >= 0x1p-100f && s <= 0x1p100f)) {
        const float y = 0x1.010102p-8f;  // RN(1/255)
        const float q0 = __fmul_rn(s, y);
        const float r = __fmaf_rn(-q0, 255.0f, s);
        return __fmaf_rn(r, y, q0);
    }
    return __fdiv_rn(s, 255.0f);
}

// The absmax value at flat index i of a double-quantized absmax array: 8-bit
// code q[i] times the step RN(scale / 255) of its group, in one correctly
// rounded fp32 product (the value bnb4_dequant_absmax writes).
__device__ __forceinline__ float dq_absmax(const uint8_t *__restrict__ q, const float *__restrict__ scales,
                                           int log2G, int64_t i) {
    return __fmul_rn((float)__ldg(q + i), div255_rn(__ldg(scales + (i >> log2G))));
}

// The loads behind one absmax value, before any arithmetic: the fp32 value,
// or the 8-bit code and its group's scale.  Kernels that fetch a stage ahead
// hold these in registers, so no use of a load sits next to its issue.
struct AbsmaxRaw {
    uint32_t code;
    float v;  // the fp32 absmax, or the group scale when the source is 8-bit
};

// One absmax value of a weight: fp32, or rebuilt from 8-bit statistics when
// q is given.
struct AbsmaxSrc {
    const float *f32;
    const uint8_t *q;
    const float *scales;
    int log2G;
    __device__ __forceinline__ float operator()(int64_t i) const {
        return q ? dq_absmax(q, scales, log2G, i) : __ldg(f32 + i);
    }
    __device__ __forceinline__ AbsmaxRaw raw(int64_t i) const {
        if (q) return AbsmaxRaw{(uint32_t)__ldg(q + i), __ldg(scales + (i >> log2G))};
        return AbsmaxRaw{0u, __ldg(f32 + i)};
    }
    // the same value as operator() on the same index
    __device__ __forceinline__ float finish(const AbsmaxRaw &r) const {
        return q ? __fmul_rn((float)r.code, div255_rn(r.v)) : r.v;
    }
};

}  // namespace bnb4
