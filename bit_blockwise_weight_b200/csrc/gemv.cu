// gemv.cu -- gemv_4bit (M == 1): y = x @ dequant(W)^T (+ bias), CUDA cores.
//
// "Feat/mps gemm 4bit bf16", What runs natively now: gemv_4bit is a fused
// dequant + dot kernel; the bias epilogue is added before the one rounding of
// the output (section Correctness).  The weight stream (0.5 B per weight plus
// 4 B of absmax per block) is the whole cost, so the kernel is built around
// reading it once, coalesced, with enough bytes in flight and as few
// shared-memory wavefronts per weight as possible.
//
// Work split (persistent, one CTA per SM):
//   * CTA c owns rows [N c / G, N (c+1) / G) (balanced to one row) and all of
//     K; x is copied once into shared memory (16-bit, swizzled so that the
//     per-lane reads below never conflict);
//   * the CTA's work is a list of units (quad of 4 rows, 1024-element segment
//     of K), split into 16 equal contiguous ranges, one per warp;
//   * lane l of a warp owns 32 weights (16 packed bytes) of each row of the
//     unit: 512 contiguous bytes per row per warp;
//   * every lane streams its own bytes (and their block absmax) through a
//     3-slot cp.async ring in shared memory, so two units are in flight per
//     warp without holding registers;
//   * decode: a 256-entry table, replicated once per bank, maps a packed byte
//     to its two codes as a bf16x2 / f16x2 word (one conflict-free lookup per
//     two weights); each code is multiplied by x with a mixed-precision FMA
//     (16-bit operands, fp32 accumulate), so nothing is unpacked;
//   * the lane's 32 weights lie in one quantization block: their sum is
//     scaled by the block absmax once, in fp32;
//   * when a warp leaves a quad, its 4 row sums are reduced across lanes with
//     xor-shuffles and stored to shared memory; quads shared by neighbouring
//     warps are added in warp order at the end (the result is the same bits
//     on every run).
// The codes enter as 16-bit values (the code table rounded once to bf16 /
// fp16), as in the small-M kernel.  No global scratch.
//
// Double-quantized absmax ("mps-bitsandbytes 0.4.7", Functional API, Double
// Quantization): with DQ the absmax array arrives as 8-bit codes plus one fp32
// scale per group of consecutive blocks.  Lanes 2i and 2i+1 share a block
// (blocks hold 64 or more weights); for the unit's 4 rows the even lane copies
// the aligned 32-bit words holding the block's codes and the odd lane the
// scales, into their two 16-byte slot entries (the slot keeps its size).  Both
// lanes rebuild absmax = RN(float(code) * RN(scale / 255)), the value the
// inverse of the double quantization gives, so the product is the plain
// gemv's with that absmax.  The weight stream shrinks from 4.5 to about 4.13
// bits per weight at blocks of 64.
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace bnb4 {

namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kSeg = 1024;       // elements per unit per row (32 lanes x 32)
constexpr int STAGES = 3;
constexpr int kSlot = 4 * 32 * 16 + 32 * 16;  // W [4 rows][32 lanes] 16 B + absmax [32 lanes][4]
constexpr int kLut = 256 * 32 * 4;            // 32 KB
constexpr int kMaxRows = 1024;   // rows per CTA
constexpr int kMaxK = 32768;
constexpr int kXv = kMaxK / 8 / kThreads;     // 16-byte pieces of x per thread

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

// 4-byte copy of the first `n` bytes (0..4) at src, zero-filling the rest
__device__ __forceinline__ void cp_async4_n(uint32_t dst, const void *src, int n) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(n));
}

template <int BYTES>
__device__ __forceinline__ void cp_async(uint32_t dst, const void *src, bool valid) {
    const int n = valid ? BYTES : 0;
    if (BYTES == 16)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n));
    else
        asm volatile("cp.async.ca.shared.global [%0], [%1], %2, %3;" ::"r"(dst), "l"(src),
                     "n"(BYTES), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// acc += code.lo * x.lo + code.hi * x.hi with 16-bit operands and an fp32 accumulator
template <typename D> struct Fma2;
template <> struct Fma2<BF16> {
    __device__ static __forceinline__ void run(float &a0, float &a1, uint32_t c, uint32_t x) {
        asm("{\n\t.reg .b16 c0, c1, x0, x1;\n\t"
            "mov.b32 {c0, c1}, %2;\n\tmov.b32 {x0, x1}, %3;\n\t"
            "fma.rn.f32.bf16 %0, c0, x0, %0;\n\tfma.rn.f32.bf16 %1, c1, x1, %1;\n\t}"
            : "+f"(a0), "+f"(a1)
            : "r"(c), "r"(x));
    }
};
template <> struct Fma2<F16> {
    __device__ static __forceinline__ void run(float &a0, float &a1, uint32_t c, uint32_t x) {
        asm("{\n\t.reg .b16 c0, c1, x0, x1;\n\t"
            "mov.b32 {c0, c1}, %2;\n\tmov.b32 {x0, x1}, %3;\n\t"
            "fma.rn.f32.f16 %0, c0, x0, %0;\n\tfma.rn.f32.f16 %1, c1, x1, %1;\n\t}"
            : "+f"(a0), "+f"(a1)
            : "r"(c), "r"(x));
    }
};

// element k of x -> its 16-bit slot in shared memory.  Lane chunks of 32
// elements (64 B) hold four 16-byte pieces; piece i of chunk L sits at
// position i ^ ((L >> 1) & 3), which spreads the eight lanes of a quarter
// warp over all 32 banks.
__device__ __forceinline__ int xswz(int k) {
    const int L = k >> 5, i = (k >> 3) & 3;
    return (L << 5) | ((i ^ ((L >> 1) & 3)) << 3) | (k & 7);
}

// absmax: fp32 [N, K/B], or with DQ the 8-bit codes [N, K/B] (nq = N*K/B
// bytes) with `scales` [ceil(nq / 2^log2G)]
template <typename D, bool DQ>
__global__ void __launch_bounds__(kThreads, 1)
gemv_kernel(const uint16_t *__restrict__ x, const uint8_t *__restrict__ W,
            const void *__restrict__ absmax, const float *__restrict__ scales, int log2G,
            const uint16_t *__restrict__ bias, uint16_t *__restrict__ y, int N, int K, int log2B,
            const __grid_constant__ CodeTable tab) {
    extern __shared__ __align__(16) uint8_t smem[];
    uint32_t *lut = reinterpret_cast<uint32_t *>(smem);
    uint8_t *ring = smem + kLut;                                                  // warps x STAGES
    float *rowsum = reinterpret_cast<float *>(ring + kWarps * STAGES * kSlot);    // [kMaxRows]
    float *part = rowsum + kMaxRows;                                              // [kWarps][2][4]
    uint16_t *xs = reinterpret_cast<uint16_t *>(part + kWarps * 8);              // [K] swizzled

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = gridDim.x;
    const int r0 = (int)(((int64_t)N * blockIdx.x) / G);
    const int r1 = (int)(((int64_t)N * (blockIdx.x + 1)) / G);
    const int rows = r1 - r0;
    const int Q = (rows + 3) >> 2;
    const int S = (K + kSeg - 1) / kSeg;
    const int U = Q * S;
    const int64_t row_bytes = K >> 1;
    const int nblk = K >> log2B;

    const uint32_t lut_base = (uint32_t)__cvta_generic_to_shared(lut);
    const uint32_t lane4 = 4u * lane;
    const uint32_t my_ring = (uint32_t)__cvta_generic_to_shared(ring) + warp * STAGES * kSlot;
    const uint32_t xs_base = (uint32_t)__cvta_generic_to_shared(xs);
    const int u_lo = (int)(((int64_t)U * warp) / kWarps);
    const int u_hi = (int)(((int64_t)U * (warp + 1)) / kWarps);

    auto issue = [&](int u, int slot) {
        const uint32_t base = my_ring + slot * kSlot;
        const int q = u / S, s = u - q * S;
        const int k = s * kSeg + 32 * lane;
        const bool ok = u < u_hi && k < K;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int row = r0 + 4 * q + r;
            const bool v = ok && row < r1;
            cp_async<16>(base + (r * 32 + lane) * 16,
                         v ? W + (int64_t)row * row_bytes + (k >> 1) : W, v);
            if constexpr (DQ) {
                // even lane: the word holding the block's code; odd lane: the
                // block's group scale (one copy either way, no divergence).
                // Block indices fit in 32 bits: N * K / B <= 151552 * 512.
                const int bi = row * nblk + (k >> log2B);
                const int ws = bi & ~3, left = N * nblk - ws;
                const void *src = (lane & 1) ? static_cast<const void *>(scales + (v ? bi >> log2G : 0))
                                             : static_cast<const void *>(static_cast<const uint8_t *>(absmax) +
                                                                         (v ? ws : 0));
                cp_async4_n(base + 4 * 32 * 16 + lane * 16 + 4 * r, src,
                            !v ? 0 : (lane & 1) ? 4 : (left < 4 ? left : 4));
            } else {
                const int64_t bi = (int64_t)row * nblk + (k >> log2B);
                cp_async<4>(base + 4 * 32 * 16 + lane * 16 + 4 * r,
                            static_cast<const float *>(absmax) + (v ? bi : 0), v);
            }
        }
    };

    // the first weight copies go out before the table and x are staged, so
    // their latency overlaps the prologue (the ring is per warp, nothing else
    // touches it)
#pragma unroll
    for (int i = 0; i < STAGES - 1; ++i) {
        issue(u_lo + i, i);
        cp_async_commit();
    }
    {
        // x: all 16-byte loads issued before any store (K <= kMaxK, K % 8 == 0)
        const uint4 *x4 = reinterpret_cast<const uint4 *>(x);
        const int K8 = K >> 3;
        uint4 xv[kXv];
#pragma unroll
        for (int i = 0; i < kXv; ++i)
            if (tid + i * kThreads < K8) xv[i] = __ldg(x4 + tid + i * kThreads);
        for (int e = tid >> 3; e < 256; e += kThreads / 8) {
            const uint32_t v = Dt<D>::pack2(tab.v[e >> 4], tab.v[e & 15]);
            reinterpret_cast<uint4 *>(lut + e * 32)[tid & 7] = make_uint4(v, v, v, v);
        }
#pragma unroll
        for (int i = 0; i < kXv; ++i) {
            const int c = tid + i * kThreads;
            if (c < K8) *reinterpret_cast<uint4 *>(xs + xswz(8 * c)) = xv[i];
        }
    }
    __syncthreads();
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const int qf = U > 0 ? u_lo / S : 0, ql = U > 0 ? (u_hi - 1) / S : 0;  // this warp's first and last quads
    for (int u = u_lo; u < u_hi; ++u) {
        const int it = u - u_lo;
        issue(u + STAGES - 1, (it + STAGES - 1) % STAGES);
        cp_async_commit();
        cp_async_wait<STAGES - 1>();
        const uint32_t base = my_ring + (it % STAGES) * kSlot;
        const int q = u / S, s = u - q * S;
        const int k = s * kSeg + 32 * lane;
        // x[k .. k+32) as 16 bf16x2 / f16x2 words (zeros past the end of K)
        uint32_t xq[16];
        if (k < K) {
            const int L = k >> 5;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint4 v = lds128(xs_base + ((L << 5) | ((i ^ ((L >> 1) & 3)) << 3)) * 2);
                xq[4 * i] = v.x; xq[4 * i + 1] = v.y; xq[4 * i + 2] = v.z; xq[4 * i + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) xq[i] = 0u;
        }
        const uint4 av = lds128(base + 4 * 32 * 16 + lane * 16);
        float am[4] = {__uint_as_float(av.x), __uint_as_float(av.y), __uint_as_float(av.z),
                       __uint_as_float(av.w)};
        if constexpr (DQ) {
            // the lane pair's code words and scales (zeros for rows past the slab
            // or segments past K, whose sums are dropped or zero)
            const uint32_t pb = base + 4 * 32 * 16 + (lane & ~1) * 16;
            const uint4 cw = lds128(pb), sw = lds128(pb + 16);
            const uint32_t aw[4] = {cw.x, cw.y, cw.z, cw.w};
            const uint32_t sc[4] = {sw.x, sw.y, sw.z, sw.w};
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int bi = (r0 + 4 * q + r) * nblk + (k >> log2B);
                // byte (bi & 3) of the word into the low byte of 0x4b000000:
                // the float 2^23 + code, exact
                const float c = __uint_as_float(__byte_perm(aw[r], 0x4b000000u, 0x7440u | (bi & 3)));
                am[r] = __fmul_rn(__fsub_rn(c, 8388608.0f), div255_rn(__uint_as_float(sc[r])));
            }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const uint4 wv = lds128(base + (r * 32 + lane) * 16);
            const uint32_t w4[4] = {wv.x, wv.y, wv.z, wv.w};
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    // byte j of word qq = weights 8qq+2j (high nibble) and 8qq+2j+1
                    const uint32_t sh = j == 0 ? (w4[qq] << 7) : (w4[qq] >> (8 * j - 7));
                    const uint32_t c2 = lds32(lut_base + ((sh & 0x7f80u) | lane4));
                    Fma2<D>::run(s0, s1, c2, xq[4 * qq + j]);
                }
            }
            acc[r] = __fmaf_rn(s0 + s1, am[r], acc[r]);
        }
        // leaving this quad: reduce the lane sums.  A quad strictly inside the
        // warp's range is the warp's alone and goes straight to the row sums;
        // the first and last quads may be shared with neighbouring warps and
        // go to this warp's two partial slots, added below in warp order, so
        // that the result does not depend on which warp finishes first.
        if (u + 1 == u_hi || (u + 1) / S != q) {
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const float v = warp_sum(acc[r]);
                const int row = 4 * q + r;
                if (lane == 0) {
                    if (q == qf) part[warp * 8 + r] = v;
                    else if (q == ql) part[warp * 8 + 4 + r] = v;
                    else if (row < rows) rowsum[row] = v;
                }
                acc[r] = 0.f;
            }
        }
    }
    cp_async_wait<0>();
    __syncthreads();
    for (int r = tid; r < rows; r += kThreads) {
        // the warps whose unit ranges meet this row's quad (units [ul, uh)), in
        // order: from the warp holding unit ul to the one holding uh - 1 (unit u
        // lies in warp ceil(kWarps (u + 1) / U) - 1).  A warp starting inside the
        // quad left it in slot 0, one ending inside it in slot 1; otherwise the
        // quad is the warp's alone.
        const int q = r >> 2, ul = q * S, uh = ul + S;
        const int w0 = (kWarps * (ul + 1) + U - 1) / U - 1, w1 = (kWarps * uh + U - 1) / U - 1;
        float v = 0.f;
        for (int w = w0; w <= w1; ++w) {
            const int lo = (int)(((int64_t)U * w) / kWarps), hi = (int)(((int64_t)U * (w + 1)) / kWarps);
            if (lo >= hi) continue;
            v += lo >= ul ? part[w * 8 + (r & 3)] : hi - 1 < uh ? part[w * 8 + 4 + (r & 3)] : rowsum[r];
        }
        if (bias) v += Dt<D>::to_f32(bias[r0 + r]);
        y[r0 + r] = (uint16_t)(Dt<D>::pack2(v, 0.f) & 0xffffu);
    }
}

template <typename D, bool DQ>
cudaError_t launch_t(const void *x, const uint8_t *W, const void *absmax, const float *scales, int log2G,
                     const void *bias, void *y, int N, int K, int log2B, const CodeTable &tab,
                     cudaStream_t stream) {
    const int G = device_sm_count();
    const int kpad = ((K + 31) / 32) * 32;
    const size_t smem = kLut + (size_t)kWarps * STAGES * kSlot + kMaxRows * 4 + kWarps * 8 * 4 + (size_t)kpad * 2;
    // the limit for the largest K, set once per device (attributes belong to a
    // device's context); every launch asks for no more than that
    constexpr size_t kSmemMax = kLut + (size_t)kWarps * STAGES * kSlot + kMaxRows * 4 + kWarps * 8 * 4 + kMaxK * 2;
    static_assert(kSmemMax <= 227 * 1024, "shared memory plan at the largest K");
    static std::atomic<bool> set[64];
    const int dev = cache_device();
    if (!set[dev].load(std::memory_order_relaxed)) {
        cudaError_t e = cudaFuncSetAttribute(gemv_kernel<D, DQ>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemMax);
        if (e != cudaSuccess) return e;
        set[dev].store(true, std::memory_order_relaxed);
    }
    gemv_kernel<D, DQ><<<G, kThreads, smem, stream>>>(
        static_cast<const uint16_t *>(x), W, absmax, scales, log2G, static_cast<const uint16_t *>(bias),
        static_cast<uint16_t *>(y), N, K, log2B, tab);
    return cudaGetLastError();
}

}  // namespace

int64_t gemv_max_rows() { return (int64_t)device_sm_count() * kMaxRows; }
int64_t gemv_max_k() { return kMaxK; }

cudaError_t launch_gemv(const void *x, const uint8_t *W, const float *absmax, const uint8_t *absmax_q,
                        const float *scales, int group, const void *bias, void *y, int64_t N,
                        int64_t K, int blocksize, bnb4_quant_type qt, bnb4_dtype dt,
                        cudaStream_t stream) {
    static const CodeTable nf4 = host_code_table(BNB4_NF4);
    static const CodeTable fp4 = host_code_table(BNB4_FP4);
    const CodeTable &tab = qt == BNB4_NF4 ? nf4 : fp4;
    const int log2B = ilog2(blocksize);
    if (absmax_q) {
        const int log2G = ilog2(group);
        if (dt == BNB4_F16)
            return launch_t<F16, true>(x, W, absmax_q, scales, log2G, bias, y, (int)N, (int)K, log2B, tab,
                                       stream);
        return launch_t<BF16, true>(x, W, absmax_q, scales, log2G, bias, y, (int)N, (int)K, log2B, tab,
                                    stream);
    }
    if (dt == BNB4_F16)
        return launch_t<F16, false>(x, W, absmax, nullptr, 0, bias, y, (int)N, (int)K, log2B, tab, stream);
    return launch_t<BF16, false>(x, W, absmax, nullptr, 0, bias, y, (int)N, (int)K, log2B, tab, stream);
}

}  // namespace bnb4
