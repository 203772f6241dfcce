// gemv.cu -- gemv_4bit (M == 1): y = x @ dequant(W)^T (+ bias).
//
// "Feat/mps gemm 4bit bf16", What runs natively now: gemv_4bit is a fused
// dequant + dot kernel; the bias epilogue is added before the one rounding of
// the output (section Correctness).  The weight stream (0.5 B per weight plus
// 4 B of absmax per block) is the whole cost.  On B200 a CUDA-core loop that
// turns every weight into an fp32 FMA issues more instructions than HBM lets
// it retire, so the multiply-adds go to the tensor cores (mma.sync.m16n8k16,
// fp32 accumulation) and decoding is one byte-permute plus one conflict-free
// shared load per two weights.  Every lane loads 16 contiguous bytes of the
// weight stream per instruction (narrower loads leave B200's HBM well short
// of its bandwidth at these sizes).
//
// Units.  A unit is a quad of rows x a segment of 512 weights (8 items of 64
// weights; an item lies in one quantization block).  Row pair of items
// (2p, 2p + 1) of one row is a 64-byte "item pair".  One MMA multiplies a
// 16 x 16 A tile by a 16 x 8 B tile; eight MMAs cover a unit:
//   A row m = g (g = 0..7):  row g & 3 of the quad, item pair g >> 2      (pairs 0, 1)
//   A row m = g + 8:         row g & 3 of the quad, item pair 2 + (g >> 2) (pairs 2, 3)
// Lane (g, t) holds bytes [16t, 16t + 16) of its two item pairs (two 16-byte
// loads; a warp's load covers 4 rows x 128 contiguous bytes) and feeds, in
// MMA s, bytes 2s and 2s + 1 of each: k-slot 2t + e holds weight 4s + e and
// k-slot 2t + 8 + e holds weight 4s + 2 + e of the lane's 32 weights, which
// lie in item 2P + (t >> 1) at item offset 32 (t & 1).  Column n of B is item
// n of the segment: a lane's B slots hold x where its A bytes belong to item n
// ((t >> 1) == (n & 1)) and zeros elsewhere, so C[m, n] for n in {2P(m),
// 2P(m) + 1} is the dot product of one row over one item; the other 6
// columns of each row are never read.  Lane (g, t) holds C[g, 2t..2t+1] and
// C[g + 8, 2t..2t+1]: it is the lane with the two useful sums of A row g
// when t == g >> 2, and of A row g + 8 when t == 2 + (g >> 2).  Each sum is
// scaled by its block's absmax in fp32.  The reduction over k is a plain
// sum, so the order of the k-slots is free.
//
// Decoding: a byte holds two codes (first element in the high nibble).  A
// 256-entry table maps it to the two codes as a bf16x2 / f16x2 word (lower k
// in the low half), one copy per shared-memory bank; the table sits at a
// shared address that is a multiple of 64 KB with a 256-byte entry stride, so
// one prmt builds the lane's address (table page, byte, lane) from the packed
// word and the lookup never conflicts.  The codes enter as 16-bit values (the
// code table rounded once to bf16 / fp16), so the weight a product meets is
// RN_dtype(code) * absmax: 2^-8 (bf16) or 2^-11 (fp16) relative to the
// dequantized value.
//
// Work split: CTA c owns rows [N c / G, N (c+1) / G) (balanced to one row) and
// all of K.  Its work is a list of groups (a quad of rows x kSpan consecutive
// segments, so each row's bytes are asked for in runs of kSpan x 256 bytes:
// HBM serves long runs of few rows far better than short runs of many),
// quad major; warp w takes a contiguous, balanced range of groups.  Packed
// weights and absmax go from global memory straight into registers, one
// group ahead of the MMAs; x is staged once per CTA in shared memory (the
// 16-byte pieces of odd items rotated by two places), beside a zeroed line
// from which the lanes whose B slots must be zero read, each at a bank its
// partner lane does not use, so a warp's 16-byte reads never conflict and
// need no masking.  x sits below the table's 64 KB boundary when it fits
// there, which leaves half of the SM's L1 to the loads in flight.  A lane
// accumulates its useful sums of a quad in fp32 across segments; when a warp
// leaves a quad the sums are reduced across lanes and stored to shared
// memory, and quads that two warps share are added in warp order at the end,
// so the result is the same bits on every run.  No global scratch.
//
// Double-quantized absmax ("mps-bitsandbytes 0.4.7", Functional API, Double
// Quantization): with DQ the absmax array arrives as 8-bit codes plus one
// fp32 scale per group of blocks; the lane that scales a sum rebuilds
// absmax = RN(float(code) * RN(scale / 255)), the value the inverse of the
// double quantization gives, so the product is the plain gemv's with that
// absmax.
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace bnb4 {

__device__ unsigned int g_gemv_layout_errors = 0;  // launches that found their shared plan unusable

namespace {

// Tunables (measured on B200: 16 warps, groups of 2 segments, two units'
// MMA chains interleaved; longer groups need more registers than 512
// threads leave and spill)
#ifndef BNB4_GEMV_WARPS
#define BNB4_GEMV_WARPS 16
#endif
#ifndef BNB4_GEMV_SPAN
#define BNB4_GEMV_SPAN 2
#endif
constexpr int kWarps = BNB4_GEMV_WARPS;
constexpr int kThreads = kWarps * 32;
constexpr int kSpan = BNB4_GEMV_SPAN;     // segments per group
#ifndef BNB4_GEMV_PDL
#define BNB4_GEMV_PDL 1                   // programmatic dependent launch (prologue overlaps the previous kernel)
#endif
#ifndef BNB4_GEMV_ILV
#define BNB4_GEMV_ILV 2
#endif
constexpr int kIlv = BNB4_GEMV_ILV;       // units whose MMA chains are interleaved
static_assert(kSpan % kIlv == 0, "a group's units are computed kIlv at a time");
constexpr int kItems = 8;                 // items (64 weights) per segment
constexpr int kSegK = kItems * 64;        // 512 weights per row per segment
constexpr int kMaxRows = 1024;            // rows per CTA
constexpr int kMaxK = 32768;
constexpr uint32_t kPage = 65536;         // table alignment and size (256 entries x 256 B)
constexpr uint32_t kPrefix = kMaxRows * 4 + kWarps * 2 * 4 * 4;  // row sums + warp partials
constexpr uint32_t kZero = 256;           // zeroed bytes read by the masked B lanes
// 16-byte pieces of x per thread at the largest K (rounded up to whole groups)
constexpr int kXPieces = ((kMaxK / kSegK + kSpan - 1) / kSpan * kSpan * kSegK / 8 + kThreads - 1) / kThreads;

// shared loads / stores by 32-bit shared-window address
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ void sts128(uint32_t a, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}
__device__ __forceinline__ void sts32f(uint32_t a, float v) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}
__device__ __forceinline__ float lds32f(uint32_t a) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
    return v;
}

// 16 bytes of the weight stream, absmax words and 8-bit codes: read once,
// no L1 allocation
__device__ __forceinline__ uint4 ldg_w16(const uint8_t *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}
__device__ __forceinline__ float ldg_f32(const float *p) {
    float v;
    asm volatile("ld.global.nc.L1::no_allocate.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ uint32_t ldg_u8(const uint8_t *p) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u8 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// c += A B (run) or c = A B (first: the accumulator input is one zero register)
#define BNB4_MMA(TY)                                                                                            \
    __device__ static __forceinline__ void run(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,          \
                                               uint32_t a3, uint32_t b0, uint32_t b1) {                       \
        asm("mma.sync.aligned.m16n8k16.row.col.f32." TY "." TY ".f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, " \
            "{%0,%1,%2,%3};"                                                                                 \
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])                                                 \
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));                                         \
    }                                                                                                         \
    __device__ static __forceinline__ void first(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,        \
                                                 uint32_t a3, uint32_t b0, uint32_t b1) {                     \
        asm("mma.sync.aligned.m16n8k16.row.col.f32." TY "." TY ".f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, " \
            "{%10,%10,%10,%10};"                                                                             \
            : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])                                                 \
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));                              \
    }
template <typename D> struct Mma;
template <> struct Mma<BF16> { BNB4_MMA("bf16") };
template <> struct Mma<F16> { BNB4_MMA("f16") };
#undef BNB4_MMA

// table lookup of byte k (0..3) of w: prmt puts the lane's bank offset in
// byte 0, the packed byte in byte 1 and the table page in bytes 2..3 of the
// address (L = page | 4 lane)
template <int k>
__device__ __forceinline__ uint32_t lut(uint32_t w, uint32_t L) {
    return lds32(prmt(w, L, 0x7604u | (k << 4)));
}

__device__ __forceinline__ uint32_t word(const uint4 &v, int i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// one unit's loads (a unit is a quad x one segment): the lane's 16 bytes of
// its two item pairs and, on the lane that scales sums, the absmax (or 8-bit
// codes and group scales) of its two items
struct Unit {
    uint4 wa, wb;
    float am0, am1;
    uint32_t code0, code1;
};

}  // namespace

// absmax: fp32 [N, K/B], or with DQ the 8-bit codes [N, K/B] with `scales`
// [ceil(N K / B / 2^log2G)]
template <typename D, bool DQ>
__global__ void __launch_bounds__(kThreads, 1)
gemv_kernel(const uint16_t *__restrict__ x, const uint8_t *__restrict__ W, const void *__restrict__ absmax,
            const float *__restrict__ scales, int log2G, const uint16_t *__restrict__ bias,
            uint16_t *__restrict__ y, int N, int K, int log2B, const __grid_constant__ CodeTable tab) {
    extern __shared__ __align__(16) uint8_t smem[];
    const uint32_t base0 = (uint32_t)__cvta_generic_to_shared(smem);
    const uint32_t rowsum_a = base0;                         // float [kMaxRows]
    const uint32_t part_a = base0 + kMaxRows * 4;            // float [kWarps][2][4]
    const uint32_t zero_a = base0 + kPrefix;                 // kZero bytes of zeros
    const uint32_t lut_a = (zero_a + kZero + kPage - 1) & ~(kPage - 1);

    const int nitems = K >> 6;
    const int S = (nitems + kItems - 1) / kItems;            // segments per row
    const int SS = (S + kSpan - 1) / kSpan;                  // groups per quad
    const uint32_t xbytes = (uint32_t)SS * kSpan * kSegK * 2;
    // item i of x at xs_a + 128 i: below the table if it fits, else above it
    const uint32_t xs_a = zero_a + kZero + xbytes <= lut_a ? zero_a + kZero : lut_a + kPage;
    {
        uint32_t dyn;
        asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
        if (xs_a + xbytes > base0 + dyn || lut_a + kPage > base0 + dyn) {
            // the shared-memory plan does not fit the launch: report, write nothing
            if (threadIdx.x == 0) atomicAdd(&g_gemv_layout_errors, 1u);
            return;
        }
    }

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = gridDim.x;
    const int r0 = (int)(((int64_t)N * blockIdx.x) / G);
    const int r1 = (int)(((int64_t)N * (blockIdx.x + 1)) / G);
    const int R = r1 - r0;
    const int NQ = (R + 3) >> 2;                             // quads
    const int GU = NQ * SS;                                  // groups of this CTA
    const int g_lo = (int)(((int64_t)GU * warp) / kWarps);
    const int g_hi = (int)(((int64_t)GU * (warp + 1)) / kWarps);

    const int g8 = lane >> 2, t4 = lane & 3;
    const int rq = g8 & 3;                                   // row within the quad
    const int pA = g8 >> 2, pB = 2 + (g8 >> 2);              // the lane's item pairs
    // the lane's useful sums (two, of one A row), if any
    const bool hiC = t4 >= 2;
    const bool useful = t4 == (g8 >> 2) || t4 == 2 + (g8 >> 2);
    const int it_u = 2 * (hiC ? pB : pA);                    // first of its two items
    const int64_t row_bytes = K >> 1;
    const int nblk = K >> log2B;
    const int bsh = log2B - 6;                               // item -> block
    const uint8_t *Wt = W + (int64_t)r0 * row_bytes + 64 * pA + 16 * t4;
    const int64_t a0 = (int64_t)r0 * nblk;

    // Loads of group (q, ss).  Rows past the CTA's last row and items past K
    // are clamped to the last ones: they read real data, whose sums are never
    // stored (rows) or meet zeros of x (items), so no load is predicated.
    auto load = [&](int q, int ss, Unit (&u)[kSpan]) {
        const int rl = min(4 * q + rq, R - 1);
        const int64_t br = a0 + (int64_t)rl * nblk;
        const int j0 = ss * kSpan;
        if (!DQ && bsh == 0 && (ss + 1) * kSpan * kItems <= nitems) {
            // the common case (blocks of 64, every item of the group in K): one
            // base address per group, the units at immediate offsets
            const uint8_t *wg = Wt + (int64_t)rl * row_bytes + 256 * j0;
            const float *ag = static_cast<const float *>(absmax) + br + kItems * j0 + it_u;
#pragma unroll
            for (int sp = 0; sp < kSpan; ++sp) {
                u[sp].wa = ldg_w16(wg + 256 * sp);
                u[sp].wb = ldg_w16(wg + 256 * sp + 128);
                u[sp].am0 = ldg_f32(ag + kItems * sp);
                u[sp].am1 = ldg_f32(ag + kItems * sp + 1);
                u[sp].code0 = u[sp].code1 = 0;
            }
            return;
        }
        const uint8_t *wr = Wt + (int64_t)rl * row_bytes;
        const bool whole = (ss + 1) * kSpan * kItems <= nitems;  // every item of the group is in K
#pragma unroll
        for (int sp = 0; sp < kSpan; ++sp) {
            const int j = j0 + sp;
            if (whole) {
                u[sp].wa = ldg_w16(wr + 256 * j);
                u[sp].wb = ldg_w16(wr + 256 * j + 128);
            } else {
                // byte offsets of the lane's chunks with their items clamped to K
                const int iA = min(j * kItems + 2 * pA + (t4 >> 1), nitems - 1);
                const int iB = min(j * kItems + 2 * pB + (t4 >> 1), nitems - 1);
                const uint8_t *wc = wr - 64 * pA - 16 * t4 + 16 * (t4 & 1);
                u[sp].wa = ldg_w16(wc + 32 * iA);
                u[sp].wb = ldg_w16(wc + 32 * iB);
            }
            const int b0 = min(j * kItems + it_u, nitems - 1) >> bsh;
            const int b1 = min(j * kItems + it_u + 1, nitems - 1) >> bsh;
            if constexpr (DQ) {
                const uint8_t *q8 = static_cast<const uint8_t *>(absmax);
                u[sp].code0 = ldg_u8(q8 + br + b0);
                u[sp].code1 = ldg_u8(q8 + br + b1);
                u[sp].am0 = ldg_f32(scales + ((br + b0) >> log2G));
                u[sp].am1 = ldg_f32(scales + ((br + b1) >> log2G));
            } else {
                const float *af = static_cast<const float *>(absmax);
                u[sp].am0 = ldg_f32(af + br + b0);
                u[sp].am1 = ldg_f32(af + br + b1);
                u[sp].code0 = u[sp].code1 = 0;
            }
        }
    };

    // this warp's groups, visited in order: (quad, span) advance without divisions
    const int ng = g_hi - g_lo;
    int cq = 0, css = 0;
    if (ng > 0) {
        cq = g_lo / SS;
        css = g_lo - cq * SS;
    }
    const int q_first = ng > 0 ? cq : -1;
    const int q_last = ng > 0 ? (g_hi - 1) / SS : -1;

    Unit ua[kSpan], ub[kSpan];
#if !BNB4_GEMV_PDL
    // the first group's loads leave before the table and x are staged
    if (ng > 0) load(cq, css, ua);
#endif
    {
        // table: entry v (codes of nibbles v >> 4, v & 15) copied to words 64 v + l, l < 32
        for (int idx = tid; idx < 2048; idx += kThreads) {   // 2048 16-byte pieces
            const int v = idx >> 3, q = idx & 7;
            const uint32_t e = Dt<D>::pack2(tab.v[v >> 4], tab.v[v & 15]);
            sts128(lut_a + v * 256 + q * 16, make_uint4(e, e, e, e));
        }
        if (tid < kZero / 16) sts128(zero_a + 16 * tid, make_uint4(0, 0, 0, 0));
#if BNB4_GEMV_PDL
        // Launched as a programmatic dependent, this CTA may start while the
        // previous kernel on the stream is still finishing: the work above
        // reads only this kernel's parameters.  Every global access (inputs
        // the previous kernel may write, y it may read) comes after the wait,
        // which returns once that kernel has completed and its writes are
        // visible.
        asm volatile("griddepcontrol.wait;" ::: "memory");
        if (ng > 0) load(cq, css, ua);
#endif
        // x: 16-byte piece q of item i at position (q + 2 (i & 1)) & 7 of the
        // item's 128 bytes; zeros past K.  All of a thread's loads leave before
        // any store, so staging costs one round trip.
        const uint4 *x4 = reinterpret_cast<const uint4 *>(x);
        const int npieces = SS * kSpan * kSegK / 8;
        uint4 xv[kXPieces];
#pragma unroll
        for (int i = 0; i < kXPieces; ++i) {
            const int c = tid + i * kThreads;
            xv[i] = 8 * c < K ? __ldg(x4 + c) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int i = 0; i < kXPieces; ++i) {
            const int c = tid + i * kThreads, it = c >> 3;
            if (c < npieces) sts128(xs_a + it * 128 + ((((c & 7) + 2 * (it & 1)) & 7) << 4), xv[i]);
        }
    }
    __syncthreads();

    const uint32_t L = lut_a | (4u * lane);
    // B: x of item g8 at the lane's half (t4 & 1) of it where the lane's bytes
    // lie in that item ((t4 >> 1) == (g8 & 1)); zeros elsewhere, read from the
    // zeroed line one piece past the partner lane's bank group
    const bool bmask = (t4 >> 1) == (g8 & 1);
    const uint32_t xbase = bmask ? xs_a + g8 * 128 : zero_a;
    const uint32_t xstride = bmask ? kItems * 128 : 0;
    uint32_t xo[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t pos = (4 * (t4 & 1) + q + 2 * (g8 & 1)) & 7;
        xo[q] = (bmask ? pos : (pos + 1) & 7) << 4;
    }
    float acc = 0.f;

    // reduce the lanes' sums of quad q and store its 4 row sums
    auto flush = [&](int q) {
        float v = acc;
        v += __shfl_xor_sync(FULL, v, 16);
        v += __shfl_xor_sync(FULL, v, 1);
        v += __shfl_xor_sync(FULL, v, 2);
        if ((lane & 19) == 0) {                              // lanes 0, 4, 8, 12: rows 0..3
            const int k = (lane >> 2) & 3;
            if (q == q_first)
                sts32f(part_a + (warp * 8 + k) * 4, v);
            else if (q == q_last)
                sts32f(part_a + (warp * 8 + 4 + k) * 4, v);
            else if (4 * q + k < R)
                sts32f(rowsum_a + (4 * q + k) * 4, v);
        }
        acc = 0.f;
    };

    // kIlv units' MMA chains at a time are interleaved; rows past the CTA's
    // rows are computed on clamped data and never stored
    auto compute = [&](int ss, const Unit (&u)[kSpan]) {
#pragma unroll
        for (int h = 0; h < kSpan; h += kIlv) {
            float c[kIlv][4];
            uint32_t xr[kIlv][16];
#pragma unroll
            for (int e = 0; e < kIlv; ++e) {
                const uint32_t xa = xbase + (uint32_t)(ss * kSpan + h + e) * xstride;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint4 v = lds128(xa + xo[q]);
                    xr[e][4 * q] = v.x;
                    xr[e][4 * q + 1] = v.y;
                    xr[e][4 * q + 2] = v.z;
                    xr[e][4 * q + 3] = v.w;
                }
            }
#pragma unroll
            for (int st = 0; st < 8; ++st) {
#pragma unroll
                for (int e = 0; e < kIlv; ++e) {
                    const Unit &un = u[h + e];
                    const uint32_t wa = word(un.wa, st >> 1), wb = word(un.wb, st >> 1);
                    if (st == 0)
                        Mma<D>::first(c[e], lut<0>(wa, L), lut<0>(wb, L), lut<1>(wa, L), lut<1>(wb, L), xr[e][0],
                                      xr[e][1]);
                    else if (st & 1)
                        Mma<D>::run(c[e], lut<2>(wa, L), lut<2>(wb, L), lut<3>(wa, L), lut<3>(wb, L),
                                    xr[e][2 * st], xr[e][2 * st + 1]);
                    else
                        Mma<D>::run(c[e], lut<0>(wa, L), lut<0>(wb, L), lut<1>(wa, L), lut<1>(wb, L),
                                    xr[e][2 * st], xr[e][2 * st + 1]);
                }
            }
#pragma unroll
            for (int e = 0; e < kIlv; ++e) {
                const Unit &un = u[h + e];
                float v0 = hiC ? c[e][2] : c[e][0];
                float v1 = hiC ? c[e][3] : c[e][1];
                v0 = useful ? v0 : 0.f;
                v1 = useful ? v1 : 0.f;
                float am0 = un.am0, am1 = un.am1;
                if constexpr (DQ) {
                    am0 = __fmul_rn(__uint_as_float(0x4b000000u | un.code0) - 8388608.0f, div255_rn(am0));
                    am1 = __fmul_rn(__uint_as_float(0x4b000000u | un.code1) - 8388608.0f, div255_rn(am1));
                }
                acc = __fmaf_rn(v0, am0, acc);
                acc = __fmaf_rn(v1, am1, acc);
            }
        }
    };

    auto next = [&](int &q, int &ss) {
        if (++ss == SS) {
            ss = 0;
            ++q;
        }
    };
    // ua holds group i, ub group i + 1 (loaded while group i is computed)
    for (int i = 0; i < ng; i += 2) {
        int nq = cq, nss = css;
        next(nq, nss);
        if (i + 1 < ng) load(nq, nss, ub);
        compute(css, ua);
        if (i + 1 == ng || nq != cq) flush(cq);
        if (i + 1 < ng) {
            cq = nq;
            css = nss;
            next(nq, nss);
            if (i + 2 < ng) load(nq, nss, ua);
            compute(css, ub);
            if (i + 2 == ng || nq != cq) flush(cq);
            cq = nq;
            css = nss;
        }
    }
#if BNB4_GEMV_PDL
    // the next kernel on the stream may launch now (its CTAs take SMs as this
    // grid's leave, and wait for its completion before touching memory)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#endif
    __syncthreads();

    for (int r = tid; r < R; r += kThreads) {
        // the warps whose group ranges meet this row's quad (groups [ul, uh)),
        // in order.  A warp starting inside the quad left it in slot 0, one
        // ending inside it in slot 1; otherwise the quad is the warp's alone
        // and went to the row sums.
        const int q = r >> 2, k = r & 3, ul = q * SS, uh = ul + SS;
        const int w0 = (kWarps * (ul + 1) + GU - 1) / GU - 1, w1 = (kWarps * uh + GU - 1) / GU - 1;
        float v = 0.f;
        for (int w = w0; w <= w1; ++w) {
            const int lo = (int)(((int64_t)GU * w) / kWarps), hi = (int)(((int64_t)GU * (w + 1)) / kWarps);
            if (lo >= hi) continue;
            v += lo >= ul ? lds32f(part_a + (w * 8 + k) * 4)
                 : hi - 1 < uh ? lds32f(part_a + (w * 8 + 4 + k) * 4)
                               : lds32f(rowsum_a + r * 4);
        }
        if (bias) v += Dt<D>::to_f32(bias[r0 + r]);
        y[r0 + r] = (uint16_t)(Dt<D>::pack2(v, 0.f) & 0xffffu);
    }
}

namespace {

// shared memory the kernel asks for: the prefix, the zeroed line, x when it
// fits below the next 64 KB boundary of the shared window (the dynamic region
// starts right after the device's reserved shared memory), the table, and x
// above it otherwise
size_t smem_bytes(int K, int reserved) {
    const size_t S = ((size_t)(K >> 6) + kItems - 1) / kItems;
    const size_t SS = (S + kSpan - 1) / kSpan;
    const size_t xbytes = SS * kSpan * kSegK * 2;
    const size_t zero = (size_t)reserved + kPrefix;
    const size_t lut = (zero + kZero + kPage - 1) / kPage * kPage;
    const size_t end = zero + kZero + xbytes <= lut ? lut + kPage : lut + kPage + xbytes;
    return end - (size_t)reserved;
}

template <typename D, bool DQ>
cudaError_t launch_t(const void *x, const uint8_t *W, const void *absmax, const float *scales, int log2G,
                     const void *bias, void *y, int N, int K, int log2B, const CodeTable &tab,
                     cudaStream_t stream) {
    const int G = device_sm_count();
    // the device's reserved shared memory per block, stored plus one (0 = not read yet)
    static std::atomic<int> reserved_cache[kMaxDevices];
    const int reserved = cached_per_device(reserved_cache, [] {
        int dev = 0, v = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&v, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess) {
            (void)cudaGetLastError();
            return 0;
        }
        return v + 1;
    }) - 1;
    if (reserved < 0) return cudaErrorInvalidDevice;
    // the limit for the largest K, set once per device (attributes belong to a
    // device's context); every launch asks for no more than that
    const size_t smax = smem_bytes(kMaxK, reserved);
    if (smax > 227 * 1024) return cudaErrorInvalidConfiguration;
    static std::atomic<bool> set[kMaxDevices];
    cudaError_t e = once_per_device(set, [&] {
        return cudaFuncSetAttribute(gemv_kernel<D, DQ>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smax);
    });
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(G, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem_bytes(K, reserved);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = BNB4_GEMV_PDL;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemv_kernel<D, DQ>, static_cast<const uint16_t *>(x), W, absmax, scales, log2G,
                              static_cast<const uint16_t *>(bias), static_cast<uint16_t *>(y), N, K, log2B, tab);
}

}  // namespace

int64_t gemv_max_rows() { return (int64_t)device_sm_count() * kMaxRows; }
int64_t gemv_max_k() { return kMaxK; }

cudaError_t gemv_layout_errors_address(unsigned int **p) {
    return cudaGetSymbolAddress(reinterpret_cast<void **>(p), g_gemv_layout_errors);
}

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
