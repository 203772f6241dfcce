// gemv.cu -- gemv_4bit (M == 1): y = x @ dequant(W)^T (+ bias).
//
// "Feat/mps gemm 4bit bf16", What runs natively now: gemv_4bit is a fused
// dequant + dot kernel; the bias epilogue is added before the one rounding of
// the output (section Correctness).  The weight stream (0.5 B per weight plus
// 4 B of absmax per block) is the whole cost.  On B200 a CUDA-core loop that
// turns every weight into an fp32 FMA issues more instructions than HBM lets
// it retire, so the multiply-adds go to the tensor cores (mma.sync.m16n8k16,
// fp32 accumulation) and decoding is one byte-permute plus one conflict-free
// shared load per two weights.
//
// Packing the tensor-core tile.  One MMA multiplies a 16 x 16 A tile by a
// 16 x 8 B tile.  A row m of A holds 16 weights of row rho(m) of a row pair
// and item iota(m) of a 512-weight segment (an item is 64 consecutive weights
// of one row, so it lies in one quantization block):
//     m = g      (g = 0..7):  rho = g & 1, iota = g >> 1       (items 0..3)
//     m = g + 8:              rho = g & 1, iota = 4 + (g >> 1)  (items 4..7)
// and column n of B holds the matching 16 values of x of item n.  Entry
// C[m, iota(m)] is then a partial dot product of one row over one item: the
// other 7 columns of each row are never read.  Four MMAs cover the 64 weights
// of every item, so one unit (a row pair x a segment = 1024 weights) is four
// MMAs whose 16 useful sums are each scaled by their block's absmax in fp32.
//
// K order inside an item: lane (g, t) feeds, in MMA s, packed bytes 2s and
// 2s + 1 of its 8 bytes [8t, 8t + 8) of the item, so k-slot 2t + e holds
// weight 16t + 4s + e and k-slot 2t + 8 + e holds 16t + 4s + 2 + e; the B
// fragment takes x at the same positions.  The reduction over k is a plain
// sum, so the order is free.
//
// Decoding: a byte holds two codes (first element in the high nibble).  A
// 256-entry table maps it to the two codes as a bf16x2 / f16x2 word (lower k
// in the low half), one copy per shared-memory bank; the table sits at a
// shared address that is a multiple of 64 KB with a 256-byte entry stride, so
// one prmt builds the lane's address (table page, byte, lane) from the packed
// word and the lookup never conflicts.  The codes enter as 16-bit values (the
// code table rounded once to bf16 / fp16), so the weight a product meets is
// RN_dtype(code) * absmax: 2^-9 (bf16) or 2^-12 (fp16) relative to the
// dequantized value.
//
// Work split: CTA c owns rows [N c / G, N (c+1) / G) (balanced to one row) and
// all of K.  Its work is a list of groups (a block of 4 row pairs x one
// segment), pair-block major; warp w takes a contiguous, balanced range of
// groups.  Packed weights and absmax go from global memory straight into
// registers (8-byte loads, full 32-byte sectors), two groups ahead of the
// MMAs, so no shared-memory bandwidth is spent on staging them; x is staged
// once per CTA in shared memory (swizzled: the eight items a warp reads at
// once land in distinct banks).  A lane accumulates its useful sums per row
// pair in fp32 across segments; when a warp leaves a pair block the sums are
// reduced across lanes and stored to shared memory, and pair blocks that two
// warps share are added in warp order at the end, so the result is the same
// bits on every run.  No global scratch.
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

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kPairs = 4;                 // row pairs per pair block (8 rows)
constexpr int kItems = 8;                 // items (64 weights) per segment
constexpr int kSegK = kItems * 64;        // 512 weights per row per segment
constexpr int kMaxRows = 1024;            // rows per CTA
constexpr int kMaxK = 32768;
constexpr uint32_t kPage = 65536;         // table alignment and size (256 entries x 256 B)
constexpr uint32_t kPrefix = kMaxRows * 4 + kWarps * 2 * 8 * 4;  // row sums + warp partials

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

// 8 bytes of the weight stream (read once: no L1 allocation); zeros when !ok
__device__ __forceinline__ uint2 ldg_w8(const uint8_t *p, bool ok) {
    uint2 v;
    asm volatile(
        "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %3, 0;\n\tmov.b32 %0, 0;\n\tmov.b32 %1, 0;\n\t"
        "@q ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];\n\t}"
        : "=r"(v.x), "=r"(v.y)
        : "l"(p), "r"((int)ok));
    return v;
}
__device__ __forceinline__ float ldg_f32(const float *p, bool ok) {
    float v;
    asm volatile("{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %2, 0;\n\tmov.b32 %0, 0;\n\t"
                 "@q ld.global.nc.L1::no_allocate.f32 %0, [%1];\n\t}"
                 : "=f"(v)
                 : "l"(p), "r"((int)ok));
    return v;
}
__device__ __forceinline__ uint32_t ldg_u8(const uint8_t *p, bool ok) {
    uint32_t v;
    asm volatile("{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %2, 0;\n\tmov.b32 %0, 0;\n\t"
                 "@q ld.global.nc.L1::no_allocate.u8 %0, [%1];\n\t}"
                 : "=r"(v)
                 : "l"(p), "r"((int)ok));
    return v;
}

template <typename D> struct Mma;
template <> struct Mma<BF16> {
    __device__ static __forceinline__ void run(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
        asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
};
template <> struct Mma<F16> {
    __device__ static __forceinline__ void run(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
        asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
};

// table lookup of byte k (0..3) of w: prmt puts the lane's bank offset in
// byte 0, the packed byte in byte 1 and the table page in bytes 2..3 of the
// address (L = page | 4 lane)
template <int k>
__device__ __forceinline__ uint32_t lut(uint32_t w, uint32_t L) {
    return lds32(prmt(w, L, 0x7604u | (k << 4)));
}

// one unit's loads: 8 packed bytes of item iota(g) and of item iota(g + 8),
// and, on the lane that scales a sum, its block's absmax (or 8-bit code and
// group scale)
struct Unit {
    uint2 wa, wb;
    float am;
    uint32_t code;
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
    const uint32_t part_a = base0 + kMaxRows * 4;            // float [kWarps][2][8]
    const uint32_t lut_a = (base0 + kPrefix + kPage - 1) & ~(kPage - 1);
    const uint32_t xs_a = lut_a + kPage;

    const int nitems = K >> 6;
    const int S = (nitems + kItems - 1) / kItems;
    {
        uint32_t dyn;
        asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
        if (xs_a + (uint32_t)S * kSegK * 2 > base0 + dyn) {
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
    const int NP = (R + 1) >> 1;
    const int NPB = (NP + kPairs - 1) / kPairs;
    const int GU = NPB * S;                                  // groups of this CTA
    const int g_lo = (int)(((int64_t)GU * warp) / kWarps);
    const int g_hi = (int)(((int64_t)GU * (warp + 1)) / kWarps);

    const int g8 = lane >> 2, t4 = lane & 3;
    const int rho = g8 & 1, itA = g8 >> 1;
    // the lane's useful accumulator entry (at most one per lane)
    const bool hiC = t4 >= 2;
    const bool useful = t4 == (g8 >> 2) || t4 == 2 + (g8 >> 2);
    const bool oddC = (itA & 1) != 0;
    const int it_u = hiC ? itA + 4 : itA;
    const int64_t row_bytes = K >> 1;
    const int nblk = K >> log2B;
    const int bsh = log2B - 6;                               // item -> block

    auto load = [&](int g, Unit (&u)[kPairs]) {
        const int pb = g / S, j = g - pb * S;
        const int iA = j * kItems + itA, iB = iA + 4, iu = j * kItems + it_u;
#pragma unroll
        for (int pp = 0; pp < kPairs; ++pp) {
            const int rl = 2 * (pb * kPairs + pp) + rho;     // row within the CTA
            const bool rok = rl < R && g < g_hi;
            const int row = r0 + rl;
            const uint8_t *wr = W + (int64_t)row * row_bytes + 8 * t4;
            u[pp].wa = ldg_w8(wr + iA * 32, rok && iA < nitems);
            u[pp].wb = ldg_w8(wr + iB * 32, rok && iB < nitems);
            const bool aok = rok && useful && iu < nitems;
            const int64_t bi = (int64_t)row * nblk + (iu >> bsh);
            if constexpr (DQ) {
                u[pp].code = ldg_u8(static_cast<const uint8_t *>(absmax) + (aok ? bi : 0), aok);
                u[pp].am = ldg_f32(scales + (aok ? (bi >> log2G) : 0), aok);
            } else {
                u[pp].am = ldg_f32(static_cast<const float *>(absmax) + (aok ? bi : 0), aok);
                u[pp].code = 0;
            }
        }
    };

    Unit ua[kPairs], ub[kPairs];
    // the first two groups' loads leave before the table and x are staged
    load(g_lo, ua);
    load(g_lo + 1, ub);
    {
        // table: entry v (codes of nibbles v >> 4, v & 15) copied to words 64 v + l, l < 32
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int idx = tid + i * kThreads;              // 2048 16-byte pieces
            const int v = idx >> 3, q = idx & 7;
            const uint32_t e = Dt<D>::pack2(tab.v[v >> 4], tab.v[v & 15]);
            sts128(lut_a + v * 256 + q * 16, make_uint4(e, e, e, e));
        }
        // x: 16-byte piece q of item i at position (q + (i & 1)) & 7; zeros past K
        const uint4 *x4 = reinterpret_cast<const uint4 *>(x);
        const int npieces = S * kSegK / 8;
        for (int c = tid; c < npieces; c += kThreads) {
            const uint4 v = 8 * c < K ? __ldg(x4 + c) : make_uint4(0, 0, 0, 0);
            const int i = c >> 3, q = c & 7;
            sts128(xs_a + i * 128 + (((q + (i & 1)) & 7) << 4), v);
        }
    }
    __syncthreads();

    const uint32_t L = lut_a | (4u * lane);
    const int pb_first = g_lo < g_hi ? g_lo / S : -1;
    const int pb_last = g_lo < g_hi ? (g_hi - 1) / S : -1;
    float acc[kPairs] = {0.f, 0.f, 0.f, 0.f};

    // reduce the lanes' sums of pair block pb and store its 8 row sums
    auto flush = [&](int pb) {
        const bool b4 = (lane & 16) != 0, b3 = (lane & 8) != 0;
        // over lane bit 4: keep pairs (0, 1) or (2, 3), send the other two
        float k0 = b4 ? acc[2] : acc[0], k1 = b4 ? acc[3] : acc[1];
        const float s0 = b4 ? acc[0] : acc[2], s1 = b4 ? acc[1] : acc[3];
        k0 += __shfl_xor_sync(FULL, s0, 16);
        k1 += __shfl_xor_sync(FULL, s1, 16);
        // over lane bit 3: keep one of the two
        float q = b3 ? k1 : k0;
        q += __shfl_xor_sync(FULL, b3 ? k0 : k1, 8);
        q += __shfl_xor_sync(FULL, q, 1);
        q += __shfl_xor_sync(FULL, q, 2);
        // lanes 4 i hold pair 2 b4 + b3, row rho = bit 2
        if ((lane & 3) == 0) {
            const int k = 2 * (2 * (int)b4 + (int)b3) + ((lane >> 2) & 1);  // row within the block
            if (pb == pb_first)
                sts32f(part_a + (warp * 16 + k) * 4, q);
            else if (pb == pb_last)
                sts32f(part_a + (warp * 16 + 8 + k) * 4, q);
            else if (8 * pb + k < R)
                sts32f(rowsum_a + (8 * pb + k) * 4, q);
        }
#pragma unroll
        for (int pp = 0; pp < kPairs; ++pp) acc[pp] = 0.f;
    };

    auto compute = [&](int g, const Unit (&u)[kPairs]) {
        const int pb = g / S, j = g - pb * S;
        // x of item 8 j + g8 at this lane's 16 positions [16 t, 16 t + 16)
        const uint32_t xi = xs_a + (j * kItems + g8) * 128;
        const uint4 x0 = lds128(xi + (((2 * t4 + (g8 & 1)) & 7) << 4));
        const uint4 x1 = lds128(xi + (((2 * t4 + 1 + (g8 & 1)) & 7) << 4));
#pragma unroll
        for (int pp = 0; pp < kPairs; ++pp) {
            if (2 * (pb * kPairs + pp) < R) {                 // warp-uniform
                float c[4] = {0.f, 0.f, 0.f, 0.f};
                const uint32_t wa0 = u[pp].wa.x, wa1 = u[pp].wa.y, wb0 = u[pp].wb.x, wb1 = u[pp].wb.y;
                Mma<D>::run(c, lut<0>(wa0, L), lut<0>(wb0, L), lut<1>(wa0, L), lut<1>(wb0, L), x0.x, x0.y);
                Mma<D>::run(c, lut<2>(wa0, L), lut<2>(wb0, L), lut<3>(wa0, L), lut<3>(wb0, L), x0.z, x0.w);
                Mma<D>::run(c, lut<0>(wa1, L), lut<0>(wb1, L), lut<1>(wa1, L), lut<1>(wb1, L), x1.x, x1.y);
                Mma<D>::run(c, lut<2>(wa1, L), lut<2>(wb1, L), lut<3>(wa1, L), lut<3>(wb1, L), x1.z, x1.w);
                float v = hiC ? (oddC ? c[3] : c[2]) : (oddC ? c[1] : c[0]);
                v = useful ? v : 0.f;
                float am = u[pp].am;
                if constexpr (DQ) {
                    const float cf = __uint_as_float(0x4b000000u | u[pp].code) - 8388608.0f;
                    am = useful ? __fmul_rn(cf, div255_rn(am)) : 0.f;
                }
                acc[pp] = __fmaf_rn(v, am, acc[pp]);
            }
        }
        if (g + 1 == g_hi || (g + 1) / S != pb) flush(pb);
    };

    for (int g = g_lo; g < g_hi; g += 2) {
        compute(g, ua);
        load(g + 2, ua);
        if (g + 1 < g_hi) {
            compute(g + 1, ub);
            load(g + 3, ub);
        }
    }
    __syncthreads();

    for (int r = tid; r < R; r += kThreads) {
        // the warps whose group ranges meet this row's pair block (groups
        // [ul, uh)), in order.  A warp starting inside the block left it in
        // slot 0, one ending inside it in slot 1; otherwise the block is the
        // warp's alone and went to the row sums.
        const int pb = r >> 3, k = r & 7, ul = pb * S, uh = ul + S;
        const int w0 = (kWarps * (ul + 1) + GU - 1) / GU - 1, w1 = (kWarps * uh + GU - 1) / GU - 1;
        float v = 0.f;
        for (int w = w0; w <= w1; ++w) {
            const int lo = (int)(((int64_t)GU * w) / kWarps), hi = (int)(((int64_t)GU * (w + 1)) / kWarps);
            if (lo >= hi) continue;
            v += lo >= ul ? lds32f(part_a + (w * 16 + k) * 4)
                 : hi - 1 < uh ? lds32f(part_a + (w * 16 + 8 + k) * 4)
                               : lds32f(rowsum_a + r * 4);
        }
        if (bias) v += Dt<D>::to_f32(bias[r0 + r]);
        y[r0 + r] = (uint16_t)(Dt<D>::pack2(v, 0.f) & 0xffffu);
    }
}

namespace {

// shared memory the kernel asks for: the prefix, padding up to the next 64 KB
// boundary of the shared window (the dynamic region starts right after the
// device's reserved shared memory), the table and x
size_t smem_bytes(int K, int reserved) {
    const size_t S = ((size_t)(K >> 6) + kItems - 1) / kItems;
    const size_t lut = ((size_t)reserved + kPrefix + kPage - 1) / kPage * kPage;
    return lut - (size_t)reserved + kPage + S * kSegK * 2;
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
    gemv_kernel<D, DQ><<<G, kThreads, smem_bytes(K, reserved), stream>>>(
        static_cast<const uint16_t *>(x), W, absmax, scales, log2G, static_cast<const uint16_t *>(bias),
        static_cast<uint16_t *>(y), N, K, log2B, tab);
    return cudaGetLastError();
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
