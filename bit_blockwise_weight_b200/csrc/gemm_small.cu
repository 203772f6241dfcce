// gemm_small.cu -- gemm_4bit for small M (1 <= M <= 16): Y = X @ dequant(W)^T (+ bias).
//
// "Feat/mps gemm 4bit bf16", What runs natively now (gemm_4bit, general M)
// and Performance (small M is dominated by the weight stream).  At M <= 16
// the product is a real matrix-matrix product, but it still moves 0.5625 B
// of weight per 2*M flops, far below the tensor-core ridge: the weight stream
// sets the time.  CUDA-core FMAs cannot keep up with 16 products per decoded
// weight, so the decoded weights go straight from registers into
// mma.sync.m16n8k16 fragments (W is the 16-row A operand, X^T the 8-column B
// operand), with fp32 accumulation.
//
// Decode: a 256-entry table maps one packed byte to the two codes it holds
// as a bf16x2 / f16x2 register (first element in the low half).  The table is
// replicated once per shared-memory bank (32 KB) so that every lane reads its
// own bank: lookups never conflict.
//
// K order inside a 64-element quantization block: lane (g, t) owns weights
// [16t, 16t+16) of rows g and g+8 (8 contiguous bytes each).  For mma step s
// (0..3) it feeds bytes 2s and 2s+1 of its 8, so k-slot 2t+e holds
// k = 16t + 4s + e and k-slot 2t+8+e holds k = 16t + 4s + 2 + e; the B
// fragment takes the same k values of X.  The reduction over k is a plain sum,
// so the order is free, and every step stays inside one block: the four steps
// of a block accumulate into a block sum that is scaled by the block's absmax
// in fp32 once.
//
// Work split (persistent, one CTA per SM): CTA c owns rows
// [N c / G, N (c+1) / G) -- balanced to one row -- and all of K.  Its rows form
// T tiles of 16 (the last one partial), grouped by up to 4 per warp so that
// each X fragment feeds 4 tiles; the 8 warps split the groups and then K.
// Weights, absmax and X fragments of the next block are loaded into registers
// while the current block is multiplied.  Partial sums of the warps that
// share a group meet in shared memory.  No global scratch.
#include "common.cuh"
#include "kernels.h"

namespace bnb4 {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int MT = 4;                 // m16 tiles per warp
constexpr int kMaxTiles = 64;         // rows per CTA <= 1024
constexpr int kMaxM = 16;

template <typename D> struct Mma;
template <> struct Mma<BF16> {
    __device__ static __forceinline__ void run(float c[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
};
template <> struct Mma<F16> {
    __device__ static __forceinline__ void run(float c[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
};

__device__ __forceinline__ uint2 ld_stream8(const uint8_t *p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

// byte j (0..3) of a word -> offset of its entry in this lane's bank
// (entry e of lane l sits at word 32 e + l)
__device__ __forceinline__ uint32_t lut_off(uint32_t w, int j, uint32_t lane4) {
    const uint32_t sh = j == 0 ? (w << 7) : (w >> (8 * j - 7));
    return (sh & 0x7f80u) | lane4;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

struct Frag {
    uint2 w[MT][2];     // rows g and g+8 of each tile: 8 bytes (16 weights)
    float a[MT][2];     // their block absmax
};

template <typename D, int NT>
__global__ void __launch_bounds__(kThreads, 1)
gemm_small_kernel(const uint16_t *__restrict__ X, const uint8_t *__restrict__ W,
                  const float *__restrict__ absmax, const uint16_t *__restrict__ bias,
                  uint16_t *__restrict__ Y, int M, int N, int K, int log2B, const __grid_constant__ CodeTable tab) {
    extern __shared__ __align__(16) uint8_t smem[];
    uint32_t *lut = reinterpret_cast<uint32_t *>(smem);                 // 256 x 32 words
    float *sum = reinterpret_cast<float *>(smem + 256 * 32 * 4);        // [kMaxTiles*16][16]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3;

    // CTA rows
    const int G = gridDim.x;
    const int r0 = (int)(((int64_t)N * blockIdx.x) / G);
    const int r1 = (int)(((int64_t)N * (blockIdx.x + 1)) / G);
    const int T = (r1 - r0 + 15) >> 4;  // tiles
    const int nb = K >> 6;              // 64-element blocks along K
    const int64_t row_bytes = K >> 1;
    const int nblk = K >> log2B;

    // byte -> code pair table, one copy per bank (a thread fills 4 copies at once)
    for (int e = tid >> 3; e < 256; e += kThreads / 8) {
        const uint32_t v = Dt<D>::pack2(tab.v[e >> 4], tab.v[e & 15]);
        reinterpret_cast<uint4 *>(lut + e * 32)[tid & 7] = make_uint4(v, v, v, v);
    }
    for (int e = tid; e < T * 16 * kMaxM; e += kThreads) sum[e] = 0.f;
    __syncthreads();
    if (T == 0) return;

    const uint32_t lut_base = (uint32_t)__cvta_generic_to_shared(lut);
    const uint32_t lane4 = 4u * lane;

    // warp -> (tile group, K part)
    const int groups = (T + MT - 1) / MT;
    for (int gbase = 0; gbase < groups; gbase += kWarps) {
        const int gcount = min(kWarps, groups - gbase);
        const int kparts = kWarps / gcount;
        const int gi = gbase + warp / kparts;
        const int kp = warp % kparts;
        const bool active = warp < gcount * kparts;
        const int b_lo = active ? (int)(((int64_t)nb * kp) / kparts) : 0;
        const int b_hi = active ? (int)(((int64_t)nb * (kp + 1)) / kparts) : 0;

        int rows[MT][2];
        bool rv[MT][2];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                rows[mt][h] = r0 + 16 * (gi * MT + mt) + 8 * h + g;
                rv[mt][h] = active && (gi * MT + mt) < T && rows[mt][h] < r1;
            }
        auto fetch = [&](int b, Frag &f) {
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if (rv[mt][h]) {
                        const int64_t rb = (int64_t)rows[mt][h];
                        f.w[mt][h] = ld_stream8(W + rb * row_bytes + 32 * b + 8 * t);
                        f.a[mt][h] = __ldg(absmax + rb * nblk + ((64 * b) >> log2B));
                    } else {
                        f.w[mt][h] = make_uint2(0, 0);
                        f.a[mt][h] = 0.f;
                    }
                }
        };
        // X fragment of block b: lane (g, t) needs X[nt*8 + g][64b + 16t + 4s .. +4] for s = 0..3
        auto fetch_x = [&](int b, uint2 (&xf)[4][NT]) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int m = nt * 8 + g;
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    xf[s][nt] = (m < M) ? __ldg(reinterpret_cast<const uint2 *>(
                                              X + (int64_t)m * K + 64 * b + 16 * t + 4 * s))
                                        : make_uint2(0, 0);
            }
        };

        float acc[MT][NT][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[mt][nt][i] = 0.f;

        Frag cur, nxt;
        uint2 xc[4][NT], xn[4][NT];
        if (b_lo < b_hi) {
            fetch(b_lo, cur);
            fetch_x(b_lo, xc);
        }
        for (int b = b_lo; b < b_hi; ++b) {
            if (b + 1 < b_hi) {
                fetch(b + 1, nxt);
                fetch_x(b + 1, xn);
            }
            float blk[MT][NT][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) blk[mt][nt][i] = 0.f;
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const int wi = s >> 1, j0 = 2 * (s & 1), j1 = j0 + 1;
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    const uint32_t wg = wi ? cur.w[mt][0].y : cur.w[mt][0].x;
                    const uint32_t wg8 = wi ? cur.w[mt][1].y : cur.w[mt][1].x;
                    uint32_t a[4];
                    a[0] = lds32(lut_base + lut_off(wg, j0, lane4));
                    a[1] = lds32(lut_base + lut_off(wg8, j0, lane4));
                    a[2] = lds32(lut_base + lut_off(wg, j1, lane4));
                    a[3] = lds32(lut_base + lut_off(wg8, j1, lane4));
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) Mma<D>::run(blk[mt][nt], a, xc[s][nt].x, xc[s][nt].y);
                }
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        acc[mt][nt][i] = __fmaf_rn(blk[mt][nt][i], cur.a[mt][i >> 1], acc[mt][nt][i]);
            cur = nxt;
#pragma unroll
            for (int s = 0; s < 4; ++s)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) xc[s][nt] = xn[s][nt];
        }

        // this warp's partial sums -> shared sums (warps of a group split K)
        if (active) {
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const int tile = gi * MT + mt;
                if (tile >= T) continue;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int r = 16 * tile + 8 * (i >> 1) + g;
                        const int m = nt * 8 + 2 * t + (i & 1);
                        if (m < M) atomicAdd(&sum[r * kMaxM + m], acc[mt][nt][i]);
                    }
            }
        }
    }
    __syncthreads();
    for (int e = tid; e < T * 16 * kMaxM; e += kThreads) {
        const int r = e / kMaxM, m = e % kMaxM;
        const int row = r0 + r;
        if (m < M && row < r1) {
            float v = sum[e];
            if (bias) v += Dt<D>::to_f32(bias[row]);
            Y[(int64_t)m * N + row] = (uint16_t)(Dt<D>::pack2(v, 0.f) & 0xffffu);
        }
    }
}

size_t smem_bytes(int tiles) { return 256 * 32 * 4 + (size_t)tiles * 16 * kMaxM * 4; }

template <typename D, int NT>
cudaError_t launch_t(const void *X, const uint8_t *W, const float *absmax, const void *bias,
                     void *Y, int M, int N, int K, int log2B, const CodeTable &tab,
                     cudaStream_t stream) {
    const int G = device_sm_count();
    const int max_rows = (N + G - 1) / G;
    const int tiles = (max_rows + 15) / 16;
    if (tiles > kMaxTiles) return cudaErrorInvalidValue;
    const size_t smem = smem_bytes(tiles);
    static int smem_set = 0;  // largest dynamic shared memory size set so far
    if ((int)smem > 48 * 1024 && (int)smem > smem_set) {
        cudaError_t e = cudaFuncSetAttribute(gemm_small_kernel<D, NT>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        smem_set = (int)smem;
    }
    gemm_small_kernel<D, NT><<<G, kThreads, smem, stream>>>(
        static_cast<const uint16_t *>(X), W, absmax, static_cast<const uint16_t *>(bias),
        static_cast<uint16_t *>(Y), M, N, K, log2B, tab);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_small(const void *X, const uint8_t *W, const float *absmax,
                              const void *bias, void *Y, int64_t M, int64_t N, int64_t K,
                              int blocksize, bnb4_quant_type qt, bnb4_dtype dt,
                              cudaStream_t stream) {
    static const CodeTable nf4 = host_code_table(BNB4_NF4);
    static const CodeTable fp4 = host_code_table(BNB4_FP4);
    const CodeTable &tab = qt == BNB4_NF4 ? nf4 : fp4;
    const int log2B = ilog2(blocksize);
    const int m = (int)M, n = (int)N, k = (int)K;
    if (dt == BNB4_F16) {
        if (M <= 8) return launch_t<F16, 1>(X, W, absmax, bias, Y, m, n, k, log2B, tab, stream);
        return launch_t<F16, 2>(X, W, absmax, bias, Y, m, n, k, log2B, tab, stream);
    }
    if (M <= 8) return launch_t<BF16, 1>(X, W, absmax, bias, Y, m, n, k, log2B, tab, stream);
    return launch_t<BF16, 2>(X, W, absmax, bias, Y, m, n, k, log2B, tab, stream);
}

}  // namespace bnb4
