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
// K order inside a 128-element span: lane (g, t) owns weights [32t, 32t+32)
// of rows g and g+8 (16 contiguous bytes each).  For mma step s it feeds
// bytes 2s and 2s+1 of its chunk, so k-slot 2t+e holds k = 32t + 4s + e and
// k-slot 2t+8+e holds k = 32t + 4s + 2 + e; the B fragment takes the same k
// values of X.  The reduction over k is a plain sum, so this order is free.
//
// absmax: with blocksize 64 a span holds two blocks (lanes t < 2 carry block
// 0, t >= 2 block 1).  Two mma per step, each with the other block's B values
// zeroed, keep the two block sums apart; each is scaled by its absmax in fp32.
// For blocksize >= 128 a span lies in one block and one mma per step does.
//
// CTA: 4 warps on 32 rows; a 512-element window of K per iteration (one span
// per warp), X windows double-buffered in shared memory with cp.async, weight
// chunks double-buffered in registers.  Warps' partial sums meet in shared
// memory; K split over a thread-block cluster meets in distributed shared
// memory.  No global scratch.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace bnb4 {

namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kRows = 32;              // rows of W per CTA (two m16 tiles)
constexpr int kSpan = 128;             // K elements per warp per window
constexpr int kWin = kWarps * kSpan;   // 512
constexpr int kXStride = kWin + 16;    // bf16 elements per X row in smem (+32 B: no bank conflicts)
constexpr int kMaxM = 16;

__device__ __forceinline__ uint4 ld_stream(const uint8_t *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

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

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// byte j (0..3) of a word -> offset of its entry in this lane's bank
// (entry e of lane l sits at word 32 e + l)
__device__ __forceinline__ uint32_t lut_off(uint32_t w, int j, uint32_t lane4) {
    const uint32_t sh = j == 0 ? (w << 7) : (w >> (8 * j - 7));
    return (sh & 0x7f80u) | lane4;
}

__device__ __forceinline__ void cp_async8(void *smem, const void *gmem) {
    const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(s), "l"(gmem));
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

template <typename D, int NT>
__global__ void __launch_bounds__(kThreads)
gemm_small_kernel(const uint16_t *__restrict__ X, const uint8_t *__restrict__ W,
                  const float *__restrict__ absmax, const uint16_t *__restrict__ bias,
                  uint16_t *__restrict__ Y, int M, int N, int K, int log2B, int Kc,
                  CodeTable tab) {
    extern __shared__ __align__(16) uint8_t smem[];
    uint32_t *lut = reinterpret_cast<uint32_t *>(smem);                        // 256 x 32 words
    uint16_t *xwin = reinterpret_cast<uint16_t *>(smem + 256 * 32 * 4);        // [2][16][kXStride]
    float *red = reinterpret_cast<float *>(xwin + 2 * kMaxM * kXStride);       // [kWarps][32][16]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int ksplit = gridDim.y;
    const int k0 = blockIdx.y * Kc;
    const int k1 = min(K, k0 + Kc);
    const int row0 = blockIdx.x * kRows;
    const int64_t row_bytes = K >> 1;
    const int nblk = K >> log2B;

    // byte -> code pair table, one copy per bank
    for (int e = tid; e < 256; e += kThreads) {
        const uint32_t v = Dt<D>::pack2(tab.v[e >> 4], tab.v[e & 15]);
#pragma unroll 4
        for (int b = 0; b < 32; ++b) lut[e * 32 + b] = v;
    }

    const int nwin = (k1 - k0 + kWin - 1) / kWin;
    // X window in the order the B fragments read it: the group of 4 elements
    // k = 128 w + 32 t + 4 s (+0..3) sits at 128 w + 16 s + 4 t, so the four
    // lanes t of one step read 32 contiguous bytes
    auto load_xwin = [&](int wi, int buf) {
        const int kb = k0 + wi * kWin;
        uint16_t *dst = xwin + buf * kMaxM * kXStride;
        for (int c = tid; c < M * (kWin / 4); c += kThreads) {
            const int m = c / (kWin / 4), q = c % (kWin / 4);
            const int k = kb + q * 4;
            const int w = q >> 5, tt = (q >> 3) & 3, ss = q & 7;
            uint16_t *d = dst + m * kXStride + w * kSpan + ss * 16 + tt * 4;
            if (k < k1)
                cp_async8(d, X + (int64_t)m * K + k);
            else
                *reinterpret_cast<uint2 *>(d) = make_uint2(0, 0);
        }
        cp_async_commit();
    };
    // rows >= M of both X buffers stay zero
    for (int c = tid; c < 2 * kMaxM * kXStride / 8; c += kThreads) {
        const int m = (c * 8 / kXStride) % kMaxM;
        if (m >= M) reinterpret_cast<uint4 *>(xwin)[c] = make_uint4(0, 0, 0, 0);
    }

    // this lane's rows: tile mt, half h -> row0 + 16 mt + 8 h + g
    int rows[2][2];
    bool rv[2][2];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            rows[mt][h] = row0 + 16 * mt + 8 * h + g;
            rv[mt][h] = rows[mt][h] < N;
        }
    auto load_w = [&](int wi, uint4 (&dst)[2][2]) {
        const int kk = k0 + wi * kWin + warp * kSpan + 32 * t;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int h = 0; h < 2; ++h)
                dst[mt][h] = (rv[mt][h] && kk < k1)
                                 ? ld_stream(W + (int64_t)rows[mt][h] * row_bytes + (kk >> 1))
                                 : make_uint4(0, 0, 0, 0);
    };

    float acc[2][NT][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[mt][nt][i] = 0.f;

    const uint32_t lut_base = (uint32_t)__cvta_generic_to_shared(lut);
    const uint32_t lane4 = 4u * lane;
    const bool two_blocks = log2B == 6;  // blocksize 64: a span holds two blocks

    uint4 wcur[2][2], wnxt[2][2];
    if (nwin > 0) {
        load_xwin(0, 0);
        load_w(0, wcur);
    }
    __syncthreads();  // lut ready

    for (int wi = 0; wi < nwin; ++wi) {
        cp_async_wait_all();
        __syncthreads();  // X window wi visible; the other buffer is free
        if (wi + 1 < nwin) {
            load_xwin(wi + 1, (wi + 1) & 1);
            load_w(wi + 1, wnxt);
        }
        const int kspan = k0 + wi * kWin + warp * kSpan;
        const uint16_t *xb = xwin + (wi & 1) * kMaxM * kXStride + warp * kSpan + 4 * t;

        float plo[2][NT][4], phi[2][NT][4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) plo[mt][nt][i] = phi[mt][nt][i] = 0.f;

#pragma unroll
        for (int s = 0; s < 8; ++s) {
            uint32_t b[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const uint2 v = *reinterpret_cast<const uint2 *>(xb + (nt * 8 + g) * kXStride + 16 * s);
                b[nt][0] = v.x;
                b[nt][1] = v.y;
            }
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                const uint32_t wg = (&wcur[mt][0].x)[s >> 1];
                const uint32_t wg8 = (&wcur[mt][1].x)[s >> 1];
                const int j0 = 2 * (s & 1), j1 = j0 + 1;
                uint32_t a[4];
                a[0] = lds32(lut_base + lut_off(wg, j0, lane4));
                a[1] = lds32(lut_base + lut_off(wg8, j0, lane4));
                a[2] = lds32(lut_base + lut_off(wg, j1, lane4));
                a[3] = lds32(lut_base + lut_off(wg8, j1, lane4));
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (two_blocks) {
                        const uint32_t lo0 = t < 2 ? b[nt][0] : 0u, lo1 = t < 2 ? b[nt][1] : 0u;
                        const uint32_t hi0 = t < 2 ? 0u : b[nt][0], hi1 = t < 2 ? 0u : b[nt][1];
                        Mma<D>::run(plo[mt][nt], a, lo0, lo1);
                        Mma<D>::run(phi[mt][nt], a, hi0, hi1);
                    } else {
                        Mma<D>::run(plo[mt][nt], a, b[nt][0], b[nt][1]);
                    }
                }
            }
        }
        // block scales: rows g / g+8 of each tile, blocks of k = kspan and kspan + 64
        const int blo = kspan >> log2B;
        const int bhi = (kspan + 64) >> log2B;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            float alo[2], ahi[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float *ap = absmax + (int64_t)rows[mt][h] * nblk;
                alo[h] = (rv[mt][h] && kspan < k1) ? __ldg(ap + blo) : 0.f;
                ahi[h] = (rv[mt][h] && two_blocks && kspan + 64 < k1) ? __ldg(ap + bhi) : 0.f;
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int h = i >> 1;
                    acc[mt][nt][i] = __fmaf_rn(plo[mt][nt][i], alo[h], acc[mt][nt][i]);
                    if (two_blocks) acc[mt][nt][i] = __fmaf_rn(phi[mt][nt][i], ahi[h], acc[mt][nt][i]);
                }
        }
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int h = 0; h < 2; ++h) wcur[mt][h] = wnxt[mt][h];
    }

    // warps' partial sums -> red[warp][row][m]
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = 16 * mt + 8 * (i >> 1) + g;
                const int m = nt * 8 + 2 * t + (i & 1);
                red[(warp * kRows + r) * kMaxM + m] = acc[mt][nt][i];
            }
    __syncthreads();
    for (int e = tid; e < kRows * kMaxM; e += kThreads) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) v += red[w * kRows * kMaxM + e];
        red[e] = v;  // red[0] now holds the CTA's sums (each e read only by its owner)
    }

    auto finish = [&](int e, float v) {
        const int r = e / kMaxM, m = e % kMaxM;
        const int row = row0 + r;
        if (m < M && row < N) {
            if (bias) v += Dt<D>::to_f32(bias[row]);
            Y[(int64_t)m * N + row] = (uint16_t)(Dt<D>::pack2(v, 0.f) & 0xffffu);
        }
    };

    if (ksplit == 1) {
        __syncthreads();
        for (int e = tid; e < kRows * kMaxM; e += kThreads) finish(e, red[e]);
        return;
    }
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    const int rank = (int)cluster.block_rank();
    for (int e = tid; e < kRows * kMaxM; e += kThreads) {
        if (e % ksplit != rank) continue;
        float v = 0.f;
        for (int q = 0; q < ksplit; ++q) v += *cluster.map_shared_rank(&red[e], q);
        finish(e, v);
    }
    cluster.sync();
}

size_t smem_bytes() {
    return 256 * 32 * 4 + 2 * kMaxM * kXStride * 2 + kWarps * kRows * kMaxM * 4;
}

// choose the K split (cluster size) that fills the GPU's CTA slots most evenly
int pick_ksplit(int groups, int wins, int slots) {
    int best = 1;
    double best_eff = 0.0;
    for (int ks = 1; ks <= 8 && ks <= wins; ++ks) {
        const int per = (wins + ks - 1) / ks;
        const int ks_eff = (wins + per - 1) / per;
        if (ks_eff != ks) continue;
        const long units = (long)groups * ks;
        const long waves = (units + slots - 1) / slots;
        const double eff = (double)units / (double)(waves * slots) * (1.0 - 0.02 * (ks - 1));
        if (eff > best_eff + 1e-9) {
            best_eff = eff;
            best = ks;
        }
    }
    return best;
}

template <typename D, int NT>
cudaError_t launch_t(const void *X, const uint8_t *W, const float *absmax, const void *bias,
                     void *Y, int M, int N, int K, int log2B, const CodeTable &tab,
                     cudaStream_t stream) {
    const size_t smem = smem_bytes();
    static bool attr_set = false;  // benign race: setting it twice is harmless
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(gemm_small_kernel<D, NT>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    const int groups = (N + kRows - 1) / kRows;
    const int wins = (K + kWin - 1) / kWin;
    const int slots = device_sm_count() * 3;
    const int ks = pick_ksplit(groups, wins, slots);
    const int per = (wins + ks - 1) / ks;
    const int Kc = per * kWin;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(groups, ks, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = ks;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemm_small_kernel<D, NT>, static_cast<const uint16_t *>(X), W,
                              absmax, static_cast<const uint16_t *>(bias),
                              static_cast<uint16_t *>(Y), M, N, K, log2B, Kc, tab);
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
