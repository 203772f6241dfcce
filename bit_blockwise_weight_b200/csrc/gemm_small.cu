// gemm_small.cu -- gemm_4bit for 1 <= M <= 16, gemv included:
// Y[M, N] = X[M, K] . dequant(W)[N, K]^T (+ bias).
//
// "Feat/mps gemm 4bit bf16", What runs natively now (gemv_4bit for M == 1 and
// gemm_4bit for general M) and Performance (small M is dominated by the
// weight stream).  At M <= 16 the product moves 0.5625 B of weight per 2 M
// flops: the weight stream sets the time, and decoding the 4-bit codes at HBM
// rate is the work.  Weight tiles are small and many, so the multiply-adds go
// to mma.sync.m16n8k16 fed straight from registers (W is the 16-row A operand,
// X^T the 8-column B operand, fp32 accumulation):
//
//   * warp 0 streams, per four 64-element runs of K, the CTA's packed-weight
//     tile (rows x 128 bytes, 128-byte swizzle), its absmax tile and four
//     16-token X tiles (64 elements each, 128-byte swizzle; tokens past M
//     arrive as zeros) into a 4-slot ring with TMA;
//   * warps 1-16 each own one 16-row tile of the CTA's rows.  Per run a lane
//     reads its 8 packed bytes of two rows and its X fragments with
//     conflict-free shared loads, turns each byte into a pair of 16-bit codes
//     through a byte table replicated once per shared-memory bank, and issues
//     the MMAs; the run's sums are scaled by the block absmax in fp32.
//
// K order inside a 64-element run: lane (g, t) owns weights [16t, 16t+16) of
// rows g and g+8 (8 contiguous bytes each).  For mma step s (0..3) it feeds
// bytes 2s and 2s+1 of its 8, so k-slot 2t+e holds k = 16t + 4s + e and k-slot
// 2t+8+e holds k = 16t + 4s + 2 + e; the B fragment takes the same k values of
// X.  The reduction over k is a plain sum, so the order is free, and every
// step stays inside one run, hence one block.  So the weight a token meets is
// RN_dtype(code) * absmax, accumulated in fp32; the codes, as 16-bit values,
// lose at most 2^-8 (bf16) or 2^-11 (f16) relative.
//
// Work split: CTA (g, z) owns rows [N g / G, N (g+1) / G) (balanced to one
// row, at most 256) and the z-th of S shares of the K stages; the S CTAs of a
// cluster add their partial sums through distributed shared memory.  No
// global scratch.  Every mbarrier wait is bounded.
#include <atomic>
#include <cstring>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace bnb4 {

namespace {

constexpr int kRowsMax = 256;                     // weight rows per CTA
constexpr int RUN = 64;                           // weights per row per run (one block or less)
constexpr int RPS = 4;                            // runs per stage (128-byte weight rows)
constexpr int STAGES = 4;
constexpr int NTOK = 16;                          // tokens, zero-padded
constexpr int W_SLOT = kRowsMax * RPS * RUN / 2;  // 32 KB
constexpr int X_RUN = NTOK * RUN * 2;             // 2 KB per run
constexpr int X_SLOT = RPS * X_RUN;               // 8 KB
constexpr int AMX_SLOT = kRowsMax * 4;            // one 16-byte box per row
constexpr int NCW = 16;                           // compute warps (one 16-row tile each)
constexpr int MT = kRowsMax / 16 / NCW;           // 16-row tiles per compute warp
constexpr int THREADS = (1 + NCW) * 32;           // 544

struct Smem {
    uint8_t w[STAGES][W_SLOT];   // 1024-byte aligned (128-byte swizzle atoms)
    uint8_t x[STAGES][X_SLOT];   // 1024-byte aligned
    float amx[STAGES][AMX_SLOT];
    uint64_t full[STAGES], empty[STAGES];
    int abort;
};
static_assert(kRowsMax * NTOK * 4 <= STAGES * W_SLOT, "output staging fits in the weight ring");
static_assert(sizeof(Smem) + 1024 + 256 * 32 * 4 <= 227 * 1024, "shared memory plan");

// byte -> (code hi nibble, code lo nibble) as a 16-bit pair, one copy per
// bank: entry e of lane l at word 32 e + l
__shared__ uint32_t s_lut[256 * 32];

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
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

// offset of byte j (0..3) of w's table entry in this lane's bank
__device__ __forceinline__ uint32_t lut_off(uint32_t w, int j) {
    const uint32_t sh = j == 0 ? (w << 7) : (w >> (8 * j - 7));
    return sh & 0x7f80u;
}

// NT = 1 for M <= 8 (tokens 0..7), 2 for M <= 16.  GMODE: how absmax
// arrives (0: 16-byte boxes by TMA; else the producer warp gathers it, see
// below).
template <typename D, int NT, int GMODE>
__global__ void __launch_bounds__(THREADS, 1)
gemm_small_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_amx,
                  const __grid_constant__ CUtensorMap tmap_x, const AbsmaxSrc absmax,
                  const uint16_t *__restrict__ bias, uint16_t *__restrict__ Y, int M, int N, int K,
                  int log2B, int rbox, const __grid_constant__ CodeTable tab) {
    constexpr bool amx_tma = GMODE == 0;
    extern __shared__ uint8_t smem_raw[];
    Smem &s = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                        ~(uintptr_t)1023);
    volatile int *abort = &s.abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x;
    const int r0 = (int)(((int64_t)N * blockIdx.x) / G), r1 = (int)(((int64_t)N * (blockIdx.x + 1)) / G);
    const int R = r1 - r0;
    const int S = gridDim.z, z = blockIdx.z;
    const int nb = K / RUN;
    // K split in whole stages, so that a stage's absmax box starts on a
    // 4-scale boundary
    const int nq = (nb + RPS - 1) / RPS;
    const int b_lo = RPS * (int)(((int64_t)nq * z) / S);
    const int b_hi = min(nb, RPS * (int)(((int64_t)nq * (z + 1)) / S));
    const int iters = b_hi > b_lo ? b_hi - b_lo : 0;  // runs
    const int stages = (iters + RPS - 1) / RPS;
    const int nblk = K >> log2B;

    for (int e = threadIdx.x; e < 256 * 8; e += THREADS) {  // one entry's copies for 4 lanes
        const uint32_t v = Dt<D>::pack2(tab.v[(e >> 3) >> 4], tab.v[(e >> 3) & 15]);
        reinterpret_cast<uint4 *>(s_lut)[e] = make_uint4(v, v, v, v);
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], NCW);  // one arrival per compute warp
        }
        s.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    float acc[MT][NT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[mt][nt][i] = 0.0f;
    const int g = lane >> 2, t = lane & 3, wc = warp - 1;

    if (warp == 0) {
        // ------------------------------------ TMA producer: weights, X, absmax
        const uint32_t tx = (uint32_t)rbox * (RPS * RUN / 2) + X_SLOT + (amx_tma ? (uint32_t)rbox * 16u : 0u);
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_w)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_x)) : "memory");
        }
        // Absmax rows not 16-byte pitched, or 8-bit statistics: the lanes
        // gather each stage's scales themselves.  GMODE 1 (fp32) and 2 (8-bit
        // codes of blocks of 64: one 32-bit word of four codes and one group
        // scale per row) load a stage ahead into registers, and the values are
        // finished when the stage is written, so the loads of stage q + 1 are
        // in flight while the ring waits for a free slot.  GMODE 3 (other
        // 8-bit layouts) gathers and finishes at the stage itself.
        constexpr int GR = GMODE == 1 || GMODE == 2 ? kRowsMax / 32 : 1;
        float gv[GR][GMODE == 1 ? RPS : 1];
        uint32_t gw[GMODE == 2 ? GR : 1];
        auto gather = [&](int q) {
            const int b = b_lo + q * RPS;
#pragma unroll
            for (int pi = 0; pi < GR; ++pi) {
                const int p = lane + 32 * pi;
                if constexpr (GMODE == 1) {
#pragma unroll
                    for (int j = 0; j < RPS; ++j) {
                        const int blk = ((b + j) * RUN) >> log2B;
                        gv[pi][j] = (p < R && b + j < b_hi) ? __ldg(absmax.f32 + (int64_t)(r0 + p) * nblk + blk) : 0.0f;
                    }
                } else if constexpr (GMODE == 2) {
                    // blocks b .. b + 3 of the row: four codes of one word, one group
                    const int64_t f = (int64_t)(r0 + p) * nblk + b;
                    const bool in = p < R && b < b_hi;
                    gw[pi] = in ? __ldg(reinterpret_cast<const uint32_t *>(absmax.q + f)) : 0u;
                    gv[pi][0] = in ? __ldg(absmax.scales + (f >> absmax.log2G)) : 0.0f;
                }
            }
        };
        if (GMODE != 0 && stages > 0) gather(0);
        int issued = 0;
        for (int q = 0; q < stages; ++q) {
            const int st = q % STAGES;
            bool ok = true;
            if (q >= STAGES) ok = mbar_wait(&s.empty[st], ((q / STAGES) - 1) & 1, abort);
            if (!__all_sync(FULL, ok)) break;
            const int b = b_lo + q * RPS;                  // first run of the stage
            const int x0 = ((b * RUN) >> log2B) & ~3;      // first scale of the absmax box
            if constexpr (GMODE == 1) {
#pragma unroll
                for (int pi = 0; pi < GR; ++pi)
#pragma unroll
                    for (int j = 0; j < RPS; ++j) {
                        const int p = lane + 32 * pi;
                        const int blk = ((b + j) * RUN) >> log2B;
                        if (p < R && b + j < b_hi) s.amx[st][p * 4 + (blk - x0)] = gv[pi][j];
                    }
            } else if constexpr (GMODE == 2) {
#pragma unroll
                for (int pi = 0; pi < GR; ++pi) {
                    const int p = lane + 32 * pi;
                    if (p < R) {
                        const float step = div255_rn(gv[pi][0]);
#pragma unroll
                        for (int j = 0; j < RPS; ++j)
                            if (b + j < b_hi) s.amx[st][p * 4 + j] = __fmul_rn((float)((gw[pi] >> (8 * j)) & 255u), step);
                    }
                }
            } else if constexpr (GMODE == 3) {
                for (int p = lane; p < R; p += 32)
                    for (int j = 0; j < RPS && b + j < b_hi; ++j) {
                        const int blk = ((b + j) * RUN) >> log2B;
                        s.amx[st][p * 4 + (blk - x0)] = absmax((int64_t)(r0 + p) * nblk + blk);
                    }
            }
            if (GMODE != 0 && q + 1 < stages) gather(q + 1);
            __syncwarp();  // the gathered scales are written before lane 0 arrives
            if (lane == 0) {
                mbar_arrive_expect_tx(&s.full[st], tx);
                tma_load_2d(&tmap_w, &s.full[st], s.w[st], b * (RUN / 2), r0);
#pragma unroll
                for (int j = 0; j < RPS; ++j)  // runs past K arrive as zeros
                    tma_load_2d(&tmap_x, &s.full[st], s.x[st] + j * X_RUN, (b + j) * RUN, 0);
                if (amx_tma) tma_load_2d(&tmap_amx, &s.full[st], s.amx[st], x0, r0);
            }
            issued = q + 1;
        }
        if (lane == 0)
            for (int q = (issued > STAGES ? issued - STAGES : 0); q < issued; ++q)
                mbar_drain(&s.full[q % STAGES], (q / STAGES) & 1);
    } else {
        // ------------------------------------------------ compute warps
        const uint32_t lut = smem_u32(s_lut) + 4u * lane;
        const uint32_t w_base = smem_u32(s.w[0]), x_base = smem_u32(s.x[0]), amx_base = smem_u32(s.amx[0]);
        // tiles of this warp present in the CTA's rows
        int ntl = 0;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
            if (16 * (wc + NCW * mt) < R) ntl = mt + 1;
        for (int q = 0; q < stages; ++q) {
            const int st = q % STAGES;
            if (!__all_sync(FULL, mbar_wait(&s.full[st], (q / STAGES) & 1, abort))) break;
            const int b = b_lo + q * RPS;
            const int x0 = ((b * RUN) >> log2B) & ~3;
            const uint32_t ws = w_base + st * W_SLOT, xs = x_base + st * X_SLOT, as = amx_base + st * (AMX_SLOT * 4);
#pragma unroll 1
            for (int j = 0; j < RPS; ++j) {
                if (b + j >= b_hi) break;
                // X fragments of run j: token nt*8 + g, k = 16t + 4s .. +3 (8 bytes)
                uint2 xf[4][NT];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int m = nt * 8 + g;
                    const uint32_t row = xs + j * X_RUN + (m >> 3) * 1024 + (m & 7) * 128;
#pragma unroll
                    for (int s4 = 0; s4 < 4; ++s4)
                        xf[s4][nt] = lds64(row + ((((uint32_t)(2 * t + (s4 >> 1))) ^ (uint32_t)(m & 7)) << 4) +
                                           8 * (s4 & 1));
                }
                const uint32_t aoff = 4u * (uint32_t)((((b + j) * RUN) >> log2B) - x0);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    if (mt >= ntl) break;
                    const int rr0 = 16 * (wc + NCW * mt) + g, rr1 = rr0 + 8;
                    const uint32_t chunk = (uint32_t)(2 * j + (t >> 1));
                    const uint2 w0 = lds64(ws + rr0 * 128 + ((chunk ^ (uint32_t)(rr0 & 7)) << 4) + 8 * (t & 1));
                    const uint2 w1 = lds64(ws + rr1 * 128 + ((chunk ^ (uint32_t)(rr1 & 7)) << 4) + 8 * (t & 1));
                    const float a0 = __uint_as_float(lds32(as + rr0 * 16 + aoff));
                    const float a1 = __uint_as_float(lds32(as + rr1 * 16 + aoff));
                    float blk[NT][4];
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int i = 0; i < 4; ++i) blk[nt][i] = 0.0f;
#pragma unroll
                    for (int s4 = 0; s4 < 4; ++s4) {
                        const int wi = s4 >> 1, j0 = 2 * (s4 & 1), j1 = j0 + 1;
                        const uint32_t wg = wi ? w0.y : w0.x;
                        const uint32_t wg8 = wi ? w1.y : w1.x;
                        uint32_t a[4];
                        a[0] = lds32(lut + lut_off(wg, j0));
                        a[1] = lds32(lut + lut_off(wg8, j0));
                        a[2] = lds32(lut + lut_off(wg, j1));
                        a[3] = lds32(lut + lut_off(wg8, j1));
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) Mma<D>::run(blk[nt], a, xf[s4][nt].x, xf[s4][nt].y);
                    }
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            acc[mt][nt][i] = __fmaf_rn(blk[nt][i], (i >> 1) ? a1 : a0, acc[mt][nt][i]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.empty[st]);  // one arrival per warp, after all its reads
        }
    }

    // ----------------- output: stage the sums, add the cluster's partials
    // (S > 1) and store.  Every thread of every CTA of the cluster passes the
    // same barriers.  The ring is idle: every stage was consumed or drained.
    __syncthreads();
    float *stg = reinterpret_cast<float *>(&s.w[0][0]);  // [kRowsMax][NTOK]
    if (warp >= 1) {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int rr = 16 * (wc + NCW * mt) + g + 8 * (i >> 1);
                    stg[rr * NTOK + nt * 8 + 2 * t + (i & 1)] = acc[mt][nt][i];
                }
    }
    if (S > 1) cluster_sync_all();
    else __syncthreads();
    const uint32_t stg_addr = smem_u32(stg);
    const int q_lo = (int)(((int64_t)R * z) / S), q_hi = (int)(((int64_t)R * (z + 1)) / S);
    const int nr = q_hi - q_lo;
    for (int v = threadIdx.x; v < nr * NT * 8; v += THREADS) {
        const int m = v / nr, lr = q_lo + v % nr;  // consecutive threads: consecutive rows
        if (m >= M) continue;
        float sum;
        if (S > 1) {
            float p[8];
            const uint32_t la = stg_addr + (uint32_t)(lr * NTOK + m) * 4;
#pragma unroll
            for (int q2 = 0; q2 < 8; ++q2)
                if (q2 < S) p[q2] = ld_dsmem_f32(la, (uint32_t)q2);
            sum = p[0];
#pragma unroll
            for (int q2 = 1; q2 < 8; ++q2)
                if (q2 < S) sum += p[q2];
        } else {
            sum = stg[lr * NTOK + m];
        }
        const int row = r0 + lr;
        if (bias) sum += Dt<D>::to_f32(bias[row]);
        Y[(int64_t)m * N + row] = (uint16_t)(Dt<D>::pack2(sum, 0.f) & 0xffffu);
    }
    if (S > 1) cluster_sync_all();
}

constexpr size_t kSmemBytes = sizeof(Smem) + 1024;

template <typename D, int NT>
cudaError_t set_smem_attr() {
    static std::atomic<bool> done[kMaxDevices];  // per device: attributes belong to a device's context
    return once_per_device(done, [] {
        const void *k[4] = {(const void *)gemm_small_kernel<D, NT, 0>, (const void *)gemm_small_kernel<D, NT, 1>,
                            (const void *)gemm_small_kernel<D, NT, 2>, (const void *)gemm_small_kernel<D, NT, 3>};
        for (const void *f : k) {
            const cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    });
}

cudaLaunchConfig_t make_cfg(dim3 grid, int S, cudaStream_t stream, cudaLaunchAttribute *attr) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = S;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

// CTAs in clusters of S (1, 2, 4, 8) resident at once on the current device
template <typename D, int NT>
int cluster_capacity(int S) {
    static std::atomic<int> cache[4][kMaxDevices];
    const int ci = S == 1 ? 0 : S == 2 ? 1 : S == 4 ? 2 : 3;
    return cached_per_device(cache[ci], [&] {
        int n = 0;
        cudaLaunchAttribute attr[1];
        cudaLaunchConfig_t cfg = make_cfg(dim3(1, 1, S), S, 0, attr);
        if (set_smem_attr<D, NT>() != cudaSuccess ||
            cudaOccupancyMaxActiveClusters(&n, gemm_small_kernel<D, NT, 0>, &cfg) != cudaSuccess || n <= 0) {
            (void)cudaGetLastError();
            n = device_sm_count() / S;
        }
        return n * S;
    });
}

// Row groups G and K split S.  A CTA's time is taken as its runs times
// max(rows, kRowsMax), plus a fixed cost per split for the reduction: each
// compute warp owns a 16-row tile and its chain of loads, lookups and MMAs
// is latency-bound, so a stage takes about as long with few rows as with
// 256 (measured on B200: 28672 x 8192 at M = 2 ran 59.6 us as 74 groups of
// 111 rows split 2 ways, 46.3 us as 37 groups of 222 rows split 4 ways).
struct Plan {
    int G, S;
};

template <typename D, int NT>
Plan make_plan(int N, int nb) {
    Plan best{1, 1};
    double best_t = 1e300;
    const int nq = (nb + RPS - 1) / RPS;  // stages of RPS runs; a split takes whole stages
    for (int S = 1; S <= 8 && S <= nq; S *= 2) {
        const int cap = cluster_capacity<D, NT>(S);
        long G = cap / S;
        if (G > (N + 15) / 16) G = (N + 15) / 16;  // at least 16 rows per group
        if (G < 1) G = 1;
        if ((N + G - 1) / G > kRowsMax) G = (N + kRowsMax - 1) / kRowsMax;
        const long rows = (N + G - 1) / G;
        const long waves = (G * S + cap - 1) / cap;
        const double t = (double)waves * (RPS * ((nq + S - 1) / S) * (double)(rows > kRowsMax ? rows : kRowsMax) +
                                          (S > 1 ? 4.0 * 64 : 0.0));
        if (t < best_t - 1e-9) {
            best_t = t;
            best = Plan{(int)G, S};
        }
    }
    return best;
}

template <typename D, int NT>
cudaError_t launch_t(const void *X, const uint8_t *W, const AbsmaxSrc &absmax, const void *bias, void *Y,
                     int M, int N, int K, int log2B, const CodeTable &tab, cudaStream_t stream) {
    if (!get_encode()) return cudaErrorNotSupported;
    const int nb = K / RUN;
    const Plan plan = make_plan<D, NT>(N, nb);
    const int rbox = (N + plan.G - 1) / plan.G;
    const CUtensorMapDataType xt = std::is_same<D, BF16>::value ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                                : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUtensorMap map_w, map_x, map_amx;
    const uint64_t row_bytes = (uint64_t)K / 2;
    if (encode_2d(&map_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, W, row_bytes, N, row_bytes, RPS * RUN / 2, rbox,
                  CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS ||
        encode_2d(&map_x, xt, X, K, M, (uint64_t)K * 2, RUN, NTOK, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    // absmax by 16-byte TMA boxes when its row pitch allows, else (or for
    // 8-bit statistics) gathered by the producer warp
    const int nblk = K >> log2B;
    int amx_tma = (nblk % 4 == 0 && !absmax.q) ? 1 : 0;
    std::memset(&map_amx, 0, sizeof(map_amx));
    if (amx_tma && encode_2d(&map_amx, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, absmax.f32, nblk, N, (uint64_t)nblk * 4, 4,
                             rbox, CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
        amx_tma = 0;
    cudaError_t e = set_smem_attr<D, NT>();
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = make_cfg(dim3(plan.G, 1, plan.S), plan.S, stream, attr);
    // absmax gathered by the producer: fp32 (1); 8-bit codes of blocks of 64
    // with rows of whole 4-code words and groups of at least 4 (2); other
    // 8-bit layouts (3)
    const int gmode = amx_tma ? 0 : !absmax.q ? 1 : (log2B == 6 && nblk % 4 == 0 && absmax.log2G >= 2) ? 2 : 3;
    const uint16_t *b16 = static_cast<const uint16_t *>(bias);
    uint16_t *y16 = static_cast<uint16_t *>(Y);
    switch (gmode) {
    case 0:
        return cudaLaunchKernelEx(&cfg, gemm_small_kernel<D, NT, 0>, map_w, map_amx, map_x, absmax, b16, y16, M, N,
                                  K, log2B, rbox, tab);
    case 1:
        return cudaLaunchKernelEx(&cfg, gemm_small_kernel<D, NT, 1>, map_w, map_amx, map_x, absmax, b16, y16, M, N,
                                  K, log2B, rbox, tab);
    case 2:
        return cudaLaunchKernelEx(&cfg, gemm_small_kernel<D, NT, 2>, map_w, map_amx, map_x, absmax, b16, y16, M, N,
                                  K, log2B, rbox, tab);
    default:
        return cudaLaunchKernelEx(&cfg, gemm_small_kernel<D, NT, 3>, map_w, map_amx, map_x, absmax, b16, y16, M, N,
                                  K, log2B, rbox, tab);
    }
}

}  // namespace

cudaError_t gemm_small_timeouts_address(unsigned int **p) { return wait_timeouts_address(p); }

cudaError_t launch_gemm_small(const void *X, const uint8_t *W, const float *absmax_f32, const uint8_t *absmax_q,
                              const float *scales, int group, const void *bias, void *Y, int64_t M, int64_t N,
                              int64_t K, int blocksize, bnb4_quant_type qt, bnb4_dtype dt,
                              cudaStream_t stream) {
    static const CodeTable nf4 = host_code_table(BNB4_NF4);
    static const CodeTable fp4 = host_code_table(BNB4_FP4);
    const CodeTable &tab = qt == BNB4_NF4 ? nf4 : fp4;
    const AbsmaxSrc absmax{absmax_f32, absmax_q, scales, absmax_q ? ilog2(group) : 0};
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
