// gemm_tc.cu -- gemm_4bit for large M and gemm_4bit_backward on the 5th-gen
// tensor cores (tcgen05, accumulators in TMEM).
//
// "Feat/mps gemm 4bit bf16", What runs natively now (gemm_4bit for general M;
// gemm_4bit_backward, grad_input = grad_output @ dequantize_4bit(B)) and
// Performance (at large M the GEMM itself dominates).  The pages' design
// dequantizes weight chunks into a scratch buffer and calls a library GEMM;
// here the weight never exists in dequantized form outside shared memory:
//
//   forward   D[M, N] = A[M, K] . W[N, K]^T   (A = X,  reduction over K)
//   backward  D[M, K] = A[M, N] . W[N, K]     (A = dY, reduction over N)
//
// One CTA computes a 256 x BN output tile (BN = 256, or forward a narrower
// multiple of 16 down to 160 when that fills the SMs better) as two M=128
// tcgen05.mma accumulators (2 x BN TMEM columns)
// that share one B operand:
//   * warp 0, one thread: TMA loads of A (two 128 x 64 boxes per stage,
//     128-byte swizzle) into a 3-slot ring;
//   * warp 10: TMA loads of the stage's packed weight tile (BN rows x 32 bytes,
//     32-byte swizzle, forward; 64 rows x 128 bytes, 128-byte swizzle,
//     backward) and of the matching absmax tile (16 bytes per weight row) into
//     a 4-slot ring.  When the absmax row pitch is not a multiple of 16 bytes
//     the warp gathers the absmax values with ordinary loads instead;
//   * warps 2-9: each thread reads one 64-element weight run (32 packed bytes
//     + its block absmax) from the ring, decodes it by byte permutation from
//     the block's 16 scaled values (no shuffles) and writes one 128-byte row
//     of the B tile in the canonical 128-byte-swizzled layout: K-major rows for
//     the forward, MN-major rows for the backward (so neither needs a
//     transpose), fences the writes to the async proxy and arrives on the stage
//     barrier of a 2-slot B ring;
//   * warp 1, one thread: waits for A and B of a stage, issues 2 x 4
//     tcgen05.mma (K = 16 each) and commits the slots back to the producers;
//   * after the last stage warps 2-9 read the accumulators (tcgen05.ld), add
//     the bias in fp32, round once and store.
// Each decoded weight is RN_dtype(fp32(code * absmax)), the exact value the
// dequantize kernel produces, so the MMA consumes the dequantized weight.
// Packed-weight bytes that the tensor map clips (rows past N, bytes past K/2)
// arrive as zeros; the absmax tile is clipped the same way, so rows past N
// decode to +-0, and columns past K meet zero-filled A columns.
//
// Every mbarrier wait is bounded (about one second of %globaltimer); a wait
// that runs out raises the library's device error word, makes the CTA skip
// the rest of its work, and still frees its TMEM before returning.
#include <atomic>
#include <cstring>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace bnb4 {

namespace {

constexpr int BM = 256;           // two M=128 accumulators
constexpr int BN_MAX = 256;       // output columns per tile (256, or narrower to fill the SMs)
constexpr int BK = 64;            // reduction per stage (one 128-byte swizzle row)
constexpr int A_STAGES = 3;
constexpr int B_STAGES = 2;
constexpr int W_STAGES = 4;
constexpr int A_HALF = 128 * BK * 2;             // 16 KB per 128-row box
constexpr int A_STAGE = 2 * A_HALF;              // 32 KB
constexpr int B_STAGE = BN_MAX * BK * 2;         // 32 KB
constexpr int W_SLOT = BN_MAX * BK / 2;          // 8 KB of packed weights per stage
constexpr int AMX_SLOT = BN_MAX * 4;             // 4 floats per weight row
constexpr int RED_CW = 64;                       // columns per reduction chunk (split K)
constexpr int RED_PITCH = RED_CW + 4;            // fp32 staging row pitch
constexpr int NUM_DQ_WARPS = 8;
constexpr int W_WARP = 2 + NUM_DQ_WARPS;          // weight-tile producer
constexpr int THREADS = (3 + NUM_DQ_WARPS) * 32;  // 352

struct Smem {
    uint8_t a[A_STAGES][A_STAGE];   // 1024-byte aligned (swizzle atoms)
    uint8_t b[B_STAGES][B_STAGE];
    uint8_t w[W_STAGES][W_SLOT];
    float amx[W_STAGES][AMX_SLOT];
    uint64_t full_a[A_STAGES], empty_a[A_STAGES];
    uint64_t full_b[B_STAGES], empty_b[B_STAGES];
    uint64_t full_w[W_STAGES], empty_w[W_STAGES];
    uint64_t tmem_full;
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(Smem) + 1024 <= 227 * 1024, "shared memory plan");
static_assert(BM * RED_PITCH * 4 <= A_STAGES * A_STAGE, "split-K staging fits in the A ring");

template <typename D, int CNT>
__device__ __forceinline__ void store_out(uint16_t *out, int64_t row, int n_out, int col,
                                          const float *v, const uint16_t *bias, bool add_bias) {
    uint16_t *dst = out + row * n_out + col;
    float w[CNT];
#pragma unroll
    for (int e = 0; e < CNT; ++e) {
        w[e] = v[e];
        if (add_bias && bias && col + e < n_out) w[e] += Dt<D>::to_f32(bias[col + e]);
    }
    if (col + CNT <= n_out && ((reinterpret_cast<uintptr_t>(dst) & 15) == 0) && CNT % 8 == 0) {
#pragma unroll
        for (int e = 0; e < CNT; e += 8) {
            uint4 p;
            p.x = Dt<D>::pack2(w[e], w[e + 1]);
            p.y = Dt<D>::pack2(w[e + 2], w[e + 3]);
            p.z = Dt<D>::pack2(w[e + 4], w[e + 5]);
            p.w = Dt<D>::pack2(w[e + 6], w[e + 7]);
            *reinterpret_cast<uint4 *>(dst + e) = p;
        }
    } else if (col + CNT <= n_out && ((reinterpret_cast<uintptr_t>(dst) & 7) == 0) && CNT % 4 == 0) {
#pragma unroll
        for (int e = 0; e < CNT; e += 4)
            *reinterpret_cast<uint2 *>(dst + e) =
                make_uint2(Dt<D>::pack2(w[e], w[e + 1]), Dt<D>::pack2(w[e + 2], w[e + 3]));
    } else {
#pragma unroll
        for (int e = 0; e < CNT; ++e)
            if (col + e < n_out) dst[e] = (uint16_t)(Dt<D>::pack2(w[e], 0.f) & 0xffffu);
    }
}

template <typename D, bool BWD, int BN>
__global__ void __launch_bounds__(THREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_w,
               const __grid_constant__ CUtensorMap tmap_amx, const AbsmaxSrc absmax,
               const uint16_t *__restrict__ bias, uint16_t *__restrict__ out, int M, int N, int K,
               int log2B, int amx_tma, const __grid_constant__ CodeTable tab) {
    extern __shared__ uint8_t smem_raw[];
    Smem &s = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                        ~(uintptr_t)1023);
    volatile int *abort = &s.abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_out = BWD ? K : N;  // output columns
    const int red = BWD ? N : K;    // reduction length
    const int c0 = blockIdx.x * BN;  // first output column of the tile
    const int m0 = blockIdx.y * BM;
    // split of the reduction over the CTAs of a cluster (gridDim.z of them)
    const int C = gridDim.z, z = blockIdx.z;
    const int iters_all = (red + BK - 1) / BK;
    const int i_lo = (int)(((int64_t)iters_all * z) / C);
    const int iters = (int)(((int64_t)iters_all * (z + 1)) / C) - i_lo;
    const int nblk = K >> log2B;
    // first absmax column of the 16-byte box that holds a stage's scales
    // (backward: fixed per tile; forward: per stage)
    const int bwd_x0 = (c0 >> log2B) & ~3;

    if (threadIdx.x == 0) {
        for (int i = 0; i < A_STAGES; ++i) {
            mbar_init(&s.full_a[i], 1);
            mbar_init(&s.empty_a[i], 1);
        }
        for (int i = 0; i < B_STAGES; ++i) {
            mbar_init(&s.full_b[i], NUM_DQ_WARPS * 32);
            mbar_init(&s.empty_b[i], 1);
        }
        for (int i = 0; i < W_STAGES; ++i) {
            mbar_init(&s.full_w[i], 32);
            mbar_init(&s.empty_w[i], NUM_DQ_WARPS * 32);
        }
        mbar_init(&s.tmem_full, 1);
        s.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {  // whole warp: allocate all 512 TMEM columns
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                         smem_u32(&s.tmem_base))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s.tmem_base;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (A)
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_a))
                         : "memory");
            int issued = 0;
            for (int i = 0; i < iters; ++i) {
                const int st = i % A_STAGES;
                if (i >= A_STAGES && !mbar_wait(&s.empty_a[st], ((i / A_STAGES) - 1) & 1, abort)) break;
                mbar_arrive_expect_tx(&s.full_a[st], A_STAGE);
                tma_load_2d(&tmap_a, &s.full_a[st], s.a[st], (i_lo + i) * BK, m0);
                tma_load_2d(&tmap_a, &s.full_a[st], s.a[st] + A_HALF, (i_lo + i) * BK, m0 + 128);
                issued = i + 1;
            }
            // do not leave while a load may still be landing in this CTA's memory
            for (int i = (issued > A_STAGES ? issued - A_STAGES : 0); i < issued; ++i)
                mbar_drain(&s.full_a[i % A_STAGES], (i / A_STAGES) & 1);
        }
    } else if (warp == W_WARP) {
        // ---------------------------------- TMA producer (packed weights, absmax)
        constexpr int W_ROWS = BWD ? BK : BN;  // weight rows per stage
        constexpr uint32_t W_BYTES = W_ROWS * (BWD ? BN_MAX / 2 : BK / 2);
        const uint32_t tx = W_BYTES + (amx_tma ? W_ROWS * 16u : 0u);
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_w))
                         : "memory");
            if (amx_tma)
                asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_amx))
                             : "memory");
        }
        // Without absmax boxes (rows not 16-byte pitched, or 8-bit
        // statistics) the lanes gather each stage's scales into the same
        // [row][4] layout the tensor map would produce, one stage ahead: the
        // loads of stage i + 1 are in flight while the ring waits for a slot.
        // Element p (lane + 32 pi) of a stage: forward, row c0 + p of the
        // stage's block; backward, row it BK + (p & 63), block column p >> 6.
        AbsmaxRaw gv[8];
        auto slot_of = [&](int it, int p, int &row, int &blk, int &at) {
            if (BWD) {
                row = it * BK + (p & 63);
                blk = (c0 + 64 * (p >> 6)) >> log2B;
                at = (p & 63) * 4 + (blk - bwd_x0);
            } else {
                row = c0 + p;
                blk = (it * BK) >> log2B;
                at = p * 4 + (blk & 3);
            }
        };
        auto gather = [&](int i) {
            const int it = i_lo + i;
#pragma unroll
            for (int pi = 0; pi < 8; ++pi) {
                const int p = lane + 32 * pi;
                int row, blk, at;
                slot_of(it, p, row, blk, at);
                const bool in = BWD ? (row < N && blk < nblk) : (p < BN && row < N);
                gv[pi] = in ? absmax.raw((int64_t)row * nblk + blk) : AbsmaxRaw{0u, 0.0f};
            }
        };
        if (!amx_tma && iters > 0) gather(0);
        int issued = 0;
        for (int i = 0; i < iters; ++i) {
            const int st = i % W_STAGES;
            bool ok = true;
            if (i >= W_STAGES) ok = mbar_wait(&s.empty_w[st], ((i / W_STAGES) - 1) & 1, abort);
            if (!__all_sync(FULL, ok)) break;
            const int it = i_lo + i;
            if (!amx_tma) {
                float *dst = s.amx[st];
#pragma unroll
                for (int pi = 0; pi < 8; ++pi) {
                    const int p = lane + 32 * pi;
                    int row, blk, at;
                    slot_of(it, p, row, blk, at);
                    if (BWD || p < BN) dst[at] = absmax.finish(gv[pi]);
                }
                if (i + 1 < iters) gather(i + 1);
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(&s.full_w[st], tx);
                if (BWD) {
                    tma_load_2d(&tmap_w, &s.full_w[st], s.w[st], c0 >> 1, it * BK);
                    if (amx_tma) tma_load_2d(&tmap_amx, &s.full_w[st], s.amx[st], bwd_x0, it * BK);
                } else {
                    tma_load_2d(&tmap_w, &s.full_w[st], s.w[st], it * (BK / 2), c0);
                    if (amx_tma)
                        tma_load_2d(&tmap_amx, &s.full_w[st], s.amx[st], ((it * BK) >> log2B) & ~3, c0);
                }
            } else {
                mbar_arrive(&s.full_w[st]);
            }
            issued = i + 1;
        }
        if (lane == 0)
            for (int i = (issued > W_STAGES ? issued - W_STAGES : 0); i < issued; ++i)
                mbar_drain(&s.full_w[i % W_STAGES], (i / W_STAGES) & 1);
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = make_idesc<BN, 128>(std::is_same<D, BF16>::value, BWD);
            bool ok = true;
            for (int i = 0; i < iters && ok; ++i) {
                const int sa = i % A_STAGES, sb = i % B_STAGES;
                ok = mbar_wait(&s.full_a[sa], (i / A_STAGES) & 1, abort) &&
                     mbar_wait(&s.full_b[sb], (i / B_STAGES) & 1, abort);
                if (!ok) break;
                tc_fence_after();
                const uint32_t a_base = smem_u32(s.a[sa]);
                const uint32_t b_base = smem_u32(s.b[sb]);
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    // B: K-major rows of 128 B (forward), or MN-major with the four
                    // 64-column atoms 1 KB apart and 8-row groups 4 KB apart (backward)
                    const uint64_t bdesc =
                        BWD ? smem_desc(b_base + kk * 2 * 4096, 1024, 4096)
                            : smem_desc(b_base + kk * 32, 16, 1024);
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt) {
                        const uint64_t adesc = smem_desc(a_base + mt * A_HALF + kk * 32, 16, 1024);
                        tc_mma(tmem + mt * BN, adesc, bdesc, idesc, (i > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                tc_commit(&s.empty_a[sa]);  // slots free once these MMAs have read them
                tc_commit(&s.empty_b[sb]);
            }
            if (ok) tc_commit(&s.tmem_full);
        }
    } else {
        // ---------------------------------------- weight dequant warps
        // 256 runs of 64 weights per stage, one per thread
        const int t = threadIdx.x - 64;
        // forward: row t of the tile (output column c0 + t) over the stage's 64
        // reduction indices; backward: reduction row (t & 63) of the stage over
        // output columns c0 + 64 (t >> 6) ... + 63
        const bool active = BWD || t < BN;
        // source of the run in a weight slot, as two swizzled 16-byte chunks
        uint32_t src0, src1;
        if (BWD) {
            const uint32_t r = t & 63, g = t >> 6;
            src0 = r * 128 + (((2 * g) ^ (r & 7)) << 4);
            src1 = r * 128 + (((2 * g + 1) ^ (r & 7)) << 4);
        } else {
            src0 = t * 32 + ((0u ^ ((t >> 2) & 1)) << 4);
            src1 = t * 32 + ((1u ^ ((t >> 2) & 1)) << 4);
        }
        // absmax slot index: [row][4], the column inside the 16-byte box
        const int amx_row = BWD ? (t & 63) : t;
        const int bwd_idx = ((c0 + 64 * (t >> 6)) >> log2B) - bwd_x0;
        // destination row of this run in the B tile
        uint32_t row_base, row_sw;
        if (BWD) {
            const uint32_t r = t & 63, atom = t >> 6;
            row_base = atom * 1024 + (r >> 3) * 4096 + (r & 7) * 128;
            row_sw = r;
        } else {
            row_base = (t >> 3) * 1024 + (t & 7) * 128;
            row_sw = t;
        }
        auto load = [&](int i, uint32_t (&w)[8], float &a) -> bool {
            const int ws = i % W_STAGES;
            if (!mbar_wait(&s.full_w[ws], (i / W_STAGES) & 1, abort)) return false;
            if (active) {
                const uint4 v0 = *reinterpret_cast<const uint4 *>(s.w[ws] + src0);
                const uint4 v1 = *reinterpret_cast<const uint4 *>(s.w[ws] + src1);
                w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
                w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
                const int idx = BWD ? bwd_idx : (((i_lo + i) * BK) >> log2B) & 3;
                a = s.amx[ws][amx_row * 4 + idx];
            } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) w[q] = 0u;
                a = 0.0f;
            }
            mbar_arrive(&s.empty_w[ws]);
            return true;
        };
        uint32_t w[8], nw[8];
        float a = 0.0f, na = 0.0f;
        bool ok = iters > 0 && load(0, w, a);
        for (int i = 0; i < iters && ok; ++i) {
            const int sb = i % B_STAGES;
            if (i + 1 < iters) ok = load(i + 1, nw, na);
            if (i >= B_STAGES && !mbar_wait(&s.empty_b[sb], ((i / B_STAGES) - 1) & 1, abort)) break;
            uint8_t *bt = s.b[sb];
            const ScaledPlanes sp = scaled_planes<D>(tab, a);
#pragma unroll
            for (int j = 0; j < 8; ++j) {  // chunk j = weights 8j .. 8j+7 = bytes 4j..4j+3
                uint32_t o[4];
                decode4(sp, w[j], o[0], o[1]);
                decode4(sp, w[j] >> 16, o[2], o[3]);
                if (active)
                    *reinterpret_cast<uint4 *>(bt + swz(row_base, row_sw, j)) = make_uint4(o[0], o[1], o[2], o[3]);
            }
            fence_proxy_async();
            mbar_arrive(&s.full_b[sb]);
#pragma unroll
            for (int q = 0; q < 8; ++q) w[q] = nw[q];
            a = na;
        }

        // ------------------------------------------------ direct epilogue
        if (C == 1) {
            __syncwarp();
            if (mbar_wait(&s.tmem_full, 0, abort)) {
                __syncwarp();
                tc_fence_after();
                // warp 2 + ew: TMEM lane quadrant warp & 3 (the one it may read),
                // accumulator ew >> 2
                const int ew = warp - 2;
                const int q = warp & 3;
                const int mt = (ew >> 2) & 1;
                const int row = m0 + mt * 128 + q * 32 + lane;
                const uint32_t tbase = tmem + mt * BN + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
                for (int cc = 0; cc < BN; cc += 16) {
                    uint32_t r[16];
                    tmem_ld16(tbase + cc, r);
                    tmem_ld_wait();
                    const int col = c0 + cc;
                    if (row < M && col < n_out) {
                        float v[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] = __uint_as_float(r[e]);
                        store_out<D, 16>(out, row, n_out, col, v, bias, !BWD);
                    }
                }
            }
        }
    }

    // ------------------- split reduction: add the cluster's partial tiles
    // Every thread of every CTA of the cluster passes the same cluster
    // barriers, whatever happened before, so none can be left waiting.
    if (C > 1) {
        __syncwarp();
        const bool dq = warp >= 2 && warp < W_WARP;
        bool have = false;
        if (dq) {
            have = __all_sync(FULL, mbar_wait(&s.tmem_full, 0, abort));
            if (have) tc_fence_after();
        }
        // the A ring is free once the last MMA has completed: fp32 staging of
        // one 256 x 64 chunk of this CTA's partial tile
        float *stg = reinterpret_cast<float *>(&s.a[0][0]);
        const uint32_t stg_addr = smem_u32(stg);
        const int rows_per = BM / C;
#pragma unroll 1
        for (int cb = 0; cb < BN; cb += RED_CW) {
            if (dq && have) {
                const int ew = warp - 2;
                const int q = warp & 3, mt = (ew >> 2) & 1;
                const int lrow = mt * 128 + q * 32 + lane;
                const uint32_t tbase = tmem + mt * BN + ((uint32_t)(q * 32) << 16);
#pragma unroll
                for (int cc = 0; cc < RED_CW; cc += 16) {
                    if (cb + cc >= BN) break;  // a narrower tile ends inside the last chunk
                    uint32_t r[16];
                    tmem_ld16(tbase + cb + cc, r);
                    tmem_ld_wait();
                    float4 *d = reinterpret_cast<float4 *>(stg + lrow * RED_PITCH + cc);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        d[e] = make_float4(__uint_as_float(r[4 * e]), __uint_as_float(r[4 * e + 1]),
                                           __uint_as_float(r[4 * e + 2]), __uint_as_float(r[4 * e + 3]));
                }
            }
            cluster_sync_all();
            if (dq) {
                const int e0 = threadIdx.x - 64;
                for (int v = e0; v < rows_per * (RED_CW / 4); v += NUM_DQ_WARPS * 32) {
                    const int lr = z * rows_per + v / (RED_CW / 4);
                    const int c4 = (v % (RED_CW / 4)) * 4;
                    if (cb + c4 >= BN) continue;
                    const uint32_t la = stg_addr + (uint32_t)(lr * RED_PITCH + c4) * 4;
                    // all C partials in flight before the first add (C <= 8)
                    float4 p[8];
#pragma unroll
                    for (int q2 = 0; q2 < 8; ++q2)
                        if (q2 < C) p[q2] = ld_dsmem_f4(la, (uint32_t)q2);
                    float4 acc = p[0];
#pragma unroll
                    for (int q2 = 1; q2 < 8; ++q2)
                        if (q2 < C) {
                            acc.x += p[q2].x; acc.y += p[q2].y; acc.z += p[q2].z; acc.w += p[q2].w;
                        }
                    const int row = m0 + lr, col = c0 + cb + c4;
                    if (row < M && col < n_out) {
                        const float vv[4] = {acc.x, acc.y, acc.z, acc.w};
                        store_out<D, 4>(out, row, n_out, col, vv, bias, !BWD);
                    }
                }
            }
            cluster_sync_all();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
    }
}

constexpr size_t kSmemBytes = sizeof(Smem) + 1024;

template <typename D, bool BWD, int BN>
cudaError_t set_smem_attr() {
    static std::atomic<bool> done[kMaxDevices];  // per device: attributes belong to a device's context
    return once_per_device(done, [] {
        return cudaFuncSetAttribute(gemm_tc_kernel<D, BWD, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    });
}

cudaLaunchConfig_t make_cfg(dim3 grid, int C, cudaStream_t stream, cudaLaunchAttribute *attr) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = C;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

// CTAs of clusters of C (1, 2, 4, 8) that can be resident at once on the
// current device: clusters must fit inside one GPC, so this can be below the
// SM count.  Queried once per device and cluster size.
template <typename D, bool BWD, int BN>
int cluster_capacity(int C) {
    static std::atomic<int> cache[4][kMaxDevices];
    const int ci = C == 1 ? 0 : C == 2 ? 1 : C == 4 ? 2 : 3;
    return cached_per_device(cache[ci], [&] {
        int n = 0;
        cudaLaunchAttribute attr[1];
        cudaLaunchConfig_t cfg = make_cfg(dim3(1, 1, C), C, 0, attr);
        if (set_smem_attr<D, BWD, BN>() != cudaSuccess ||
            cudaOccupancyMaxActiveClusters(&n, gemm_tc_kernel<D, BWD, BN>, &cfg) != cudaSuccess || n <= 0) {
            (void)cudaGetLastError();
            n = device_sm_count() / C;
        }
        return n * C;
    });
}

template <typename D, bool BWD, int BN>
cudaError_t launch_bn(const CUtensorMap &map_a, const CUtensorMap &map_w, const CUtensorMap &map_amx,
                      const AbsmaxSrc &absmax, const void *bias, void *out, int M, int N, int K,
                      int log2B, int amx_tma, const CodeTable &tab, int C, cudaStream_t stream) {
    cudaError_t e = set_smem_attr<D, BWD, BN>();
    if (e != cudaSuccess) return e;
    const int n_out = BWD ? K : N;
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = make_cfg(dim3((n_out + BN - 1) / BN, (M + BM - 1) / BM, C), C, stream, attr);
    return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<D, BWD, BN>, map_a, map_w, map_amx, absmax,
                              static_cast<const uint16_t *>(bias), static_cast<uint16_t *>(out), M,
                              N, K, log2B, amx_tma, tab);
}

// Tile width and reduction split: the pair minimising
//   waves x (stages per CTA + fixed cost) x (kWidthFixed + width),
// the fixed cost (prologue, epilogue; the cluster reduction when split) in
// stage units.  A stage's time grows with the width (the MMAs) on top of a
// part that does not (the dequant warps convert all 256 rows of a stage
// either way); measured on B200 at M = 2048, 160-wide tiles took 61 us per
// wave and 256-wide 69 us, about 600 columns' worth of fixed time.  A split
// keeps at least 8 stages per CTA.
constexpr double kWidthFixed = 600.0;
struct Plan {
    int bn, C;
};

template <typename D, bool BWD>
Plan make_plan(long mt, int n_out, int iters) {
    Plan best{256, 1};
    double best_t = 1e300;
    for (int bn : {256, 224, 208, 192, 176, 160}) {
        if (BWD && bn != 256) continue;  // the MN-major tile is built from 64-column atoms
        const long tiles = mt * ((n_out + bn - 1) / bn);
        for (int C = 1; C <= 8; C *= 2) {
            if (C > 1 && iters / C < 8) break;
            // residency does not depend on the width (shared memory is sized for 256)
            const int cap = cluster_capacity<D, BWD, 256>(C);
            const long waves = (tiles * C + cap - 1) / cap;
            const double t = (double)waves * ((iters + C - 1) / C + (C == 1 ? 4 : 8)) * (kWidthFixed + bn);
            if (t < best_t - 1e-9) {
                best_t = t;
                best = Plan{bn, C};
            }
        }
    }
    return best;
}

template <typename D, bool BWD>
cudaError_t launch_t(const void *A, const uint8_t *W, const AbsmaxSrc &absmax, const void *bias,
                     void *out, int M, int N, int K, int log2B, const CodeTable &tab,
                     cudaStream_t stream) {
    if (!get_encode()) return cudaErrorNotSupported;
    const int red = BWD ? N : K;
    const int n_out = BWD ? K : N;
    // A: [M rows, red columns] row-major; TMA needs a 16-byte row pitch
    if ((red * 2) % 16 != 0) return cudaErrorInvalidValue;
    const CUtensorMapDataType a_type = std::is_same<D, BF16>::value ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                                    : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUtensorMap map_a, map_w, map_amx;
    if (encode_2d(&map_a, a_type, A, red, M, (uint64_t)red * 2, BK, 128, CU_TENSOR_MAP_SWIZZLE_128B) !=
        CUDA_SUCCESS)
        return cudaErrorInvalidValue;

    const long mt = (M + BM - 1) / BM;
    const int iters = (red + BK - 1) / BK;
    const Plan plan = make_plan<D, BWD>(mt, n_out, iters);
    const int bn = plan.bn, C = plan.C;
    // packed weights [N rows, K/2 bytes]: per stage BN rows x 32 bytes (forward)
    // or 64 rows x 128 bytes (backward)
    const uint64_t row_bytes = (uint64_t)K / 2;  // a multiple of 16: K % 32 == 0
    const CUresult rw =
        BWD ? encode_2d(&map_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, W, row_bytes, N, row_bytes, BN_MAX / 2, BK,
                        CU_TENSOR_MAP_SWIZZLE_128B)
            : encode_2d(&map_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, W, row_bytes, N, row_bytes, BK / 2, bn,
                        CU_TENSOR_MAP_SWIZZLE_32B);
    if (rw != CUDA_SUCCESS) return cudaErrorInvalidValue;
    // absmax [N rows, K / blocksize]: 16-byte boxes when its row pitch allows,
    // otherwise (or when it arrives as 8-bit statistics) gathered by the
    // producer warp
    const int nblk = K >> log2B;
    int amx_tma = (nblk % 4 == 0 && !absmax.q) ? 1 : 0;
    memset(&map_amx, 0, sizeof(map_amx));
    if (amx_tma &&
        encode_2d(&map_amx, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, absmax.f32, nblk, N, (uint64_t)nblk * 4, 4,
                  BWD ? BK : bn, CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
        amx_tma = 0;

    if constexpr (!BWD) {
        switch (bn) {
        case 224: return launch_bn<D, BWD, 224>(map_a, map_w, map_amx, absmax, bias, out, M, N, K, log2B, amx_tma, tab, C, stream);
        case 208: return launch_bn<D, BWD, 208>(map_a, map_w, map_amx, absmax, bias, out, M, N, K, log2B, amx_tma, tab, C, stream);
        case 192: return launch_bn<D, BWD, 192>(map_a, map_w, map_amx, absmax, bias, out, M, N, K, log2B, amx_tma, tab, C, stream);
        case 176: return launch_bn<D, BWD, 176>(map_a, map_w, map_amx, absmax, bias, out, M, N, K, log2B, amx_tma, tab, C, stream);
        case 160: return launch_bn<D, BWD, 160>(map_a, map_w, map_amx, absmax, bias, out, M, N, K, log2B, amx_tma, tab, C, stream);
        default: break;
        }
    }
    return launch_bn<D, BWD, 256>(map_a, map_w, map_amx, absmax, bias, out, M, N, K, log2B, amx_tma,
                                  tab, C, stream);
}

// A wait that nothing completes, bounded at limit_ns: exercises the timeout
// path (error count raised, no fault, the kernel returns).
__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, &abort_flag, limit_ns);
}

}  // namespace

cudaError_t launch_selftest_wait_timeout(cudaStream_t stream) {
    wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(1000000ull);  // 1 ms
    return cudaGetLastError();
}

cudaError_t gemm_tc_timeouts_address(unsigned int **p) { return wait_timeouts_address(p); }

cudaError_t launch_gemm_tc(const void *A, const uint8_t *W, const float *absmax_f32, const uint8_t *absmax_q,
                           const float *scales, int group, const void *bias,
                           void *D, int64_t M, int64_t N, int64_t K, int blocksize,
                           bnb4_quant_type qt, bnb4_dtype dt, bool backward, cudaStream_t stream) {
    static const CodeTable nf4 = host_code_table(BNB4_NF4);
    static const CodeTable fp4 = host_code_table(BNB4_FP4);
    const CodeTable &tab = qt == BNB4_NF4 ? nf4 : fp4;
    const AbsmaxSrc absmax{absmax_f32, absmax_q, scales, absmax_q ? ilog2(group) : 0};
    const int log2B = ilog2(blocksize);
    const int m = (int)M, n = (int)N, k = (int)K;
    if (dt == BNB4_F16)
        return backward ? launch_t<F16, true>(A, W, absmax, bias, D, m, n, k, log2B, tab, stream)
                        : launch_t<F16, false>(A, W, absmax, bias, D, m, n, k, log2B, tab, stream);
    return backward ? launch_t<BF16, true>(A, W, absmax, bias, D, m, n, k, log2B, tab, stream)
                    : launch_t<BF16, false>(A, W, absmax, bias, D, m, n, k, log2B, tab, stream);
}

}  // namespace bnb4
