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
// One CTA computes a 256 x 256 output tile as two M=128 tcgen05.mma
// accumulators (2 x 256 TMEM columns = all 512) that share one B operand:
//   * warp 0, one thread: TMA loads of A (two 128 x 64 boxes per stage,
//     128-byte swizzle) into a 3-stage ring;
//   * warps 2-9: each thread decodes one 64-element weight run per
//     stage (32 packed bytes + its block absmax) into a 128-byte row of the B tile
//     in the canonical 128-byte-swizzled layout: K-major rows for the forward,
//     MN-major rows for the backward (so neither needs a transpose), then
//     fences the writes to the async proxy and arrives on the stage barrier;
//   * warp 1, one thread: waits for both halves of a stage, issues 2 x 4
//     tcgen05.mma (K = 16 each) and commits the stage back to the producers;
//   * after the last stage warps 2-9 read the accumulators (tcgen05.ld), add
//     the bias in fp32, round once and store.
// Each decoded weight is RN_dtype(fp32(code * absmax)), the exact value the
// dequantize kernel produces, so the MMA consumes the dequantized weight.
//
// Every mbarrier wait is bounded (about one second of %globaltimer); a wait
// that runs out raises the library's device error word, makes the CTA skip
// the rest of its work, and still frees its TMEM before returning.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace bnb4 {

__device__ unsigned int g_device_error = 0;  // raised by a timed-out wait

namespace {

constexpr int BM = 256;           // two M=128 accumulators
constexpr int BN_MAX = 256;       // output columns per tile (256, or 224 to fill the SMs)
constexpr int BK = 64;            // reduction per stage (one 128-byte swizzle row)
constexpr int STAGES = 3;
constexpr int A_HALF = 128 * BK * 2;             // 16 KB per 128-row box
constexpr int A_STAGE = 2 * A_HALF;              // 32 KB
constexpr int B_STAGE = BN_MAX * BK * 2;         // 32 KB
constexpr int RED_CW = 64;                       // columns per reduction chunk (split K)
constexpr int RED_PITCH = RED_CW + 4;            // fp32 staging row pitch
constexpr int NUM_DQ_WARPS = 8;
constexpr int THREADS = (2 + NUM_DQ_WARPS) * 32;  // 320
constexpr int RUN_PARTS = NUM_DQ_WARPS / 8;       // threads per 64-weight run
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // ~1 s

struct Smem {
    uint8_t a[STAGES][A_STAGE];   // 1024-byte aligned (swizzle atoms)
    uint8_t b[STAGES][B_STAGE];
    uint64_t full_a[STAGES];
    uint64_t full_b[STAGES];
    uint64_t empty[STAGES];
    uint64_t tmem_full;
    uint32_t tmem_base;
    int abort;
};

// ------------------------------------------------------------------ PTX

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait: false (and the error word raised, the CTA told to abort) when
// the barrier did not reach the phase within the limit or another thread of
// the CTA already gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (global_ns() - t0 > kWaitLimitNs) {
            *abort = 1;
            atomicAdd(&g_device_error, 1u);
            return false;
        }
    }
}

__device__ __forceinline__ void tma_load_2d(const CUtensorMap *map, uint64_t *bar, void *dst,
                                            int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t shfl_idx(uint32_t v, uint32_t lane_bits) {
    uint32_t r;
    asm volatile("shfl.sync.idx.b32 %0, %1, %2, 0x1f, 0xffffffff;"
                 : "=r"(r)
                 : "r"(v), "r"(lane_bits));
    return r;
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm100 version 1.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3fff);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3fff) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3fff) << 32;
    d |= (uint64_t)1 << 46;  // version
    d |= (uint64_t)2 << 61;  // SWIZZLE_128B
    return d;
}

// Instruction descriptor for kind::f16: fp32 accumulate, M = 128, N = BN.
template <int BN>
__host__ __device__ constexpr uint32_t make_idesc(bool bf16, bool b_mn_major) {
    return (1u << 4)                              // D format: F32
           | ((bf16 ? 1u : 0u) << 7)              // A format
           | ((bf16 ? 1u : 0u) << 10)             // B format
           | ((b_mn_major ? 1u : 0u) << 16)       // B major (A is K-major)
           | ((uint32_t)(BN >> 3) << 17)          // N
           | ((uint32_t)(128 >> 4) << 24);        // M
}

// Byte offset of the 16-byte chunk j of 128-byte row `row` inside a
// 128-byte-swizzled region whose 8-row atoms sit `atom_stride` apart:
// physical chunk = j ^ (row mod 8).
__device__ __forceinline__ uint32_t swz(uint32_t row_base, uint32_t row, uint32_t j) {
    return row_base + ((j ^ (row & 7u)) << 4);
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t local_addr, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(remote)
                 : "memory");
    return v;
}

template <typename D>
__device__ __forceinline__ void store_out(uint16_t *out, int64_t row, int n_out, int col,
                                          const float *v, int cnt, const uint16_t *bias, bool add_bias) {
    uint16_t *dst = out + row * n_out + col;
    float w[16];
    for (int e = 0; e < cnt; ++e) {
        w[e] = v[e];
        if (add_bias && bias && col + e < n_out) w[e] += Dt<D>::to_f32(bias[col + e]);
    }
    if (col + cnt <= n_out && cnt % 8 == 0 && ((reinterpret_cast<uintptr_t>(dst) & 15) == 0)) {
        for (int e = 0; e < cnt; e += 8) {
            uint4 p;
            p.x = Dt<D>::pack2(w[e], w[e + 1]);
            p.y = Dt<D>::pack2(w[e + 2], w[e + 3]);
            p.z = Dt<D>::pack2(w[e + 4], w[e + 5]);
            p.w = Dt<D>::pack2(w[e + 6], w[e + 7]);
            *reinterpret_cast<uint4 *>(dst + e) = p;
        }
    } else {
        for (int e = 0; e < cnt && col + e < n_out; ++e) dst[e] = (uint16_t)(Dt<D>::pack2(w[e], 0.f) & 0xffffu);
    }
}

template <typename D, bool BWD, int BN>
__global__ void __launch_bounds__(THREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_a, const uint8_t *__restrict__ W,
               const float *__restrict__ absmax, const uint16_t *__restrict__ bias,
               uint16_t *__restrict__ out, int M, int N, int K, int log2B, CodeTable tab) {
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
    const int64_t row_bytes = K >> 1;
    const int nblk = K >> log2B;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&s.full_a[i], 1);
            mbar_init(&s.full_b[i], NUM_DQ_WARPS * 32);
            mbar_init(&s.empty[i], 1);
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
            for (int i = 0; i < iters; ++i) {
                const int st = i % STAGES;
                if (i >= STAGES && !mbar_wait(&s.empty[st], ((i / STAGES) - 1) & 1, abort)) break;
                mbar_arrive_expect_tx(&s.full_a[st], A_STAGE);
                tma_load_2d(&tmap_a, &s.full_a[st], s.a[st], (i_lo + i) * BK, m0);
                tma_load_2d(&tmap_a, &s.full_a[st], s.a[st] + A_HALF, (i_lo + i) * BK, m0 + 128);
            }
            // do not leave while a load may still be landing in this CTA's memory
            for (int i = (iters > STAGES ? iters - STAGES : 0); i < iters; ++i)
                if (!mbar_wait(&s.full_a[i % STAGES], (i / STAGES) & 1, abort)) break;
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = make_idesc<BN>(std::is_same<D, BF16>::value, BWD);
            bool ok = true;
            for (int i = 0; i < iters && ok; ++i) {
                const int st = i % STAGES;
                const uint32_t par = (i / STAGES) & 1;
                ok = mbar_wait(&s.full_a[st], par, abort) && mbar_wait(&s.full_b[st], par, abort);
                if (!ok) break;
                tc_fence_after();
                const uint32_t a_base = smem_u32(s.a[st]);
                const uint32_t b_base = smem_u32(s.b[st]);
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
                tc_commit(&s.empty[st]);  // stage free once these MMAs have read it
            }
            if (ok) tc_commit(&s.tmem_full);
        }
    } else {
        // ---------------------------------------- weight dequant warps
        // 256 runs of 64 weights per stage; RUN_PARTS threads share a run, each
        // decoding 32 / RUN_PARTS packed bytes into 8 / RUN_PARTS of its chunks
        const int part = (threadIdx.x - 64) >> 8;
        const int t = (threadIdx.x - 64) & 255;
        constexpr int WORDS = 8 / RUN_PARTS;
        const uint32_t my_code = __float_as_uint(tab.v[lane & 15]);
        // run geometry: forward row t of the tile (output column c0 + t) over the
        // stage's 64 reduction indices; backward reduction row (t & 63) of the
        // stage over output columns c0 + 64 (t >> 6) ... + 63
        auto src = [&](int i, int &wrow, int &kcol) {
            if (BWD) {
                wrow = (i_lo + i) * BK + (t & 63);
                kcol = c0 + 64 * (t >> 6);
            } else {
                wrow = t < BN ? c0 + t : N;  // threads past the tile width decode nothing
                kcol = (i_lo + i) * BK;
            }
        };
        auto fetch = [&](int i, uint32_t (&w)[WORDS], float &a) {
            int wrow, kcol;
            src(i, wrow, kcol);
            if (wrow < N && kcol < K) {
                const uint4 *p = reinterpret_cast<const uint4 *>(W + (int64_t)wrow * row_bytes + (kcol >> 1)) +
                                 part * (WORDS / 4);
#pragma unroll
                for (int q = 0; q < WORDS / 4; ++q) {
                    const uint4 v = __ldg(p + q);
                    w[4 * q] = v.x; w[4 * q + 1] = v.y; w[4 * q + 2] = v.z; w[4 * q + 3] = v.w;
                }
                a = __ldg(absmax + (int64_t)wrow * nblk + (kcol >> log2B));
            } else {
#pragma unroll
                for (int q = 0; q < WORDS; ++q) w[q] = 0u;
                a = 0.0f;  // zero weights past the edges
            }
        };
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
        uint32_t w[WORDS], nw[WORDS];
        float a, na;
        if (iters > 0) fetch(0, w, a);
        for (int i = 0; i < iters; ++i) {
            const int st = i % STAGES;
            if (i + 1 < iters) fetch(i + 1, nw, na);
            if (i >= STAGES && !mbar_wait(&s.empty[st], ((i / STAGES) - 1) & 1, abort)) break;
            uint8_t *bt = s.b[st];
#pragma unroll
            for (int jj = 0; jj < WORDS; ++jj) {  // chunk j = weights 8j .. 8j+7 = bytes 4j..4j+3
                const int j = WORDS * part + jj;
                uint32_t o[4];
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const uint32_t byte_sh = 8 * h;  // byte h of word j
                    const float ch = __uint_as_float(shfl_idx(my_code, w[jj] >> (byte_sh + 4)));
                    const float cl = __uint_as_float(shfl_idx(my_code, w[jj] >> byte_sh));
                    o[h] = Dt<D>::pack2(__fmul_rn(ch, a), __fmul_rn(cl, a));
                }
                if (BWD || t < BN)
                    *reinterpret_cast<uint4 *>(bt + swz(row_base, row_sw, j)) = make_uint4(o[0], o[1], o[2], o[3]);
            }
            fence_proxy_async();
            mbar_arrive(&s.full_b[st]);
#pragma unroll
            for (int q = 0; q < WORDS; ++q) w[q] = nw[q];
            a = na;
        }

        // ------------------------------------------------ direct epilogue
        if (C == 1) {
            __syncwarp();
            if (mbar_wait(&s.tmem_full, 0, abort)) {
                __syncwarp();
                tc_fence_after();
                // warp 2 + ew: TMEM lane quadrant warp & 3 (the one it may read),
                // accumulator (ew >> 2) & 1, column part ew >> 3
                const int ew = warp - 2;
                const int q = warp & 3;
                const int mt = (ew >> 2) & 1;
                const int row = m0 + mt * 128 + q * 32 + lane;
                const uint32_t tbase = tmem + mt * BN + ((uint32_t)(q * 32) << 16);
                const int cbeg = (ew >> 3) * (BN / RUN_PARTS);
#pragma unroll 1
                for (int cc = cbeg; cc < cbeg + BN / RUN_PARTS; cc += 16) {
                    uint32_t r[16];
                    tmem_ld16(tbase + cc, r);
                    tmem_ld_wait();
                    const int col = c0 + cc;
                    if (row < M && col < n_out) {
                        float v[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] = __uint_as_float(r[e]);
                        store_out<D>(out, row, n_out, col, v, 16, bias, !BWD);
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
        bool have = false;
        if (warp >= 2) {
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
            if (warp >= 2 && have) {
                const int ew = warp - 2;
                const int q = warp & 3, mt = (ew >> 2) & 1;
                const int lrow = mt * 128 + q * 32 + lane;
                const uint32_t tbase = tmem + mt * BN + ((uint32_t)(q * 32) << 16);
                const int cbeg = (ew >> 3) * (RED_CW / RUN_PARTS);
#pragma unroll
                for (int cc = cbeg; cc < cbeg + RED_CW / RUN_PARTS; cc += 16) {
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
            if (warp >= 2) {
                const int e0 = threadIdx.x - 64;
                for (int v = e0; v < rows_per * (RED_CW / 4); v += NUM_DQ_WARPS * 32) {
                    const int lr = z * rows_per + v / (RED_CW / 4);
                    const int c4 = (v % (RED_CW / 4)) * 4;
                    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                    const uint32_t la = stg_addr + (uint32_t)(lr * RED_PITCH + c4) * 4;
                    for (int q2 = 0; q2 < C; ++q2) {
                        const float4 p = ld_dsmem_f4(la, (uint32_t)q2);
                        acc.x += p.x; acc.y += p.y; acc.z += p.z; acc.w += p.w;
                    }
                    const int row = m0 + lr, col = c0 + cb + c4;
                    if (row < M && col < n_out) {
                        const float vv[4] = {acc.x, acc.y, acc.z, acc.w};
                        store_out<D>(out, row, n_out, col, vv, 4, bias, !BWD);
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

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

template <typename D, bool BWD, int BN>
cudaError_t launch_bn(const CUtensorMap &map, const uint8_t *W, const float *absmax,
                      const void *bias, void *out, int M, int N, int K, int log2B,
                      const CodeTable &tab, int C, cudaStream_t stream) {
    const size_t smem = sizeof(Smem) + 1024;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<D, BWD, BN>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    const int n_out = BWD ? K : N;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((n_out + BN - 1) / BN, (M + BM - 1) / BM, C);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = C;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<D, BWD, BN>, map, W, absmax,
                              static_cast<const uint16_t *>(bias), static_cast<uint16_t *>(out), M,
                              N, K, log2B, tab);
}

// fraction of the SM slots that the last wave of `tiles` one-SM CTAs leaves busy
double wave_eff(long tiles, int sms) {
    const long waves = (tiles + sms - 1) / sms;
    return (double)tiles / (double)(waves * sms);
}

template <typename D, bool BWD>
cudaError_t launch_t(const void *A, const uint8_t *W, const float *absmax, const void *bias,
                     void *out, int M, int N, int K, int log2B, const CodeTable &tab,
                     cudaStream_t stream) {
    auto encode = get_encode();
    if (!encode) return cudaErrorNotSupported;
    const int red = BWD ? N : K;
    const int n_out = BWD ? K : N;
    // A: [M rows, red columns] row-major; TMA needs a 16-byte row pitch
    if ((red * 2) % 16 != 0) return cudaErrorInvalidValue;
    CUtensorMap map;
    cuuint64_t dims[2] = {(cuuint64_t)red, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)red * 2};
    cuuint32_t box[2] = {BK, 128};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(&map, std::is_same<D, BF16>::value ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                           : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                        2, const_cast<void *>(A), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;

    const int sms = device_sm_count();
    const long mt = (M + BM - 1) / BM;
    // tile width: 224 when it fills the SMs better (forward only; the backward's
    // MN-major weight tile is built from 64-column atoms)
    int bn = 256;
    if (!BWD && wave_eff(mt * ((n_out + 223) / 224), sms) > wave_eff(mt * ((n_out + 255) / 256), sms) + 0.02)
        bn = 224;
    const long tiles = mt * ((n_out + bn - 1) / bn);
    // split the reduction over a cluster when the tiles alone leave SMs idle
    // and every CTA keeps at least 16 stages
    const int iters = (red + BK - 1) / BK;
    int C = 1;
    while (C < 8 && tiles * (2 * C) <= sms && iters / (2 * C) >= 16) C *= 2;
    if constexpr (!BWD) {
        if (bn == 224)
            return launch_bn<D, BWD, 224>(map, W, absmax, bias, out, M, N, K, log2B, tab, C, stream);
    }
    return launch_bn<D, BWD, 256>(map, W, absmax, bias, out, M, N, K, log2B, tab, C, stream);
}

}  // namespace

cudaError_t launch_gemm_tc(const void *A, const uint8_t *W, const float *absmax, const void *bias,
                           void *D, int64_t M, int64_t N, int64_t K, int blocksize,
                           bnb4_quant_type qt, bnb4_dtype dt, bool backward, cudaStream_t stream) {
    static const CodeTable nf4 = host_code_table(BNB4_NF4);
    static const CodeTable fp4 = host_code_table(BNB4_FP4);
    const CodeTable &tab = qt == BNB4_NF4 ? nf4 : fp4;
    const int log2B = ilog2(blocksize);
    const int m = (int)M, n = (int)N, k = (int)K;
    if (dt == BNB4_F16)
        return backward ? launch_t<F16, true>(A, W, absmax, bias, D, m, n, k, log2B, tab, stream)
                        : launch_t<F16, false>(A, W, absmax, bias, D, m, n, k, log2B, tab, stream);
    return backward ? launch_t<BF16, true>(A, W, absmax, bias, D, m, n, k, log2B, tab, stream)
                    : launch_t<BF16, false>(A, W, absmax, bias, D, m, n, k, log2B, tab, stream);
}

}  // namespace bnb4
