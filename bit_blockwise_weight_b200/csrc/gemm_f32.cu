// gemm_f32.cu -- the 4-bit matmuls in fp32: x, bias and y in float32, and the
// weight a product meets is the exact fp32 dequantized value RN32(code *
// absmax) ("Feat/mps gemm 4bit bf16", Performance: gemv_4bit is measured
// across fp16, bf16 and fp32).  Products and sums are fp32 FMAs on the CUDA
// cores: the tensor cores' fp32 input path (tf32) keeps 10 mantissa bits,
// which this dtype's accuracy rules out.
//
//   gemv_f32_kernel   M == 1.  CTA c owns rows [N c / G, N (c+1) / G) and all
//                     of K; its work is a list of units (a quad of rows x 1024
//                     weights of K), quad major, split into contiguous,
//                     balanced ranges, one per warp.  Lane l holds 32
//                     consecutive weights of each row of the unit (16-byte
//                     loads, one group of loads ahead of the arithmetic) and
//                     the matching 32 values of x, read once from shared
//                     memory for the four rows.  Each code comes from a
//                     16-entry table replicated once per bank (conflict-free),
//                     is multiplied by its block's absmax (the exact fp32
//                     weight) and accumulated with an FMA.  Row sums are
//                     reduced across lanes when a warp leaves a quad; quads
//                     that two warps share are added in warp order, so the
//                     result is the same bits on every run.
//   gemm_f32_smallm_kernel  2 <= M <= 16, forward (below).
//   gemm_f32_kernel   M > 16 and the backward.  A classic shared-memory tiled
//                     product: BM x 64 output tiles, 64-wide reduction steps;
//                     the step's weight tile is dequantized into shared memory
//                     as fp32 (transposed for the forward, as stored for the
//                     backward), the activations tile is staged beside it,
//                     and each thread accumulates a 4 x 4 block of outputs
//                     (256 threads per 64-row tile, 64 per 16-row tile).
//
// No global scratch.
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace bnb4 {

namespace {

// ------------------------------------------------------------------ gemv

constexpr int kVWarps = 16;
constexpr int kVThreads = kVWarps * 32;
constexpr int kVUnitK = 1024;                 // weights per row per unit (32 lanes x 32)
constexpr int kVMaxRows = 1024;               // rows per CTA
constexpr int kVMaxK = 32768;

__device__ __forceinline__ uint4 ldg_nc16(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// the value of `v` held by lane (lane_bits & 31)
__device__ __forceinline__ uint32_t shfl_idx(uint32_t v, uint32_t lane_bits) {
    uint32_t r;
    asm volatile("shfl.sync.idx.b32 %0, %1, %2, 0x1f, 0xffffffff;" : "=r"(r) : "r"(v), "r"(lane_bits));
    return r;
}

__global__ void __launch_bounds__(kVThreads, 1)
gemv_f32_kernel(const float *__restrict__ x, const uint8_t *__restrict__ W, const float *__restrict__ absmax,
                const float *__restrict__ bias, float *__restrict__ y, int N, int K, int log2B,
                const __grid_constant__ CodeTable tab) {
    extern __shared__ __align__(16) float vsm[];
    float *code = vsm;                                 // [16][32]: entry e, copy l at 32 e + l
    float *rowsum = code + 16 * 32;                    // [kVMaxRows]
    float *part = rowsum + kVMaxRows;                  // [kVWarps][2][4]
    float *xs = part + kVWarps * 8;                    // [K rounded up to kVUnitK]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = gridDim.x;
    const int r0 = (int)(((int64_t)N * blockIdx.x) / G);
    const int r1 = (int)(((int64_t)N * (blockIdx.x + 1)) / G);
    const int R = r1 - r0;
    const int NQ = (R + 3) >> 2;
    const int S = (K + kVUnitK - 1) / kVUnitK;         // units per quad
    const int GU = NQ * S;
    const int u_lo = (int)(((int64_t)GU * warp) / kVWarps);
    const int u_hi = (int)(((int64_t)GU * (warp + 1)) / kVWarps);
    const int64_t row_bytes = K >> 1;
    const int nblk = K >> log2B;

    for (int i = tid; i < 16 * 32; i += kVThreads) code[i] = tab.v[i >> 5];
    const int Kp = S * kVUnitK;
    for (int i = tid; i < Kp / 4; i += kVThreads)
        reinterpret_cast<float4 *>(xs)[i] = 4 * i < K ? __ldg(reinterpret_cast<const float4 *>(x) + i)
                                                      : make_float4(0.f, 0.f, 0.f, 0.f);

    // the lane's 32 weights of each row of unit (q, s): rows past the CTA's
    // last row are clamped to it (their sums are never stored), weights past
    // K are clamped in place (they meet zeros of x)
    struct Rows {
        uint4 w[4];
        float a[4];
    };
    auto load = [&](int u, Rows &rw) {
        const int q = u / S, s = u - q * S;
        const int k = min(s * kVUnitK + 32 * lane, K - 32);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int rl = min(4 * q + r, R - 1);
            const int64_t row = r0 + rl;
            rw.w[r] = ldg_nc16(W + row * row_bytes + (k >> 1));
            rw.a[r] = __ldg(absmax + row * nblk + (k >> log2B));
        }
    };

    Rows cur, nxt;
    if (u_lo < u_hi) load(u_lo, cur);
    __syncthreads();

    const int q_first = u_lo < u_hi ? u_lo / S : -1;
    const int q_last = u_lo < u_hi ? (u_hi - 1) / S : -1;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int u = u_lo; u < u_hi; ++u) {
        if (u + 1 < u_hi) load(u + 1, nxt);
        const int q = u / S, s = u - q * S;
        const int k = s * kVUnitK + 32 * lane;
        float xv[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 v = reinterpret_cast<const float4 *>(xs + k)[i];
            xv[4 * i] = v.x;
            xv[4 * i + 1] = v.y;
            xv[4 * i + 2] = v.z;
            xv[4 * i + 3] = v.w;
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const uint32_t w4[4] = {cur.w[r].x, cur.w[r].y, cur.w[r].z, cur.w[r].w};
            float sacc = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint32_t b = (w4[i >> 2] >> (8 * (i & 3))) & 255u;
                // first element of the byte in its high nibble; the exact weight RN32(code * absmax)
                const float w0 = __fmul_rn(code[((b >> 4) << 5) + lane], cur.a[r]);
                const float w1 = __fmul_rn(code[((b & 15u) << 5) + lane], cur.a[r]);
                sacc = __fmaf_rn(xv[2 * i], w0, sacc);
                sacc = __fmaf_rn(xv[2 * i + 1], w1, sacc);
            }
            acc[r] += sacc;
        }
        if (u + 1 == u_hi || (u + 1) / S != q) {
            // reduce the 4 row sums over the 32 lanes: halve over bits 4 and 3,
            // then plain sums over bits 2, 1, 0; lanes 0, 8, 16, 24 end with rows 0..3
            const bool b4 = (lane & 16) != 0, b3 = (lane & 8) != 0;
            float k0 = b4 ? acc[2] : acc[0], k1 = b4 ? acc[3] : acc[1];
            k0 += __shfl_xor_sync(FULL, b4 ? acc[0] : acc[2], 16);
            k1 += __shfl_xor_sync(FULL, b4 ? acc[1] : acc[3], 16);
            float v = b3 ? k1 : k0;
            v += __shfl_xor_sync(FULL, b3 ? k0 : k1, 8);
            v += __shfl_xor_sync(FULL, v, 4);
            v += __shfl_xor_sync(FULL, v, 2);
            v += __shfl_xor_sync(FULL, v, 1);
            if ((lane & 7) == 0) {
                const int rr = 2 * (int)b4 + (int)b3;
                if (q == q_first) part[warp * 8 + rr] = v;
                else if (q == q_last) part[warp * 8 + 4 + rr] = v;
                else if (4 * q + rr < R) rowsum[4 * q + rr] = v;
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) acc[r] = 0.f;
        }
        if (u + 1 < u_hi) cur = nxt;
    }
    __syncthreads();
    for (int r = tid; r < R; r += kVThreads) {
        const int q = r >> 2, rr = r & 3, ul = q * S, uh = ul + S;
        const int w0 = (kVWarps * (ul + 1) + GU - 1) / GU - 1, w1 = (kVWarps * uh + GU - 1) / GU - 1;
        float v = 0.f;
        for (int w = w0; w <= w1; ++w) {
            const int lo = (int)(((int64_t)GU * w) / kVWarps), hi = (int)(((int64_t)GU * (w + 1)) / kVWarps);
            if (lo >= hi) continue;
            v += lo >= ul ? part[w * 8 + rr] : hi - 1 < uh ? part[w * 8 + 4 + rr] : rowsum[r];
        }
        if (bias) v += bias[r0 + r];
        y[r0 + r] = v;
    }
}

// -------------------------------------------------------------- tiled gemm

constexpr int kBN = 64;   // output columns per tile (weight rows forward, K columns backward)
constexpr int kBK = 64;   // reduction step

// cluster barrier and a load from another CTA's shared memory (split reduction)
__device__ __forceinline__ void cluster_barrier() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t local_addr, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}

// BWD == false: Y[m, n] = sum_k A[m, k] W[n, k] (+ bias[n]), A = X [M, K], tile over (m, n), step over k.
// BWD == true:  Y[m, k] = sum_n A[m, n] W[n, k], A = dY [M, N], tile over (m, k), step over n.
// Every thread accumulates a 4 x 4 block (4 m x 4 output columns): per
// reduction index two 16-byte shared loads feed 16 FMAs.  BM = 64 uses 256
// threads per tile, BM = 16 (M <= 16) 64, several tiles per SM.  With
// gridDim.z = S > 1 the S CTAs of a cluster split the reduction steps; their
// partial tiles meet in shared memory and are added in rank order (the same
// bits on every run), each rank storing a share of the tile's rows.
template <int BM, bool BWD>
__global__ void __launch_bounds__(BM * 4)
gemm_f32_kernel(const float *__restrict__ A, const uint8_t *__restrict__ W, const float *__restrict__ absmax,
                const float *__restrict__ bias, float *__restrict__ Y, int M, int N, int K, int log2B,
                const __grid_constant__ CodeTable tab) {
    constexpr int TM = 4;                          // outputs per thread along m
    constexpr int kGThreads = BM * 4;              // 16 column groups x BM / 4 row groups
    __shared__ __align__(16) float As[kBK][BM + 4];     // [reduction][m]
    __shared__ __align__(16) float Bs[kBK][kBN + 4];    // [reduction][output column]
    __shared__ float code[16];
    const int tid = threadIdx.x;
    if (tid < 16) code[tid] = tab.v[tid];
    const int m0 = blockIdx.y * BM;
    const int c0 = blockIdx.x * kBN;               // first output column of the tile
    const int ncols = BWD ? K : N;                 // output columns
    const int red = BWD ? N : K;                   // reduction length
    const int tx = tid & 15, ty = tid >> 4;        // columns 4 tx .. 4 tx + 3, rows TM ty .. TM ty + 3
    const int64_t row_bytes = K >> 1;
    const int nblk = K >> log2B;
    float acc[TM][4];
#pragma unroll
    for (int i = 0; i < TM; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    __syncthreads();

    const int S = gridDim.z, z = blockIdx.z;
    const int nsteps = (red + kBK - 1) / kBK;
    const int st_lo = (int)(((int64_t)nsteps * z) / S), st_hi = (int)(((int64_t)nsteps * (z + 1)) / S);
    for (int r0 = st_lo * kBK; r0 < st_hi * kBK; r0 += kBK) {
        // activations: A[m0 + i][r0 + j] -> As[j][i], zeros outside
        for (int e = tid; e < BM * kBK; e += kGThreads) {
            const int i = e / kBK, j = e % kBK;
            const int m = m0 + i, r = r0 + j;
            As[j][i] = (m < M && r < red) ? A[(int64_t)m * red + r] : 0.f;
        }
        // weight tile: 64 weight rows x 64 weights, in pieces of (row, 16 weights)
        for (int pc = tid; pc < 256; pc += kGThreads) {
            const int lr = pc >> 2, part = pc & 3;     // tile row, quarter of the 64 weights
            int wrow, wk;                               // weight row and first k of this thread's 16
            if (!BWD) { wrow = c0 + lr; wk = r0 + 16 * part; }
            else { wrow = r0 + lr; wk = c0 + 16 * part; }
            float v[16];
            if (wrow < N && wk < K) {
                const uint2 p = __ldg(reinterpret_cast<const uint2 *>(W + (int64_t)wrow * row_bytes + (wk >> 1)));
                const float a = __ldg(absmax + (int64_t)wrow * nblk + (wk >> log2B));
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint32_t b = ((i < 4 ? p.x : p.y) >> (8 * (i & 3))) & 255u;
                    v[2 * i] = __fmul_rn(code[b >> 4], a);
                    v[2 * i + 1] = __fmul_rn(code[b & 15u], a);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = 0.f;
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                if (!BWD) Bs[16 * part + i][lr] = v[i];       // [k][n]
                else Bs[lr][16 * part + i] = v[i];            // [n][k]
            }
        }
        __syncthreads();
#pragma unroll 8
        for (int j = 0; j < kBK; ++j) {
            const float4 aq = *reinterpret_cast<const float4 *>(&As[j][TM * ty]);
            const float a[TM] = {aq.x, aq.y, aq.z, aq.w};
            const float4 bq = *reinterpret_cast<const float4 *>(&Bs[j][4 * tx]);
            const float b[4] = {bq.x, bq.y, bq.z, bq.w};
#pragma unroll
            for (int i = 0; i < TM; ++i)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[i][c] = __fmaf_rn(a[i], b[c], acc[i][c]);
        }
        __syncthreads();
    }
    if (S == 1) {
#pragma unroll
        for (int i = 0; i < TM; ++i) {
            const int m = m0 + TM * ty + i;
            if (m >= M) continue;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int col = c0 + 4 * tx + c;
                if (col >= ncols) continue;
                float v = acc[i][c];
                if (!BWD && bias) v += bias[col];
                Y[(int64_t)m * ncols + col] = v;
            }
        }
        return;
    }
    // split: this CTA's partial tile [BM][kBN] in the (now idle) A tile, then
    // rank z adds rows [BM z / S, BM (z+1) / S) over the ranks in order
    static_assert(BM * kBN <= kBK * (BM + 4), "partial tile fits in the A tile");
    float *Ps = &As[0][0];
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) Ps[(TM * ty + i) * kBN + 4 * tx + c] = acc[i][c];
    cluster_barrier();
    const int rlo = (BM * z) / S, rhi = (BM * (z + 1)) / S;
    const uint32_t ps_addr = (uint32_t)__cvta_generic_to_shared(Ps);
    for (int e = tid; e < (rhi - rlo) * kBN; e += kGThreads) {
        const int lr = rlo + e / kBN, lc = e % kBN;
        const uint32_t la = ps_addr + (uint32_t)(lr * kBN + lc) * 4u;
        float v = 0.f;
        for (int q = 0; q < S; ++q) v += ld_cluster_f32(la, (uint32_t)q);
        const int m = m0 + lr, col = c0 + lc;
        if (m < M && col < ncols) {
            if (!BWD && bias) v += bias[col];
            Y[(int64_t)m * ncols + col] = v;
        }
    }
    cluster_barrier();  // no CTA leaves while its partial tile may still be read
}

// ------------------------------------------------- small M, forward
//
// M <= 16 (rows padded to MT): every weight is decoded once and meets all MT
// rows of x in registers, and all lanes of a warp step through K together, so
// each x value is one broadcast shared-memory read.  A CTA owns 128 TN weight
// rows (thread i rows t * 128 + i, t < TN).  Per step of 128 weights the CTA
// copies 64 contiguous bytes of each of its rows into shared memory
// (asynchronous 16-byte copies, four threads per row) together with the
// step's x, one step ahead of the arithmetic; a thread then reads its rows 16
// bytes (32 weights) at a time (rows padded to 80 bytes: the reads of 8 lanes
// fall in distinct banks), takes each code by a shuffle from a lane-held table
// and multiplies it by the block's absmax (the exact fp32 weight).  56 KB of
// shared memory leaves room for 4 CTAs per SM (measured on B200: 128-weight
// steps beat 256-weight ones, which hold only 2).  With gridDim.z = S > 1 the
// S CTAs of a cluster split K and add their partial tiles in rank order; S is
// chosen for the fewest waves per unit of work.
constexpr int kSMThreads = 128;
constexpr int kSMStep = 128;                  // weights of a row per step
constexpr int kSMRowPitch = kSMStep / 2 + 16; // bytes per staged row (padded by 16)
constexpr int kSMPieces = kSMStep / 32;       // 16-byte pieces per row per step

__host__ __device__ constexpr size_t sm_w_bytes(int TN) { return (size_t)kSMThreads * TN * kSMRowPitch; }
__host__ __device__ constexpr size_t sm_x_bytes(int MT) { return (size_t)kSMStep * MT * sizeof(float); }
__host__ __device__ constexpr size_t sm_smem(int MT, int TN) { return 2 * (sm_w_bytes(TN) + sm_x_bytes(MT)); }

__device__ __forceinline__ void cp_async4(uint32_t dst, const float *src, bool valid) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(valid ? 4 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}

template <int MT, int TN>
__global__ void __launch_bounds__(kSMThreads)
gemm_f32_smallm_kernel(const float *__restrict__ X, const uint8_t *__restrict__ W, const float *__restrict__ absmax,
                       const float *__restrict__ bias, float *__restrict__ Y, int M, int N, int K, int log2B,
                       const __grid_constant__ CodeTable tab) {
    static_assert(MT % 4 == 0 && MT <= 16, "rows in float4 groups");
    constexpr int kRows = kSMThreads * TN;        // weight rows (output columns) per CTA
    static_assert(MT * kRows * sizeof(float) <= sm_smem(MT, TN), "partial tile fits in the buffers");
    // [2] weight stages [kRows][kSMRowPitch], then [2] x stages [kSMStep][MT];
    // the partial tile at the end
    extern __shared__ __align__(16) uint8_t smb[];
    const uint32_t sm_a = (uint32_t)__cvta_generic_to_shared(smb);
    const uint32_t w_a = sm_a, x_a = sm_a + 2 * (uint32_t)sm_w_bytes(TN);
    const float *xsm = reinterpret_cast<const float *>(smb + 2 * sm_w_bytes(TN));
    const int tid = threadIdx.x, lane = tid & 31;
    const uint32_t my_code = __float_as_uint(tab.v[lane & 15]);
    const int c0 = blockIdx.x * kRows;
    const int S = gridDim.z, z = blockIdx.z;
    const int n64 = K / 64;                       // K is a multiple of the blocksize (>= 64)
    const int k_lo = (int)(((int64_t)n64 * z) / S) * 64;
    const int k_hi = (int)(((int64_t)n64 * (z + 1)) / S) * 64;
    const int64_t row_bytes = K >> 1;
    const int nblk = K >> log2B;
    const float *arow[TN];
#pragma unroll
    for (int t = 0; t < TN; ++t) arow[t] = absmax + (int64_t)min(c0 + t * kSMThreads + tid, N - 1) * nblk;
    float acc[MT][TN];
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int t = 0; t < TN; ++t) acc[m][t] = 0.f;

    // one step's weights (the CTA's rows, 16-byte pieces of [kb, kb + kn)) and
    // x (x[m][kb + kk] -> [kk][m], zeros past M and past kn); rows past N are
    // clamped to the last one (their sums are never stored)
    auto stage = [&](int kb, int buf) {
        const int kn = min(kSMStep, k_hi - kb);
        const int pieces = kn / 32;               // 16-byte pieces per row
        for (int c = tid; c < kRows * kSMPieces; c += kSMThreads) {
            const int r = c / kSMPieces, pc = c % kSMPieces;
            if (pc < pieces) {
                const int n = min(c0 + r, N - 1);
                cp_async16(w_a + (uint32_t)(buf * sm_w_bytes(TN) + r * kSMRowPitch + 16 * pc),
                           W + (int64_t)n * row_bytes + (kb >> 1) + 16 * pc);
            }
        }
        for (int e = tid; e < MT * kSMStep; e += kSMThreads) {
            const int m = e / kSMStep, kk = e % kSMStep;
            const bool valid = m < M && kk < kn;
            cp_async4(x_a + (uint32_t)(buf * sm_x_bytes(MT) + (kk * MT + m) * sizeof(float)),
                      valid ? X + (int64_t)m * K + kb + kk : X, valid);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    if (k_lo < k_hi) stage(k_lo, 0);
    int buf = 0;
    for (int kb = k_lo; kb < k_hi; kb += kSMStep) {
        if (kb + kSMStep < k_hi) {
            stage(kb + kSMStep, buf ^ 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();  // every thread's copies of this step have landed
        const int pieces = min(kSMStep, k_hi - kb) / 32;
        const uint32_t wrow0 = w_a + (uint32_t)(buf * sm_w_bytes(TN) + tid * kSMRowPitch);
        const float *xs = xsm + buf * (sm_x_bytes(MT) / sizeof(float));
        for (int pc = 0; pc < pieces; ++pc) {
            uint4 w[TN];
            float a[TN];
#pragma unroll
            for (int t = 0; t < TN; ++t) {
                w[t] = lds128(wrow0 + (uint32_t)(t * kSMThreads * kSMRowPitch + 16 * pc));
                a[t] = __ldg(arow[t] + ((kb + 32 * pc) >> log2B));
            }
            // byte j holds reduction indices 2j (high nibble) and 2j + 1
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                float wv[2][TN];
#pragma unroll
                for (int t = 0; t < TN; ++t) {
                    const uint32_t wd = (j >> 2) == 0 ? w[t].x : (j >> 2) == 1 ? w[t].y : (j >> 2) == 2 ? w[t].z : w[t].w;
                    const int sh = 8 * (j & 3);
                    // the shuffle reads lane (index & 31); lanes 16..31 repeat the table
                    wv[0][t] = __fmul_rn(__uint_as_float(shfl_idx(my_code, wd >> (sh + 4))), a[t]);
                    wv[1][t] = __fmul_rn(__uint_as_float(shfl_idx(my_code, wd >> sh)), a[t]);
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float *xr = xs + (32 * pc + 2 * j + h) * MT;
#pragma unroll
                    for (int q = 0; q < MT / 4; ++q) {
                        const float4 xv = *reinterpret_cast<const float4 *>(xr + 4 * q);
#pragma unroll
                        for (int t = 0; t < TN; ++t) {
                            acc[4 * q][t] = __fmaf_rn(xv.x, wv[h][t], acc[4 * q][t]);
                            acc[4 * q + 1][t] = __fmaf_rn(xv.y, wv[h][t], acc[4 * q + 1][t]);
                            acc[4 * q + 2][t] = __fmaf_rn(xv.z, wv[h][t], acc[4 * q + 2][t]);
                            acc[4 * q + 3][t] = __fmaf_rn(xv.w, wv[h][t], acc[4 * q + 3][t]);
                        }
                    }
                }
            }
        }
        __syncthreads();  // this buffer is free for the step after next
        buf ^= 1;
    }
    if (S == 1) {
#pragma unroll
        for (int t = 0; t < TN; ++t) {
            const int n = c0 + t * kSMThreads + tid;
            if (n >= N) continue;
            const float bv = bias ? bias[n] : 0.f;
#pragma unroll
            for (int m = 0; m < MT; ++m)
                if (m < M) Y[(int64_t)m * N + n] = bias ? acc[m][t] + bv : acc[m][t];
        }
        return;
    }
    // split: the partial tile [MT][kRows] in the buffers (idle since the last
    // barrier), then rank z adds rows [MT z / S, MT (z+1) / S) over the ranks
    // in order
    float *ps = reinterpret_cast<float *>(smb);
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int t = 0; t < TN; ++t) ps[m * kRows + t * kSMThreads + tid] = acc[m][t];
    cluster_barrier();
    const int rlo = (MT * z) / S, rhi = (MT * (z + 1)) / S;
    for (int e = tid; e < (rhi - rlo) * kRows; e += kSMThreads) {
        const int m = rlo + e / kRows, col = e % kRows, n = c0 + col;
        const uint32_t la = sm_a + (uint32_t)(m * kRows + col) * 4u;
        float v = 0.f;
        for (int q = 0; q < S; ++q) v += ld_cluster_f32(la, (uint32_t)q);
        if (m < M && n < N) Y[(int64_t)m * N + n] = bias ? v + bias[n] : v;
    }
    cluster_barrier();  // no CTA leaves while its partial tile may still be read
}

template <int MT, int TN>
cudaError_t launch_smallm(const float *A, const uint8_t *W, const float *absmax, const float *bias, float *Y, int M,
                          int N, int K, int log2B, const CodeTable &tab, cudaStream_t stream) {
    const int SMs = device_sm_count();
    constexpr int kRows = kSMThreads * TN;
    constexpr size_t smem = sm_smem(MT, TN);
    static std::atomic<bool> set[kMaxDevices];
    cudaError_t e = once_per_device(set, [] {
        return cudaFuncSetAttribute(gemm_f32_smallm_kernel<MT, TN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)smem);
    });
    if (e != cudaSuccess) return e;
    const int tiles = (N + kRows - 1) / kRows;
    static std::atomic<int> occ_cache[kMaxDevices];
    const int per_sm = cached_per_device(occ_cache, [] {
        int v = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, gemm_f32_smallm_kernel<MT, TN>, kSMThreads, smem) !=
                cudaSuccess || v < 1) {
            (void)cudaGetLastError();
            v = 1;
        }
        return v;
    });
    const int64_t slots = (int64_t)SMs * per_sm;
    // the split (a cluster of at most 8, at least 4 steps each) with the
    // fewest waves per unit of work: waves(S) / S, ties to the smaller S
    int S = 1;
    double best = 1e30;
    for (int s = 1; s <= 8; ++s) {
        if (s > 1 && K / (kSMStep * s) < 4) break;
        const double cost = (double)((tiles * (int64_t)s + slots - 1) / slots) / s;
        if (cost < best - 1e-9) {
            best = cost;
            S = s;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(tiles, 1, S);
    cfg.blockDim = dim3(kSMThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = S;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemm_f32_smallm_kernel<MT, TN>, A, W, absmax, bias, Y, M, N, K, log2B, tab);
}

size_t gemv_f32_smem(int K) {
    const size_t Kp = ((size_t)K + kVUnitK - 1) / kVUnitK * kVUnitK;
    return (16 * 32 + kVMaxRows + kVWarps * 8 + Kp) * sizeof(float);
}

}  // namespace

int64_t gemv_f32_max_rows() { return (int64_t)device_sm_count() * kVMaxRows; }
int64_t gemv_f32_max_k() { return kVMaxK; }

cudaError_t launch_gemv_f32(const float *x, const uint8_t *W, const float *absmax, const float *bias, float *y,
                            int64_t N, int64_t K, int blocksize, bnb4_quant_type qt, cudaStream_t stream) {
    static const CodeTable nf4 = host_code_table(BNB4_NF4);
    static const CodeTable fp4 = host_code_table(BNB4_FP4);
    const CodeTable &tab = qt == BNB4_NF4 ? nf4 : fp4;
    static std::atomic<bool> set[kMaxDevices];
    cudaError_t e = once_per_device(set, [] {
        return cudaFuncSetAttribute(gemv_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)gemv_f32_smem(kVMaxK));
    });
    if (e != cudaSuccess) return e;
    gemv_f32_kernel<<<device_sm_count(), kVThreads, gemv_f32_smem((int)K), stream>>>(
        x, W, absmax, bias, y, (int)N, (int)K, ilog2(blocksize), tab);
    return cudaGetLastError();
}

cudaError_t launch_gemm_f32(const float *A, const uint8_t *W, const float *absmax, const float *bias, float *Y,
                            int64_t M, int64_t N, int64_t K, int blocksize, bnb4_quant_type qt, bool backward,
                            cudaStream_t stream) {
    static const CodeTable nf4 = host_code_table(BNB4_NF4);
    static const CodeTable fp4 = host_code_table(BNB4_FP4);
    const CodeTable &tab = qt == BNB4_NF4 ? nf4 : fp4;
    if (!backward && M <= 16) {
        const int log2B_ = ilog2(blocksize);
        const int m_ = (int)M, n_ = (int)N, k_ = (int)K;
        if (M <= 4) return launch_smallm<4, 2>(A, W, absmax, bias, Y, m_, n_, k_, log2B_, tab, stream);
        if (M <= 8) return launch_smallm<8, 2>(A, W, absmax, bias, Y, m_, n_, k_, log2B_, tab, stream);
        return launch_smallm<16, 2>(A, W, absmax, bias, Y, m_, n_, k_, log2B_, tab, stream);
    }
    const int ncols = (int)(backward ? K : N);
    const int log2B = ilog2(blocksize);
    // reduction split S (a cluster of S CTAs along z): enough CTAs for about
    // 4 per SM, at least 8 reduction steps each, S a power of two up to 8
    const int BM = M <= 16 ? 16 : 64;
    const int64_t tiles = (int64_t)((ncols + kBN - 1) / kBN) * ((M + BM - 1) / BM);
    const int nsteps = (int)((backward ? N : K) + kBK - 1) / kBK;
    int S = 1;
    while (S < 8 && tiles * S < 4LL * device_sm_count() && nsteps / (2 * S) >= 8) S *= 2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((ncols + kBN - 1) / kBN, (unsigned)((M + BM - 1) / BM), S);
    cfg.blockDim = dim3(BM * 4, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = S;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const int m = (int)M, n = (int)N, k = (int)K;
    if (BM == 16) {
        if (backward) return cudaLaunchKernelEx(&cfg, gemm_f32_kernel<16, true>, A, W, absmax, (const float *)nullptr, Y, m, n, k, log2B, tab);
        return cudaLaunchKernelEx(&cfg, gemm_f32_kernel<16, false>, A, W, absmax, bias, Y, m, n, k, log2B, tab);
    }
    if (backward) return cudaLaunchKernelEx(&cfg, gemm_f32_kernel<64, true>, A, W, absmax, (const float *)nullptr, Y, m, n, k, log2B, tab);
    return cudaLaunchKernelEx(&cfg, gemm_f32_kernel<64, false>, A, W, absmax, bias, Y, m, n, k, log2B, tab);
}

}  // namespace bnb4
