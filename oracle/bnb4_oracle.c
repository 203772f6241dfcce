/*
 * bnb4_oracle.c -- plain CPU oracle for 4-bit blockwise quantization and the
 * 4-bit matmuls.  TEST INFRASTRUCTURE ONLY (see bnb4_oracle.h): the product
 * library never links it.
 *
 * Build: cc -O1 -std=c11 -fno-fast-math -ffp-contract=off -shared -fPIC.
 * Contraction is disabled so that every float operation below is the single
 * IEEE operation it is written as.
 *
 * Readings of the pages where they are silent (each one is also listed in the
 * design notes):
 *   R1 NF4 values: the 16 decimal literals given with the 4096x4096 gemv
 *      workload, each rounded to the nearest fp32 (the pages only name NF4:
 *      "mps-bitsandbytes 0.4.7", Features table, and the credit to QLoRA).
 *   R2 FP4 values: E2M1 (1 sign, 2 exponent, 1 mantissa bit), exponent bias 1
 *      with subnormals, magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6} divided by 6 so
 *      the largest code is 1; index = s<<3 | e<<1 | m.  The pages define no
 *      FP4 table ("mps-bitsandbytes 0.4.7", Features table, names FP4 only).
 *   R3 absmax of a block is max |x| in fp32; the last block holds n mod B
 *      elements when B does not divide n.
 *   R4 normalisation is the IEEE fp32 quotient x / absmax; an all-zero block
 *      (absmax == 0) normalises every element to 0.
 *   R5 nearest code: argmin_i |v - c_i| evaluated in float64, ties go to the
 *      smallest index.  Exact search, never a lookup table ("Feat/mps gemm
 *      4bit bf16", Correctness: the 65536-point LUT snap that missed 1365 of
 *      1,048,576 values).
 *   R6 packing: byte j = idx[2j] << 4 | idx[2j+1] (first element in the high
 *      nibble); an odd tail leaves the low nibble 0.
 *   R7 dequantisation: one fp32 product code * absmax, then one
 *      round-to-nearest-even conversion to the output dtype.
 *   R8 matmul reference: float64 sum over k of x * fp32(code * absmax), plus
 *      bias, with no rounding of the result.
 *   R9 double quantization of absmax (see oracle_double_quant).
 *   R10 8-bit blockwise: steps R3-R5 and R7 with a caller's 256-entry code
 *      table and one code index per byte (see oracle_quantize_8bit); the
 *      nearest entry is decided on exact distances (a caller's table may
 *      hold -c and +c, where float64 distances would tie tiny quotients).
 *   R11 4-bit embedding lookup: rows of a table quantized as one flat array
 *      (see oracle_embedding_4bit).
 */
#include "bnb4_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- tables */

int oracle_code_table(int qtype, float out[16])
{
    if (qtype == ORACLE_NF4) {
        /* R1: decimal literals, rounded to fp32 by the compiler. */
        static const float nf4[16] = {
            -1.0f,       -0.6961928f, -0.5250731f, -0.3949175f,
            -0.2844414f, -0.1848074f, -0.0910500f, 0.0f,
            0.0795803f,  0.1609302f,  0.2461123f,  0.3379152f,
            0.4407098f,  0.5626170f,  0.7229568f,  1.0f};
        memcpy(out, nf4, sizeof(nf4));
        return 0;
    }
    if (qtype == ORACLE_FP4) {
        /* R2: decode the E2M1 bit fields, then scale by 1/6. */
        for (int idx = 0; idx < 16; ++idx) {
            int s = (idx >> 3) & 1, e = (idx >> 1) & 3, m = idx & 1;
            double mag = (e == 0) ? 0.5 * m : (1.0 + 0.5 * m) * ldexp(1.0, e - 1);
            double v = mag / 6.0;
            out[idx] = (float)(s ? -v : v);
        }
        return 0;
    }
    return -1;
}

/* ----------------------------------------------------------- conversions */

float oracle_bf16_to_f32(uint16_t h)
{
    /* bfloat16 is by definition the upper half of an IEEE binary32. */
    uint32_t bits = (uint32_t)h << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return f;
}

float oracle_f16_to_f32(uint16_t h)
{
    int s = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);
    return (float)(s ? -v : v);
}

/* Round a finite double holding an fp32 value to a binary format with p
 * significand bits, minimum normal exponent emin and largest finite value
 * maxf, ties to even.  Returns +-inf on overflow.  All steps are exact
 * power-of-two scalings plus one rint() in the default (nearest-even) mode. */
static double round_to_format(double f, int p, int emin, double maxf)
{
    if (f == 0.0 || isnan(f) || isinf(f))
        return f;
    double a = fabs(f);
    int e;
    frexp(a, &e);
    int lead = e - 1;
    if (lead < emin)
        lead = emin;
    double quantum = ldexp(1.0, lead - (p - 1));
    double r = nearbyint(a / quantum) * quantum;
    if (r > maxf)
        r = INFINITY;
    return f < 0 ? -r : r;
}

static uint16_t encode_format(double r, int mant_bits, int bias, int emin,
                              int exp_all_ones)
{
    uint16_t sign = signbit(r) ? (uint16_t)(1u << 15) : 0;
    if (isnan(r))
        return (uint16_t)(sign | (exp_all_ones << mant_bits) | (1u << (mant_bits - 1)));
    double a = fabs(r);
    if (a == 0.0)
        return sign;
    if (isinf(a))
        return (uint16_t)(sign | (exp_all_ones << mant_bits));
    int e;
    frexp(a, &e);
    int lead = e - 1;
    if (lead < emin) { /* subnormal: integer multiple of the smallest quantum */
        double mant = a / ldexp(1.0, emin - mant_bits);
        return (uint16_t)(sign | (uint16_t)mant);
    }
    double mant = (a / ldexp(1.0, lead) - 1.0) * ldexp(1.0, mant_bits);
    return (uint16_t)(sign | ((uint16_t)(lead + bias) << mant_bits) | (uint16_t)mant);
}

uint16_t oracle_f32_to_f16_rne(float f)
{
    double r = round_to_format((double)f, 11, -14, 65504.0);
    return encode_format(r, 10, 15, -14, 31);
}

uint16_t oracle_f32_to_bf16_rne(float f)
{
    double maxf = ldexp(2.0 - ldexp(1.0, -7), 127);
    double r = round_to_format((double)f, 8, -126, maxf);
    return encode_format(r, 7, 127, -126, 255);
}

static float load_elem(const void *x, int dtype, int64_t i)
{
    switch (dtype) {
    case ORACLE_F32: return ((const float *)x)[i];
    case ORACLE_F16: return oracle_f16_to_f32(((const uint16_t *)x)[i]);
    case ORACLE_BF16: return oracle_bf16_to_f32(((const uint16_t *)x)[i]);
    default: return NAN;
    }
}

static void store_elem(void *out, int dtype, int64_t i, float v)
{
    switch (dtype) {
    case ORACLE_F32: ((float *)out)[i] = v; break;
    case ORACLE_F16: ((uint16_t *)out)[i] = oracle_f32_to_f16_rne(v); break;
    case ORACLE_BF16: ((uint16_t *)out)[i] = oracle_f32_to_bf16_rne(v); break;
    default: break;
    }
}

static int valid_dtype(int d) { return d == ORACLE_F32 || d == ORACLE_F16 || d == ORACLE_BF16; }

int oracle_to_f32_array(const void *in, int dtype, int64_t n, float *out)
{
    if (!valid_dtype(dtype) || n < 0)
        return -1;
    for (int64_t i = 0; i < n; ++i)
        out[i] = load_elem(in, dtype, i);
    return 0;
}

int oracle_from_f32_array(const float *in, int64_t n, int dtype, void *out)
{
    if (!valid_dtype(dtype) || n < 0)
        return -1;
    for (int64_t i = 0; i < n; ++i)
        store_elem(out, dtype, i, in[i]);
    return 0;
}

/* ------------------------------------------------------------- quantize */

/* R5: exact nearest code, ties to the smallest index. */
static int nearest_code(float v, const float code[16])
{
    int best = 0;
    double bd = fabs((double)v - (double)code[0]);
    for (int j = 1; j < 16; ++j) {
        double d = fabs((double)v - (double)code[j]);
        if (d < bd) {
            bd = d;
            best = j;
        }
    }
    return best;
}

int oracle_quantize(const void *x, int dtype, int64_t n, int blocksize,
                    int qtype, uint8_t *packed, float *absmax)
{
    float code[16];
    if (oracle_code_table(qtype, code) != 0 || !valid_dtype(dtype) ||
        blocksize <= 0 || n < 0)
        return -1;
    memset(packed, 0, (size_t)((n + 1) / 2));
    int64_t nblocks = (n + blocksize - 1) / blocksize;
    for (int64_t b = 0; b < nblocks; ++b) {
        int64_t lo = b * blocksize;
        int64_t hi = lo + blocksize < n ? lo + blocksize : n; /* R3 tail */
        /* step 1 (R3): block absmax */
        float amax = 0.0f;
        for (int64_t i = lo; i < hi; ++i) {
            float a = fabsf(load_elem(x, dtype, i));
            if (a > amax)
                amax = a;
        }
        absmax[b] = amax;
        for (int64_t i = lo; i < hi; ++i) {
            /* step 2 (R4): normalise to [-1, 1] */
            float v = (amax == 0.0f) ? 0.0f : load_elem(x, dtype, i) / amax;
            /* step 3 (R5): nearest code */
            int idx = nearest_code(v, code);
            /* step 4 (R6): pack, first element high nibble */
            if ((i & 1) == 0)
                packed[i >> 1] |= (uint8_t)(idx << 4);
            else
                packed[i >> 1] |= (uint8_t)idx;
        }
    }
    return 0;
}

/* ----------------------------------------------------------- dequantize */

static int code_index(const uint8_t *packed, int64_t i)
{
    uint8_t byte = packed[i >> 1];
    return (i & 1) ? (byte & 15) : (byte >> 4);
}

/* R7: one fp32 product. */
static float dequant_f32(const uint8_t *packed, const float *absmax, int64_t i,
                         int blocksize, const float code[16])
{
    float c = code[code_index(packed, i)];
    float a = absmax[i / blocksize];
    float p = c * a;
    return p;
}

int oracle_dequantize(const uint8_t *packed, const float *absmax, int64_t n,
                      int blocksize, int qtype, int out_dtype, void *out)
{
    float code[16];
    if (oracle_code_table(qtype, code) != 0 || !valid_dtype(out_dtype) ||
        blocksize <= 0 || n < 0)
        return -1;
    for (int64_t i = 0; i < n; ++i)
        store_elem(out, out_dtype, i, dequant_f32(packed, absmax, i, blocksize, code));
    return 0;
}

/* --------------------------------------------------------------- matmul */

static int matmul_args_ok(int dtype, int qtype, int blocksize, int64_t M,
                          int64_t N, int64_t K, float code[16])
{
    return oracle_code_table(qtype, code) == 0 && valid_dtype(dtype) &&
           blocksize > 0 && M >= 0 && N >= 0 && K >= 0;
}

/* R8: one output of the forward product; weight row j is the flat range
 * [j*K, (j+1)*K) of the quantized array. */
static double forward_entry(const void *X, int x_dtype, const uint8_t *packed,
                            const float *absmax, const void *bias, int64_t N,
                            int64_t K, int blocksize, const float code[16],
                            int64_t m, int64_t j)
{
    (void)N;
    double acc = 0.0;
    for (int64_t k = 0; k < K; ++k) {
        double xv = (double)load_elem(X, x_dtype, m * K + k);
        double wv = (double)dequant_f32(packed, absmax, j * K + k, blocksize, code);
        acc += xv * wv;
    }
    if (bias)
        acc += (double)load_elem(bias, x_dtype, j);
    return acc;
}

int oracle_matmul(const void *X, int x_dtype, const uint8_t *packed,
                  const float *absmax, const void *bias, int64_t M, int64_t N,
                  int64_t K, int blocksize, int qtype, double *Y)
{
    float code[16];
    if (!matmul_args_ok(x_dtype, qtype, blocksize, M, N, K, code))
        return -1;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t j = 0; j < N; ++j)
            Y[m * N + j] = forward_entry(X, x_dtype, packed, absmax, bias, N, K,
                                         blocksize, code, m, j);
    return 0;
}

int oracle_matmul_entries(const void *X, int x_dtype, const uint8_t *packed,
                          const float *absmax, const void *bias, int64_t M,
                          int64_t N, int64_t K, int blocksize, int qtype,
                          const int64_t *ms, const int64_t *js, int64_t count,
                          double *Y)
{
    float code[16];
    if (!matmul_args_ok(x_dtype, qtype, blocksize, M, N, K, code))
        return -1;
    for (int64_t i = 0; i < count; ++i) {
        if (ms[i] < 0 || ms[i] >= M || js[i] < 0 || js[i] >= N)
            return -1;
        Y[i] = forward_entry(X, x_dtype, packed, absmax, bias, N, K, blocksize,
                             code, ms[i], js[i]);
    }
    return 0;
}

/* The backward product (grad_input = grad_output @ dequantize(W)), one entry. */
static double backward_entry(const void *dY, int dy_dtype, const uint8_t *packed,
                             const float *absmax, int64_t N, int64_t K,
                             int blocksize, const float code[16], int64_t m,
                             int64_t k)
{
    double acc = 0.0;
    for (int64_t j = 0; j < N; ++j) {
        double g = (double)load_elem(dY, dy_dtype, m * N + j);
        double wv = (double)dequant_f32(packed, absmax, j * K + k, blocksize, code);
        acc += g * wv;
    }
    return acc;
}

int oracle_matmul_backward(const void *dY, int dy_dtype, const uint8_t *packed,
                           const float *absmax, int64_t M, int64_t N, int64_t K,
                           int blocksize, int qtype, double *dX)
{
    float code[16];
    if (!matmul_args_ok(dy_dtype, qtype, blocksize, M, N, K, code))
        return -1;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k)
            dX[m * K + k] = backward_entry(dY, dy_dtype, packed, absmax, N, K,
                                           blocksize, code, m, k);
    return 0;
}

int oracle_matmul_backward_entries(const void *dY, int dy_dtype,
                                   const uint8_t *packed, const float *absmax,
                                   int64_t M, int64_t N, int64_t K,
                                   int blocksize, int qtype, const int64_t *ms,
                                   const int64_t *ks, int64_t count, double *dX)
{
    float code[16];
    if (!matmul_args_ok(dy_dtype, qtype, blocksize, M, N, K, code))
        return -1;
    for (int64_t i = 0; i < count; ++i) {
        if (ms[i] < 0 || ms[i] >= M || ks[i] < 0 || ks[i] >= K)
            return -1;
        dX[i] = backward_entry(dY, dy_dtype, packed, absmax, N, K, blocksize,
                               code, ms[i], ks[i]);
    }
    return 0;
}

/* ------------------------------------------------ double quantization (R9) */

int oracle_double_quant(const float *absmax, int64_t n, int group, uint8_t *q,
                        float *scales)
{
    if (group < 1 || n < 0)
        return -1;
    for (int64_t g0 = 0; g0 < n; g0 += group) {
        const int64_t g1 = g0 + group < n ? g0 + group : n;
        float s = 0.0f;
        for (int64_t i = g0; i < g1; ++i)
            if (absmax[i] > s)
                s = absmax[i];
        scales[g0 / group] = s;
        for (int64_t i = g0; i < g1; ++i) {
            uint8_t code = 0;
            if (s > 0.0f) {
                const float v = absmax[i] / s;  /* fp32 quotient */
                const float t = v * 255.0f;     /* fp32 product */
                const float r = rintf(t);       /* ties to even */
                if (r > 0.0f)                   /* NaN and r <= 0 give 0 */
                    code = r >= 255.0f ? (uint8_t)255 : (uint8_t)r;
            }
            q[i] = code;
        }
    }
    return 0;
}

int oracle_dequant_absmax(const uint8_t *q, const float *scales, int64_t n,
                          int group, float *out)
{
    if (group < 1 || n < 0)
        return -1;
    for (int64_t i = 0; i < n; ++i) {
        const float step = scales[i / group] / 255.0f;  /* fp32 quotient */
        out[i] = (float)q[i] * step;                    /* fp32 product */
    }
    return 0;
}

/* ---------------------------------------- 8-bit blockwise quantization (R10) */

/* A caller's table is usable when it is strictly ascending, finite, inside
 * [-1, 1], and every entry is 0 or at least 2^-24 in magnitude.  With the
 * last condition every comparison of |v - c| that can decide an index is
 * exact in float64: a close call sits at a midpoint of two entries, which is
 * then at least 2^-25 in magnitude, and the differences of fp32 values that
 * large span fewer than 53 bits. */
static int code8_usable(const float *code)
{
    for (int j = 0; j < 256; ++j) {
        const float c = code[j];
        if (!(c >= -1.0f && c <= 1.0f))
            return 0;
        if (c != 0.0f && fabsf(c) < 0x1p-24f)
            return 0;
        if (j > 0 && !(code[j - 1] < c))
            return 0;
    }
    return 1;
}

/* |v - c| exactly, as hi + lo with hi = RN(|v - c|) in float64 and lo the
 * rounding error (Knuth's TwoSum; exact, no underflow for fp32 inputs).  A
 * plain float64 difference is not exact once |v| is below 2^-53 |c|: with a
 * table holding -c and +c (a decision threshold of exactly 0) it would call
 * every tiny v a tie. */
struct dist2 {
    double hi, lo;
};
static struct dist2 exact_distance(float v, float c)
{
    const double a = v, b = -(double)c;
    const double s = a + b, bb = s - a;
    const double err = (a - (s - bb)) + (b - bb);
    struct dist2 d = {s, err};
    if (s < 0.0) {
        d.hi = -s;
        d.lo = -err;
    }
    return d;
}
/* x < y for exact values hi + lo: hi is the rounded value, so hi decides
 * unless the two are equal */
static int dist_less(struct dist2 x, struct dist2 y)
{
    return x.hi < y.hi || (x.hi == y.hi && x.lo < y.lo);
}

/* R10 (as R5): exact nearest of the 256 entries, ties to the smallest index. */
static int nearest_code8(float v, const float *code)
{
    int best_j = 0;
    struct dist2 best_d = exact_distance(v, code[0]);
    for (int j = 1; j < 256; ++j) {
        const struct dist2 dist = exact_distance(v, code[j]);
        if (dist_less(dist, best_d)) {
            best_d = dist;
            best_j = j;
        }
    }
    return best_j;
}

int oracle_quantize_8bit(const void *x, int dtype, int64_t n, int blocksize,
                         const float *code, uint8_t *q, float *absmax)
{
    if (!code8_usable(code) || !valid_dtype(dtype) || blocksize <= 0 || n < 0)
        return -1;
    const int64_t nblocks = (n + blocksize - 1) / blocksize;
    for (int64_t b = 0; b < nblocks; ++b) {
        const int64_t lo = b * blocksize;
        const int64_t hi = lo + blocksize < n ? lo + blocksize : n; /* R3 tail */
        /* step 1 (R3): block absmax */
        float amax = 0.0f;
        for (int64_t i = lo; i < hi; ++i) {
            const float mag = fabsf(load_elem(x, dtype, i));
            if (mag > amax)
                amax = mag;
        }
        absmax[b] = amax;
        for (int64_t i = lo; i < hi; ++i) {
            /* step 2 (R4): normalise */
            const float xi = load_elem(x, dtype, i);
            const float v = (amax == 0.0f) ? 0.0f : xi / amax;
            /* step 3 (R10): nearest entry, one byte per element */
            q[i] = (uint8_t)nearest_code8(v, code);
        }
    }
    return 0;
}

int oracle_dequantize_8bit(const uint8_t *q, const float *absmax, int64_t n,
                           int blocksize, const float *code, int out_dtype,
                           void *out)
{
    if (!code8_usable(code) || !valid_dtype(out_dtype) || blocksize <= 0 || n < 0)
        return -1;
    for (int64_t i = 0; i < n; ++i) {
        /* R7: one fp32 product, then the output rounding */
        const float entry = code[q[i]];
        const float scale = absmax[i / blocksize];
        store_elem(out, out_dtype, i, entry * scale);
    }
    return 0;
}

/* ------------------------------------------ 4-bit embedding lookup (R11) */

int oracle_embedding_4bit(const uint8_t *packed, const float *absmax, int64_t V,
                          int64_t D, int blocksize, int qtype,
                          const int64_t *idx, int64_t n_idx, int out_dtype,
                          void *out)
{
    float code[16];
    if (oracle_code_table(qtype, code) != 0 || !valid_dtype(out_dtype) ||
        blocksize <= 0 || V < 0 || D < 0 || n_idx < 0)
        return -1;
    for (int64_t r = 0; r < n_idx; ++r) /* every index checked before any output */
        if (idx[r] < 0 || idx[r] >= V)
            return -1;
    for (int64_t r = 0; r < n_idx; ++r)
        for (int64_t k = 0; k < D; ++k) {
            /* element k of table row idx[r] is element idx[r]*D + k of the flat array */
            const int64_t e = idx[r] * D + k;
            store_elem(out, out_dtype, r * D + k, dequant_f32(packed, absmax, e, blocksize, code));
        }
    return 0;
}
