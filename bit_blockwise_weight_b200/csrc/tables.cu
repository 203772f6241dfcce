// tables.cu -- host construction of the code tables and of the decision
// tables that the quantize kernel searches (see common.cuh).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <vector>
#include <cstdlib>
#include <cstring>

#include "common.cuh"

namespace bnb4 {

CodeTable host_code_table(bnb4_quant_type qt) {
    CodeTable t{};
    if (qt == BNB4_NF4) {
        static const float nf4[16] = {
            -1.0f,       -0.6961928f, -0.5250731f, -0.3949175f, -0.2844414f, -0.1848074f,
            -0.0910500f, 0.0f,        0.0795803f,  0.1609302f,  0.2461123f,  0.3379152f,
            0.4407098f,  0.5626170f,  0.7229568f,  1.0f};
        for (int i = 0; i < 16; ++i) t.v[i] = nf4[i];
    } else {
        // E2M1 -> value / 6
        for (int i = 0; i < 16; ++i) {
            const int sign = i >> 3, e = (i >> 1) & 3, m = i & 1;
            const double mag = e ? std::ldexp(2.0 + m, e - 2) : 0.5 * m;
            t.v[i] = (float)((sign ? -mag : mag) / 6.0);
        }
    }
    return t;
}

// cell index of an fp32 value, exactly as the device computes it:
// rn(13 v + 13) with ties to even (13 v + 13 is exact in double).
static int host_cell(float v) { return (int)std::nearbyint(13.0 * (double)v + 13.0); }

QuantTables host_quant_tables(bnb4_quant_type qt) {
    const CodeTable c = host_code_table(qt);
    // distinct values in ascending order, each with the smallest index holding it
    float val[16];
    int idx[16];
    int nd = 0;
    for (int i = 0; i < 16; ++i) {
        bool seen = false;
        for (int j = 0; j < nd; ++j)
            if (val[j] == c.v[i]) seen = true;  // +0 == -0: keeps index 0
        if (!seen) {
            val[nd] = c.v[i];
            idx[nd] = i;
            ++nd;
        }
    }
    for (int a = 1; a < nd; ++a)  // insertion sort by value
        for (int b = a; b > 0 && val[b - 1] > val[b]; --b) {
            float tv = val[b]; val[b] = val[b - 1]; val[b - 1] = tv;
            int ti = idx[b]; idx[b] = idx[b - 1]; idx[b - 1] = ti;
        }
    // thresholds: v > thr[r]  <=>  rank(v) >= r + 1
    float thr[16];
    for (int r = 0; r + 1 < nd; ++r) {
        const double mid = 0.5 * ((double)val[r] + (double)val[r + 1]);  // exact
        const bool tie_up = idx[r + 1] < idx[r];  // a tie goes to the smaller index
        float t = (float)mid;
        if ((double)t > mid) t = std::nextafter(t, -INFINITY);
        if (tie_up && (double)t == mid) t = std::nextafter(t, -INFINITY);
        thr[r] = t;
    }
    QuantTables q{};
    q.valid = 1;
    for (int k = 0; k < 32; ++k) {
        int base = 0, inside = -1;
        for (int r = 0; r + 1 < nd; ++r) {
            const int cr = host_cell(thr[r]);
            if (cr < k) ++base;
            if (cr == k) {
                if (inside >= 0) q.valid = 0;  // the cell search needs one threshold per cell
                inside = r;
            }
        }
        const int lo = idx[base];
        const int hi = inside >= 0 ? idx[base + 1] : lo;
        q.thr[k] = inside >= 0 ? thr[inside] : 2.0f;  // 2 > every |v| <= 1
        q.lohi[k] = (uint32_t)lo | ((uint32_t)hi << 4);
        uint32_t key;
        if (inside >= 0) {
            std::memcpy(&key, &thr[inside], 4);
            key = (key & ~15u) | (uint32_t)(base + 1);
        } else {
            const float below_all = -0x1p100f;
            std::memcpy(&key, &below_all, 4);
            key |= (uint32_t)base;
        }
        q.key[k] = key;
        q.rank_lohi[k] = (uint32_t)base | ((uint32_t)(inside >= 0 ? base + 1 : base) << 4);
    }
    // The screen is exact when (a) every threshold lies in (-1, 1), so the
    // key moves it by less than 16 ulp <= 2^-20, and (b) no threshold lies
    // within 2^-16 of a cell boundary (j - 12.5) / 13, so a cell index taken
    // from an approximate quotient (relative error ~2^-22) can only differ
    // from the exact one where the nearest code does not change.
    bool ok = true;
    for (int r = 0; r + 1 < nd; ++r) {
        if (!(std::fabs(thr[r]) < 1.0f)) ok = false;
        for (int j = 0; j <= 26; ++j)
            if (std::fabs((double)thr[r] - (j - 12.5) / 13.0) <= 0x1p-16) ok = false;
    }
    bool ident = true, fold = true;
    for (int r = 0; r < nd; ++r) {
        if (idx[r] != r) ident = false;
        if (idx[r] != (r >= 7 ? r - 7 : 15 - r)) fold = false;
    }
    q.fast = !ok ? 0 : ident ? 1 : fold ? 2 : 0;
    return q;
}

// FP4 with 16-bit inputs.  The codes are E2M1 / 6, so the nominal decision
// points are T = k / 24 (k in {1, 3, 5, 7, 10, 14, 20}, either sign); the
// fp32 codes move each midpoint from T by about 1e-9.  For x and a with p-bit
// significands (x = X 2^ex, a = A 2^ea, X, A < 2^p, a >= 2^(ea+p-1) when
// normal), 24 x - k a is a multiple of 2^min(ex, ea), so a ratio x / a that
// is not exactly T lies at least 2^(min(ex, ea) - ea - p) / 24 from it; near
// T, x / a < 2^(ex - ea + 1) forces ex - ea >= e_T, the smallest integer
// above log2 |T| - 1, which gives the gap g_T = 2^(e_T - p) / 24 (a
// subnormal a only widens it).  So every element is either exactly on T or
// at least g_T away, and a key placed about g_T / 2 from T, on the side that
// sends an exact tie where the IEEE quotient RN(T) sends it, decides every
// element of a block with absmax in the screen's range: the screen's own
// error, with r = RN(1/a) from the exact reciprocal, is below |x / a| 2^-24.
// The key keeps the rank above in its low mantissa nibble (a shift of at
// most 8 ulps, inside the margins checked below).
bool host_fp4_exact_tables(int p, QuantTables &q) {
    q = host_quant_tables(BNB4_FP4);
    if (!q.valid || q.fast != 2) return false;
    // the distinct values in rank order, as numerators over 12
    static const int n12[15] = {-12, -8, -6, -4, -3, -2, -1, 0, 1, 2, 3, 4, 6, 8, 12};
    const CodeTable c = host_code_table(BNB4_FP4);
    float val[15];
    for (int r = 0; r < 15; ++r) {
        val[r] = (float)(n12[r] / 12.0);
        bool found = false;
        for (int i = 0; i < 16; ++i) found |= c.v[i] == val[r];
        if (!found) return false;  // the codes are these values rounded once
    }
    for (int k = 0; k < 32; ++k) {
        if (q.thr[k] == 2.0f) continue;  // no threshold in the cell: the key stays below every value
        const int R = (int)((q.rank_lohi[k] >> 4) & 15u);  // rank just above the threshold
        if (R < 1 || R > 14) return false;
        const double T = (n12[R - 1] + n12[R]) / 24.0;
        const double mid = 0.5 * ((double)val[R - 1] + (double)val[R]);
        // an exact tie x / a == T has the IEEE quotient RN(T) (T is not a
        // float midpoint), which goes above the threshold iff RN(T) > thr
        const bool up = (float)T > q.thr[k];
        const int e = (int)std::floor(std::log2(std::fabs(T)) - 1.0 - 1e-9) + 1;
        const double gap = std::ldexp(1.0, e - p) / 24.0;
        const double err = std::fabs(T) * 0x1p-24 * (1.0 + 0x1p-20) + 0x1p-60;
        // the midpoint next to T, and the gap wide against an ulp, so a ratio
        // a gap from T also has its IEEE quotient on its own side of thr
        const double ulp = std::ldexp(1.0, (int)std::floor(std::log2(std::fabs(T))) - 23);
        if (std::fabs(mid - T) > gap / 64 || gap < 16 * ulp) return false;
        float K = (float)(up ? T - gap / 2 : T + gap / 2);
        uint32_t kb;
        std::memcpy(&kb, &K, 4);
        int64_t cand = (int64_t)((kb & ~15u) | (uint32_t)R);
        if (cand - (int64_t)kb > 8) cand -= 16;
        if ((int64_t)kb - cand > 8) cand += 16;
        kb = (uint32_t)cand;
        std::memcpy(&K, &kb, 4);
        const double Kd = K;
        // ties and every other ratio stay on their sides of the key, with
        // room for the screen's error
        if (up ? !(Kd > T - gap + err && Kd < T - err) : !(Kd > T + err && Kd < T + gap - err)) return false;
        for (int j = 0; j <= 26; ++j)  // and the cell is still exact
            if (std::fabs(Kd - (j - 12.5) / 13.0) <= 0x1p-16) return false;
        q.key[k] = kb;
    }
    return true;
}

// A table whose decision thresholds no ratio of two p-bit values comes near
// (NF4 with bf16 inputs: every ratio x / a with |x| <= a lies at least 15 ulps
// from every NF4 midpoint; fp16 ratios come within a fraction of an ulp, and
// FP4's midpoints lie a fraction of an ulp from the ratios k / 24).  The
// ratios are enumerated (X / A 2^d: X < 2^p, A in [2^(p-1), 2^p), d down to
// where no threshold is reached; a subnormal absmax is outside the screen's
// range anyway); each key is put inside the
// gap between the nearest ratios below and above its threshold, clear of
// both by the screen's error with r = RN(1/a) (below |x / a| 2^-24), with the
// rank nibble kept.  Returns false, leaving q unusable, where a gap is too
// narrow.
bool host_ratio_exact_tables(bnb4_quant_type qt, int p, QuantTables &q) {
    q = host_quant_tables(qt);
    if (!q.valid || q.fast == 0 || p < 2 || p > 11) return false;
    const CodeTable c = host_code_table(qt);
    std::vector<double> ratio;
    ratio.reserve((size_t)1 << (2 * p - 1));
    for (int A = 1 << (p - 1); A < (1 << p); ++A)
        for (int X = 0; X < (1 << p); ++X) ratio.push_back((double)X / A);
    std::sort(ratio.begin(), ratio.end());
    for (int k = 0; k < 32; ++k) {
        if (q.thr[k] == 2.0f) continue;  // no threshold in the cell
        const int R = (int)((q.rank_lohi[k] >> 4) & 15u);
        // the exact midpoint of the two codes the threshold separates
        float lo_v = -2.0f, hi_v = 2.0f;
        for (int i = 0; i < 16; ++i) {
            if (c.v[i] <= q.thr[k] && c.v[i] > lo_v) lo_v = c.v[i];
            if (c.v[i] > q.thr[k] && c.v[i] < hi_v) hi_v = c.v[i];
        }
        const double mid = 0.5 * ((double)lo_v + (double)hi_v), m = std::fabs(mid);
        if (!(m > 0.0) || hi_v > 1.0f || lo_v < -1.0f) return false;
        // nearest ratio magnitudes below and above |mid|, over the scalings
        // that reach it (ratios below 2^-20 |mid| cannot)
        double below = 0.0, above = 4.0;
        for (int d = 1; d >= -40; --d) {
            const double sc = std::ldexp(1.0, d);
            if (2.0 * sc < m * 0x1p-20) break;
            const double t = m / sc;
            auto it = std::lower_bound(ratio.begin(), ratio.end(), t);
            if (it != ratio.end()) {
                if (*it == t) return false;  // a ratio on the midpoint
                above = std::min(above, *it * sc);
            }
            if (it != ratio.begin()) below = std::max(below, *(it - 1) * sc);
        }
        // every ratio at least two ulps of the midpoint away, so its IEEE
        // quotient (half an ulp off) falls on the same side of the threshold
        // (within an ulp of the midpoint) as the ratio itself
        const double u = std::ldexp(1.0, (int)std::floor(std::log2(m)) - 23);
        if (m - below < 2 * u || above - m < 2 * u) return false;
        const double err = above * 0x1p-24 * (1.0 + 0x1p-20) + 0x1p-60;
        // the key (signed like the threshold) inside (below + err, above - err)
        const double target = 0.5 * (below + above);
        float K = (float)(mid < 0 ? -target : target);
        uint32_t kb;
        std::memcpy(&kb, &K, 4);
        int64_t cand = (int64_t)((kb & ~15u) | (uint32_t)R);
        if (cand - (int64_t)kb > 8) cand -= 16;
        if ((int64_t)kb - cand > 8) cand += 16;
        kb = (uint32_t)cand;
        std::memcpy(&K, &kb, 4);
        const double Km = std::fabs((double)K);
        if (!(Km > below + err && Km < above - err)) return false;
        for (int j = 0; j <= 26; ++j)  // and the cell is still exact
            if (std::fabs((double)K - (j - 12.5) / 13.0) <= 0x1p-16) return false;
        q.key[k] = kb;
    }
    return true;
}

}  // namespace bnb4
