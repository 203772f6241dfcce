// Prints the quantize kernel's exact-screen tables as the library's host code
// builds them (tables.cu), for tests/test_exact_keys_host.py: per case a line
// "case <name> <ok>", the 16 codes as fp32 bits, then per cell with a
// threshold "cell <k> <key bits> <thr bits> <lohi>".  Host code only.
#include <cstdio>
#include <cstring>

#include "common.cuh"

static unsigned bits(float f) {
    unsigned u;
    std::memcpy(&u, &f, 4);
    return u;
}

int main() {
    struct Case {
        const char *name;
        int ratio;  // 0: host_fp4_exact_tables, 1: host_ratio_exact_tables
        bnb4_quant_type qt;
        int p;
    } cases[] = {{"fp4_bf16", 0, BNB4_FP4, 8}, {"fp4_f16", 0, BNB4_FP4, 11}, {"nf4_bf16", 1, BNB4_NF4, 8},
                 {"nf4_f16", 1, BNB4_NF4, 11}};
    for (const Case &c : cases) {
        bnb4::QuantTables q;
        const bool ok = c.ratio ? bnb4::host_ratio_exact_tables(c.qt, c.p, q) : bnb4::host_fp4_exact_tables(c.p, q);
        std::printf("case %s %d\n", c.name, ok ? 1 : 0);
        const bnb4::CodeTable t = bnb4::host_code_table(c.qt);
        std::printf("codes");
        for (int i = 0; i < 16; ++i) std::printf(" %08x", bits(t.v[i]));
        std::printf("\n");
        if (!ok) continue;
        for (int k = 0; k < 32; ++k)
            if (q.thr[k] != 2.0f) std::printf("cell %d %08x %08x %u\n", k, q.key[k], bits(q.thr[k]), q.lohi[k]);
    }
    return 0;
}
