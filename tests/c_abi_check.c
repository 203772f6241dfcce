/* Plain C99 client of include/bnb4.h: compiles with warnings as errors, links
 * libbnb4.so and exercises the calls that return before any device work
 * (version, status strings, argument checks).  Exit code 0 = all as expected. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "bnb4.h"

static int failures = 0;

static void expect(int got, int want, const char *what) {
    if (got != want) {
        fprintf(stderr, "%s: got %d, want %d\n", what, got, want);
        ++failures;
    }
}

int main(void) {
    void *a = (void *)(uintptr_t)4096; /* aligned, never dereferenced */
    float code[256];
    int j;
    for (j = 0; j < 256; ++j) code[j] = (float)(j - 128) / 128.0f;

    expect(bnb4_version() >= 10000, 1, "version");
    expect(strcmp(bnb4_status_string(BNB4_OK), "ok") == 0, 1, "status string");
    expect(bnb4_quantize(a, (uint8_t *)a, (float *)a, -1, 64, BNB4_NF4, BNB4_BF16, 0), BNB4_ERR_SHAPE, "quantize n<0");
    expect(bnb4_quantize(a, (uint8_t *)a, (float *)a, 8, 48, BNB4_NF4, BNB4_BF16, 0), BNB4_ERR_BLOCKSIZE,
           "quantize blocksize");
    expect(bnb4_dequantize((const uint8_t *)a, (const float *)a, 0, 8, 64, BNB4_FP4, BNB4_F16, 0), BNB4_ERR_NULL,
           "dequantize null out");
    expect(bnb4_gemv(a, (const uint8_t *)a, (const float *)a, 0, a, 64, 100, 64, BNB4_NF4, BNB4_BF16, 0),
           BNB4_ERR_SHAPE, "gemv K%32");
    expect(bnb4_gemm(a, (const uint8_t *)a, (const float *)a, 0, a, 2, 64, 128, 64, BNB4_NF4, (bnb4_dtype)7, 0),
           BNB4_ERR_DTYPE, "gemm dtype");
    expect(bnb4_gemm_backward(a, (const uint8_t *)a, (const float *)a, a, 2, 60, 128, 64, BNB4_NF4, BNB4_BF16, 0),
           BNB4_ERR_SHAPE, "backward N%8");
    expect(bnb4_double_quant((const float *)a, 10, 100, (uint8_t *)a, (float *)a, 0), BNB4_ERR_BLOCKSIZE,
           "double_quant group");
    expect(bnb4_gemv_dq(a, (const uint8_t *)a, (const uint8_t *)a, 0, 256, 0, a, 64, 128, 64, BNB4_NF4,
                        BNB4_BF16, 0), BNB4_ERR_NULL, "gemv_dq null scales");
    code[7] = 2.0f;
    expect(bnb4_quantize_8bit(a, (uint8_t *)a, (float *)a, 8, 64, code, BNB4_F32, 0), BNB4_ERR_CODE, "8-bit table");
    expect(bnb4_embedding_4bit((const uint8_t *)a, (const float *)a, 10, 0, 64, BNB4_NF4, (const int64_t *)a, 3, a,
                               BNB4_BF16, 0), BNB4_ERR_SHAPE, "embedding D<1");
    if (failures == 0) printf("c abi ok\n");
    return failures != 0;
}
