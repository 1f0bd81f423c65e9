/* A C consumer of include/q4.h: compiles as C99 against the header, links
 * libq4.so, and exercises calls that return before any CUDA work (version,
 * status strings, argument validation), so it runs without a GPU. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "q4.h"

#define CHECK(cond)                                                   \
    do {                                                              \
        if (!(cond)) {                                                \
            fprintf(stderr, "failed: %s (line %d)\n", #cond, __LINE__); \
            return 1;                                                 \
        }                                                             \
    } while (0)

int main(void) {
    const void* A16 = (const void*)(uintptr_t)0x10000; /* never dereferenced */
    CHECK(strstr(q4_version(), "sm_100a") != NULL);
    CHECK(strcmp(q4_status_string(Q4_OK), "Q4_OK") == 0);
    CHECK(strcmp(q4_status_string(Q4_ERR_WORKSPACE), "Q4_ERR_WORKSPACE") == 0);

    q4_weight w;
    memset(&w, 0, sizeof(w));
    w.qweight = (const uint8_t*)A16;
    w.scales = A16;
    w.out = 64;
    w.in = 256;
    w.group_size = 128;
    w.bits = 8; /* only 4 is supported */
    w.symmetric = 1;
    CHECK(q4_gemv(&w, A16, Q4_BF16, 1, (void*)A16, Q4_BF16, NULL, 0, NULL) == Q4_ERR_UNSUPPORTED);
    w.bits = 4;
    CHECK(q4_gemv(&w, A16, Q4_BF16, 9, (void*)A16, Q4_BF16, NULL, 0, NULL) == Q4_ERR_SHAPE);
    CHECK(q4_gemv(&w, A16, Q4_BF16, 1, (void*)A16, Q4_BF16, NULL, 0, NULL) == Q4_ERR_WORKSPACE);
    CHECK(q4_quantize_pack(A16, Q4_F16, 8, 100, 128, 4, 1, (uint8_t*)A16, (void*)A16, NULL, NULL) ==
          Q4_ERR_SHAPE);
    CHECK(q8_gemv((const int8_t*)A16, (const float*)A16, 64, 120, A16, Q4_BF16, 1, (void*)A16,
                  Q4_BF16, NULL, 0, NULL) == Q4_ERR_SHAPE);
    CHECK(kv_quantize_int8(A16, Q4_F32, 4, 128, (int8_t*)A16, (void*)A16, NULL) == Q4_ERR_UNSUPPORTED);
    CHECK(mxfp4_quantize(A16, Q4_BF16, 4, 48, (uint8_t*)A16, (uint8_t*)A16, NULL) == Q4_ERR_SHAPE);
    CHECK(nvfp4_quantize(A16, Q4_BF16, 0, 64, (uint8_t*)A16, (uint8_t*)A16, (float*)A16, NULL) == Q4_OK);
    printf("c abi ok\n");
    return 0;
}
