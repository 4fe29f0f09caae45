/* A plain C11 client of the library's C ABI (include/nvfp4.h), built and run by
 * tests/test_c_abi.py. It needs no GPU: it checks the layout-size functions against their
 * definitions, the status strings, and that argument errors return before any device work. */
#include <stdio.h>
#include <string.h>

#include "nvfp4.h"

static int failures = 0;

#define CHECK(cond)                                                 \
    do {                                                            \
        if (!(cond)) {                                              \
            fprintf(stderr, "FAILED: %s (line %d)\n", #cond, __LINE__); \
            ++failures;                                             \
        }                                                           \
    } while (0)

int main(void) {
    CHECK(nvfp4_version() >= 100);

    /* codes: 16 bytes per 32 elements; linear scales: one byte per 16 elements;
     * tensor-core scales: 512-byte atoms of 128 rows x 4 scales */
    CHECK(nvfp4_codes_pitch(3072) == 1536);
    CHECK(nvfp4_codes_pitch(17) == 16);
    CHECK(nvfp4_sf_bytes(4680, 3072, NVFP4_SF_LINEAR) == 4680LL * 192);
    CHECK(nvfp4_sf_bytes(4680, 3072, NVFP4_SF_MMA) == 37LL * 48 * 512);
    CHECK(nvfp4_sf_bytes(4680, 3072, 7) == -1);
    CHECK(nvfp4_kv_cache_bytes(30, 24, 128, 12, 4680, 0) == 30LL * 12 * 4680 * 3072 / 2);
    CHECK(nvfp4_kv_cache_bytes(30, 24, 128, 12, 4680, 1) == 30LL * 12 * 4680 * 3072 / 16);
    CHECK(nvfp4_kv_cache_bytes(30, 24, 128, 12, 4680, 2) == 30LL * 12 * 4);

    for (int s = 0; s <= 5; ++s) {
        const char *msg = nvfp4_status_string(s);
        CHECK(msg != NULL && strlen(msg) > 0);
    }

    /* argument errors are synchronous and need no device */
    nvfp4_tensor t;
    memset(&t, 0, sizeof t);
    t.rows = 4;
    t.cols = 32;
    t.sf_layout = NVFP4_SF_MMA;
    CHECK(nvfp4_quantize(NULL, 4, 32, 32, NVFP4_ROWWISE, NULL, &t, NULL, 0, NULL, NULL) == NVFP4_ERR_INVALID_ARG);
    CHECK(nvfp4_gemm(NULL, NULL, NULL, NULL, NULL, 0, 0, NULL, NULL) == NVFP4_ERR_INVALID_ARG);
    CHECK(kv_dequant(NULL, 0, NULL, 0, NULL, NULL, NULL, NULL) == NVFP4_ERR_INVALID_ARG);
    CHECK(kv_attention(NULL, 0, NULL, 0, NULL, 0, 0, 1.0f, NULL, 0, NULL, NULL) == NVFP4_ERR_INVALID_ARG);

    if (failures == 0) printf("c abi ok\n");
    return failures == 0 ? 0 : 1;
}
