/*
 * A plain C99 consumer of include/nvfp4decode.h: the header must compile as C
 * (not only C++) with warnings as errors, and the library must link and answer
 * its host-side calls from C.  Only calls that touch no device are made: sizes,
 * status text, argument errors (returned before any device work), the host
 * model of one packed unit, and the verify and top-k work splits.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "nvfp4decode.h"

#define CHECK(cond)                                                      \
    do {                                                                 \
        if (!(cond)) {                                                   \
            fprintf(stderr, "failed at line %d: %s\n", __LINE__, #cond); \
            return 1;                                                    \
        }                                                                \
    } while (0)

int main(void)
{
    size_t nq = 0, ns = 0;
    /* 100 x 208 pads to 4 tiles of 32 rows x 4 chunks of 64 columns */
    CHECK(nvfp4_packed_bytes(100, 208, &nq, &ns) == NVFP4_OK);
    CHECK(nq == 16 * 1024 && ns == 16 * 128);
    CHECK(nvfp4_packed_bytes(0, 64, &nq, &ns) == NVFP4_ERR_SHAPE);
    CHECK(nvfp4_packed_bytes(100, 200, &nq, &ns) == NVFP4_ERR_SHAPE); /* K % 16 != 0 */
    CHECK(nvfp4_version() >= 100);
    CHECK(strlen(nvfp4_status_string(NVFP4_ERR_M)) > 0);

    /* an aligned stand-in pointer: argument errors come back before it is used */
    void* p = (void*)(uintptr_t)(1u << 20);
    CHECK(nvfp4_gemm_decode(p, 0, p, p, 1.0f, p, 32, 64, NULL) == NVFP4_ERR_M);
    CHECK(nvfp4_gemm_decode(NULL, 1, p, p, 1.0f, p, 32, 64, NULL) == NVFP4_ERR_ARG);
    CHECK(nvfp4_gemm_decode(p, 1, p, p, 1.0f, p, 32, 40, NULL) == NVFP4_ERR_SHAPE);
    CHECK(nvfp4_stream_read(p, 64, p, 0, NULL) == NVFP4_ERR_ARG);
    CHECK(nvfp4_round_replay(NULL, 1, NULL) == NVFP4_ERR_ARG);
    CHECK(nvfp4_round_destroy(NULL) == NVFP4_OK);

    /* host model of the layout: a 32 x 64 matrix of code 2 (1.0) with scale
     * byte 0x38 (1.0) packs into one unit that dequantises to gscale everywhere */
    static uint8_t q[32 * 32], s[32 * 4], qu[1024], su[128];
    static float W[32 * 64];
    memset(q, 0x22, sizeof q);
    memset(s, 0x38, sizeof s);
    CHECK(nvfp4_host_pack_unit(q, s, 32, 64, 0, 0, qu, su) == NVFP4_OK);
    CHECK(nvfp4_host_dequant_unit(qu, su, 0.5f, W) == NVFP4_OK);
    for (int i = 0; i < 32 * 64; ++i) CHECK(W[i] == 0.5f);

    int64_t ctas = 0, units = 0;
    int nl = 0;
    CHECK(nvfp4_verify_geometry(40, 151936, 5120, 148, &ctas, &units, &nl) == NVFP4_OK);
    CHECK(nl == 48 && ctas >= 1 && ctas <= 148 && units >= ctas);

    int splits = 0, slice = 0;
    CHECK(nvfp4_topk_splits(8, 151936, 8, 148, &splits, &slice) == NVFP4_OK);
    CHECK(splits >= 1 && (int64_t)splits * slice >= 151936);

    printf("ok\n");
    return 0;
}
