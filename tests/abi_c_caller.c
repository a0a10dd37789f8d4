/*
 * A plain C99 caller of libcsa: compiled against include/csa.h with gcc -std=c99 -pedantic and
 * linked to libcsa.so by tests/test_abi_c_caller.py.  It checks, without a GPU, what the header
 * promises on the host side: version and status strings, workspace sizes, the documented error
 * codes for bad arguments, and CSA_OK for calls with nothing to compute.  The pointers are
 * never dereferenced: every call below returns during its argument checks.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>

#include "csa.h"

static int failures = 0;

#define EXPECT(expr, want)                                                                   \
    do {                                                                                     \
        long got_ = (long)(expr);                                                            \
        if (got_ != (long)(want)) {                                                          \
            fprintf(stderr, "line %d: %s = %ld, expected %ld\n", __LINE__, #expr, got_,      \
                    (long)(want));                                                           \
            failures++;                                                                      \
        }                                                                                    \
    } while (0)

int main(void)
{
    void *f = (void *)(uintptr_t)0x100000;          /* 16-byte aligned stand-in, never read */
    void *mis = (void *)(uintptr_t)0x100004;        /* misaligned stand-in */
    const float *ff = (const float *)f;
    csa_kv_rows kv0 = {(uint8_t *)f, (uint16_t *)f, (float *)f, 0, 512, 64};
    csa_kv_rows win_small = {(uint8_t *)f, (uint16_t *)f, (float *)f, 10, 512, 64};
    csa_fp4_rows q4 = {(uint8_t *)f, (uint8_t *)f, 0, 128};
    csa_fp4_rows k4 = {(uint8_t *)f, (uint8_t *)f, 1000, 128};
    int status;

    EXPECT(csa_abi_version(), 101);
    EXPECT(csa_last_path(), CSA_PATH_NONE);
    for (status = 0; status >= -6; status--) {
        const char *s = csa_status_string(status);
        if (!s || !s[0]) {
            fprintf(stderr, "status %d has no description\n", status);
            failures++;
        }
    }
    EXPECT(indexer_topk_workspace_size(10, 7, 4) >= 10 * 8 * 4, 1);
    EXPECT(hybrid_attn_decode_workspace_size(2, 64, 512, 1024, 128, 262144, 1) > 0, 1);
    EXPECT(indexer_topk_static_capacity(), (16 << 20) + 256);

    /* bad arguments */
    EXPECT(csa_compress(NULL, f, f, f, ff, 8, 16, 4, CSA_F32, f, CSA_F32, NULL, NULL, NULL), CSA_ERR_INVALID_ARG);
    EXPECT(csa_compress(f, f, f, f, ff, 8, 18, 4, CSA_F32, f, CSA_F32, NULL, NULL, NULL), CSA_ERR_UNSUPPORTED);
    EXPECT(csa_compress(f, f, f, f, ff, 8, 16, 65, CSA_F32, f, CSA_F32, NULL, NULL, NULL), CSA_ERR_INVALID_ARG);
    EXPECT(csa_compress(f, f, f, f, ff, 8, 16, 4, CSA_F32, NULL, CSA_F32, NULL, NULL, NULL), CSA_ERR_INVALID_ARG);
    EXPECT(csa_compress(f, f, f, f, ff, 8, 16, 4, CSA_F32, mis, CSA_F32, NULL, NULL, NULL), CSA_ERR_INVALID_ARG);
    EXPECT(hca_compress(f, f, ff, 4096, 512, 2048, CSA_BF16, f, CSA_F32, NULL, NULL), CSA_ERR_INVALID_ARG);
    EXPECT(csa_quantize_kv(f, CSA_F32, 4, 512, 32, &kv0, NULL), CSA_ERR_INVALID_ARG);
    EXPECT(csa_quantize_fp4(f, CSA_F32, 4, 48, &q4, NULL), CSA_ERR_INVALID_ARG);
    EXPECT(indexer_topk(&q4, ff, &k4, CSA_FP4, NULL, NULL, 1000, 1, 64, 128, 4, 0, 250, (int32_t *)f, NULL,
                        f, 1 << 20, NULL), CSA_ERR_UNSUPPORTED);
    EXPECT(indexer_topk(&q4, ff, &k4, CSA_FP4, NULL, NULL, 1000, 1, 64, 128, 4, 64, 250, (int32_t *)f, NULL,
                        f, 16, NULL), CSA_ERR_WORKSPACE);
    EXPECT(indexer_topk(&q4, ff, &k4, 7, NULL, NULL, 1000, 1, 64, 128, 4, 64, 250, (int32_t *)f, NULL,
                        f, 1 << 20, NULL), CSA_ERR_INVALID_ARG);
    EXPECT(hybrid_attn_prefill(f, f, f, 4, NULL, 0, ff, 1.0f, 16, 64, 96, 4, 128, CSA_BF16, f, NULL, NULL),
           CSA_ERR_UNSUPPORTED);
    EXPECT(hybrid_attn_prefill(f, f, f, 4, NULL, 0, ff, NAN, 16, 64, 512, 4, 128, CSA_BF16, f, NULL, NULL),
           CSA_ERR_INVALID_ARG);
    EXPECT(hybrid_attn_prefill(f, f, NULL, 4, NULL, 0, ff, 1.0f, 16, 64, 512, 4, 128, CSA_BF16, f, NULL, NULL),
           CSA_ERR_INVALID_ARG);
    EXPECT(hybrid_attn_decode(f, &kv0, (const int64_t *)f, (const int64_t *)f, &win_small, (const int32_t *)f,
                              (const int32_t *)f, 1024, ff, 1.0f, 2, 64, 512, 4, 128, 1000, f, NULL, f, 1 << 30,
                              NULL), CSA_ERR_INVALID_ARG);
    EXPECT(csa_decode_glue(f, f, NULL, 256, 512, 128, f, &q4, NULL), CSA_ERR_INVALID_ARG);
    EXPECT(csa_device_error(NULL, NULL), CSA_ERR_INVALID_ARG);

    /* nothing to compute */
    EXPECT(csa_compress(f, f, f, f, ff, 3, 128, 4, CSA_F32, f, CSA_F32, NULL, NULL, NULL), CSA_OK);
    EXPECT(hca_compress(f, f, ff, 127, 512, 128, CSA_BF16, f, CSA_F32, NULL, NULL), CSA_OK);
    EXPECT(csa_quantize_kv(f, CSA_F32, 0, 512, 64, &kv0, NULL), CSA_OK);
    EXPECT(csa_quantize_fp4(f, CSA_F32, 0, 128, &q4, NULL), CSA_OK);
    EXPECT(indexer_topk(&q4, ff, &k4, CSA_FP4, NULL, NULL, 1000, 0, 64, 128, 4, 1024, 250, (int32_t *)f, NULL,
                        NULL, 0, NULL), CSA_OK);
    EXPECT(indexer_topk_static(&q4, ff, &k4, CSA_FP4, NULL, NULL, 1000, 0, 64, 128, 4, 1024, 250, (int32_t *)f,
                               NULL, NULL), CSA_OK);
    EXPECT(hybrid_attn_prefill(f, f, f, 0, NULL, 0, ff, 1.0f, 0, 64, 512, 128, 128, CSA_BF16, f, NULL, NULL),
           CSA_OK);
    EXPECT(hybrid_attn_decode(f, &kv0, (const int64_t *)f, (const int64_t *)f, &kv0, (const int32_t *)f,
                              (const int32_t *)f, 1024, ff, 1.0f, 0, 64, 512, 4, 128, 0, f, NULL, NULL, 0, NULL),
           CSA_OK);
    EXPECT(csa_decode_glue(f, f, NULL, 0, 512, 0, f, NULL, NULL), CSA_OK);

    if (failures) {
        fprintf(stderr, "%d check(s) failed\n", failures);
        return 1;
    }
    printf("ok\n");
    return 0;
}
