/*
 * c_consumer.c -- a plain C99 program against include/pa.h and libpa.so.
 * Built and run by tests/test_c_consumer.py on the CPU: it calls only the
 * host-side entry points (sizes, host validation, status strings, the block
 * manager), which need no GPU, and exits 0 when every check holds.
 */
#include <stdio.h>
#include <string.h>

#include "pa.h"

static int failures = 0;

#define CHECK(cond)                                                     \
    do {                                                                \
        if (!(cond)) {                                                  \
            fprintf(stderr, "check failed (line %d): %s\n", __LINE__, #cond); \
            ++failures;                                                 \
        }                                                               \
    } while (0)

int main(void) {
    int64_t slots[16], copies[8];
    int32_t table[8];
    int ncopies = -1, ncached = -1, nblocks = -1;
    int64_t ntokens = -1;
    const int32_t prompt[7] = {11, 12, 13, 14, 15, 16, 17};
    const int32_t next_a[1] = {21}, next_b[1] = {22};
    pa_block_manager* m;

    CHECK(pa_version() >= 100);
    CHECK(strstr(pa_status_string(PA_ERR_WORKSPACE), "workspace") != NULL);
    CHECK(pa_decode_workspace_bytes(64, 32, 128, 2048, 512) > 0);
    CHECK(pa_decode_workspace_bytes(64, 32, 128, 2048, 0) == 0);   /* bad partition size */

    /* host validation: nothing is launched, no GPU needed */
    CHECK(pa_decode(NULL, PA_F32, NULL, NULL, NULL, NULL, NULL, 1, 32, 8, 128, 16, 64, 4, 0, 0.1f, 512,
                    NULL, 0, PA_BF16, NULL, NULL) == PA_ERR_INVALID_ARG);
    CHECK(pa_decode(NULL, PA_F32, NULL, NULL, NULL, NULL, NULL, 1, 32, 8, 96, 16, 64, 4, 0, 0.1f, 512,
                    NULL, 0, PA_BF16, NULL, NULL) == PA_ERR_UNSUPPORTED);   /* head_dim 96 */
    /* the one-call step checks its scatter, copy and decode arguments first */
    CHECK(pa_decode_step(NULL, PA_F32, NULL, NULL, NULL, NULL, NULL, NULL, 4, NULL, 0, NULL, NULL, 1, 32, 8,
                         128, 16, 64, 4, 0, 0.1f, 512, NULL, 0, PA_BF16, NULL, NULL) == PA_ERR_INVALID_ARG);
    CHECK(pa_decode_step(NULL, PA_F32, NULL, NULL, NULL, NULL, NULL, NULL, -1, NULL, 0, NULL, NULL, 1, 32, 8,
                         128, 16, 64, 4, 0, 0.1f, 512, NULL, 0, PA_BF16, NULL, NULL) == PA_ERR_INVALID_ARG);
    CHECK(pa_reshape_and_cache(NULL, NULL, NULL, NULL, NULL, 1, 8, 128, 16, 64, PA_BF16, NULL, NULL) ==
          PA_ERR_INVALID_ARG);
    CHECK(pa_copy_blocks(NULL, NULL, NULL, 0, 16, 4, NULL, NULL) == PA_OK);       /* no pairs: no-op */
    CHECK(pa_selftest_bounded_wait(NULL, 1000, NULL) == PA_ERR_INVALID_ARG);

    /* the block manager: 8 blocks of 4 tokens, prefix cache on */
    m = pa_bm_create(8, 4, NULL, 1);
    CHECK(m != NULL);
    if (m == NULL) return 1;
    CHECK(pa_bm_add_sequence(m, 0) == PA_OK);
    CHECK(pa_bm_add_sequence(m, 0) == PA_ERR_INVALID_ARG);                      /* duplicate id */
    CHECK(pa_bm_append(m, 0, prompt, 7, slots, copies, 4, &ncopies, &ncached) == PA_OK);
    CHECK(ncopies == 0 && ncached == 0);
    CHECK(pa_bm_block_table(m, 0, table, 8, &nblocks, &ntokens) == PA_OK);
    CHECK(nblocks == 2 && ntokens == 7);
    CHECK(slots[0] == (int64_t)table[0] * 4 && slots[6] == (int64_t)table[1] * 4 + 2);
    CHECK(pa_bm_num_free(m) == 6);

    /* parallel sampling: fork, then both samples write into the shared partial block */
    CHECK(pa_bm_fork(m, 0, 1) == PA_OK);
    CHECK(pa_bm_ref_count(m, table[1]) == 2);
    CHECK(pa_bm_append(m, 0, next_a, 1, slots, copies, 4, &ncopies, NULL) == PA_OK);
    CHECK(ncopies == 1 && copies[0] == table[1]);   /* the first writer copies the shared block */
    CHECK(pa_bm_ref_count(m, table[1]) == 1);
    CHECK(pa_bm_append(m, 1, next_b, 1, slots, copies, 4, &ncopies, NULL) == PA_OK);
    CHECK(ncopies == 0 && slots[0] == (int64_t)table[1] * 4 + 3);   /* the last sharer writes in place */

    /* a new request with the same first block of prompt finds it cached */
    CHECK(pa_bm_add_sequence(m, 2) == PA_OK);
    CHECK(pa_bm_append(m, 2, prompt, 7, slots, copies, 4, &ncopies, &ncached) == PA_OK);
    CHECK(ncached == 4 && slots[0] == -1 && slots[3] == -1 && slots[4] >= 0);

    CHECK(pa_bm_free(m, 0) == PA_OK && pa_bm_free(m, 1) == PA_OK && pa_bm_free(m, 2) == PA_OK);
    CHECK(pa_bm_num_free(m) == 8);
    pa_bm_destroy(m);

    if (failures == 0) printf("c consumer ok\n");
    return failures == 0 ? 0 : 1;
}
