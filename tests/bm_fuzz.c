/*
 * bm_fuzz.c -- random histories through the host block manager (pa_bm_*),
 * built with the address and undefined-behaviour sanitizers by
 * tests/test_block_manager_sanitized.py (CPU only: the block manager makes no
 * CUDA call).  After every operation the manager's state is checked against
 * what the pages fix:
 *   - a sequence of n tokens holds ceil(n / B) blocks (a block is taken only
 *     when a token crosses into it);
 *   - every block's reference count is the number of block tables naming it;
 *   - the free blocks are exactly those with count 0;
 *   - every slot an append returns is block * B + offset of that token's
 *     position in the sequence's table, or -1 for a token found in the
 *     prefix cache.
 * Usage: bm_fuzz <seed> <operations>; exit status 0 when every check holds.
 */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "pa.h"

enum { NB = 24, B = 4, MAX_SEQS = 12, MAX_TOK = 64, MAX_COPIES = 16 };

static int failures = 0;
#define CHECK(cond)                                                                     \
    do {                                                                                \
        if (!(cond)) {                                                                  \
            if (failures < 20) fprintf(stderr, "check failed (line %d): %s\n", __LINE__, #cond); \
            ++failures;                                                                 \
        }                                                                               \
    } while (0)

static unsigned long long rng_state;
static unsigned rnd(unsigned n) { /* xorshift64*, uniform enough for a fuzzer */
    rng_state ^= rng_state >> 12;
    rng_state ^= rng_state << 25;
    rng_state ^= rng_state >> 27;
    return (unsigned)((rng_state * 2685821657736338717ull) >> 33) % n;
}

static long n_hits = 0, n_copies = 0, n_full = 0;   /* coverage, printed with -v */
static int64_t live[MAX_SEQS];
static int num_live = 0;
static int64_t next_id = 0;

static int table_of(pa_block_manager* m, int64_t id, int32_t* out, int* nblocks, int64_t* ntokens) {
    return pa_bm_block_table(m, id, out, MAX_TOK, nblocks, ntokens);
}

static void check_state(pa_block_manager* m) {
    int refs[NB];
    int32_t table[MAX_TOK];
    int i, k, nblocks, nfree = 0;
    int64_t ntokens;
    memset(refs, 0, sizeof(refs));
    for (i = 0; i < num_live; ++i) {
        CHECK(table_of(m, live[i], table, &nblocks, &ntokens) == PA_OK);
        CHECK(nblocks == (int)((ntokens + B - 1) / B));
        for (k = 0; k < nblocks; ++k) {
            CHECK(table[k] >= 0 && table[k] < NB);
            if (table[k] >= 0 && table[k] < NB) ++refs[table[k]];
        }
    }
    for (k = 0; k < NB; ++k) {
        CHECK(pa_bm_ref_count(m, k) == refs[k]);
        nfree += refs[k] == 0;
    }
    CHECK(pa_bm_num_free(m) == nfree);
}

/* The slots of the tokens appended to `id` from position n0 on. */
static void check_slots(pa_block_manager* m, int64_t id, int64_t n0, const int64_t* slots) {
    int32_t table[MAX_TOK];
    int nblocks;
    int64_t ntokens, p;
    if (table_of(m, id, table, &nblocks, &ntokens) != PA_OK) {
        CHECK(0);
        return;
    }
    for (p = n0; p < ntokens; ++p) {
        const int64_t s = slots[p - n0];
        CHECK(s == -1 || s == (int64_t)table[p / B] * B + p % B);
    }
}

static int64_t length_of(pa_block_manager* m, int64_t id) {
    int nblocks;
    int64_t ntokens = -1;
    pa_bm_block_table(m, id, NULL, 0, &nblocks, &ntokens);
    return ntokens;
}

static void remove_live(int i) {
    live[i] = live[--num_live];
}

int main(int argc, char** argv) {
    const unsigned long long seed = argc > 1 ? strtoull(argv[1], NULL, 10) : 1;
    const int ops = argc > 2 ? atoi(argv[2]) : 2000;
    /* three prompts that repeat, so that the prefix cache gets hits */
    static const int32_t prompts[3][12] = {{1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 12},
                                           {1, 2, 3, 4, 9, 9, 9, 9, 5, 5, 5, 5},
                                           {7, 7, 7, 7, 1, 2, 3, 4, 8, 8, 8, 8}};
    int cache, op;
    rng_state = seed * 0x9e3779b97f4a7c15ull + 1;
    for (cache = 0; cache <= 1; ++cache) {
        pa_block_manager* m = pa_bm_create(NB, B, NULL, cache);
        CHECK(m != NULL);
        if (!m) return 1;
        num_live = 0;
        for (op = 0; op < ops; ++op) {
            int32_t toks[16];
            int64_t slots[32], copies[2 * MAX_COPIES];
            int ncopies = 0, ncached = 0, rc, n, i;
            const unsigned kind = rnd(5);
            if (kind == 0 && num_live < MAX_SEQS) {            /* a new request with a prompt */
                const int64_t id = next_id++;
                const int which = (int)rnd(4);
                n = 1 + (int)rnd(12);
                for (i = 0; i < n; ++i) toks[i] = which < 3 ? prompts[which][i] : 1 + (int)rnd(50);
                CHECK(pa_bm_add_sequence(m, id) == PA_OK);
                live[num_live++] = id;
                rc = pa_bm_append(m, id, toks, n, slots, copies, MAX_COPIES, &ncopies, &ncached);
                CHECK(rc == PA_OK || rc == PA_ERR_WORKSPACE);
                CHECK(ncached >= 0 && ncached <= n && ncached % B == 0);
                n_hits += ncached / B;
                n_full += rc == PA_ERR_WORKSPACE;
                check_slots(m, id, 0, slots);
            } else if (kind == 1 && num_live > 0) {             /* decode: 1-3 tokens */
                const int64_t id = live[rnd((unsigned)num_live)];
                const int64_t n0 = length_of(m, id);
                n = 1 + (int)rnd(3);
                if (n0 + n > MAX_TOK) continue;
                for (i = 0; i < n; ++i) toks[i] = 1 + (int)rnd(50);
                rc = pa_bm_append(m, id, toks, n, slots, copies, MAX_COPIES, &ncopies, NULL);
                CHECK(rc == PA_OK || rc == PA_ERR_WORKSPACE);
                CHECK(ncopies >= 0 && ncopies <= 1);
                n_copies += ncopies;
                n_full += rc == PA_ERR_WORKSPACE;
                for (i = 0; i < ncopies; ++i)
                    CHECK(copies[2 * i] != copies[2 * i + 1] && copies[2 * i] >= 0 && copies[2 * i] < NB);
                check_slots(m, id, n0, slots);
            } else if (kind == 2 && num_live > 0 && num_live < MAX_SEQS) {   /* parallel sample */
                const int64_t parent = live[rnd((unsigned)num_live)], child = next_id++;
                CHECK(pa_bm_fork(m, parent, child) == PA_OK);
                live[num_live++] = child;
                CHECK(length_of(m, child) == length_of(m, parent));
            } else if (kind == 3 && num_live > 0) {             /* a finished request */
                const int i_free = (int)rnd((unsigned)num_live);
                CHECK(pa_bm_free(m, live[i_free]) == PA_OK);
                remove_live(i_free);
            } else if (kind == 4 && num_live > 0) {             /* one decode step of several sequences */
                int64_t ids[6], n0[6];
                int32_t counts[6];
                int k = 0, at = 0, j, total = 0;
                const int want = 1 + (int)rnd(6);
                for (j = 0; j < num_live && k < want; ++j) {
                    if (rnd(2) == 0 && length_of(m, live[j]) + 2 <= MAX_TOK) {
                        ids[k] = live[j];
                        n0[k] = length_of(m, live[j]);
                        counts[k] = 1 + (int)rnd(2);
                        total += counts[k];
                        ++k;
                    }
                }
                for (i = 0; i < total; ++i) toks[i] = 1 + (int)rnd(50);
                rc = pa_bm_append_batch(m, k, ids, counts, toks, slots, copies, MAX_COPIES, &ncopies, &ncached);
                CHECK(rc == PA_OK || rc == PA_ERR_WORKSPACE);
                n_copies += ncopies;
                n_full += rc == PA_ERR_WORKSPACE;
                if (rc == PA_OK) {
                    for (j = 0; j < k; ++j) {
                        CHECK(length_of(m, ids[j]) == n0[j] + counts[j]);
                        check_slots(m, ids[j], n0[j], slots + at);
                        at += counts[j];
                    }
                }
            }
            check_state(m);
        }
        /* bad arguments change nothing */
        CHECK(pa_bm_append(m, -12345, NULL, 1, NULL, NULL, 0, NULL, NULL) == PA_ERR_INVALID_ARG);
        CHECK(pa_bm_fork(m, -12345, next_id) == PA_ERR_INVALID_ARG);
        CHECK(pa_bm_ref_count(m, NB) == -1 && pa_bm_ref_count(m, -1) == -1);
        check_state(m);
        while (num_live > 0) {
            CHECK(pa_bm_free(m, live[num_live - 1]) == PA_OK);
            --num_live;
        }
        CHECK(pa_bm_num_free(m) == NB);
        pa_bm_destroy(m);
    }
    if (argc > 3 && strcmp(argv[3], "-v") == 0)
        printf("prefix-cache hits %ld, copy-on-write copies %ld, pool-exhausted appends %ld\n", n_hits, n_copies,
               n_full);
    if (failures) fprintf(stderr, "%d check(s) failed\n", failures);
    return failures ? 1 : 0;
}
