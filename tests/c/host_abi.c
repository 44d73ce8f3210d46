/* The library's host calls used from plain C11: a block manager with
 * fork, copy-on-write and free ("vLLM推理加速框架：PagedAttention与连续批处理技术解析"
 * 2.1-2.2), and a scheduler step admitting through the prefix cache with a C
 * token function ("大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置",
 * section "Prefix Caching前缀复用优化").  Every expected value is worked by hand
 * from the free-list rule (blocks taken from the end of the list) and the
 * slot rule slot = block * block_size + offset.  No device call is made.
 * Prints "ok" and returns 0 when every check holds. */
#include <stdint.h>
#include <stdio.h>

#include "pa.h"

static int failures = 0;

#define CHECK(cond)                                                  \
    do {                                                             \
        if (!(cond)) {                                               \
            fprintf(stderr, "line %d: check failed: %s\n", __LINE__, #cond); \
            ++failures;                                              \
        }                                                            \
    } while (0)

static int32_t next_token(void* ctx, int64_t seq_id, int64_t position) {
    (void)ctx;
    return (int32_t)((seq_id + position) % 5);
}

static void block_manager_case(void) {
    const int32_t order[8] = {0, 1, 2, 3, 4, 5, 6, 7};
    pa_bm* bm = NULL;
    int32_t table[8];
    int n = 0, count = 0, nfree = 0, used = 0, ctx = 0;
    int64_t slot = 0;
    int32_t src = 0, dst = 0;
    CHECK(pa_bm_create(8, 4, order, &bm) == PA_OK);
    CHECK(pa_bm_allocate(bm, 1, 6) == PA_OK);              /* two blocks: 7, then 6 */
    CHECK(pa_bm_block_table(bm, 1, table, 8, &n) == PA_OK && n == 2 && table[0] == 7 && table[1] == 6);
    CHECK(pa_bm_fork(bm, 1, 2) == PA_OK);
    CHECK(pa_bm_ref_count(bm, 6, &count) == PA_OK && count == 2);
    /* position 6 of seq 2 lands in the shared, partly filled block 6: copy it to block 5 */
    CHECK(pa_bm_append_slot(bm, 2, &slot, &src, &dst) == PA_OK);
    CHECK(slot == 5 * 4 + 2 && src == 6 && dst == 5);
    CHECK(pa_bm_ref_count(bm, 6, &count) == PA_OK && count == 1);
    CHECK(pa_bm_stats(bm, 2, &nfree, &used, &ctx) == PA_OK && nfree == 5 && used == 3 && ctx == 7);
    CHECK(pa_bm_free(bm, 1) == PA_OK);                     /* block 6 back on the list, 7 still held */
    CHECK(pa_bm_append_slot(bm, 2, &slot, &src, &dst) == PA_OK && slot == 5 * 4 + 3 && src == -1);
    CHECK(pa_bm_append_slot(bm, 2, &slot, &src, &dst) == PA_OK && slot == 6 * 4 + 0);
    CHECK(pa_bm_free(bm, 1) == PA_ERR_INVALID_ARG);        /* already freed */
    pa_bm_destroy(bm);
}

static void scheduler_case(void) {
    pa_bm* bm = NULL;
    pa_sched* s = NULL;
    const int32_t prefix[3] = {1, 2, 3};
    const int32_t prompt[3] = {3, 0, 1};
    int cached = -1;
    pa_sched_counts c;
    int32_t kind[8];
    int64_t a[8], b[8], cc[8], running[2];
    int32_t lens[2];
    int i;
    CHECK(pa_bm_create(16, 2, NULL, &bm) == PA_OK);
    CHECK(pa_bm_enable_prefix_cache(bm, 1) == PA_OK);
    /* holder: blocks 15 (tokens 1 2, cached) and 14 (token 3, partly filled) */
    CHECK(pa_bm_allocate_prefix(bm, 100, prefix, 3, &cached) == PA_OK && cached == 0);
    CHECK(pa_sched_create(bm, 4, 100, &s) == PA_OK);
    CHECK(pa_sched_add_request(s, 7, 1, 1, 0, -1, 0) == PA_OK);   /* plain mode: accepted */
    pa_sched_destroy(s);
    CHECK(pa_sched_create(bm, 4, 100, &s) == PA_OK);
    CHECK(pa_sched_enable_prefix_cache(s, prefix, 3, next_token, NULL) == PA_OK);
    CHECK(pa_sched_add_request(s, 1, 3, 2, 1, -1, 0) == PA_ERR_INVALID_ARG);   /* ids required */
    CHECK(pa_sched_add_request_tokens(s, 1, prompt, 3, 2, 1, -1, 0) == PA_OK);
    CHECK(pa_sched_step(s) == PA_OK);
    CHECK(pa_sched_counts_get(s, &c) == PA_OK && c.num_admitted == 1 && c.num_ops == 5 && c.num_running == 1);
    if (c.num_ops == 5 && c.num_running == 1) {
        CHECK(pa_sched_record(s, NULL, NULL, NULL, kind, a, b, cc, running, lens) == PA_OK);
        /* history 1 2 3 3 0 1: block 15 found for (1 2); (3 3) -> block 13, (0 1) -> 12;
         * writes for positions 2..5, then the decode token (1 + 6) % 5 = 2 at position 6
         * opens block 11 */
        const int64_t want[5] = {13 * 2, 13 * 2 + 1, 12 * 2, 12 * 2 + 1, 11 * 2};
        for (i = 0; i < 5; ++i) CHECK(kind[i] == 0 && a[i] == 1 && b[i] == 2 + i && cc[i] == want[i]);
        CHECK(running[0] == 1 && lens[0] == 7);
    }
    pa_sched_destroy(s);
    pa_bm_destroy(bm);
}

int main(void) {
    block_manager_case();
    scheduler_case();
    CHECK(pa_status_string(PA_ERR_NO_BLOCKS) != NULL);
    if (failures) return 1;
    printf("ok\n");
    return 0;
}
