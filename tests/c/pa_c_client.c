/*
 * A plain C99 client of libpa.so: the public header compiles as C and the
 * host-side calls work through the C ABI with no GPU (plans built for
 * inspection, device = -1; argument checks that reject calls before any work
 * is queued).  Exit status 0 when every check holds; otherwise the number of
 * the first failed check.
 */
#include <stdio.h>
#include <string.h>

#include "pa.h"

#define CHECK(n, cond)                                   \
    do {                                                 \
        if (!(cond)) {                                   \
            fprintf(stderr, "check %d failed: %s\n", n, #cond); \
            return n;                                    \
        }                                                \
    } while (0)

int main(void) {
    /* three requests: two decodes (16 and 39 prior tokens) and a fresh
       6-token prefill, 4 query heads on 2 kv heads, head_dim 64 */
    const int32_t cu[4] = {0, 1, 2, 8};
    const int32_t seq[3] = {17, 40, 6};
    pa_dims d;
    memset(&d, 0, sizeof d);
    d.num_tokens = 8;
    d.num_seqs = 3;
    d.num_q_heads = 4;
    d.num_kv_heads = 2;
    d.head_dim = 64;
    d.num_blocks = 64;
    d.max_blocks_per_seq = 3;
    d.block_size = 16;

    pa_plan *plan = NULL;
    CHECK(1, pa_plan_build(cu, seq, NULL, &d, -1, &plan) == PA_OK && plan != NULL);

    pa_plan_info info;
    CHECK(2, pa_plan_get_info(plan, &info) == PA_OK);
    /* every query row of a segment with q_len <= 16 is a decode row, per kv
       head: 8 tokens x 2 kv heads */
    CHECK(3, info.num_decode_rows == 16);
    /* blocks the rows read: ceil(17/16) + ceil(40/16) + sum_j ceil((j+1)/16) for j < 6, per kv head */
    CHECK(4, info.decode_kv_blocks == (2 + 3 + 6) * 2);
    /* keys without last-block padding: 17 + 40 + (1 + 2 + ... + 6), per kv head */
    CHECK(4, info.decode_kv_keys == (17 + 40 + 21) * 2);
    CHECK(5, info.num_prefill_tiles == 0 && info.num_sms == 148);
    CHECK(6, pa_plan_workspace_bytes(plan) == info.workspace_bytes && info.workspace_bytes >= 256);
    CHECK(7, info.attention_launches == 1);

    /* the plan is rebuilt in place */
    pa_plan *same = plan;
    CHECK(8, pa_plan_build(cu, seq, NULL, &d, -1, &plan) == PA_OK && plan == same);

    /* host-checkable errors, before any work */
    const int32_t bad_cu[4] = {0, 1, 2, 9};
    pa_plan *p2 = NULL;
    CHECK(9, pa_plan_build(bad_cu, seq, NULL, &d, -1, &p2) == PA_ERR_SHAPE && p2 == NULL);
    pa_dims d2 = d;
    d2.head_dim = 96;
    CHECK(10, pa_plan_build(cu, seq, NULL, &d2, -1, &p2) == PA_ERR_UNSUPPORTED);
    CHECK(11, pa_reshape_and_cache(NULL, NULL, NULL, NULL, NULL, &d, NULL) == PA_ERR_NULL);
    /* a host-only plan is refused by the compute calls */
    char *fake = (char *)(uintptr_t)0x10000;
    CHECK(12, pa_attention_varlen(fake, fake, fake, (const int32_t *)fake, (const int32_t *)fake,
                                  (const int32_t *)fake, 0.125f, fake, &d, plan, fake, (size_t)1 << 20,
                                  NULL) == PA_ERR_PLAN);

    CHECK(13, strcmp(pa_status_string(PA_OK), "") != 0 && pa_version() != NULL);
    pa_plan_destroy(plan);
    pa_plan_destroy(NULL);
    printf("C client ok: %d decode rows, %lld blocks, workspace %llu bytes\n", info.num_decode_rows,
           (long long)info.decode_kv_blocks, (unsigned long long)info.workspace_bytes);
    return 0;
}
