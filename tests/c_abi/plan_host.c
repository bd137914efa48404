/* A plain C caller of the library's C ABI (include/bca.h), no GPU needed: a host-only
 * plan for one video of 2 chunks x 2 latent frames x 8 x 8 tokens (128 tokens per
 * chunk), block-causal by default (no slice list), 4 query / 2 KV heads, D = 48.
 * Prints "<num_q> <num_k> <visible_pairs> <row0_visible> <row255_visible>" and checks the
 * error paths; exit status 0 on success. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include "bca.h"

static int expect(int got, int want, const char *what) {
    if (got != want) {
        fprintf(stderr, "%s: got %d (%s), want %d\n", what, got, bca_error_string(got), want);
        return 1;
    }
    return 0;
}

int main(void) {
    bca_video video = {2, 2, 8, 8, 0};
    bca_problem p = {0};
    p.num_q_heads = 4;
    p.num_kv_heads = 2;
    p.head_dim = 48;
    p.num_videos = 1;
    p.videos = &video;
    p.num_cache_keys = 0;
    p.num_slices = 0;
    p.slices = NULL;
    p.rope_base[0] = p.rope_base[1] = p.rope_base[2] = 10000.0f;
    p.norm_eps = 1e-6f;
    p.flags = BCA_PLAN_HOST_ONLY;

    bca_plan_t plan = NULL;
    int fails = expect(bca_plan_create(&p, &plan), BCA_OK, "bca_plan_create");
    if (fails) return 1;
    bca_plan_info info;
    fails += expect(bca_plan_get_info(plan, &info), BCA_OK, "bca_plan_get_info");

    uint8_t *rows = (uint8_t *)malloc((size_t)info.num_k * 256);
    fails += expect(bca_plan_expand_rows(plan, 0, 256, rows), BCA_OK, "bca_plan_expand_rows");
    int64_t first = 0, last = 0;
    for (int64_t j = 0; j < info.num_k; ++j) {
        first += rows[j];
        last += rows[(size_t)255 * info.num_k + j];
    }
    /* a host-only plan launches nothing */
    fails += expect(bca_fwd(plan, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL),
                    BCA_ERR_HOST_ONLY_PLAN, "bca_fwd on a host-only plan");
    bca_plan_destroy(plan);
    free(rows);

    /* an unsupported head dim and a bad slice are refused, with no plan left behind */
    p.head_dim = 40;
    plan = NULL;
    fails += expect(bca_plan_create(&p, &plan), BCA_ERR_UNSUPPORTED, "head_dim 40");
    fails += expect(plan == NULL, 1, "no plan after a refusal");
    p.head_dim = 48;
    bca_slice bad = {0, 300, 0, 10, BCA_SLICE_FULL};   /* q_end beyond Nq = 256 */
    p.num_slices = 1;
    p.slices = &bad;
    fails += expect(bca_plan_create(&p, &plan), BCA_ERR_BAD_SLICE, "slice out of range");

    printf("%lld %lld %lld %lld %lld\n", (long long)info.num_q, (long long)info.num_k,
           (long long)info.visible_pairs, (long long)first, (long long)last);
    return fails ? 1 : 0;
}
