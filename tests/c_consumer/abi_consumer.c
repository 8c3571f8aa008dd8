/* A plain C99 program that uses the library through include/tsp.h and
 * include/tsp_testing.h only.  It builds a plan and reads the zigzag map and
 * both shard schedules, checking the properties they must have:
 *   - the map is a permutation;
 *   - every rank gets the same number of causal (query, key) pairs;
 *   - each schedule gives every rank every shard once.
 * It also queries sizes and FLOPs, and checks error reporting.  Needs no GPU.
 * Exit status 0 on success; otherwise the number of the failed check. */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "tsp.h"
#include "tsp_testing.h"

#define CHECK(n, cond)                                    \
    do {                                                  \
        if (!(cond)) {                                    \
            fprintf(stderr, "check %d failed: %s\n", n, #cond); \
            return n;                                     \
        }                                                 \
    } while (0)

static int run(int h, int heads, int ffn, int64_t S, int D) {
    tsp_plan_t plan = NULL;
    CHECK(1, tsp_plan(h, heads, ffn, S, D, &plan) == TSP_OK && plan != NULL);

    int32_t *map = (int32_t *)malloc((size_t)S * sizeof(int32_t));
    char *seen = (char *)calloc((size_t)S, 1);
    CHECK(2, map && seen);
    CHECK(3, tsp_zigzag_map(plan, map) == TSP_OK);
    for (int64_t i = 0; i < S; ++i) {
        CHECK(4, map[i] >= 0 && map[i] < S && !seen[map[i]]);
        seen[map[i]] = 1;
    }
    /* equal causal work: a query at position p sees p + 1 keys */
    const int64_t L = S / D;
    int64_t pairs0 = -1;
    for (int r = 0; r < D; ++r) {
        int64_t pairs = 0;
        for (int64_t i = 0; i < L; ++i) pairs += (int64_t)map[r * L + i] + 1;
        if (r == 0) pairs0 = pairs;
        CHECK(5, pairs == pairs0);
    }

    int32_t *sched = (int32_t *)malloc((size_t)D * D * sizeof(int32_t));
    CHECK(6, sched != NULL);
    for (int phase = 0; phase < 2; ++phase) {
        CHECK(7, tsp_shard_schedule(plan, phase, sched) == TSP_OK);
        for (int r = 0; r < D; ++r) {
            memset(seen, 0, (size_t)D);
            for (int t = 0; t < D; ++t) {
                const int s = sched[t * D + r];
                CHECK(8, s >= 0 && s < D && !seen[s]);
                seen[s] = 1;
            }
        }
    }
    CHECK(9, tsp_shard_schedule(plan, 2, sched) == TSP_ERR_INVALID_ARG);

    size_t ws = 0, saved = 0, ring_ws = 0;
    CHECK(10, tsp_workspace_size(plan, 1, &ws, &saved) == TSP_OK && ws > 0 && saved > 0);
    CHECK(11, tsp_workspace_size(plan, 0, &ws, &saved) == TSP_OK && ws > 0 && saved == 0);
    CHECK(12, tsp_ring_mlp_workspace_size(plan, &ring_ws) == TSP_OK && ring_ws > 0);
    const double f = tsp_layer_flops(plan, 0), fb = tsp_layer_flops(plan, 1);
    CHECK(13, f > 0.0 && fb == 2.0 * f);  /* backward = 2 x forward */

    /* arguments are refused before anything touches the device */
    CHECK(14, tsp_layer_forward(plan, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL) ==
                  TSP_ERR_INVALID_ARG);

    free(sched);
    free(seen);
    free(map);
    tsp_plan_destroy(plan);
    return 0;
}

int main(void) {
    int rc = run(128, 4, 512, 256, 2);
    if (rc == 0) rc = run(4096, 32, 16384, 8192, 8);
    if (rc == 0) rc = run(2048, 16, 4096, 4096, 16);
    if (rc) return rc;

    tsp_plan_t bad = NULL;
    if (tsp_plan(128, 4, 512, 250, 2, &bad) != TSP_ERR_INDIVISIBLE || bad != NULL) return 20;
    if (strcmp(tsp_status_string(TSP_ERR_TIMEOUT), "TSP_ERR_TIMEOUT") != 0) return 21;
    tsp_plan_destroy(NULL);
    printf("ok\n");
    return 0;
}
