/*
 * tsp_testing.h - test hooks of the TSP layer library.
 *
 * These entry points exist so that tests can check one kernel at a time and
 * look at intermediate tensors; the layer itself is driven through tsp.h.
 * The paper pages describe no such calls: they are infrastructure of this
 * library.
 */
#ifndef TSP_TESTING_H
#define TSP_TESTING_H

#include <stddef.h>
#include <stdint.h>

#include "tsp.h"

#ifdef __cplusplus
extern "C" {
#endif

/* C[M][N] (float32, row stride ldc) = sum_k A[m][k] * B[n][k] with the layer's
 * tcgen05 GEMM kernel, fp32 accumulation; A and B are both bf16 (f16 == 0) or
 * both fp16 (f16 != 0).
 *   a_mn == 0: A is [M][K] (row stride lda); a_mn != 0: A is stored [K][M].
 *   b_mn == 0: B is [N][K] (row stride ldb); b_mn != 0: B is stored [K][N].
 * M % 128 == 0, N % 128 == 0, K % 64 == 0 (TSP_ERR_UNSUPPORTED otherwise);
 * device pointers, 16-byte aligned.  force_bn128 != 0 selects the 128-column
 * tile even where the 256-column tile applies.  Asynchronous on `stream`. */
tsp_status tsp_test_gemm(int a_mn, int b_mn, int M, int N, int K, const void *A, int64_t lda, const void *B,
                         int64_t ldb, float *C, int64_t ldc, int force_bn128, int f16, void *stream);

/* Byte offset of a named intermediate inside the `saved` buffer (names: rstd1,
 * a, q, k, v, o, lse, y, rstd2, b, u, g, wqkv_h, wo_h, w1_h, w2_h, scales) or,
 * with a "ws." prefix, inside the backward scratch (ws.du, ws.db, ws.dy,
 * ws.dyh, ws.dO, ws.delta, ws.dqkv, ws.da, ws.dy16, ws.gscales).
 * Layouts: a, q, o, b fp16 [S][h] local rows; k, v fp16 [S][h] global rows;
 * y f32 [S][h]; u bf16 [S][F]; g fp16 [S][F]; lse f32 [H][S] in log2 units
 * (scores times log2(e)/sqrt(dh)); rstd f32 [S]; the *_h weight copies fp16,
 * each the bf16 weight times 2^e_i; scales f32: [0..3] = 2^-e_i and
 * [8..11] = 2^e_i for wqkv, wo, w1, w2.  The backward's gradients (ws.du,
 * ws.db, ws.dy, ws.dyh, ws.dO, ws.dqkv, ws.da, ws.dy16) are those of the
 * layer times 2^k, with ws.gscales f32 [0] = 2^-k and [1] = 2^k.
 * TSP_ERR_INVALID_ARG for an unknown name. */
tsp_status tsp_test_buffer_offset(tsp_plan_t plan, const char *name, size_t *offset);

/* Host evaluation of the rule the dK/dV kernel uses to walk the 64-row query
 * steps that can see a key: writes to *out the first local step q >= from
 * (step q = local rows [64 q, 64 q + 64)) whose largest global position is at
 * least kv0, or S / 64 when there is none.  It is the same function the
 * kernel runs, so a test can check it against a scan of the zigzag map.
 * TSP_ERR_INVALID_ARG for from outside [0, S / 64] or kv0 outside [0, S). */
tsp_status tsp_test_next_visible(tsp_plan_t plan, int from, int kv0, int *out);

/* Host copy of a table the plan uploads for the kernels (computed on the
 * host, no GPU needed), written to out[0 .. *count) (host memory; *count
 * always receives the length).  which:
 *   0  inverse zigzag map: position -> local row, [S]
 *   1  largest position of each 128-row local query tile, [S/128]
 *   2  forward attention work order: pairs (query block * heads + head,
 *      number of 128-key tiles to visit) for 256-row query blocks
 *   3  dK/dV work order: key tile * heads + head, [S/128 * heads]
 *   4  dQ work order: query tile * heads + head, [S/128 * heads]
 * Work orders are head-major with the longest items of a head first here;
 * the plan uploads the forward and dK/dV orders paired in waves
 * (tsp_test_work_order).
 * TSP_ERR_INVALID_ARG for another `which`, a NULL pointer or a table longer
 * than `capacity`. */
tsp_status tsp_test_tables(tsp_plan_t plan, int which, int32_t *out, int64_t capacity, int64_t *count);

/* Host replay of the walk the dK/dV kernel makes over the 64-row query steps
 * that can see the key tile starting at position kv0: writes the visited
 * steps, in the kernel's order, to steps[0 .. *count) (host memory, at most
 * `capacity` entries; *count always receives the full length).  The same
 * code as the kernel's, so a test can compare it with a scan of the zigzag
 * map.  TSP_ERR_INVALID_ARG for kv0 outside [0, S), a NULL pointer, or a
 * walk longer than `capacity`. */
tsp_status tsp_test_step_walk(tsp_plan_t plan, int kv0, int32_t *steps, int capacity, int *count);

/* The same work orders (which = 2, 3, 4 as above) as the plan uploads them
 * for a device with `num_ctas` SMs: every other round of num_ctas consecutive
 * items reversed, so that the persistent CTAs, which take items i, i +
 * num_ctas, ..., draw long and short items in turn and stay in step.
 * TSP_ERR_INVALID_ARG for another `which`, num_ctas < 1, a NULL pointer or a
 * table longer than `capacity`. */
tsp_status tsp_test_work_order(tsp_plan_t plan, int which, int num_ctas, int32_t *out, int64_t capacity,
                               int64_t *count);

/* Host replay of the walk the single-pass attention backward makes over the
 * 64-row query steps that can see the key tile starting at position kv0: the
 * same steps as tsp_test_step_walk, in descending order of position (chunks
 * from the last, each from its last step down), so that every walk is a
 * prefix of the walk for kv0 = 0.  Output and errors as tsp_test_step_walk. */
tsp_status tsp_test_step_walk_desc(tsp_plan_t plan, int kv0, int32_t *steps, int capacity, int *count);

/* The same walk as tsp_test_step_walk_desc kept to one rank's query rows (its
 * chunks 2D-1-rank, then rank), as the per-rank attention backward makes it.
 * Output and errors as tsp_test_step_walk, and TSP_ERR_INVALID_ARG for a rank
 * outside [0, D). */
tsp_status tsp_test_step_walk_rank(tsp_plan_t plan, int rank, int kv0, int32_t *steps, int capacity, int *count);

/* The per-rank attention backward's work order of `rank` for num_ctas
 * persistent CTAs, as uploaded: key tile * heads + head for every key tile
 * that the rank's rows see, paired in waves.  Errors as tsp_test_work_order,
 * and TSP_ERR_INVALID_ARG for a rank outside [0, D). */
tsp_status tsp_test_rank_kv_order(tsp_plan_t plan, int rank, int num_ctas, int32_t *out, int64_t capacity,
                                  int64_t *count);

/* Self-test of the bounded device-side wait used by every kernel: launches one
 * CTA that waits on an mbarrier nothing ever completes, with a limit of
 * `limit_cycles` SM cycles.  The wait gives up, the kernel writes 0 to
 * result_dev[0] (1 would mean the wait completed) and sets the plan's error
 * flag, so the next tsp_sync_status() reports TSP_ERR_TIMEOUT.  No memory
 * copy or tensor-core work is in flight, so giving up is safe. */
/* y[i] = 2^x[i] for n device floats, by the polynomial exp2 that the
 * attention forward uses for a share of its exponentials (which = 0) or by
 * the hardware approximation it uses for the rest (which = 1).
 * TSP_ERR_INVALID_ARG for another `which`, n < 0 or a NULL pointer with
 * n > 0; TSP_ERR_CUDA for a failed launch. */
tsp_status tsp_test_exp2(const float *x, float *y, int n, int which, void *stream);

tsp_status tsp_test_wait_timeout(tsp_plan_t plan, long long limit_cycles, int *result_dev, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* TSP_TESTING_H */
