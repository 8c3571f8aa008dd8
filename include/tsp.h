/*
 * tsp.h - C ABI of the folded Tensor-Sequence-Parallel (TSP) decoder layer on
 * one NVIDIA B200 (sm_100a).
 *
 * What is computed.  "Zyphra TSP folds TP+SP onto one GPU axis, 2.6x throughput
 * on 1,024 MI300Xs" (zubnet.ai), paragraph 1: tensor parallelism (weights) and
 * sequence parallelism (tokens) share one mesh axis of size D, so each of the D
 * ranks holds 1/D of the layer's weights and 1/D of the sequence.  Paragraph 2
 * of the same page gives the schedule: attention weight shards are broadcast
 * one after another and applied by every rank to its own tokens, K/V are then
 * all-gathered under a zigzag token partition, and the MLP weight shards travel
 * a ring so that partial sums stay on their rank (no all-reduce).  Here the D
 * ranks are virtual ranks of one GPU: a broadcast, an all-gather or a ring step
 * becomes the choice of which shard, or which K/V rows, a tile reads.
 *
 * The layer (one dense pre-norm decoder layer, batch 1, no bias, no positional
 * encoding):
 *     a = RMSNorm(x; g1)            eps = 1e-5 inside the square root
 *     [Q|K|V] = a Wqkv^T            Wqkv rows: Q heads 0..H-1, then K, then V
 *     O = causal softmax(Q K^T / sqrt(dh)) V     per head, key <= query
 *     y = x + O Wo^T
 *     b = RMSNorm(y; g2)
 *     z = y + GELU_tanh(b W1^T) W2^T
 *
 * Conventions shared by every call.
 *   - Weights use the [out, in] row-major layout of a linear layer, bf16:
 *     wqkv [3h][h], wo [h][h], w1 [F][h], w2 [h][F].  Gains g1, g2: float32 [h].
 *   - Activations are row-major [tokens][features] in RANK-MAJOR ZIGZAG order:
 *     rank 0's L = S/D tokens, then rank 1's, ...  Row r*L+i holds global token
 *     tsp_zigzag_map()[r*L+i].  The caller permutes with that map.
 *   - The caller owns and allocates every buffer; the library never allocates
 *     or frees caller memory.  The plan owns its host metadata and a few small
 *     device tables, created on first use and freed by tsp_plan_destroy.
 *   - Device pointers must be 16-byte aligned (TSP_ERR_ALIGNMENT otherwise).
 *   - Outputs are overwritten, never accumulated into.
 *   - Layer calls are asynchronous on `stream` (a cudaStream_t, may be 0).
 *     Argument errors are reported synchronously and enqueue nothing.
 *   - A bounded device-side wait that ran out sets a flag in the plan; it is
 *     reported as TSP_ERR_TIMEOUT by tsp_sync_status() (layer calls do not
 *     read it: that would block on the device).  Kernels never spin without
 *     a limit.
 *   - Arithmetic: inputs and the outputs y, dx are bf16, gradients of weights
 *     and gains fp32.  Every tensor-core operand the layer computes itself
 *     (a, Q, K, V, P, O, b, GELU output, and the backward's dU, dy, dO, dS,
 *     dQ, dK, dV) is stored as fp16, whose rounding is 8x finer than bf16's,
 *     and multiplied in fp16 x fp16 MMAs at the same rate, with fp32
 *     accumulation.  bf16 weights and dY enter as exact fp16 copies scaled by
 *     powers of two chosen from their largest magnitudes (the scales are
 *     undone exactly in the epilogues); the backward runs on dY times such a
 *     power of two, so gradients of any magnitude sit inside fp16's range.  A
 *     value too large for an fp16 intermediate sets a flag in the plan,
 *     reported as TSP_ERR_RANGE by tsp_sync_status().
 */
#ifndef TSP_H
#define TSP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct tsp_plan_s *tsp_plan_t; /* opaque, host-owned */

typedef enum {
    TSP_OK = 0,
    TSP_ERR_INVALID_ARG = 1, /* NULL pointer, non-positive size, bad phase */
    TSP_ERR_INDIVISIBLE = 2, /* S % 2D, heads % D, ffn % D or h % heads != 0 */
    TSP_ERR_UNSUPPORTED = 3, /* shape outside the kernels' tiling, or device is not sm_100 */
    TSP_ERR_ALIGNMENT = 4,   /* a device pointer is not 16-byte aligned */
    TSP_ERR_CUDA = 5,        /* a CUDA runtime call or kernel launch failed */
    TSP_ERR_TIMEOUT = 6,     /* a bounded device-side wait expired */
    TSP_ERR_RANGE = 7        /* a computed value overflowed its fp16 intermediate (|v| >= 65520) */
} tsp_status;

/* Build a plan for one layer: hidden size h, `heads` attention heads (head size
 * dh = h/heads, Q and K/V heads equal), FFN width `ffn`, S tokens, D virtual
 * ranks.  Divisibility follows from the partition (2D zigzag chunks, heads and
 * FFN units split D ways): TSP_ERR_INDIVISIBLE if S % (2D), heads % D,
 * ffn % D or h % heads is non-zero.  TSP_ERR_UNSUPPORTED when the shape is
 * outside what the kernels tile: dh not in {32, 64, 128}, h % 128, S % 256,
 * (S/D) % 128, ffn % 128 or (ffn/D) % 64 non-zero; and when it is too large
 * for their 32-bit thread numbering: S > 2^28 or heads * S > 67,108,856
 * (S up to about 2.1 million tokens at 32 heads).  Needs no GPU.
 * On success *out receives a new plan. */
tsp_status tsp_plan(int h, int heads, int ffn, int64_t S, int D, tsp_plan_t *out);

/* Free a plan and its device tables.  NULL is ignored.  Not while a layer call
 * that uses the plan is still running on the GPU. */
void tsp_plan_destroy(tsp_plan_t plan);

/* Zigzag token partition ("Zyphra TSP folds TP+SP onto one GPU axis",
 * zubnet.ai, paragraph 2: zigzag partition of K/V for load balance).  The
 * sequence is cut into 2D chunks of c = S/(2D) tokens and rank r owns chunks r
 * and 2D-1-r, in ascending order, so every rank sees the same number of causal
 * (query, key) pairs.  Writes S int32 values to host memory:
 * map_host[r*L + i] = global position of rank r's i-th token.  Needs no GPU. */
tsp_status tsp_zigzag_map(tsp_plan_t plan, int32_t *map_host);

/* Shard schedule of one phase (same page, paragraph 2), D x D int32 to host
 * memory, sched_host[t*D + r] = shard that rank r applies at step t.
 * phase 0: attention broadcast, shard t at step t on every rank.
 * phase 1: MLP ring, rank r holds shard (r + t) mod D (it starts with its own
 * shard and receives rank r+1's after each step).  Attention shard t is heads
 * [t*H/D, (t+1)*H/D); MLP shard s is FFN units [s*F/D, (s+1)*F/D).
 * TSP_ERR_INVALID_ARG for another phase.  Needs no GPU. */
tsp_status tsp_shard_schedule(tsp_plan_t plan, int phase, int32_t *sched_host);

/* Bytes of device memory the layer calls need.
 *   training != 0: *saved_bytes = activations kept from forward to backward,
 *                  *ws_bytes = scratch of either call.
 *   training == 0: *saved_bytes = 0, *ws_bytes = scratch of an inference
 *                  forward (pass saved = NULL).
 * Either output pointer may be NULL.  Needs no GPU. */
tsp_status tsp_workspace_size(tsp_plan_t plan, int training, size_t *ws_bytes, size_t *saved_bytes);

/* Forward of the folded layer.  Device pointers:
 *   x    bf16 [S][h] rank-major zigzag order (input)
 *   g1, g2 float32 [h]; wqkv, wo, w1, w2 bf16 as above (inputs)
 *   y    bf16 [S][h] rank-major zigzag order (output z of the layer)
 *   saved  NULL for inference, else saved_bytes for tsp_layer_backward
 *   ws     ws_bytes of scratch (its contents are not kept)
 * Steps on the GPU: RMSNorm1; QKV projection over the attention shards in
 * broadcast order, whose epilogue writes K and V at their global rows (the
 * all-gather); causal attention of local queries over the gathered K/V;
 * out-projection with head-group partial sums in broadcast order plus the
 * residual; RMSNorm2; W1 with GELU; W2 with its K loop over FFN shards in ring
 * order (r+t) mod D, partial sums in the rank's fp32 accumulator, plus the
 * residual.  fp16 tensor-core operands (see Arithmetic above), fp32
 * accumulation, fp32 residual stream.  With `saved`, the fp16 weight copies
 * are kept there for tsp_layer_backward. */
tsp_status tsp_layer_forward(tsp_plan_t plan, const void *x, const float *g1, const void *wqkv,
                             const void *wo, const float *g2, const void *w1, const void *w2,
                             void *y, void *saved, void *ws, void *stream);

/* Inference prefill: the forward above without training state, keeping the
 * layer's keys and values as a cache for later decoding.  The review page
 * "Zyphra TSP: 2.6x Faster AI Training Review" (What's New) extends the
 * method's benefits to inference; this is the forward run for that use.
 * Device pointers:
 *   x, g1, wqkv, wo, g2, w1, w2, y  as for tsp_layer_forward
 *   k_cache, v_cache  fp16 [S][h] each (outputs, owned by the caller): the
 *       keys and values of all S tokens in GLOBAL position order (row p =
 *       token at position p, the all-gathered layout), head n in columns
 *       [n*dh, (n+1)*dh).  The attention of this call reads them there.
 *   ws  the ws_bytes that tsp_workspace_size(plan, 0, ...) reports (scratch)
 * Same kernels and arithmetic as tsp_layer_forward with saved = NULL, so y is
 * identical to that call's output and the caches hold exactly the K and V it
 * computes.  Errors: TSP_ERR_INVALID_ARG for a NULL pointer,
 * TSP_ERR_ALIGNMENT unless every pointer is 16-byte aligned (both checked
 * before anything is enqueued), TSP_ERR_UNSUPPORTED off sm_100, TSP_ERR_CUDA
 * for a failed launch. */
tsp_status tsp_layer_prefill(tsp_plan_t plan, const void *x, const float *g1, const void *wqkv,
                             const void *wo, const float *g2, const void *w1, const void *w2,
                             void *y, void *k_cache, void *v_cache, void *ws, void *stream);

/* The MLP alone, in the ring schedule with no all-reduce.  The zubnet.ai page
 * "Zyphra TSP folds TP+SP onto one GPU axis, 2.6x throughput on 1,024
 * MI300Xs" (paragraph 4) calls this part of the method worth taking on its
 * own into an existing tensor-parallel setup; it is steps W1 + GELU and W2 of
 * tsp_layer_forward on caller buffers.  For every virtual rank r (rows
 * [r*L, (r+1)*L) of the rank-major layout):
 *   out_r = resid_r + sum_{t=0}^{D-1} GELU_tanh(b_r W1[s_t]^T) W2[:, s_t]^T,
 *   s_t = (r + t) mod D (FFN shard s_t = units [s_t*F/D, (s_t+1)*F/D)),
 * the partial sums staying in the rank's fp32 accumulator.  Device pointers:
 *   b      bf16 [S][h], rank-major (input, the normalised activations; copied
 *          to fp16 unscaled, so |b| must stay below 65520: TSP_ERR_RANGE)
 *   w1     bf16 [F][h]; w2 bf16 [h][F] (inputs, copied to scaled fp16)
 *   resid  float32 [S][h], rank-major (input; pass zeros for no residual)
 *   out    bf16 [S][h], rank-major (output)
 *   ws     tsp_ring_mlp_workspace_size bytes of scratch (holds U, G and the
 *          fp16 copies)
 * Errors: TSP_ERR_INVALID_ARG for a NULL pointer, TSP_ERR_ALIGNMENT unless
 * every pointer is 16-byte aligned (both before anything is enqueued),
 * TSP_ERR_UNSUPPORTED off sm_100, TSP_ERR_CUDA for a failed launch. */
tsp_status tsp_ring_mlp_workspace_size(tsp_plan_t plan, size_t *ws_bytes);
tsp_status tsp_ring_mlp_forward(tsp_plan_t plan, const void *b, const void *w1, const void *w2,
                                const float *resid, void *out, void *ws, void *stream);

/* Backward of the folded layer (exact gradient of the forward; the pages give
 * no backward schedule, so it runs the forward's collectives in reverse:
 * weight-gradient pieces are summed over ranks in rank order, and key/value
 * gradients are summed over every rank's queries and written back at the
 * owning rank's rows).  Device pointers:
 *   dy   bf16 [S][h] upstream gradient of the layer output, rank-major order
 *   x, g1, wqkv, wo, g2, w1, w2  the forward's inputs (the weights' fp16
 *          copies that the forward kept in `saved` are what the MMAs read)
 *   saved  the buffer filled by tsp_layer_forward with the same inputs
 *   ws     ws_bytes of scratch
 * Outputs: dx bf16 [S][h] rank-major order; dg1, dg2 float32 [h];
 *   dwqkv float32 [3h][h], dwo float32 [h][h], dw1 float32 [F][h],
 *   dw2 float32 [h][F]. */
tsp_status tsp_layer_backward(tsp_plan_t plan, const void *dy, const void *x, const float *g1,
                              const void *wqkv, const void *wo, const float *g2, const void *w1,
                              const void *w2, const void *saved, void *ws, void *dx, float *dg1,
                              float *dwqkv, float *dwo, float *dg2, float *dw1, float *dw2,
                              void *stream);

/* A stack of `layers` folded layers with activation recompute: the model the
 * pages measure is such a stack (a 7B decoder of 32 of these layers, zubnet.ai
 * page "Zyphra TSP folds TP+SP onto one GPU axis, 2.6x throughput on 1,024
 * MI300Xs", paragraph 1).  Layer i has its own weights and gains; the host
 * arrays g1[i], wqkv[i], ... hold `layers` device pointers each (layouts as
 * for tsp_layer_forward).  Between layers the activations and gradients are
 * bf16 [S][h] in rank-major zigzag order, as at the layer's own boundary.
 *
 * tsp_stack_workspace_size: bytes of
 *   ws      scratch of one layer call plus three bf16 [S][h] tensors
 *   saved   one layer's saved intermediates (as tsp_workspace_size)
 *   inputs  the inputs of layers 1 .. layers-1, bf16 [layers-1][S][h]
 * Needs no GPU.  TSP_ERR_INVALID_ARG for layers < 1. */
tsp_status tsp_stack_workspace_size(tsp_plan_t plan, int layers, size_t *ws_bytes, size_t *saved_bytes,
                                    size_t *inputs_bytes);

/* Forward of the stack: z = layer_{L-1}( ... layer_0(x)).  With `saved`
 * (training) every layer's input except the first is kept in `inputs` and
 * the last layer's intermediates in `saved`, for tsp_stack_backward; with
 * saved = NULL (inference) `inputs` is not used and the layers' outputs go
 * through the scratch at the end of `ws`.  Device pointers x, z bf16 [S][h];
 * ws, saved, inputs of tsp_stack_workspace_size's sizes.  Errors as for
 * tsp_layer_forward, and TSP_ERR_INVALID_ARG for layers < 1, a NULL pointer
 * in a weight array, or saved without inputs when layers > 1. */
tsp_status tsp_stack_forward(tsp_plan_t plan, int layers, const void *x, const float *const *g1,
                             const void *const *wqkv, const void *const *wo, const float *const *g2,
                             const void *const *w1, const void *const *w2, void *z, void *inputs, void *saved,
                             void *ws, void *stream);

/* Backward of the stack after a training tsp_stack_forward with the same
 * pointers: from the last layer down, every layer but the last is run
 * forward again from its kept input (activation recompute, into `saved`),
 * then backward; the gradient of a layer's input is the next lower layer's
 * output gradient (bf16 [S][h], two scratch tensors in turn at the end of
 * `ws`).  Device pointers: dz bf16 [S][h] (gradient of z, input); dx bf16
 * [S][h] (output); per-layer gradient arrays dg1[i], dwqkv[i], dwo[i], dg2[i],
 * dw1[i], dw2[i] as for tsp_layer_backward (outputs, overwritten).  `saved`
 * is overwritten.  Errors as for tsp_layer_backward, and TSP_ERR_INVALID_ARG
 * for layers < 1, a NULL pointer in an array, or inputs = NULL when
 * layers > 1. */
tsp_status tsp_stack_backward(tsp_plan_t plan, int layers, const void *dz, const void *x, const float *const *g1,
                              const void *const *wqkv, const void *const *wo, const float *const *g2,
                              const void *const *w1, const void *const *w2, const void *inputs, void *saved,
                              void *ws, void *dx, float *const *dg1, float *const *dwqkv, float *const *dwo,
                              float *const *dg2, float *const *dw1, float *const *dw2, void *stream);

/* One rank's share of the forward, for running the folded layer on D
 * devices, one virtual rank each ("Zyphra TSP folds TP+SP onto one GPU axis,
 * 2.6x throughput on 1,024 MI300Xs", zubnet.ai, paragraphs 1-2).  Rank r
 * holds its L = S/D tokens (rows [r*L, (r+1)*L) of the rank-major layout)
 * and runs two calls, with the K/V all-gather between them:
 *
 * tsp_rank_workspace_size: bytes of one rank's workspace (its rows of every
 * intermediate, the LSE of all S local rows, the fp16 weight copies).
 *
 * tsp_rank_forward_qkv: RMSNorm1 of the rank's tokens x (bf16 [L][h]) and
 * their projection onto every attention shard (the whole Wqkv, bf16 [3h][h]:
 * the shards the broadcast schedule delivers, all present on the device).  Q
 * stays in ws; K and V are written into k, v (fp16 [S][h], global position
 * order) at the positions of the rank's own tokens only: the rank's
 * contribution to the all-gather.
 *
 * Between the calls the caller all-gathers K and V so that every rank's k, v
 * hold all S rows.  Rank j's rows are the positions of its two zigzag chunks,
 * [j*c, (j+1)*c) and [(2D-1-j)*c, (2D-j)*c), c = S/(2D): two all-gathers of
 * c-row blocks per tensor put every block in place.
 *
 * tsp_rank_forward_out: causal attention of the rank's queries over all S
 * keys, the out-projection + residual, RMSNorm2, W1 with GELU, and W2 with its
 * K loop over the FFN shards in the rank's ring order (rank + t) mod D (the
 * shards the ring delivers, all present: wo, w1, w2 whole) + residual, into z
 * (bf16 [L][h]).  x is the same rank's tokens as in the first call.
 *
 * The same kernels as tsp_layer_forward on the rank's rows, so the D ranks'
 * z rows are bit for bit the layer's.  Errors: TSP_ERR_INVALID_ARG for a rank
 * outside [0, D) or a NULL pointer, TSP_ERR_ALIGNMENT unless every pointer is
 * 16-byte aligned, TSP_ERR_UNSUPPORTED when L is not a multiple of 256 (the
 * attention's query items are 256-row blocks) or off sm_100, TSP_ERR_CUDA for
 * a failed launch; argument errors are found before anything is enqueued. */
tsp_status tsp_rank_workspace_size(tsp_plan_t plan, size_t *ws_bytes);
tsp_status tsp_rank_forward_qkv(tsp_plan_t plan, int rank, const void *x, const float *g1, const void *wqkv,
                                void *k, void *v, void *ws, void *stream);
tsp_status tsp_rank_forward_out(tsp_plan_t plan, int rank, const void *x, const void *k, const void *v,
                                const void *wo, const float *g2, const void *w1, const void *w2, void *z, void *ws,
                                void *stream);

/* One rank's share of the backward, after that rank's two forward calls with
 * the same ws, k and v (the workspace keeps the rank's activations, the
 * gathered K/V stay in k, v).  Head size 128 only.  Two calls, with the dK/dV
 * reduce-scatter between them:
 *
 * tsp_rank_backward_workspace_size: bytes of one rank's backward scratch bws.
 *
 * tsp_rank_backward_attn: from dz (bf16 [L][h], gradient of the rank's z
 * rows): the MLP backward (dW2, dW1 with the rank's rows as the contraction;
 * db with its K loop in the rank's ring order), RMSNorm2 backward (dg2), the
 * out-projection backward (dWo, dO) and the attention backward of the rank's
 * query rows over all S keys: dQ of its rows stays in bws, and its share of
 * dK and dV for every key goes out as fp32 partial sums into dk_part, dv_part
 * ([S][h], rank-major local rows of the key's owner; overwritten, keys the
 * rank's rows do not see are zero).  dwo [h][h], dg2 [h], dw1 [F][h], dw2
 * [h][F] (fp32, overwritten) are the sums over this rank's rows only.
 *
 * Between the calls the caller sums dk_part and dv_part over the ranks and
 * hands each rank its rows: a reduce-scatter of the S rows into L-row blocks
 * (block j to rank j), since the partial rows are already in rank-major
 * order.
 *
 * tsp_rank_backward_qkv: with dk, dv (fp32 [L][h], the reduced dK, dV of the
 * rank's own rows): the QKV projection backward (dWqkv [3h][h], this rank's
 * rows only) and RMSNorm1 backward + residual into dx (bf16 [L][h]) and dg1
 * [h] (this rank's rows only).  x, g1 as in the forward.
 *
 * The caller then sums dwqkv, dwo, dw1, dw2, dg1 and dg2 over the ranks
 * (all-reduce).  The gradient scale 2^k of a rank comes from its own max|dz|,
 * and the dK/dV it receives are converted into that rank's fp16 domain: a sum
 * past fp16's range there (dz of very different magnitudes across ranks)
 * is reported as TSP_ERR_RANGE by tsp_sync_status, never silently clipped.
 * Up to rounding the results are the layer backward's on the rank's rows
 * (the layer takes one scale from all rows, the fixed-point dQ sum its bound
 * from all rows, and the dK/dV partials are summed in fp32 before the fp16
 * rounding).  Errors as for the forward calls, and TSP_ERR_UNSUPPORTED for a
 * head size other than 128. */
tsp_status tsp_rank_backward_workspace_size(tsp_plan_t plan, size_t *bws_bytes);
tsp_status tsp_rank_backward_attn(tsp_plan_t plan, int rank, const void *dz, const void *k, const void *v,
                                  const float *g2, void *ws, void *bws, float *dk_part, float *dv_part, float *dwo,
                                  float *dg2, float *dw1, float *dw2, void *stream);
tsp_status tsp_rank_backward_qkv(tsp_plan_t plan, int rank, const void *x, const float *g1, const float *dk,
                                 const float *dv, void *ws, void *bws, void *dx, float *dg1, float *dwqkv,
                                 void *stream);

/* Wait for `stream`, then report TSP_ERR_CUDA for an asynchronous CUDA error,
 * TSP_ERR_TIMEOUT if a device-side wait of this plan ran out, or TSP_ERR_RANGE
 * if a value overflowed an fp16 intermediate (the flags are cleared by the
 * report). */
tsp_status tsp_sync_status(tsp_plan_t plan, void *stream);

/* Static, human-readable name of a status. */
const char *tsp_status_string(tsp_status status);

/* Kernel stages of one forward + backward (profiling ids): 0-6 the forward
 * and 7-19 the backward in launch order; 20 the forward's weight conversion
 * (first in the forward) and 21 the backward's dY conversion (first in the
 * backward).  With head size 128 the attention backward is one pass, stage
 * 22 (dK, dV and the fp32 dQ sum) and stage 23 (dQ to fp16), in place of
 * stages 15 and 16.  Stage 24 is the per-rank backward's conversion of the
 * reduced dK/dV into fp16 (tsp_rank_backward_qkv). */
#define TSP_NUM_STAGES 25

/* Per-stage timing with CUDA events.  tsp_profile_enable(plan, 1) clears the
 * record and starts bracketing every stage of later layer calls with a pair of
 * events on the call's stream; 0 stops.  tsp_profile_read waits for the
 * recorded events of one stage (0 <= stage < TSP_NUM_STAGES) and returns its
 * static name, the summed elapsed milliseconds, the number of calls recorded
 * and the kernel launches they made.  Any output pointer may be NULL. */
tsp_status tsp_profile_enable(tsp_plan_t plan, int enable);
tsp_status tsp_profile_read(tsp_plan_t plan, int stage, const char **name, double *total_ms, int64_t *calls,
                            int64_t *kernel_launches);

/* Kernels this plan has launched since it was created (every layer call adds
 * 9 for a forward and 17 for a backward). */
int64_t tsp_kernel_launches(tsp_plan_t plan);

/* RMSNorm backward plus residual that allocates nothing.  The TSP pages have
 * no counterpart: this is a library convenience.  It computes what the last
 * stage of tsp_layer_backward computes for RMSNorm1:
 *     n = x * rstd,   dn = dout * g,
 *     dx = resid + rstd * (dn - n * mean(dn * n))      (bf16 out)
 *     dg = sum over rows of dout * n                    (float32 out)
 * for callers that cannot allocate device memory (no cudaMalloc allowed in
 * their context, or no memory pool to draw scratch from).  The per-block
 * partial sums of dg live in a 16 MiB device array owned by the library, which
 * every GPU that loads the library holds until the process exits; the call
 * needs only its inputs and outputs.  Device pointers, 16-byte aligned:
 *   dout  float32 [rows][h]  gradient reaching the normalised output
 *   x     bf16    [rows][h]  the normalised input
 *   rstd  float32 [rows]     1/sqrt(mean(x^2) + eps) from the forward
 *   g     float32 [h]        gain
 *   resid float32 [rows][h]  gradient reaching x through the residual branch
 *   dx    bf16    [rows][h]  output
 *   dg    float32 [h]        output
 * Limits: h % 128 == 0 and ceil(rows / 64) * h <= 4,194,304; beyond them the
 * call returns TSP_ERR_UNSUPPORTED and enqueues nothing.  The first call on a
 * device looks up the array's device address with that device current; make
 * that first call before any stream capture.  All calls share the one array:
 * calls that overlap on the GPU (on different streams or from different host
 * threads) race, so the caller must order them.  Nothing in the array needs
 * clearing between calls, since each call writes every slot it reads.
 * Asynchronous on `stream`. */
tsp_status tsp_rmsnorm_backward_noalloc(const float *dout, const void *x, const float *rstd, const float *g,
                                        const float *resid, void *dx, float *dg, int rows, int h, void *stream);

/* Algorithmic floating-point work of one call, counting causal attention
 * pairs only and no recompute: forward = 2S(4h^2 + 2hF) + 2hS(S+1);
 * backward = 2 x forward.  Needs no GPU. */
double tsp_layer_flops(tsp_plan_t plan, int backward);

#ifdef __cplusplus
}
#endif

#endif /* TSP_H */
