// Internal (not exported) interfaces between the host plan and the kernel
// translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace tsp {

struct DevErr;

// Epilogues of the GEMM (row = thread's output row, acc = fp32 accumulator
// times the descriptor's alpha; "h" = the operand type of the GEMM: fp16 when
// GemmDesc::f16, else bf16):
enum GemmEpilogue : int {
    EPI_F32 = 0,        // out  f32[row][col] = acc
    EPI_BF16 = 1,       // out bf16[row][col] = acc
    EPI_QKV = 2,        // col < h: out (Q) at local row; h..2h: out_k at rowmap[row]; 2h..3h: out_v likewise (h)
    EPI_RESID_F32 = 3,  // out  f32 = acc + aux bf16 (residual)
    EPI_GELU = 4,       // out bf16 = acc (pre-activation U), out2 h = gelu_tanh(acc)
    EPI_RESID_BF16 = 5, // out bf16 = acc + aux f32 (residual)
    EPI_DGELU = 6,      // out h = acc * gelu_tanh'(aux bf16)
    EPI_F16 = 7,        // out fp16[row][col] = acc
};

// C[M][N] = sum_k A[m][k] B[n][k].
//   a_mn == false: A is [M][K] with row stride lda;  true: A is stored [K][M] (row stride lda).
//   b_mn == false: B is [N][K] with row stride ldb;  true: B is stored [K][N] (row stride ldb).
// M % 128 == 0, K % 64 == 0, N % 128 == 0, pointers 16-byte aligned.
// A and B are both fp16 (f16) or both bf16.  Every fp16 store of an epilogue
// checks for overflow and sets kErrRange in the error word.
struct GemmDesc {
    const void *A;
    int64_t lda;
    bool a_mn;
    const void *B;
    int64_t ldb;
    bool b_mn;
    int M, N, K;
    int epi;
    void *out;
    int64_t ldo;
    void *out2;
    int64_t ldo2;
    const void *aux;
    int64_t ldaux;
    // ring K order: rows of rank ring_rank0 + m / ring_rows start at K block
    // rank * ring_kblocks
    int ring_rows;
    int ring_kblocks;
    int ring_rank0;
    // EPI_QKV only
    const int *rowmap;
    int hsplit;
    void *out_k;
    void *out_v;
    bool force_bn128;
    bool f16;            // operand type: fp16 (else bf16)
    const float *alpha;  // device scalar multiplying the accumulator, or null for 1
};

cudaError_t launch_gemm(const GemmDesc &g, const DevErr &err, int num_sms, cudaStream_t st);

// Tensor-map encoding through the driver entry point (no libcuda link).
bool encode_tensor_map_2d(CUtensorMap *m, const void *base, CUtensorMapDataType dtype, int elem_bytes,
                          int64_t inner, int64_t outer, int64_t outer_stride_bytes, int box_inner, int box_outer,
                          CUtensorMapSwizzle swz);

// RMSNorm forward: out = x * rstd * g, rstd = 1/sqrt(mean(x^2)+eps); out is
// fp16 (overflow reported in err) or bf16 (out_f16 false).  x is bf16
// (x_f32 == nullptr) or f32.
cudaError_t launch_rmsnorm_fwd(const void *x_bf16, const float *x_f32, const float *g, void *out, bool out_f16,
                               float *rstd, int rows, int h, unsigned int *err, cudaStream_t st);

// RMSNorm backward plus residual:
//   n = x*rstd, dn = dout*g, dx = (resid*rm + rstd*(dn - n*mean(dn*n))) * xm,
//   dg = (sum over rows of dout*n) * gm,
// with rm = *resid_mul, xm = *dx_mul, gm = *dg_mul (each 1 when null).
// dout f32; x bf16 or f32; resid bf16 or f32; outputs dx_f32 and/or dx_low
// (bf16, or fp16 when low_f16, overflow reported in err); per-block partial
// sums of dout*n go to dg_partial[nblocks][h] and are reduced (in block order)
// into dg.
struct NormBwd {
    const float *dout;
    const void *x_bf16;
    const float *x_f32;
    const float *rstd;
    const float *g;
    const void *resid_bf16;
    const float *resid_f32;
    float *dx_f32;
    void *dx_low;
    bool low_f16;
    float *dg_partial;
    float *dg;
    const float *resid_mul, *dx_mul, *dg_mul;
    unsigned int *err;
    int rows, h;
};
cudaError_t launch_rmsnorm_bwd(const NormBwd &n, cudaStream_t st);
int rmsnorm_bwd_partial_blocks(int rows);

// bf16 -> fp16 conversion with a power-of-two scale taken from the tensor's
// largest magnitude: dst = fp16(src * 2^e), e chosen so that max|src| * 2^e
// lies in [2^(target-1), 2^target), so every element keeps fp16's full 11-bit
// significand far above its subnormal range.  *scale_inv = 2^-e undoes it in
// a consumer's epilogue; *scale = 2^e.  With target == kNoScale, e = 0 and a
// magnitude fp16 cannot hold sets kErrRange.  Two launches for up to
// kMaxConv tensors: block partial maxima, then the conversion (every block
// reduces the partials itself, so no atomics and no clearing).
constexpr int kNoScale = -1000;
constexpr int kMaxConv = 5;
constexpr int kConvBlocks = 296;  // blocks per tensor (2 per SM)
struct ConvTensor {
    const void *src;   // bf16, n elements, 16-byte aligned
    void *dst;         // fp16, n elements
    int64_t n;         // multiple of 8
    int target;
    float *scale_inv;  // may be null
    float *scale;      // may be null
};
struct ConvBatch {
    ConvTensor t[kMaxConv];
    int count;
    float *partial;    // kMaxConv * kConvBlocks floats of scratch
    unsigned int *err;
};
cudaError_t launch_convert_f16(const ConvBatch &b, cudaStream_t st);
// fp32 [rows][cols] -> fp16 times *mul (device scalar) into rows of stride
// ldd elements (cols, ldd multiples of 8; both pointers 16-byte aligned).
// Test hook: y = 2^x by the attention forward's polynomial (which = 0) or by
// the MUFU approximation (which = 1), n device floats.
cudaError_t launch_exp2_test(const float *x, float *y, int n, int which, cudaStream_t st);
cudaError_t launch_scale_to_f16(const float *src, int64_t rows, int cols, void *dst, int64_t ldd, const float *mul,
                                unsigned int *err, cudaStream_t st);

// Attention.  Q, K, V, O (and dO, dQ, dK, dV in the backward) are fp16.
struct AttnDesc {
    int S, L, D, H, dh, chunk;  // tokens, tokens per rank, ranks, heads, head dim, zigzag chunk
    const void *q;              // fp16 [q_rows][h]: local rows q_row0 .. q_row0 + q_rows - 1
    const void *k, *v;          // fp16 [S][h] global rows
    void *o;                    // fp16 [q_rows][h], rows as q
    float *lse;                 // f32 [H][S] local rows, log2 domain (scores pre-multiplied by log2 e / sqrt(dh))
    const int *order;           // pairs (qblock * H + head, number of 128-key tiles), in paired waves
    int num_items;
    int q_row0, q_rows;         // the local rows Q and O hold (0 and S for the whole layer)
};
cudaError_t launch_attn_fwd(const AttnDesc &a, const DevErr &err, int num_sms, cudaStream_t st);

// First local 64-row query step q >= from whose largest global position is at
// least kv0 (so at least one of its rows sees key kv0), or nq64 when there is
// none.  The local rows of rank r are its low zigzag chunk r followed by its
// high chunk 2D - 1 - r, each `chunk` rows (a multiple of 64) with ascending
// positions; so every step lies in one chunk, and within a chunk the steps
// that see kv0 form a suffix.  At most 2D chunks are examined.
__host__ __device__ inline int zz_next_visible(int from, int kv0, int D, int chunk, int nq64) {
    const int spc = chunk / 64;  // steps per chunk
    for (int lc = from / spc; lc < 2 * D; ++lc) {
        const int r = lc >> 1;
        const int start = ((lc & 1) ? 2 * D - 1 - r : r) * chunk;  // position of the chunk's first row
        // step t of the chunk ends at position start + 64 t + 63
        const int need = kv0 - 63 - start;
        const int t0 = need <= 0 ? 0 : (need + 63) / 64;
        const int lo = lc * spc;
        const int t = (from > lo ? from - lo : 0) > t0 ? (from > lo ? from - lo : 0) : t0;
        if (t < spc) return lo + t;
    }
    return nq64;
}

// Visibility of 64-row query steps to a key tile, from the zigzag layout.
struct StepVis {
    int D, chunk, nq64;
    int rank = -1;  // >= 0: only the steps of rank `rank` (chunks rank and 2D-1-rank); DescWalk only
};

// Walks the query steps that can see a key tile kv0, in ascending order.
// Within a zigzag chunk the visible steps form a suffix, so after a chunk's
// first visible step every later step of that chunk is visible too: the
// closed form runs once per chunk and a step costs one compare.  Used by the
// dK/dV kernel; host-callable so that tests can replay the walk.
struct StepWalk {
    int q;        // current step; nq64 once the walk is over
    int run_end;  // end (exclusive) of the chunk holding q
    __host__ __device__ inline void seek(const StepVis &v, int from, int kv0) {
        q = zz_next_visible(from, kv0, v.D, v.chunk, v.nq64);
        const int spc = v.chunk >> 6;
        run_end = q < v.nq64 ? (q / spc + 1) * spc : v.nq64;
    }
    __host__ __device__ inline void next(const StepVis &v, int kv0) {
        if (q + 1 < run_end) ++q;
        else seek(v, q + 1, kv0);
    }
};

// Walks the query steps that can see a key tile kv0 in descending order of
// position: position chunks from the last (2D-1) down, each chunk's steps from
// its last down to its lowest visible one.  Every walk is then a prefix of one
// common order (the steps of the highest positions, visible to every key tile,
// come first), so key tiles processed at the same time touch the same query
// rows at about the same time and those rows stay in L2.  Host-callable so
// that tests can replay the walk.
struct DescWalk {
    int q;     // current local step; nq64 once the walk is over
    int pc;    // position chunk of q: positions [pc chunk, (pc + 1) chunk)
    int t;     // step of q within its chunk
    int t_lo;  // lowest step of the chunk that reaches kv0
    __host__ __device__ inline void enter(const StepVis &v, int kv0) {
        const int spc = v.chunk >> 6;
        // step t of chunk pc ends at position pc chunk + 64 t + 63
        const int need = kv0 - 63 - pc * v.chunk;
        t_lo = need <= 0 ? 0 : (need + 63) / 64;
        if (pc < 0 || t_lo >= spc) {  // nothing here, and lower chunks lie lower still
            q = v.nq64;
            return;
        }
        t = spc - 1;
        // local rows: rank r holds chunk r, then chunk 2D-1-r
        const int lc = pc < v.D ? 2 * pc : 2 * (2 * v.D - 1 - pc) + 1;
        q = lc * spc + t;
    }
    __host__ __device__ inline void seek(const StepVis &v, int kv0) {
        pc = 2 * v.D - 1 - (v.rank < 0 ? 0 : v.rank);
        enter(v, kv0);
    }
    __host__ __device__ inline void next(const StepVis &v, int kv0) {
        if (t > t_lo) {
            --t;
            --q;
        } else {
            pc = v.rank < 0 ? pc - 1 : (pc == 2 * v.D - 1 - v.rank ? v.rank : -1);
            enter(v, kv0);
        }
    }
};

struct AttnBwdDesc {
    int S, L, D, H, dh, chunk;
    const void *q, *k, *v, *o, *dout;  // q, o, dout local rows; k, v global rows
    const float *lse;                  // as written by the forward
    float *delta;                      // f32 [H][S] scratch: rowsum(dO * O) per head, local rows
    void *dq;                          // fp16, row stride ldd, local rows
    void *dk, *dv;                     // fp16, row stride ldd, local rows of the key's owner
    unsigned int *err;                 // error word (fp16 overflow of dQ, dK, dV)
    int64_t ldd;
    const int *inv_map;                // global position -> local row
    const int *kv_order;               // work order of (head, 128-key block), in paired waves
    const int *q_order;                // work order of (head, 128-row query block), longest first per head
    int *dq_acc;                       // [S][h] scratch: dQ summed over key tiles in 32-bit fixed point
                                       // (single-pass kernel; zeroed by the Delta kernel), or null
    unsigned int *dq_bound;            // [H][3] scratch: per-head maxima bounding that sum (Delta kernel)
    // Query-row window: q, o, dout, dq and dq_acc hold the q_rows local rows
    // starting at local row q_row0 (the whole layer: 0 and S).  lse and delta
    // stay [H][S], indexed by local row.
    int q_row0, q_rows;
    // One rank's share (single-pass kernel only): rank >= 0 walks only the
    // query steps of that rank's rows, kv_order holds only the key tiles
    // those rows see, and dK / dV go out as fp32 partial sums times *dkv_mul
    // into dk_part / dv_part ([S][h], local rows of the key's owner, zeroed
    // by the launcher) instead of dk / dv.
    int rank;
    int kv_items;                      // entries of kv_order
    float *dk_part, *dv_part;
    const float *dkv_mul;
};
// Delta = rowsum(dO * O) per head; then dK/dV (key-tile items, 64-row query
// steps, visibility from zz_next_visible) and dQ (query-tile items).  zig:
// local row -> global position; qtile_maxpos: largest position of each
// 128-row local query tile.
cudaError_t launch_attn_delta(const AttnBwdDesc &a, int num_sms, cudaStream_t st);
cudaError_t launch_attn_dkdv(const AttnBwdDesc &a, const DevErr &err, int num_sms, cudaStream_t st, const int *zig);
cudaError_t launch_attn_dq(const AttnBwdDesc &a, const DevErr &err, int num_sms, cudaStream_t st, const int *zig,
                           const int *qtile_maxpos);
// Single-pass backward for dh = 128: dK, dV and the fixed-point dQ sum
// (dq_acc, integer additions: deterministic in any order) in one kernel over
// (head, 128-key tile) items; then dQ = dq_acc / sqrt(dh) as fp16 into a.dq.
bool attn_bwd_fused_supported(int dh);
cudaError_t launch_attn_bwd_fused(const AttnBwdDesc &a, const DevErr &err, int num_sms, cudaStream_t st,
                                  const int *zig);
cudaError_t launch_dq_convert(const AttnBwdDesc &a, cudaStream_t st);

}  // namespace tsp
