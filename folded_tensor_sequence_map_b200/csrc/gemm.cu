// Persistent tcgen05 GEMM for sm_100a with the layer's fused epilogues.
//
//   C[m, n] = alpha * sum_k A[m, k] * B[n, k]
//   fp16 (or bf16) operands, fp32 accumulator in TMEM; alpha is a device
//   scalar, the power of two that undoes an operand's conversion scale.
//
// A is either K-major ([M][K] rows) or MN-major ([K][M] rows, i.e. A^T stored
// row-major); the same for B.  The projections of the forward are K-major x
// K-major; data gradients (X W) are K-major x MN-major; weight gradients
// (X^T Y, contraction over tokens) are MN-major x MN-major.
//
// One CTA per SM, 6 warps:
//   warp 0      TMA producer (one elected lane): A and B tiles of BK = 64 into a
//               STAGES-deep ring of 128B-swizzled shared-memory buffers;
//   warp 1      TMEM owner and MMA issuer (one lane): 4 MMAs of 128 x BN x 16
//               per stage into one of two TMEM accumulators;
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (thread = row), the
//               fused element-wise step, and the global store; it overlaps the
//               next tile's main loop through the second accumulator.
//
// Folded-layer specifics live in the tile scheduler and the epilogue:
//   * ring K order: when ring_rows > 0, the K loop of the rows of rank
//     r = ring_rank0 + m0 / ring_rows starts at shard r's first K block and
//     wraps around (ring_rank0: the rank of row 0, for a GEMM over one
//     rank's rows),
//     so the partial sums over FFN shards are added in ring order (r+t) mod D
//     inside the rank's own accumulator ("Zyphra TSP folds TP+SP onto one GPU
//     axis", zubnet.ai, paragraph 2: the MLP ring removes the all-reduce);
//   * QKV epilogue: Q columns go to the rank-local rows, K/V columns go to the
//     token's global row (the K/V all-gather of the same paragraph).
#include "common.cuh"
#include "internal.h"

namespace tsp {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kThreads = 192;
constexpr int kGroupM = 16;  // rasterisation: 16 row blocks share each B column sweep

struct GemmArgs {
    int M, N, K;
    int ring_rows, ring_kblocks, ring_rank0;
    int epi;
    void *out;
    int64_t ldo;
    void *out2;
    int64_t ldo2;
    const void *aux;
    int64_t ldaux;
    const int *rowmap;
    int hsplit;
    void *out_k;
    void *out_v;
    const float *alpha;
    uint32_t idesc;  // instruction descriptor (operand type, majors, 128 x BN)
    bool f16;        // fp16 operands, and fp16 for the "h" outputs of the epilogues
    DevErr err;
};

template <int BN>
struct Cfg {
    static constexpr int STAGES = (BN == 256) ? 4 : 6;
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_BYTES = BN * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int TMEM_COLS = 2 * BN;
    static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
    static_assert(SMEM <= kMaxDynSmem, "GEMM stages exceed the shared-memory limit");
    // full/empty[STAGES], acc_full/empty[2], TMEM slot + abort flag, spare, drain
    static_assert(8 * (2 * STAGES + 7) <= 256, "GEMM barriers exceed their slot");
};

__device__ __forceinline__ void tile_coords(int t, int mt, int nt, int &mb, int &nb) {
    int group = t / (kGroupM * nt);
    int first = group * kGroupM;
    int gm = min(kGroupM, mt - first);
    int idx = t - group * kGroupM * nt;
    nb = idx / gm;
    mb = first + idx % gm;
}

// Bounded wait that ignores the abort flag: used while draining at exit.
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity, long long limit) {
    long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > limit) return;
    }
}

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16 *dst, const float (&v)[32]) {
    uint4 *d = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint4 w;
        w.x = pack_bf16(v[8 * j + 0], v[8 * j + 1]);
        w.y = pack_bf16(v[8 * j + 2], v[8 * j + 3]);
        w.z = pack_bf16(v[8 * j + 4], v[8 * j + 5]);
        w.w = pack_bf16(v[8 * j + 6], v[8 * j + 7]);
        d[j] = w;
    }
}
// fp16 store of 32 values; an overflow is reported, not hidden.
__device__ __forceinline__ void store_f16x32(__half *dst, const float (&v)[32], unsigned int *err) {
    flag_range(maxabs32(v), err);
    uint4 *d = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint4 w;
        w.x = pack_f16(v[8 * j + 0], v[8 * j + 1]);
        w.y = pack_f16(v[8 * j + 2], v[8 * j + 3]);
        w.z = pack_f16(v[8 * j + 4], v[8 * j + 5]);
        w.w = pack_f16(v[8 * j + 6], v[8 * j + 7]);
        d[j] = w;
    }
}
// Store in the GEMM's operand type (fp16 or bf16).
__device__ __forceinline__ void store_hx32(bool f16, void *base, int64_t off, const float (&v)[32],
                                           unsigned int *err) {
    if (f16)
        store_f16x32(static_cast<__half *>(base) + off, v, err);
    else
        store_bf16x32(static_cast<__nv_bfloat16 *>(base) + off, v);
}

__device__ __forceinline__ void load_bf16x32(const __nv_bfloat16 *src, float (&v)[32]) {
    const uint4 *s = reinterpret_cast<const uint4 *>(src);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint4 w = s[j];
        v[8 * j + 0] = bf16_lo(w.x);
        v[8 * j + 1] = bf16_hi(w.x);
        v[8 * j + 2] = bf16_lo(w.y);
        v[8 * j + 3] = bf16_hi(w.y);
        v[8 * j + 4] = bf16_lo(w.z);
        v[8 * j + 5] = bf16_hi(w.z);
        v[8 * j + 6] = bf16_lo(w.w);
        v[8 * j + 7] = bf16_hi(w.w);
    }
}

__device__ __forceinline__ void epilogue_chunk(const GemmArgs &p, int row, int col, float (&v)[32]) {
    const int64_t r = row;
    switch (p.epi) {
        case EPI_F32: {
            float4 *d = reinterpret_cast<float4 *>(static_cast<float *>(p.out) + r * p.ldo + col);
#pragma unroll
            for (int j = 0; j < 8; ++j) d[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
            break;
        }
        case EPI_BF16:
            store_bf16x32(static_cast<__nv_bfloat16 *>(p.out) + r * p.ldo + col, v);
            break;
        case EPI_F16:
            store_f16x32(static_cast<__half *>(p.out) + r * p.ldo + col, v, p.err.word);
            break;
        case EPI_QKV: {
            int which = col / p.hsplit;
            int c = col - which * p.hsplit;
            if (which == 0) {
                store_hx32(p.f16, p.out, r * p.ldo + c, v, p.err.word);
            } else {
                const int64_t g = p.rowmap[row];
                store_hx32(p.f16, which == 1 ? p.out_k : p.out_v, g * p.ldo + c, v, p.err.word);
            }
            break;
        }
        case EPI_RESID_F32: {
            float rs[32];
            load_bf16x32(static_cast<const __nv_bfloat16 *>(p.aux) + r * p.ldaux + col, rs);
            float4 *d = reinterpret_cast<float4 *>(static_cast<float *>(p.out) + r * p.ldo + col);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                d[j] = make_float4(v[4 * j] + rs[4 * j], v[4 * j + 1] + rs[4 * j + 1], v[4 * j + 2] + rs[4 * j + 2],
                                   v[4 * j + 3] + rs[4 * j + 3]);
            break;
        }
        case EPI_GELU: {
            store_bf16x32(static_cast<__nv_bfloat16 *>(p.out) + r * p.ldo + col, v);
            float g[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) g[j] = gelu_tanh(v[j]);
            store_hx32(p.f16, p.out2, r * p.ldo2 + col, g, p.err.word);
            break;
        }
        case EPI_RESID_BF16: {
            const float4 *q4 = reinterpret_cast<const float4 *>(static_cast<const float *>(p.aux) + r * p.ldaux + col);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float4 q = q4[j];
                v[4 * j] += q.x;
                v[4 * j + 1] += q.y;
                v[4 * j + 2] += q.z;
                v[4 * j + 3] += q.w;
            }
            store_bf16x32(static_cast<__nv_bfloat16 *>(p.out) + r * p.ldo + col, v);
            break;
        }
        case EPI_DGELU: {
            float u[32];
            load_bf16x32(static_cast<const __nv_bfloat16 *>(p.aux) + r * p.ldaux + col, u);
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] *= gelu_tanh_grad(u[j]);
            store_hx32(p.f16, p.out, r * p.ldo + col, v, p.err.word);
            break;
        }
        default:
            break;
    }
}

template <int BN, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                const GemmArgs p) {
    using C = Cfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t *sA = smem;
    uint8_t *sB = smem + C::STAGES * C::A_BYTES;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::STAGES * C::STAGE_BYTES);
    uint64_t *empty = full + C::STAGES;
    uint64_t *acc_full = empty + C::STAGES;
    uint64_t *acc_empty = acc_full + 2;
    uint32_t *tmem_base_slot = reinterpret_cast<uint32_t *>(acc_empty + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_base_slot + 1);
    uint64_t *drain_bar = acc_empty + 4;

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int mt = p.M / BM, nt = p.N / BN, nk = p.K / BK;
    const int ntiles = mt * nt;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 128);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&mapA);
        tma_prefetch_desc(&mapB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_base_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_slot;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued_parity[C::STAGES];
            for (int s = 0; s < C::STAGES; ++s) issued_parity[s] = -1;
            bool ok = true;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                int mb, nb;
                tile_coords(t, mt, nt, mb, nb);
                const int m0 = mb * BM, n0 = nb * BN;
                int kstart = 0;
                if (p.ring_rows > 0) kstart = ((m0 / p.ring_rows + p.ring_rank0) * p.ring_kblocks) % nk;
                for (int i = 0; i < nk; ++i) {
                    int kb = kstart + i;
                    if (kb >= nk) kb -= nk;
                    const int k0 = kb * BK;
                    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_tx(&full[stage], C::STAGE_BYTES);
                    issued_parity[stage] = static_cast<int>(phase);
                    uint8_t *a = sA + stage * C::A_BYTES;
                    uint8_t *b = sB + stage * C::B_BYTES;
                    if (A_MN) {
                        tma_load_2d(a, &mapA, &full[stage], m0, k0);
                        tma_load_2d(a + 64 * 128, &mapA, &full[stage], m0 + 64, k0);
                    } else {
                        tma_load_2d(a, &mapA, &full[stage], k0, m0);
                    }
                    if (B_MN) {
#pragma unroll
                        for (int j = 0; j < BN / 64; ++j)
                            tma_load_2d(b + j * 64 * 128, &mapB, &full[stage], n0 + 64 * j, k0);
                    } else {
                        tma_load_2d(b, &mapB, &full[stage], k0, n0);
                    }
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // Every load this thread issued must land before the CTA exits.
            for (int s = 0; s < C::STAGES; ++s)
                if (issued_parity[s] >= 0) drain_wait(&full[s], static_cast<uint32_t>(issued_parity[s]), p.err.wait_limit);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = p.idesc;
            int stage = 0;
            uint32_t phase = 0;
            uint32_t acc_phase[2] = {0, 0};
            int tile_iter = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++tile_iter) {
                const int buf = tile_iter & 1;
                if (!mbar_wait(&acc_empty[buf], acc_phase[buf] ^ 1u, abort_flag, p.err)) break;
                acc_phase[buf] ^= 1u;
                tc_fence_after();
                const uint32_t d = tmem + static_cast<uint32_t>(buf * BN);
                for (int i = 0; i < nk; ++i) {
                    if (!mbar_wait(&full[stage], phase, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a = smem_u32(sA + stage * C::A_BYTES);
                    const uint32_t b = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        uint64_t ad = A_MN ? sdesc(a + kk * 2048, 64 * 128, 1024, kSwizzle128)
                                           : sdesc(a + kk * 32, 16, 1024, kSwizzle128);
                        uint64_t bd = B_MN ? sdesc(b + kk * 2048, 64 * 128, 1024, kSwizzle128)
                                           : sdesc(b + kk * 32, 16, 1024, kSwizzle128);
                        umma_ss(d, ad, bd, idesc, (i | kk) != 0);
                    }
                    umma_commit(&empty[stage]);
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                umma_commit(&acc_full[buf]);
            }
            // No MMA may still be writing TMEM when the CTA frees it: after an
            // abort, wait (bounded) for everything issued so far.
            if (!ok || *abort_flag) {
                umma_commit(drain_bar);
                drain_wait(drain_bar, 0, p.err.wait_limit);
            }
        }
    } else {
        // Epilogue warps 2..5; TMEM lane quarter is fixed by warp % 4.
        const int quarter = warp & 3;
        const int row_in_tile = quarter * 32 + lane;
        const float alpha = p.alpha ? *p.alpha : 1.0f;
        uint32_t acc_phase[2] = {0, 0};
        int tile_iter = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++tile_iter) {
            const int buf = tile_iter & 1;
            int mb, nb;
            tile_coords(t, mt, nt, mb, nb);
            const int m0 = mb * BM, n0 = nb * BN;
            if (!warp_wait(&acc_full[buf], acc_phase[buf], abort_flag, p.err)) break;
            acc_phase[buf] ^= 1u;
            tc_fence_after();
            const uint32_t base = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(buf * BN);
            const int row = m0 + row_in_tile;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                float v[32];
                tmem_ld32(base + c * 32, v);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] *= alpha;
                epilogue_chunk(p, row, n0 + c * 32, v);
            }
            tc_fence_before();
            mbar_arrive(&acc_empty[buf]);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

// Host: a 2D fp16 or bf16 tensor map over a row-major [rows][cols] matrix with
// row stride `ld` elements, box {64 columns, box_rows rows}, 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, int64_t ld, int box_rows, bool f16) {
    return encode_tensor_map_2d(m, base, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                                cols, rows, ld * 2, 64, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int BN, bool A_MN, bool B_MN>
cudaError_t launch_impl(const GemmDesc &g, const GemmArgs &p, int num_sms, cudaStream_t st) {
    using C = Cfg<BN>;
    CUtensorMap ma, mb;
    bool ok = A_MN ? make_map(&ma, g.A, g.K, g.M, g.lda, 64, g.f16) : make_map(&ma, g.A, g.M, g.K, g.lda, BM, g.f16);
    ok = ok && (B_MN ? make_map(&mb, g.B, g.K, g.N, g.ldb, 64, g.f16) : make_map(&mb, g.B, g.N, g.K, g.ldb, BN, g.f16));
    if (!ok) return cudaErrorInvalidValue;
    auto kern = gemm_kernel<BN, A_MN, B_MN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    const int ntiles = (g.M / BM) * (g.N / BN);
    const int grid = ntiles < num_sms ? ntiles : num_sms;
    kern<<<grid, kThreads, C::SMEM, st>>>(ma, mb, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(const GemmDesc &g, const DevErr &err, int num_sms, cudaStream_t st) {
    if (g.M % BM || g.K % BK || g.M <= 0 || g.N <= 0 || g.K <= 0) return cudaErrorInvalidValue;
    GemmArgs p{};
    p.M = g.M;
    p.N = g.N;
    p.K = g.K;
    p.ring_rows = g.ring_rows;
    p.ring_kblocks = g.ring_kblocks;
    p.ring_rank0 = g.ring_rank0;
    p.epi = g.epi;
    p.out = g.out;
    p.ldo = g.ldo;
    p.out2 = g.out2;
    p.ldo2 = g.ldo2;
    p.aux = g.aux;
    p.ldaux = g.ldaux;
    p.rowmap = g.rowmap;
    p.hsplit = g.hsplit > 0 ? g.hsplit : g.N;
    p.out_k = g.out_k;
    p.out_v = g.out_v;
    p.alpha = g.alpha;
    p.f16 = g.f16;
    p.err = err;
    const bool bn256 = (g.N % 256 == 0) && (g.epi != EPI_QKV || g.hsplit % 256 == 0) && !g.force_bn128;
    if (!bn256 && g.N % 128) return cudaErrorInvalidValue;
    p.idesc = idesc_mma(BM, bn256 ? 256 : 128, g.a_mn, g.b_mn, g.f16);
    if (!g.a_mn && !g.b_mn)
        return bn256 ? launch_impl<256, false, false>(g, p, num_sms, st) : launch_impl<128, false, false>(g, p, num_sms, st);
    if (!g.a_mn && g.b_mn)
        return bn256 ? launch_impl<256, false, true>(g, p, num_sms, st) : launch_impl<128, false, true>(g, p, num_sms, st);
    if (g.a_mn && g.b_mn)
        return bn256 ? launch_impl<256, true, true>(g, p, num_sms, st) : launch_impl<128, true, true>(g, p, num_sms, st);
    return bn256 ? launch_impl<256, true, false>(g, p, num_sms, st) : launch_impl<128, true, false>(g, p, num_sms, st);
}

}  // namespace tsp
