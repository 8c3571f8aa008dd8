// Causal flash attention forward on tcgen05 for the folded layer.
//
// Queries are the ranks' local tokens (rank-major zigzag rows); keys and values
// are the all-gathered K/V in global order ("Zyphra TSP folds TP+SP onto one
// GPU axis", zubnet.ai, paragraph 2).  Every query row carries its own global
// position p (from the zigzag map), and key k is visible iff k <= p.
//
// Work item = (head, block of 256 local query rows) = two 128-row query tiles.
// CTA layout (10 warps, persistent, one CTA per SM):
//   warp 0     TMA producer: the two Q tiles of the item, then K_j / V_j tiles
//              of 128 keys (K ring of 2, V ring of 2).
//   warp 1     TMEM owner and MMA issuer: S_w = Q_w K_j^T (128x128, fp32 in
//              TMEM) and O_w += P_w V_j (128 x dh, fp32 in TMEM) for w = 0, 1,
//              ordered so that S of the next tile overlaps the softmax of the
//              other tile (ping-pong between the two softmax groups).
//   warps 2-5  softmax group 0 (query tile 0), warps 6-9 group 1: thread =
//              query row; online softmax in the log2 domain; P written back
//              into TMEM as packed fp16 over the first half of S_w's
//              columns, where the P V MMA reads it as its A operand; O
//              rescaled in TMEM when the running max grows by more than 2^8; final
//              O / l written as fp16 and LSE (log2 domain) as fp32.
// Q, K, V, P and O are fp16.  P carries a factor 2^kPOff (exact: it is added
// to the exponent), which O / l cancels and the LSE takes out again: with the
// lazy rescale P stays below 2^(8 + kPOff) = 2^15 < 65504, and probabilities
// down to 2^-(14 + kPOff) stay normal fp16 numbers, which matters at long
// sequences, where most of a row's probabilities are small.
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256,256+dh), O1 [384,384+dh);
// P_w overwrites the first 64 columns of S_w once S_w is in registers.
#include "common.cuh"
#include "internal.h"

namespace tsp {
namespace {

constexpr int kFwdThreads = 320;
constexpr float kPOff = 7.0f;  // log2 of the factor carried by the fp16 P

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^x on the FMA pipe, for a share of the softmax's exponentials (the MUFU
// unit needs as many cycles per 128x128 tile as the tile's two MMAs).  The
// argument is split as x = n + f with n = round(x): adding 1.5 * 2^23 leaves
// n in the low mantissa bits of the sum, and f = x - n lies in [-1/2, 1/2]
// (the argument reduction of Cody and Waite, "Software Manual for the
// Elementary Functions", 1980).  2^f is a degree-5 polynomial fitted by the
// Remez exchange for least maximum relative error (csrc/fit_exp2.py: 2.1e-7
// evaluated in fp32), and 2^n enters by an integer add to the exponent
// field.  Valid for x < 128; x <= -127 (-inf included) gives 0 or a denormal
// below 2^-126.
__device__ __forceinline__ float exp2_poly(float x) {
    constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
    x = fmaxf(x, -127.0f);
    const float t = __fadd_rn(x, kShift);
    const float f = __fsub_rn(x, __fsub_rn(t, kShift));
    float p = fmaf(f, 0x1.5c08e6p-10f, 0x1.3d0c52p-7f);
    p = fmaf(p, f, 0x1.c6b6e4p-5f);
    p = fmaf(p, f, 0x1.ebf918p-3f);
    p = fmaf(p, f, 0x1.62e428p-1f);
    p = fmaf(p, f, 0x1.000002p+0f);
    return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// Which of a row's 128 exponentials per key tile take exp2_poly: key k of
// the tile when k % kPolyEvery == kPolyEvery - 1 (0: none).  Measured on the
// 7B layer at S=131072 (forward attention, ms per step, same box): none
// 154-159, one in 8 167-175, one in 5 185-187, one in 4 190-192, one in 3
// 190-195.  The softmax is not limited by the MUFU's rate, and each
// polynomial costs ten issue slots where the MUFU costs one, so none is used.
constexpr int kPolyEvery = 0;
__host__ __device__ constexpr bool poly_key(int k) { return kPolyEvery > 0 && k % kPolyEvery == kPolyEvery - 1; }

// Global position of local (rank-major) row i under the zigzag partition.
__device__ __forceinline__ int zig_pos(int i, int L, int D, int c) {
    const int r = i / L;
    const int j = i - r * L;
    return (j < c) ? r * c + j : (2 * D - 1 - r) * c + (j - c);
}

template <int DH>
struct FwdCfg {
    static constexpr int SWB = DH * 2 < 128 ? DH * 2 : 128;   // swizzle span in bytes
    static constexpr int ATOM_COLS = SWB / 2;                 // 16-bit columns per swizzle atom
    static constexpr int NATOM = DH / ATOM_COLS;
    static constexpr int TILE_BYTES = 128 * DH * 2;           // one 128-row tile of Q, K or V
    static constexpr int ATOM_BYTES = 128 * SWB;
    static constexpr uint32_t LAYOUT = SWB == 128 ? kSwizzle128 : (SWB == 64 ? kSwizzle64 : kSwizzle32);
    static constexpr int KST = 2;
    static constexpr int VST = 2;
    // smem map (1024-aligned pieces); P lives in TMEM
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + 2 * TILE_BYTES;
    static constexpr int OFF_V = OFF_K + KST * TILE_BYTES;
    static constexpr int OFF_BAR = OFF_V + VST * TILE_BYTES;
    static constexpr int SMEM = OFF_BAR + 256 + 1024;
    static_assert(SMEM <= kMaxDynSmem, "forward tiles exceed the shared-memory limit");
    // q_full/empty, k_full/empty[KST], v_full/empty[VST], s_full[2], p_full[2], o_done[2], drain
    // + TMEM slot + abort flag
    static_assert(8 * (2 * KST + 2 * VST + 9) + 8 <= 256, "forward barriers exceed their slot");
    static_assert(384 + DH <= 512, "forward TMEM columns: S0 0, S1 128, O0 256, O1 384");
};

// K-major descriptor of a [128 rows][DH] 16-bit tile for K step kk (16 columns).
template <int DH>
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int kk) {
    using C = FwdCfg<DH>;
    const int col = kk * 16;
    const uint32_t off = (col / C::ATOM_COLS) * C::ATOM_BYTES + (col % C::ATOM_COLS) * 2;
    return sdesc(base + off, 16, 8 * C::SWB, C::LAYOUT);
}
// MN-major descriptor of V[128 keys][DH] (N = DH contiguous) for K step kk (16 keys).
template <int DH>
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t base, int kk) {
    using C = FwdCfg<DH>;
    return sdesc(base + kk * 16 * C::SWB, C::ATOM_BYTES, 8 * C::SWB, C::LAYOUT);
}
// Byte offsets of K step kk from step 0 in the two layouts above, so the issue
// loop builds each descriptor once per tile and advances it (desc_plus).
template <int DH>
__host__ __device__ constexpr uint32_t kmajor_off(int kk) {
    return (kk * 16 / FwdCfg<DH>::ATOM_COLS) * FwdCfg<DH>::ATOM_BYTES + (kk * 16 % FwdCfg<DH>::ATOM_COLS) * 2;
}
template <int DH>
__host__ __device__ constexpr uint32_t mnmajor_off(int kk) {
    return kk * 16 * FwdCfg<DH>::SWB;
}

template <int DH>
__global__ void __launch_bounds__(kFwdThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                    const __grid_constant__ CUtensorMap mapV, const AttnDesc a, const DevErr err) {
    using C = FwdCfg<DH>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *q_full = bars + 0;
    uint64_t *q_empty = bars + 1;
    uint64_t *k_full = bars + 2;            // [KST]
    uint64_t *k_empty = k_full + C::KST;    // [KST]
    uint64_t *v_full = k_empty + C::KST;    // [VST]
    uint64_t *v_empty = v_full + C::VST;    // [VST]
    uint64_t *s_full = v_empty + C::VST;    // [2]
    uint64_t *p_full = s_full + 2;          // [2]
    uint64_t *o_done = p_full + 2;          // [2]
    uint64_t *drain = o_done + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int h = a.H * DH;
    const float sl2 = 1.4426950408889634f * rsqrtf(static_cast<float>(DH));

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < C::KST; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < C::VST; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int w = 0; w < 2; ++w) {
            mbar_init(&s_full[w], 1);
            mbar_init(&p_full[w], 128);
            mbar_init(&o_done[w], 1);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&mapQ);
        tma_prefetch_desc(&mapK);
        tma_prefetch_desc(&mapV);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int kcount = 0, vcount = 0, item_iter = 0;
            bool ok = true;
            for (int it = blockIdx.x; it < a.num_items && ok; it += gridDim.x, ++item_iter) {
                const int qb = a.order[2 * it] / a.H, head = a.order[2 * it] % a.H, nkv = a.order[2 * it + 1];
                if (!mbar_wait(q_empty, (item_iter & 1) ^ 1, abort_flag, err)) break;
                mbar_arrive_tx(q_full, 2 * C::TILE_BYTES);
                for (int w = 0; w < 2; ++w)
                    for (int t = 0; t < C::NATOM; ++t)
                        tma_load_2d(smem + C::OFF_Q + w * C::TILE_BYTES + t * C::ATOM_BYTES, &mapQ, q_full,
                                    head * DH + t * C::ATOM_COLS, qb * 256 + w * 128 - a.q_row0);
                for (int j = 0; j < nkv; ++j) {
                    const int ks = kcount % C::KST;
                    if (!mbar_wait(&k_empty[ks], ((kcount / C::KST) & 1) ^ 1, abort_flag, err)) { ok = false; break; }
                    mbar_arrive_tx(&k_full[ks], C::TILE_BYTES);
                    for (int t = 0; t < C::NATOM; ++t)
                        tma_load_2d(smem + C::OFF_K + ks * C::TILE_BYTES + t * C::ATOM_BYTES, &mapK, &k_full[ks],
                                    head * DH + t * C::ATOM_COLS, j * 128);
                    ++kcount;
                    const int vs = vcount % C::VST;
                    if (!mbar_wait(&v_empty[vs], ((vcount / C::VST) & 1) ^ 1, abort_flag, err)) { ok = false; break; }
                    mbar_arrive_tx(&v_full[vs], C::TILE_BYTES);
                    for (int t = 0; t < C::NATOM; ++t)
                        tma_load_2d(smem + C::OFF_V + vs * C::TILE_BYTES + t * C::ATOM_BYTES, &mapV, &v_full[vs],
                                    head * DH + t * C::ATOM_COLS, j * 128);
                    ++vcount;
                }
            }
            // Drain: every issued load has landed before exit.
            for (int s = 0; s < C::KST; ++s)
                if (kcount > s) {
                    const int last = kcount - 1 - ((kcount - 1 - s) % C::KST);
                    long long t0 = clock64();
                    while (!mbar_try_wait(&k_full[s], (last / C::KST) & 1) && clock64() - t0 < err.wait_limit) {}
                }
            for (int s = 0; s < C::VST; ++s)
                if (vcount > s) {
                    const int last = vcount - 1 - ((vcount - 1 - s) % C::VST);
                    long long t0 = clock64();
                    while (!mbar_try_wait(&v_full[s], (last / C::VST) & 1) && clock64() - t0 < err.wait_limit) {}
                }
            if (item_iter > 0) {
                long long t0 = clock64();
                while (!mbar_try_wait(q_full, (item_iter - 1) & 1) && clock64() - t0 < err.wait_limit) {}
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs this loop (warp-uniform control flow); one
        // elected lane polls the barriers and issues every MMA and commit (a
        // commit tracks the MMAs of the thread that issues it).  Descriptors
        // are built once per tile and advanced by compile-time offsets.
        {
            const bool leader = elect_one();
            const int leader_lane = __ffs(__ballot_sync(0xffffffffu, leader)) - 1;
            constexpr uint32_t idS = idesc_f16(128, 128, false, false);
            constexpr uint32_t idO = idesc_f16(128, DH, false, true);
            const uint32_t qbase = smem_u32(smem + C::OFF_Q);
            const uint64_t dQa = kmajor_desc<DH>(qbase, 0), dQb = kmajor_desc<DH>(qbase + C::TILE_BYTES, 0);
            int kcount = 0, vcount = 0, tcount = 0, item_iter = 0;
            bool ok = true;
            // S_w = Q_w K^T for the K tile in stage ks
            auto issue_s = [&](int w, int ks) {
                const uint64_t dK0 = kmajor_desc<DH>(smem_u32(smem + C::OFF_K + ks * C::TILE_BYTES), 0);
                const uint64_t dQ0 = w ? dQb : dQa;
#pragma unroll
                for (int kk = 0; kk < DH / 16; ++kk)
                    umma_ss(tmem + w * 128, desc_plus(dQ0, kmajor_off<DH>(kk)), desc_plus(dK0, kmajor_off<DH>(kk)),
                              idS, kk > 0);
                umma_commit(&s_full[w]);
            };
            for (int it = blockIdx.x; it < a.num_items && ok; it += gridDim.x, ++item_iter) {
                const int nkv = a.order[2 * it + 1];
                if (!lead_wait(leader, leader_lane, q_full, item_iter & 1, abort_flag, err)) break;
                // prologue: S_w for key tile 0
                {
                    const int ks = kcount % C::KST;
                    if (!lead_wait(leader, leader_lane, &k_full[ks], (kcount / C::KST) & 1, abort_flag, err)) break;
                    if (leader) {
                        tc_fence_after();
                        issue_s(0, ks);
                        issue_s(1, ks);
                        umma_commit(&k_empty[ks]);
                    }
                    ++kcount;
                }
                for (int j = 0; j < nkv && ok; ++j, ++tcount) {
                    const int vs = vcount % C::VST;
                    if (!lead_wait(leader, leader_lane, &v_full[vs], (vcount / C::VST) & 1, abort_flag, err)) {
                        ok = false;
                        break;
                    }
                    const uint64_t dV0 = mnmajor_desc<DH>(smem_u32(smem + C::OFF_V + vs * C::TILE_BYTES), 0);
                    const int ks = kcount % C::KST;
                    for (int w = 0; w < 2; ++w) {
                        if (!lead_wait(leader, leader_lane, &p_full[w], tcount & 1, abort_flag, err)) { ok = false; break; }
                        if (leader) {
                            tc_fence_after();
                            // P_w sits in TMEM columns [128 w, 128 w + 64): 16 keys per 8 columns
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk)
                                umma_ts(tmem + 256 + w * 128, tmem + w * 128 + kk * 8, desc_plus(dV0, mnmajor_off<DH>(kk)),
                                             idO, (j > 0 || kk > 0) ? 1u : 0u);
                            umma_commit(&o_done[w]);
                        }
                        if (j + 1 < nkv) {
                            if (w == 0 &&
                                !lead_wait(leader, leader_lane, &k_full[ks], (kcount / C::KST) & 1, abort_flag, err)) {
                                ok = false;
                                break;
                            }
                            if (leader) {
                                tc_fence_after();
                                issue_s(w, ks);
                                if (w == 1) umma_commit(&k_empty[ks]);
                            }
                            if (w == 1) ++kcount;
                        }
                    }
                    if (!ok) break;
                    if (leader) umma_commit(&v_empty[vs]);
                    ++vcount;
                }
                if (leader) umma_commit(q_empty);
            }
            const bool bad = __any_sync(0xffffffffu, !ok || *abort_flag);
            if (bad && leader) {
                umma_commit(drain);
                long long t0 = clock64();
                while (!mbar_try_wait(drain, 0) && clock64() - t0 < err.wait_limit) {}
            }
            __syncwarp();
        }
    } else {
        // ------------------------------------------------------------ softmax groups
        const int w = (warp - 2) / 4;
        const int quarter = warp & 3;
        const int trow = quarter * 32 + lane;  // row within the 128-row tile = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t s_addr = tmem + lane_off + w * 128;
        const uint32_t o_addr = tmem + lane_off + 256 + w * 128;
        int tcount = 0;
        for (int it = blockIdx.x; it < a.num_items; it += gridDim.x) {
            const int qb = a.order[2 * it] / a.H, head = a.order[2 * it] % a.H, nkv = a.order[2 * it + 1];
            const int lrow = qb * 256 + w * 128 + trow;
            const int pos = zig_pos(lrow, a.L, a.D, a.chunk);
            float m = -INFINITY, l = 0.f;
            bool ok = true;
            for (int j = 0; j < nkv; ++j, ++tcount) {
                if (!warp_wait(&s_full[w], tcount & 1, abort_flag, err)) { ok = false; break; }
                tc_fence_after();
                float s[128];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float t[32];
                    tmem_ld32(s_addr + c * 32, t);
#pragma unroll
                    for (int e = 0; e < 32; ++e) s[c * 32 + e] = t[e];
                }
                tmem_ld_wait();
                const int kv0 = j * 128;
                // Row max on the raw scores (the scale is positive), masking
                // only on tiles that reach past this row's position.  `full` is
                // warp-uniform: it selects code paths that end in warp-collective
                // TMEM stores, which must never run on a partial warp.
                const bool full = __all_sync(0xffffffffu, kv0 + 127 <= pos);
                // eight independent partial maxima: no 128-long dependency chain
                float mx[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) mx[e] = -INFINITY;
                if (full) {
#pragma unroll
                    for (int c = 0; c < 128; ++c) mx[c & 7] = fmaxf(mx[c & 7], s[c]);
                } else {
#pragma unroll
                    for (int c = 0; c < 128; ++c) {
                        if (kv0 + c > pos) s[c] = -INFINITY;
                        mx[c & 7] = fmaxf(mx[c & 7], s[c]);
                    }
                }
                float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                 fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
                mt *= sl2;
                const float m_new = fmaxf(m, mt);
                const float m_use = (j == 0 || m_new - m > 8.0f) ? m_new : m;
                if (j > 0) {
                    if (!warp_wait(&o_done[w], (tcount - 1) & 1, abort_flag, err)) { ok = false; break; }
                    tc_fence_after();
                    // TMEM loads/stores are warp-collective: rescale the whole
                    // warp's rows when any row's max moved (alpha = 1 elsewhere).
                    if (__any_sync(0xffffffffu, m_use != m)) {
                        const float alpha = ex2(m - m_use);
                        l *= alpha;
#pragma unroll 1
                        for (int c = 0; c < DH / 32; ++c) {
                            float o[32];
                            tmem_ld32(o_addr + c * 32, o);
                            tmem_ld_wait();
#pragma unroll
                            for (int e = 0; e < 32; ++e) o[e] *= alpha;
                            tmem_st32(o_addr + c * 32, o);
                        }
                        tmem_st_wait();
                    }
                }
                m = m_use;
                if (!warp_converged("softmax TMEM store")) { ok = false; break; }
                // eight independent partial sums
                float ls[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) ls[e] = 0.f;
                const float neg_m = kPOff - m;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    // 64 keys -> 32 TMEM columns of packed fp16 pairs (even key in the low half)
                    float pk[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int k0 = half * 64 + 2 * c;
                        const float x0 = fmaf(s[k0], sl2, neg_m), x1 = fmaf(s[k0 + 1], sl2, neg_m);
                        const float p0 = poly_key(k0) ? exp2_poly(x0) : ex2(x0);
                        const float p1 = poly_key(k0 + 1) ? exp2_poly(x1) : ex2(x1);
                        ls[(2 * c) & 7] += p0;
                        ls[(2 * c + 1) & 7] += p1;
                        pk[c] = __uint_as_float(pack_f16(p0, p1));
                    }
                    tmem_st32(s_addr + half * 32, pk);
                }
                tmem_st_wait();
                l += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
                tc_fence_before();
                mbar_arrive(&p_full[w]);
            }
            if (!ok) break;
            // epilogue: wait for the last P V of this tile
            if (!warp_wait(&o_done[w], (tcount - 1) & 1, abort_flag, err)) break;
            tc_fence_after();
            const float inv = 1.0f / l;
            __half *orow = static_cast<__half *>(a.o) + static_cast<int64_t>(lrow - a.q_row0) * h + head * DH;
#pragma unroll 1
            for (int c = 0; c < DH / 32; ++c) {
                float o[32];
                tmem_ld32(o_addr + c * 32, o);
                tmem_ld_wait();
                uint4 *d = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint4 v;
                    v.x = pack_f16(o[8 * q + 0] * inv, o[8 * q + 1] * inv);
                    v.y = pack_f16(o[8 * q + 2] * inv, o[8 * q + 3] * inv);
                    v.z = pack_f16(o[8 * q + 4] * inv, o[8 * q + 5] * inv);
                    v.w = pack_f16(o[8 * q + 6] * inv, o[8 * q + 7] * inv);
                    d[q] = v;
                }
            }
            // l sums the offset probabilities: log2(l) - kPOff is the true log-sum
            a.lse[static_cast<int64_t>(head) * a.S + lrow] = m + (__log2f(l) - kPOff);
            tc_fence_before();
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int DH>
cudaError_t launch_fwd_impl(const AttnDesc &a, const DevErr &err, int num_sms, cudaStream_t st) {
    using C = FwdCfg<DH>;
    const int h = a.H * DH;
    const CUtensorMapSwizzle swz = C::SWB == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                   : C::SWB == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                  : CU_TENSOR_MAP_SWIZZLE_32B;
    CUtensorMap mq, mk, mv;
    bool ok = encode_tensor_map_2d(&mq, a.q, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, h, a.q_rows, int64_t(h) * 2,
                                   C::ATOM_COLS, 128, swz);
    ok = ok && encode_tensor_map_2d(&mk, a.k, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, h, a.S, int64_t(h) * 2,
                                    C::ATOM_COLS, 128, swz);
    ok = ok && encode_tensor_map_2d(&mv, a.v, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, h, a.S, int64_t(h) * 2,
                                    C::ATOM_COLS, 128, swz);
    if (!ok) return cudaErrorInvalidValue;
    auto kern = attn_fwd_kernel<DH>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    const int grid = a.num_items < num_sms ? a.num_items : num_sms;
    kern<<<grid, kFwdThreads, C::SMEM, st>>>(mq, mk, mv, a, err);
    return cudaGetLastError();
}

__global__ void exp2_test_kernel(const float *x, float *y, int n, int which) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) y[i] = which == 0 ? exp2_poly(x[i]) : ex2(x[i]);
}

}  // namespace

cudaError_t launch_exp2_test(const float *x, float *y, int n, int which, cudaStream_t st) {
    if (n < 0 || (which != 0 && which != 1)) return cudaErrorInvalidValue;
    if (n == 0) return cudaSuccess;
    exp2_test_kernel<<<(n + 255) / 256, 256, 0, st>>>(x, y, n, which);
    return cudaGetLastError();
}

cudaError_t launch_attn_fwd(const AttnDesc &a, const DevErr &err, int num_sms, cudaStream_t st) {
    switch (a.dh) {
        case 32: return launch_fwd_impl<32>(a, err, num_sms, st);
        case 64: return launch_fwd_impl<64>(a, err, num_sms, st);
        case 128: return launch_fwd_impl<128>(a, err, num_sms, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace tsp
