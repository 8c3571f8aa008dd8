// Causal attention backward on tcgen05 for the folded layer.
//
// With s = q.k / sqrt(dh) (log2-domain LSE from the forward), per head:
//   P = exp(s - LSE),  Delta_q = rowsum(dO * O),  dS = P * (dO V^T - Delta),
//   dV = P^T dO,  dK = dS^T Q / sqrt(dh),  dQ = dS K / sqrt(dh).
// Key-side gradients gather contributions from every rank's queries and are
// written at the key owner's local row: the reverse of the forward's K/V
// all-gather ("Zyphra TSP folds TP+SP onto one GPU axis", zubnet.ai,
// paragraph 2 gives the forward exchange; its reverse is the reading taken
// for the backward).
//
// Kernels (every result deterministic: no floating-point atomics):
//   attn_delta   Delta[h][row] = sum_d dO * O (fp16 inputs, fp32 sum); for the
//                single-pass kernel it also clears the integer dQ sum and takes
//                the per-head maxima that set its fixed-point scale.
//   attn_bwd_fused (head size 128) one item = (head, 128-key tile); steps of 64
//                query rows walked from the top position down.  S^T, dP^T,
//                then P^T / dS^T and dQ^T share two TMEM step buffers; dV and
//                dK accumulate in TMEM; dQ^T is added to a 32-bit fixed-point
//                sum in global memory with integer reductions (the same bits in
//                any order), which dq_convert turns into fp16 dQ.
//   attn_dkdv2, attn_dq2 (head sizes 32, 64) the two-kernel backward: a
//                key-tile kernel for dK, dV (P^T and dS^T go back into TMEM as
//                packed fp16 over the columns they were read from) and a
//                query-tile kernel for dQ (S and dP recomputed).
// Q, K, V, O, dO and the outputs dQ, dK, dV are fp16 (gradients in the
// backward's scaled domain).  The P^T feeding dV carries a factor 2^kPOff so
// small probabilities stay normal fp16 numbers; the dV epilogue takes it out.
// Warp roles of each kernel are described above its definition.
#include "common.cuh"
#include "internal.h"

namespace tsp {
namespace {

constexpr float kPOff = 7.0f;                 // log2 of the factor carried by the fp16 P^T

// Fractional bits of a head's fixed-point dQ sum.  With P >= 0 summing to 1
// over a query's keys, sum_k |dS_qk| = sum_k P_qk |dP_qk - Delta_q|
// <= 2 max_k |dP_qk| <= 2 |dO_q| max_k |V_k|, so every partial sum of
// dQ_q = sum_k dS_qk K_k / sqrt(dh) is at most B = 2 max|dO| max|V| max|K_j| / sqrt(dh)
// in magnitude (|.| the Euclidean norm over the head's dims, |K_j| the
// largest element).  F is chosen so that B 2^F < 2^29: sums stay below 2^30
// however the contributions' roundings add.  `b` holds the head's maxima of
// |dO_q|^2, |V_k|^2 and |K_j| as float bits.  The same function gives the
// same F in every kernel that calls it.
__device__ __forceinline__ int dq_frac_bits(const unsigned int *b, int dh) {
    const float bound = 2.0f * sqrtf(__uint_as_float(b[0])) * sqrtf(__uint_as_float(b[1])) * __uint_as_float(b[2]) *
                        rsqrtf(static_cast<float>(dh));
    if (!(bound > 0.0f) || bound > 1.0e30f) return 0;
    int E = 0;
    frexpf(bound, &E);  // bound < 2^E
    return min(max(29 - E, -60), 60);
}
constexpr float kPOffInv = 1.0f / 128.0f;     // 2^-kPOff

__device__ __forceinline__ float ex2b(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void spin_drain(uint64_t *bar, uint32_t parity, long long limit) {
    long long t0 = clock64();
    while (!mbar_try_wait(bar, parity) && clock64() - t0 < limit) {
    }
}

template <int DH>
struct BCfg {
    static constexpr int SWB = DH * 2 < 128 ? DH * 2 : 128;
    static constexpr int ATOM_COLS = SWB / 2;
    static constexpr int NATOM = DH / ATOM_COLS;
    static constexpr int TILE_BYTES = 128 * DH * 2;
    static constexpr int ATOM_BYTES = 128 * SWB;
    static constexpr uint32_t LAYOUT = SWB == 128 ? kSwizzle128 : (SWB == 64 ? kSwizzle64 : kSwizzle32);
};

template <int DH>
__device__ __forceinline__ uint64_t kdesc(uint32_t base, int kk) {
    using C = BCfg<DH>;
    const int col = kk * 16;
    return sdesc(base + (col / C::ATOM_COLS) * C::ATOM_BYTES + (col % C::ATOM_COLS) * 2, 16, 8 * C::SWB, C::LAYOUT);
}
template <int DH>
CUtensorMapSwizzle swz_of() {
    return BCfg<DH>::SWB == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
           : BCfg<DH>::SWB == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                 : CU_TENSOR_MAP_SWIZZLE_32B;
}

// ---------------------------------------------------------------------------
// Delta[h][row] = sum_d dO * O per (row, head).  A warp takes 256 contiguous
// elements of one row per item of a grid-stride loop: dh/8 lanes per head,
// 16-byte loads, so a warp covers 256/dh heads (lanes past the last head sit
// out).  For the single-pass kernel (acc non-null) it also clears the
// (row, head) slice of the integer dQ sum and takes, per head, the largest
// |dO_row|^2, |V_row|^2 and |K|_max that bound the sum (dq_frac_bits): per
// block in shared memory, then one atomicMax per head and block into `bound`
// (cleared before the launch; non-negative float bits order like unsigned
// integers, so the maxima do not depend on the order).  The O / dO rows
// (q_rows of them, local rows from q_row0) and the K / V rows (all S, read
// only for the bounds) are separate ranges of the same loop.
__device__ __forceinline__ float dot8(const uint4 &a, const uint4 &b) {
    return f16_lo(a.x) * f16_lo(b.x) + f16_hi(a.x) * f16_hi(b.x) + f16_lo(a.y) * f16_lo(b.y) +
           f16_hi(a.y) * f16_hi(b.y) + f16_lo(a.z) * f16_lo(b.z) + f16_hi(a.z) * f16_hi(b.z) +
           f16_lo(a.w) * f16_lo(b.w) + f16_hi(a.w) * f16_hi(b.w);
}
__device__ __forceinline__ float absmax8(const uint4 &a) {
    float m = fmaxf(fabsf(f16_lo(a.x)), fabsf(f16_hi(a.x)));
    m = fmaxf(m, fmaxf(fabsf(f16_lo(a.y)), fabsf(f16_hi(a.y))));
    m = fmaxf(m, fmaxf(fabsf(f16_lo(a.z)), fabsf(f16_hi(a.z))));
    return fmaxf(m, fmaxf(fabsf(f16_lo(a.w)), fabsf(f16_hi(a.w))));
}

__global__ void attn_delta_kernel(const __half *o, const __half *dout, const __half *kk, const __half *vv,
                                  float *delta, int *acc, unsigned int *bound, int S, int H, int dh, int q_row0,
                                  int q_rows, int kv_rows) {
    extern __shared__ unsigned int smax[];  // [H][3]
    const bool fused = acc != nullptr;
    if (fused) {
        for (int i = threadIdx.x; i < 3 * H; i += blockDim.x) smax[i] = 0u;
        __syncthreads();
    }
    const int lane = threadIdx.x % 32;
    const int lph = dh / 8;                   // lanes per head (4, 8 or 16)
    const int hpw = 32 / lph;                 // heads per warp item
    const int groups = (H + hpw - 1) / hpw;   // warp items per row
    const int head_in = lane / lph;
    const int col = (lane % lph) * 8;
    const int64_t h = static_cast<int64_t>(H) * dh;
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x / 32);
    // rows [0, q_rows) of O and dO (local rows q_row0 + row), rows [0, kv_rows) of K and V
    const int64_t nrows = q_rows > kv_rows ? q_rows : kv_rows;
    for (int64_t wi = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 32;
         wi < nrows * groups; wi += nwarps) {
        const int64_t row = wi / groups;
        const int head = static_cast<int>(wi - row * groups) * hpw + head_in;
        const bool on = head < H;
        const bool qrow = on && row < q_rows;
        const int64_t at = row * h + static_cast<int64_t>(head) * dh + col;
        float s = 0.f, n2 = 0.f, v2 = 0.f, km = 0.f;
        if (qrow) {
            const uint4 a = *reinterpret_cast<const uint4 *>(o + at);
            const uint4 b = *reinterpret_cast<const uint4 *>(dout + at);
            s = dot8(a, b);
            if (fused) n2 = dot8(b, b);
        }
        if (fused && on && row < kv_rows) {
            const uint4 kw = *reinterpret_cast<const uint4 *>(kk + at);
            const uint4 vw = *reinterpret_cast<const uint4 *>(vv + at);
            v2 = dot8(vw, vw);
            km = absmax8(kw);
        }
        for (int off = lph / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        const bool first = on && col == 0;
        if (first && row < q_rows) delta[static_cast<int64_t>(head) * S + q_row0 + row] = s;
        if (fused) {
            for (int off = lph / 2; off > 0; off >>= 1) {
                n2 += __shfl_xor_sync(0xffffffffu, n2, off);
                v2 += __shfl_xor_sync(0xffffffffu, v2, off);
                km = fmaxf(km, __shfl_xor_sync(0xffffffffu, km, off));
            }
            if (first) {
                atomicMax(&smax[3 * head + 0], __float_as_uint(n2));
                atomicMax(&smax[3 * head + 1], __float_as_uint(v2));
                atomicMax(&smax[3 * head + 2], __float_as_uint(km));
            }
            if (qrow) {
                int4 *z = reinterpret_cast<int4 *>(acc + at);
                z[0] = make_int4(0, 0, 0, 0);
                z[1] = make_int4(0, 0, 0, 0);
            }
        }
    }
    if (fused) {
        __syncthreads();
        for (int i = threadIdx.x; i < 3 * H; i += blockDim.x)
            if (smax[i]) atomicMax(&bound[i], smax[i]);
    }
}

// ---------------------------------------------------------------------------
struct BwdParams {
    AttnBwdDesc d;
    const int *zig;          // local row -> global position (device copy of the map)
    const int *qtile_maxpos; // per 128-row local query tile, largest global position
    int num_items;
};

// ---------------------------------------------------------------------------
// Pipelined dK/dV kernel: steps of 64 query rows.
//   TMEM: S^T buffers [2] at columns 0 / 64, dP^T buffers [2] at 128 / 192,
//         dV at 256, dK at 384 (128 key lanes each).
//   The MMA warp issues S^T/dP^T of step g+1 before dV/dK of step g, so the
//   tensor core works on the next step while the element-wise warps (four
//   groups of four, 16 query columns each: four warps per SM sub-partition
//   to hide TMEM and barrier latency) turn step g into P^T and dS^T.  P^T and
//   dS^T go back into TMEM as packed fp16 (two queries per column) in the
//   columns their S^T / dP^T values came from, where the dV / dK MMAs read
//   them as the A operand.
template <int DH>
struct KvCfg {
    using C = BCfg<DH>;
    static constexpr int BQ = 64;
    static constexpr int QST = 3;
    static constexpr int QTILE = BQ * DH * 2;
    static constexpr int QATOM = BQ * C::SWB;
    static constexpr int VEC_BYTES = 3 * BQ * 4;  // lse, delta, pos of one step
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + C::TILE_BYTES;
    static constexpr int OFF_Q = OFF_V + C::TILE_BYTES;
    static constexpr int OFF_DO = OFF_Q + QST * QTILE;
    static constexpr int OFF_VEC = OFF_DO + QST * QTILE;
    static constexpr int OFF_BAR = OFF_VEC + QST * VEC_BYTES;
    static constexpr int SMEM = OFF_BAR + 256 + 1024;
    static_assert(SMEM <= kMaxDynSmem, "dK/dV tiles exceed the shared-memory limit");
    // kv_full/empty, q_full/empty[QST], s_full[2], p_full[2], acc_full, drain + TMEM slot + abort flag
    static_assert(8 * (2 * QST + 8) + 8 <= 256, "dK/dV barriers exceed their slot");
    static_assert(384 + DH <= 512, "dK/dV TMEM columns: S^T/dP^T buffers 0-255, dV 256, dK 384");
};

// K-major descriptor of a [64 rows][DH] sub-tile for K step kk (16 columns of DH).
template <int DH>
__device__ __forceinline__ uint64_t kdesc64(uint32_t base, int kk) {
    using C = BCfg<DH>;
    using K = KvCfg<DH>;
    const int col = kk * 16;
    return sdesc(base + (col / C::ATOM_COLS) * K::QATOM + (col % C::ATOM_COLS) * 2, 16, 8 * C::SWB, C::LAYOUT);
}
// MN-major descriptor of a [64 rows (K)][DH (N)] sub-tile for K step kk (16 rows).
template <int DH>
__device__ __forceinline__ uint64_t mndesc64(uint32_t base, int kk) {
    using C = BCfg<DH>;
    using K = KvCfg<DH>;
    return sdesc(base + kk * 16 * C::SWB, K::QATOM, 8 * C::SWB, C::LAYOUT);
}
// Byte offsets of K step kk from step 0 in the three operand layouts above,
// so an issue loop builds each descriptor once and advances it (desc_plus).
template <int DH>
__host__ __device__ constexpr uint32_t kdesc_off(int kk) {
    return (kk * 16 / BCfg<DH>::ATOM_COLS) * BCfg<DH>::ATOM_BYTES + (kk * 16 % BCfg<DH>::ATOM_COLS) * 2;
}
template <int DH>
__host__ __device__ constexpr uint32_t kdesc64_off(int kk) {
    return (kk * 16 / BCfg<DH>::ATOM_COLS) * (64 * BCfg<DH>::SWB) + (kk * 16 % BCfg<DH>::ATOM_COLS) * 2;
}
template <int DH>
__host__ __device__ constexpr uint32_t mndesc64_off(int kk) {
    return kk * 16 * BCfg<DH>::SWB;
}

struct KvParams {
    AttnBwdDesc d;
    const int *zig;
    int num_items;
};

// Two-kernel path: warp 0 TMA, warp 1 TMEM owner and MMA issuer, warps 2-17
// element-wise (four groups of four; thread = TMEM lane = row of the 128-row
// tile).
constexpr int kEwGroups = 4;                          // element-wise groups of four warps
constexpr int kBwdThreads2 = 64 + 128 * kEwGroups;     // + TMA warp + MMA warp

template <int DH>
__global__ void __launch_bounds__(kBwdThreads2, 1)
    attn_dkdv2_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                      const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mdO,
                      const KvParams kp, const DevErr err) {
    using C = BCfg<DH>;
    using K = KvCfg<DH>;
    const AttnBwdDesc &a = kp.d;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + K::OFF_BAR);
    uint64_t *kv_full = bars + 0, *kv_empty = bars + 1;
    uint64_t *q_full = bars + 2;                 // [QST]
    uint64_t *q_empty = q_full + K::QST;         // [QST]
    uint64_t *s_full = q_empty + K::QST;         // [2] S^T / dP^T of a step ready
    uint64_t *p_full = s_full + 2;               // [2] P^T / dS^T of a step packed
    uint64_t *acc_full = p_full + 2;             // dV / dK of an item complete
    uint64_t *drain = acc_full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int nq64 = a.S / 64;
    const StepVis vis{a.D, a.chunk, nq64};
    const float sl2 = 1.4426950408889634f * rsqrtf(static_cast<float>(DH));
    const float scale = rsqrtf(static_cast<float>(DH));

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        mbar_init(kv_empty, 1);
        for (int s = 0; s < K::QST; ++s) {
            mbar_init(&q_full[s], 1);
            mbar_init(&q_empty[s], 1);
        }
        mbar_init(&s_full[0], 1);
        mbar_init(&s_full[1], 1);
        // One P barrier per S buffer: a group that has finished step g may take
        // step g + 1 (its S is issued early) while others still work on g, so
        // the two steps' arrivals must not land on the same barrier.  Step
        // g + 2 cannot start before every group has arrived for g.
        mbar_init(&p_full[0], 128 * kEwGroups);
        mbar_init(&p_full[1], 128 * kEwGroups);
        mbar_init(acc_full, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
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
        if (lane == 0) {
            int item_iter = 0, g = 0;
            bool ok = true;
            for (int it = blockIdx.x; it < kp.num_items && ok; it += gridDim.x, ++item_iter) {
                const int kt = a.kv_order[it] / a.H, head = a.kv_order[it] % a.H;
                if (!mbar_wait(kv_empty, (item_iter & 1) ^ 1, abort_flag, err)) break;
                mbar_arrive_tx(kv_full, 2 * C::TILE_BYTES);
                for (int t = 0; t < C::NATOM; ++t) {
                    tma_load_2d(smem + K::OFF_K + t * C::ATOM_BYTES, &mK, kv_full, head * DH + t * C::ATOM_COLS, kt * 128);
                    tma_load_2d(smem + K::OFF_V + t * C::ATOM_BYTES, &mV, kv_full, head * DH + t * C::ATOM_COLS, kt * 128);
                }
                StepWalk w;
                for (w.seek(vis, 0, kt * 128); w.q < nq64; w.next(vis, kt * 128), ++g) {
                    const int q = w.q;
                    const int s = g % K::QST;
                    if (!mbar_wait(&q_empty[s], ((g / K::QST) & 1) ^ 1, abort_flag, err)) { ok = false; break; }
                    mbar_arrive_tx(&q_full[s], 2 * K::QTILE + K::VEC_BYTES);
                    for (int t = 0; t < C::NATOM; ++t) {
                        tma_load_2d(smem + K::OFF_Q + s * K::QTILE + t * K::QATOM, &mQ, &q_full[s],
                                    head * DH + t * C::ATOM_COLS, q * 64);
                        tma_load_2d(smem + K::OFF_DO + s * K::QTILE + t * K::QATOM, &mdO, &q_full[s],
                                    head * DH + t * C::ATOM_COLS, q * 64);
                    }
                    float *vec = reinterpret_cast<float *>(smem + K::OFF_VEC + s * K::VEC_BYTES);
                    bulk_load(vec, a.lse + static_cast<int64_t>(head) * a.S + q * 64, 256, &q_full[s]);
                    bulk_load(vec + 64, a.delta + static_cast<int64_t>(head) * a.S + q * 64, 256, &q_full[s]);
                    bulk_load(vec + 128, kp.zig + q * 64, 256, &q_full[s]);
                }
            }
            if (item_iter > 0) spin_drain(kv_full, (item_iter - 1) & 1, err.wait_limit);
            for (int s = 0; s < K::QST; ++s)
                if (g > s) {
                    const int last = g - 1 - ((g - 1 - s) % K::QST);
                    spin_drain(&q_full[s], (last / K::QST) & 1, err.wait_limit);
                }
        }
    } else if (warp == 1) {
        // The whole warp runs the issue loop (warp-uniform control flow); one
        // elected lane polls the barriers and issues every MMA and commit.
        // Operand descriptors are built once per tile and advanced by
        // compile-time offsets.
        {
            const bool leader = elect_one();
            const int leader_lane = __ffs(__ballot_sync(0xffffffffu, leader)) - 1;
            constexpr uint32_t idS = idesc_f16(128, 64, false, false);
            constexpr uint32_t idG = idesc_f16(128, DH, false, true);
            const uint64_t dK0 = kdesc<DH>(smem_u32(smem + K::OFF_K), 0);
            const uint64_t dV0 = kdesc<DH>(smem_u32(smem + K::OFF_V), 0);
            int item_iter = 0, g = 0;
            bool ok = true;
            auto issue_sdp = [&](int gi) -> bool {
                const int s = gi % K::QST, b = gi & 1;
                if (!lead_wait(leader, leader_lane, &q_full[s], (gi / K::QST) & 1, abort_flag, err)) return false;
                if (leader) {
                    tc_fence_after();
                    const uint64_t dQ0 = kdesc64<DH>(smem_u32(smem + K::OFF_Q + s * K::QTILE), 0);
                    const uint64_t dO0 = kdesc64<DH>(smem_u32(smem + K::OFF_DO + s * K::QTILE), 0);
#pragma unroll
                    for (int kk = 0; kk < DH / 16; ++kk)
                        umma_ss(tmem + 64 * b, desc_plus(dK0, kdesc_off<DH>(kk)), desc_plus(dQ0, kdesc64_off<DH>(kk)),
                                  idS, kk > 0);
#pragma unroll
                    for (int kk = 0; kk < DH / 16; ++kk)
                        umma_ss(tmem + 128 + 64 * b, desc_plus(dV0, kdesc_off<DH>(kk)),
                                  desc_plus(dO0, kdesc64_off<DH>(kk)), idS, kk > 0);
                    umma_commit(&s_full[b]);
                }
                return true;
            };
            for (int it = blockIdx.x; it < kp.num_items && ok; it += gridDim.x, ++item_iter) {
                const int kv0 = (a.kv_order[it] / a.H) * 128;
                if (!lead_wait(leader, leader_lane, kv_full, item_iter & 1, abort_flag, err)) break;
                if (leader) tc_fence_after();
                StepWalk w;
                w.seek(vis, 0, kv0);
                if (w.q < nq64 && !issue_sdp(g)) break;
                bool first = true;
                while (w.q < nq64) {
                    StepWalk wn = w;
                    wn.next(vis, kv0);
                    if (wn.q < nq64 && !issue_sdp(g + 1)) { ok = false; break; }
                    if (!lead_wait(leader, leader_lane, &p_full[g & 1], (g >> 1) & 1, abort_flag, err)) {
                        ok = false;
                        break;
                    }
                    if (leader) {
                        tc_fence_after();
                        const int s = g % K::QST, b = g & 1;
                        const uint64_t gQ0 = mndesc64<DH>(smem_u32(smem + K::OFF_Q + s * K::QTILE), 0);
                        const uint64_t gO0 = mndesc64<DH>(smem_u32(smem + K::OFF_DO + s * K::QTILE), 0);
                        // A operands from TMEM: queries 16 kk .. 16 kk + 15 packed at column 16 kk
#pragma unroll
                        for (int kk = 0; kk < K::BQ / 16; ++kk)
                            umma_ts(tmem + 256, tmem + 64 * b + kk * 16, desc_plus(gO0, mndesc64_off<DH>(kk)), idG,
                                         (!first || kk > 0) ? 1u : 0u);
#pragma unroll
                        for (int kk = 0; kk < K::BQ / 16; ++kk)
                            umma_ts(tmem + 384, tmem + 128 + 64 * b + kk * 16, desc_plus(gQ0, mndesc64_off<DH>(kk)),
                                         idG, (!first || kk > 0) ? 1u : 0u);
                        umma_commit(&q_empty[s]);
                    }
                    first = false;
                    ++g;
                    w = wn;
                }
                // one commit per item that had steps, so the element-wise warps'
                // wait for it is exact (a per-step commit would let a wait on
                // the last step's parity pass while an earlier step runs)
                if (leader) {
                    if (ok && !first) umma_commit(acc_full);
                    umma_commit(kv_empty);
                }
            }
            const bool bad = __any_sync(0xffffffffu, !ok || *abort_flag);
            if (bad && leader) {
                umma_commit(drain);
                spin_drain(drain, 0, err.wait_limit);
            }
            __syncwarp();
        }
    } else {
        const int grp = (warp - 2) / 4;         // query columns [16 grp, 16 grp + 16) of a step
        const int quarter = warp & 3;
        const int trow = quarter * 32 + lane;   // key row of the tile = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        int g = 0, acc_iter = 0;
        for (int it = blockIdx.x; it < kp.num_items; it += gridDim.x) {
            const int kt = a.kv_order[it] / a.H, head = a.kv_order[it] % a.H;
            const int kv0 = kt * 128;
            const int key = kv0 + trow;
            bool ok = true, any = false;
            StepWalk w;
            for (w.seek(vis, 0, kv0); w.q < nq64; w.next(vis, kv0), ++g) {
                any = true;
                const int b = g & 1, s = g % K::QST;
                if (!warp_wait(&s_full[b], (g >> 1) & 1, abort_flag, err)) { ok = false; break; }
                tc_fence_after();
                float sv[16], dp[16];
                tmem_ld16(tmem + lane_off + 64 * b + 16 * grp, sv);
                tmem_ld16(tmem + lane_off + 128 + 64 * b + 16 * grp, dp);
                tmem_ld_wait();
                const float *vec = reinterpret_cast<const float *>(smem + K::OFF_VEC + s * K::VEC_BYTES);
                const int *pos = reinterpret_cast<const int *>(vec + 128);
                // the 64 query rows of a step lie in one zigzag chunk (chunks are
                // multiples of 64 rows), so their positions are consecutive: this
                // key is visible to column e of the group iff e >= key - pos0
                const int first_vis = key - pos[16 * grp];
                const float4 *lse4 = reinterpret_cast<const float4 *>(vec + 16 * grp);
                const float4 *dl4 = reinterpret_cast<const float4 *>(vec + 64 + 16 * grp);
                uint32_t pk[8], dk[8];
#pragma unroll
                for (int e4 = 0; e4 < 4; ++e4) {
                    const float4 l = lse4[e4], d = dl4[e4];
                    const int e = 4 * e4;
                    // p = 2^kPOff P (the offset rides in the exponent)
                    float p0 = ex2b(fmaf(sv[e], sl2, kPOff - l.x)), p1 = ex2b(fmaf(sv[e + 1], sl2, kPOff - l.y));
                    float p2 = ex2b(fmaf(sv[e + 2], sl2, kPOff - l.z)), p3 = ex2b(fmaf(sv[e + 3], sl2, kPOff - l.w));
                    if (first_vis > 0) {
                        p0 = e >= first_vis ? p0 : 0.f;
                        p1 = e + 1 >= first_vis ? p1 : 0.f;
                        p2 = e + 2 >= first_vis ? p2 : 0.f;
                        p3 = e + 3 >= first_vis ? p3 : 0.f;
                    }
                    pk[2 * e4] = pack_f16(p0, p1);
                    pk[2 * e4 + 1] = pack_f16(p2, p3);
                    // dS = P (dP - Delta), without the offset
                    p0 *= kPOffInv;
                    p1 *= kPOffInv;
                    p2 *= kPOffInv;
                    p3 *= kPOffInv;
                    dk[2 * e4] = pack_f16(p0 * (dp[e] - d.x), p1 * (dp[e + 1] - d.y));
                    dk[2 * e4 + 1] = pack_f16(p2 * (dp[e + 2] - d.z), p3 * (dp[e + 3] - d.w));
                }
                // each group packs its 16 queries into the first 8 of the 16
                // columns it has just read, so no group writes what another
                // still has to read
                if (!warp_converged("P^T/dS^T TMEM store")) { ok = false; break; }
                tmem_st8u(tmem + lane_off + 64 * b + 16 * grp, pk);
                tmem_st8u(tmem + lane_off + 128 + 64 * b + 16 * grp, dk);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&p_full[b]);
            }
            if (!ok) break;
            if (!any) continue;
            if (!warp_wait(acc_full, acc_iter & 1, abort_flag, err)) break;
            ++acc_iter;
            tc_fence_after();
            // groups 0, 1 write dV (offset removed) and groups 2, 3 write dK
            // (scaled), at the key owner's local row; each pair splits the
            // 32-column chunks
            const int lrow = a.inv_map[key];
            const int which = grp >> 1;
            void *dst = which == 0 ? a.dv : a.dk;
            const float f = which == 0 ? kPOffInv : scale;
            __half *row = static_cast<__half *>(dst) + static_cast<int64_t>(lrow) * a.ldd + head * DH;
#pragma unroll 1
            for (int c = grp & 1; c < DH / 32; c += 2) {
                float v[32];
                tmem_ld32(tmem + lane_off + 256 + 128 * which + c * 32, v);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] *= f;
                flag_range(maxabs32(v), a.err);
                uint4 *d4 = reinterpret_cast<uint4 *>(row + c * 32);
#pragma unroll
                for (int qq = 0; qq < 4; ++qq)
                    d4[qq] = make_uint4(pack_f16(v[8 * qq], v[8 * qq + 1]), pack_f16(v[8 * qq + 2], v[8 * qq + 3]),
                                        pack_f16(v[8 * qq + 4], v[8 * qq + 5]), pack_f16(v[8 * qq + 6], v[8 * qq + 7]));
            }
            tc_fence_before();
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// Pipelined dQ kernel: one item = (head, 128-row query tile); steps of 64 keys.
//   TMEM: S buffers [2] at columns 0 / 64, dP buffers [2] at 128 / 192, dQ at
//   256 (128 query lanes).  The MMA warp issues S/dP of step j+1 before dQ of
//   step j, so the tensor core works while the element-wise warps (two groups
//   of four, 32 key columns each) turn step j into dS, which goes back into
//   TMEM as packed fp16 in the S columns it came from (the dQ MMA's A).
template <int DH>
struct Dq2Cfg {
    using C = BCfg<DH>;
    static constexpr int BK = 64;
    static constexpr int KST = 3;
    static constexpr int KTILE = BK * DH * 2;   // one K or V sub-tile of 64 keys
    static constexpr int KATOM = BK * C::SWB;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_DO = OFF_Q + C::TILE_BYTES;
    static constexpr int OFF_K = OFF_DO + C::TILE_BYTES;
    static constexpr int OFF_V = OFF_K + KST * KTILE;
    static constexpr int OFF_BAR = OFF_V + KST * KTILE;
    static constexpr int SMEM = OFF_BAR + 256 + 1024;
    static_assert(SMEM <= kMaxDynSmem, "dQ tiles exceed the shared-memory limit");
    // q_full/empty, k_full/empty[KST], s_full[2], p_full[2], acc_full, drain + TMEM slot + abort flag
    static_assert(8 * (2 * KST + 8) + 8 <= 256, "dQ barriers exceed their slot");
    static_assert(256 + DH <= 512, "dQ TMEM columns: S/dP buffers 0-255, dQ 256");
};

template <int DH>
__global__ void __launch_bounds__(kBwdThreads2, 1)
    attn_dq2_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                    const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mdO,
                    const BwdParams bp, const DevErr err) {
    using C = BCfg<DH>;
    using Q = Dq2Cfg<DH>;
    const AttnBwdDesc &a = bp.d;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Q::OFF_BAR);
    uint64_t *q_full = bars + 0, *q_empty = bars + 1;
    uint64_t *k_full = bars + 2;            // [KST]
    uint64_t *k_empty = k_full + Q::KST;    // [KST]
    uint64_t *s_full = k_empty + Q::KST;    // [2] S / dP of a step ready
    uint64_t *p_full = s_full + 2;          // [2] dS of a step packed
    uint64_t *acc_full = p_full + 2;        // dQ of an item complete
    uint64_t *drain = acc_full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const float sl2 = 1.4426950408889634f * rsqrtf(static_cast<float>(DH));
    const float scale = rsqrtf(static_cast<float>(DH));

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < Q::KST; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        mbar_init(&s_full[0], 1);
        mbar_init(&s_full[1], 1);
        // per-buffer dS barriers and a per-item accumulator barrier, for the
        // reasons given in the dK/dV kernel
        mbar_init(&p_full[0], 128 * kEwGroups);
        mbar_init(&p_full[1], 128 * kEwGroups);
        mbar_init(acc_full, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto nkv64 = [&](int qt) { return bp.qtile_maxpos[qt] / 64 + 1; };

    if (warp == 0) {
        if (lane == 0) {
            int item_iter = 0, g = 0;
            bool ok = true;
            for (int it = blockIdx.x; it < bp.num_items && ok; it += gridDim.x, ++item_iter) {
                const int qt = a.q_order[it] / a.H, head = a.q_order[it] % a.H;
                if (!mbar_wait(q_empty, (item_iter & 1) ^ 1, abort_flag, err)) break;
                mbar_arrive_tx(q_full, 2 * C::TILE_BYTES);
                for (int t = 0; t < C::NATOM; ++t) {
                    tma_load_2d(smem + Q::OFF_Q + t * C::ATOM_BYTES, &mQ, q_full, head * DH + t * C::ATOM_COLS, qt * 128);
                    tma_load_2d(smem + Q::OFF_DO + t * C::ATOM_BYTES, &mdO, q_full, head * DH + t * C::ATOM_COLS, qt * 128);
                }
                const int n = nkv64(qt);
                for (int j = 0; j < n; ++j, ++g) {
                    const int s = g % Q::KST;
                    if (!mbar_wait(&k_empty[s], ((g / Q::KST) & 1) ^ 1, abort_flag, err)) { ok = false; break; }
                    mbar_arrive_tx(&k_full[s], 2 * Q::KTILE);
                    for (int t = 0; t < C::NATOM; ++t) {
                        tma_load_2d(smem + Q::OFF_K + s * Q::KTILE + t * Q::KATOM, &mK, &k_full[s],
                                    head * DH + t * C::ATOM_COLS, j * 64);
                        tma_load_2d(smem + Q::OFF_V + s * Q::KTILE + t * Q::KATOM, &mV, &k_full[s],
                                    head * DH + t * C::ATOM_COLS, j * 64);
                    }
                }
            }
            if (item_iter > 0) spin_drain(q_full, (item_iter - 1) & 1, err.wait_limit);
            for (int s = 0; s < Q::KST; ++s)
                if (g > s) {
                    const int last = g - 1 - ((g - 1 - s) % Q::KST);
                    spin_drain(&k_full[s], (last / Q::KST) & 1, err.wait_limit);
                }
        }
    } else if (warp == 1) {
        // warp-uniform issue loop: one elected lane polls and issues, with
        // descriptors advanced by constant offsets (as in the dK/dV kernel)
        {
            const bool leader = elect_one();
            const int leader_lane = __ffs(__ballot_sync(0xffffffffu, leader)) - 1;
            constexpr uint32_t idS = idesc_f16(128, 64, false, false);
            constexpr uint32_t idG = idesc_f16(128, DH, false, true);
            const uint64_t dQ0 = kdesc<DH>(smem_u32(smem + Q::OFF_Q), 0);
            const uint64_t dO0 = kdesc<DH>(smem_u32(smem + Q::OFF_DO), 0);
            int item_iter = 0, g = 0;
            bool ok = true;
            auto issue_sdp = [&](int gi) -> bool {
                const int s = gi % Q::KST, b = gi & 1;
                if (!lead_wait(leader, leader_lane, &k_full[s], (gi / Q::KST) & 1, abort_flag, err)) return false;
                if (leader) {
                    tc_fence_after();
                    const uint64_t dK0 = kdesc64<DH>(smem_u32(smem + Q::OFF_K + s * Q::KTILE), 0);
                    const uint64_t dV0 = kdesc64<DH>(smem_u32(smem + Q::OFF_V + s * Q::KTILE), 0);
#pragma unroll
                    for (int kk = 0; kk < DH / 16; ++kk)
                        umma_ss(tmem + 64 * b, desc_plus(dQ0, kdesc_off<DH>(kk)), desc_plus(dK0, kdesc64_off<DH>(kk)),
                                  idS, kk > 0);
#pragma unroll
                    for (int kk = 0; kk < DH / 16; ++kk)
                        umma_ss(tmem + 128 + 64 * b, desc_plus(dO0, kdesc_off<DH>(kk)),
                                  desc_plus(dV0, kdesc64_off<DH>(kk)), idS, kk > 0);
                    umma_commit(&s_full[b]);
                }
                return true;
            };
            for (int it = blockIdx.x; it < bp.num_items && ok; it += gridDim.x, ++item_iter) {
                const int qt = a.q_order[it] / a.H;
                if (!lead_wait(leader, leader_lane, q_full, item_iter & 1, abort_flag, err)) break;
                if (leader) tc_fence_after();
                const int n = nkv64(qt);
                if (!issue_sdp(g)) break;
                for (int j = 0; j < n; ++j, ++g) {
                    if (j + 1 < n && !issue_sdp(g + 1)) { ok = false; break; }
                    if (!lead_wait(leader, leader_lane, &p_full[g & 1], (g >> 1) & 1, abort_flag, err)) {
                        ok = false;
                        break;
                    }
                    if (leader) {
                        tc_fence_after();
                        const int s = g % Q::KST, b = g & 1;
                        const uint64_t gK0 = mndesc64<DH>(smem_u32(smem + Q::OFF_K + s * Q::KTILE), 0);
                        // A = dS from TMEM: keys 16 kk .. 16 kk + 15 packed at column 16 kk
#pragma unroll
                        for (int kk = 0; kk < Q::BK / 16; ++kk)
                            umma_ts(tmem + 256, tmem + 64 * b + kk * 16, desc_plus(gK0, mndesc64_off<DH>(kk)), idG,
                                         (j > 0 || kk > 0) ? 1u : 0u);
                        umma_commit(&k_empty[s]);
                    }
                }
                if (leader) {
                    if (ok) umma_commit(acc_full);
                    umma_commit(q_empty);
                }
            }
            const bool bad = __any_sync(0xffffffffu, !ok || *abort_flag);
            if (bad && leader) {
                umma_commit(drain);
                spin_drain(drain, 0, err.wait_limit);
            }
            __syncwarp();
        }
    } else {
        const int grp = (warp - 2) / 4;         // key columns [16 grp, 16 grp + 16) of a step
        const int quarter = warp & 3;
        const int trow = quarter * 32 + lane;   // query row of the tile = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        int g = 0;
        for (int it = blockIdx.x, item_iter = 0; it < bp.num_items; it += gridDim.x, ++item_iter) {
            const int qt = a.q_order[it] / a.H, head = a.q_order[it] % a.H;
            const int lrow = qt * 128 + trow;
            const int pos = bp.zig[lrow];
            const float lse = a.lse[static_cast<int64_t>(head) * a.S + lrow];
            const float dl = a.delta[static_cast<int64_t>(head) * a.S + lrow];
            const int n = nkv64(qt);
            bool ok = true;
            for (int j = 0; j < n; ++j, ++g) {
                const int b = g & 1;
                if (!warp_wait(&s_full[b], (g >> 1) & 1, abort_flag, err)) { ok = false; break; }
                tc_fence_after();
                float sv[16], dp[16];
                tmem_ld16(tmem + lane_off + 64 * b + 16 * grp, sv);
                tmem_ld16(tmem + lane_off + 128 + 64 * b + 16 * grp, dp);
                tmem_ld_wait();
                const int k0 = j * 64 + 16 * grp;
                uint32_t pk[8];
#pragma unroll
                for (int e = 0; e < 16; e += 2) {
                    const float p0 = (k0 + e <= pos) ? ex2b(fmaf(sv[e], sl2, -lse)) : 0.f;
                    const float p1 = (k0 + e + 1 <= pos) ? ex2b(fmaf(sv[e + 1], sl2, -lse)) : 0.f;
                    pk[e / 2] = pack_f16(p0 * (dp[e] - dl), p1 * (dp[e + 1] - dl));
                }
                // packed into the first 8 of the 16 columns this group just read
                if (!warp_converged("dS TMEM store")) { ok = false; break; }
                tmem_st8u(tmem + lane_off + 64 * b + 16 * grp, pk);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&p_full[b]);
            }
            if (!ok) break;
            if (!warp_wait(acc_full, item_iter & 1, abort_flag, err)) break;
            tc_fence_after();
            {
                __half *dqrow = static_cast<__half *>(a.dq) + static_cast<int64_t>(lrow) * a.ldd + head * DH;
#pragma unroll 1
                for (int c = grp; c < DH / 32; c += kEwGroups) {
                    float v[32];
                    tmem_ld32(tmem + lane_off + 256 + c * 32, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] *= scale;
                    flag_range(maxabs32(v), a.err);
                    uint4 *d4 = reinterpret_cast<uint4 *>(dqrow + c * 32);
#pragma unroll
                    for (int qq = 0; qq < 4; ++qq)
                        d4[qq] = make_uint4(pack_f16(v[8 * qq], v[8 * qq + 1]), pack_f16(v[8 * qq + 2], v[8 * qq + 3]),
                                            pack_f16(v[8 * qq + 4], v[8 * qq + 5]), pack_f16(v[8 * qq + 6], v[8 * qq + 7]));
                }
            }
            tc_fence_before();
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// Single-pass backward (dh = 128).  One item = (head, 128-key tile kt); steps
// of 64 query rows over the steps that see the tile, in descending order of
// position (DescWalk): the items that run at the same time walk the same
// query rows in step, which keeps Q, dO and the dQ sum of those rows in L2.
//   TMEM columns (128 key lanes unless noted):
//     dV [0,128)  dK [128,256)                       accumulated per item
//     R[0] [256,384), R[1] [384,512): the buffer of steps g with g % 2 = b.
//     Within R[b], one step's columns are used three times over:
//       [0,64) S^T fp32      -> [0,32) P^T and [32,64) dS^T packed fp16
//                               (A operands of dV += P^T dO, dK += dS^T Q)
//       [64,128) dP^T fp32   -> dQ^T: lanes = head dims, columns = the
//                               step's 64 queries
//   Step g: warp 1 issues S^T = K Q^T into R[g%2] once step g-2's dV / dK /
//   dQ^T MMAs (which read P^T / dS^T there) are complete, and dP^T = V dO^T
//   once step g-2's dQ^T has been drained (both operands from shared memory);
//   the element-wise warps turn S^T into P^T while dP^T is computed, then
//   read dP^T and, after the four groups of a TMEM lane quarter have all read
//   S^T (a named barrier), write P^T and dS^T packed over S^T and dS^T also
//   to shared memory (one tile per buffer);
//   warp kMmaGWarp issues dV += P^T dO, dK += dS^T Q (A from TMEM) and
//   dQ^T = K^T dS^T over dP^T's columns (both operands from shared memory,
//   MN-major).  With two buffers the element-wise work of step g+1 overlaps
//   the dV / dK / dQ^T MMAs of step g, and nothing waits on a previous
//   step's MMAs except the reuse of a buffer two steps later.
//   Four drain warps (one per TMEM lane quarter) take dQ^T of step g out of
//   TMEM once its MMAs are complete, which frees the buffer, and add it to
//   the step's rows of the integer dQ sum in global memory as 32-bit fixed
//   point (value times 2^F_head, rounded), one global reduction per element
//   (a warp's reductions for one query row cover one 128-byte line).  Integer
//   addition is associative, so
//   the sum is the same bits whatever order the CTAs' additions reach L2 in:
//   the result is deterministic with no ordering between CTAs.  F_head comes
//   from a bound that holds for every partial sum of the head's dQ
//   (dq_frac_bits), so no sum can overflow.
template <int DH>
struct FusedCfg {
    using C = BCfg<DH>;
    static_assert(DH == 128, "the single-pass backward computes dQ^T with M = dh = 128");
    static constexpr int BQ = 64;
    static constexpr int QST = 3;
    static constexpr int QTILE = BQ * DH * 2;
    static constexpr int QATOM = BQ * C::SWB;
    static constexpr int VEC_BYTES = 3 * BQ * 4;
    static constexpr int DST_BYTES = 128 * BQ * 2;   // dS^T [128 keys][64 queries] fp16, 128-byte swizzle
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + C::TILE_BYTES;
    static constexpr int OFF_Q = OFF_V + C::TILE_BYTES;
    static constexpr int OFF_DO = OFF_Q + QST * QTILE;
    static constexpr int OFF_VEC = OFF_DO + QST * QTILE;
    static constexpr int OFF_DST = (OFF_VEC + QST * VEC_BYTES + 1023) / 1024 * 1024;   // [2] tiles
    static constexpr int OFF_BAR = OFF_DST + 2 * DST_BYTES;
    static constexpr int SMEM = OFF_BAR + 256 + 1024;
    static_assert(SMEM <= kMaxDynSmem, "single-pass backward tiles exceed the shared-memory limit");
    // kv_full/empty, q_full/empty[QST], s_full[2], dp_full[2], p_full[2], mma_done[2], buf_free[2],
    // acc_empty, drain, drain2 + TMEM slot + abort flag
    static_assert(8 * (2 + 2 * QST + 13) + 8 <= 256, "single-pass backward barriers exceed their slot");
    static constexpr uint32_t T_DV = 0, T_DK = 128, T_R = 256, R_COLS = 128;
    static constexpr uint32_t R_S = 0, R_PP = 0, R_PDS = 32, R_DP = 64, R_DQ = 64;
    static_assert(T_R + 2 * R_COLS <= 512, "single-pass backward TMEM columns");
};

constexpr int kEwThreads = 128 * kEwGroups;
// TMA warp, S^T/dP^T MMA warp, element-wise groups, 4 drain warps, dV/dK/dQ^T MMA warp
constexpr int kFusedThreads = 64 + kEwThreads + 128 + 32;

struct FusedParams {
    AttnBwdDesc d;
    const int *zig;
    int num_items;
};

// PART: one rank's share (AttnBwdDesc::rank >= 0), a separate instance so
// that the whole-layer instance carries none of its code.
template <int DH, bool PART>
__global__ void __launch_bounds__(kFusedThreads, 1)
    attn_bwd_fused_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                          const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mdO,
                          const FusedParams fp, const DevErr err) {
    using C = BCfg<DH>;
    using F = FusedCfg<DH>;
    const AttnBwdDesc &a = fp.d;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + F::OFF_BAR);
    uint64_t *kv_full = bars + 0, *kv_empty = bars + 1;
    uint64_t *q_full = bars + 2;                // [QST]
    uint64_t *q_empty = q_full + F::QST;        // [QST]
    uint64_t *s_full = q_empty + F::QST;        // [2] S^T of a step in R[b]
    uint64_t *dp_full = s_full + 2;             // [2] dP^T of a step in R[b]
    uint64_t *p_full = dp_full + 2;             // [2] P^T / dS^T of a step packed in R[b], dS^T in smem
    uint64_t *mma_done = p_full + 2;            // [2] dV / dK / dQ^T MMAs of a step complete
    uint64_t *buf_free = mma_done + 2;          // [2] dQ^T of a step read out of R[b]
    uint64_t *acc_empty = buf_free + 2;         // dV / dK of an item read out
    uint64_t *drain = acc_empty + 1;            // error path: each issuer's MMAs complete
    uint64_t *drain2 = drain + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain2 + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int nq64 = a.S / 64;
    const StepVis vis{a.D, a.chunk, nq64, PART ? a.rank : -1};
    const int q_row0 = PART ? a.q_row0 : 0;
    const float sl2 = 1.4426950408889634f * rsqrtf(static_cast<float>(DH));
    const float scale = rsqrtf(static_cast<float>(DH));
    constexpr int kDrainWarp = 2 + 4 * kEwGroups;
    constexpr int kMmaGWarp = kDrainWarp + 4;

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        mbar_init(kv_empty, 1);
        for (int s = 0; s < F::QST; ++s) {
            mbar_init(&q_full[s], 1);
            mbar_init(&q_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&dp_full[b], 1);
            mbar_init(&p_full[b], kEwThreads / 32);
            mbar_init(&mma_done[b], 1);
            mbar_init(&buf_free[b], 4);
        }
        mbar_init(acc_empty, kEwThreads / 32);
        mbar_init(drain, 1);
        mbar_init(drain2, 1);
        *abort_flag = 0;
        fence_mbar_init();
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
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int item_iter = 0, g = 0;
            bool ok = true;
            for (int it = blockIdx.x; it < fp.num_items && ok; it += gridDim.x, ++item_iter) {
                const int kt = a.kv_order[it] / a.H, head = a.kv_order[it] % a.H;
                if (!mbar_wait(kv_empty, (item_iter & 1) ^ 1, abort_flag, err)) break;
                mbar_arrive_tx(kv_full, 2 * C::TILE_BYTES);
                for (int t = 0; t < C::NATOM; ++t) {
                    tma_load_2d(smem + F::OFF_K + t * C::ATOM_BYTES, &mK, kv_full, head * DH + t * C::ATOM_COLS, kt * 128);
                    tma_load_2d(smem + F::OFF_V + t * C::ATOM_BYTES, &mV, kv_full, head * DH + t * C::ATOM_COLS, kt * 128);
                }
                DescWalk w;
                for (w.seek(vis, kt * 128); w.q < nq64; w.next(vis, kt * 128), ++g) {
                    const int q = w.q;
                    const int s = g % F::QST;
                    if (!mbar_wait(&q_empty[s], ((g / F::QST) & 1) ^ 1, abort_flag, err)) { ok = false; break; }
                    mbar_arrive_tx(&q_full[s], 2 * F::QTILE + F::VEC_BYTES);
                    for (int t = 0; t < C::NATOM; ++t) {
                        tma_load_2d(smem + F::OFF_Q + s * F::QTILE + t * F::QATOM, &mQ, &q_full[s],
                                    head * DH + t * C::ATOM_COLS, q * 64 - q_row0);
                        tma_load_2d(smem + F::OFF_DO + s * F::QTILE + t * F::QATOM, &mdO, &q_full[s],
                                    head * DH + t * C::ATOM_COLS, q * 64 - q_row0);
                    }
                    float *vec = reinterpret_cast<float *>(smem + F::OFF_VEC + s * F::VEC_BYTES);
                    bulk_load(vec, a.lse + static_cast<int64_t>(head) * a.S + q * 64, 256, &q_full[s]);
                    bulk_load(vec + 64, a.delta + static_cast<int64_t>(head) * a.S + q * 64, 256, &q_full[s]);
                    bulk_load(vec + 128, fp.zig + q * 64, 256, &q_full[s]);
                }
            }
            if (item_iter > 0) spin_drain(kv_full, (item_iter - 1) & 1, err.wait_limit);
            for (int s = 0; s < F::QST; ++s)
                if (g > s) {
                    const int last = g - 1 - ((g - 1 - s) % F::QST);
                    spin_drain(&q_full[s], (last / F::QST) & 1, err.wait_limit);
                }
        }
    } else if (warp == 1 || warp == kMmaGWarp) {
        // ------------------------------------------------------------ MMA issuers
        // Two warps issue: warp 1 the S^T / dP^T MMAs of each step, warp
        // kMmaGWarp the dV / dK / dQ^T MMAs.  Their MMAs are ordered by the
        // barriers alone (S^T/dP^T of step g complete -> s_full -> element-wise
        // -> p_full -> dV/dK/dQ^T of step g -> mma_done -> drain -> buf_free ->
        // S^T/dP^T of step g+2), so neither issuer waits behind the other's
        // queue.  In each warp the whole warp runs the loop; one elected lane
        // polls and issues (a commit tracks the MMAs of the thread that issues
        // it).
        const bool leader = elect_one();
        const int leader_lane = __ffs(__ballot_sync(0xffffffffu, leader)) - 1;
        int item_iter = 0, g = 0;
        bool ok = true;
        if (warp == 1) {
            constexpr uint32_t idS = idesc_f16(128, 64, false, false);
            const uint64_t dK0 = kdesc<DH>(smem_u32(smem + F::OFF_K), 0);
            const uint64_t dV0 = kdesc<DH>(smem_u32(smem + F::OFF_V), 0);
            for (int it = blockIdx.x; it < fp.num_items && ok; it += gridDim.x, ++item_iter) {
                const int kv0 = (a.kv_order[it] / a.H) * 128;
                if (!lead_wait(leader, leader_lane, kv_full, item_iter & 1, abort_flag, err)) break;
                DescWalk w;
                for (w.seek(vis, kv0); w.q < nq64; w.next(vis, kv0), ++g) {
                    const int s = g % F::QST, b = g & 1, n = g >> 1;
                    const uint32_t rb = tmem + F::T_R + b * F::R_COLS;
                    // S^T goes over step g-2's P^T / dS^T, free once its MMAs
                    // are complete
                    if (n > 0 && !lead_wait(leader, leader_lane, &mma_done[b], (n - 1) & 1, abort_flag, err)) {
                        ok = false;
                        break;
                    }
                    if (!lead_wait(leader, leader_lane, &q_full[s], (g / F::QST) & 1, abort_flag, err)) {
                        ok = false;
                        break;
                    }
                    if (leader) {
                        tc_fence_after();
                        const uint64_t dQ0 = kdesc64<DH>(smem_u32(smem + F::OFF_Q + s * F::QTILE), 0);
#pragma unroll
                        for (int kk = 0; kk < DH / 16; ++kk)
                            umma_ss(rb + F::R_S, desc_plus(dK0, kdesc_off<DH>(kk)),
                                    desc_plus(dQ0, kdesc64_off<DH>(kk)), idS, kk > 0);
                        umma_commit(&s_full[b]);
                    }
                    // dP^T goes over step g-2's dQ^T, free once drained
                    if (n > 0 && !lead_wait(leader, leader_lane, &buf_free[b], (n - 1) & 1, abort_flag, err)) {
                        ok = false;
                        break;
                    }
                    if (leader) {
                        tc_fence_after();
                        const uint64_t dO0 = kdesc64<DH>(smem_u32(smem + F::OFF_DO + s * F::QTILE), 0);
#pragma unroll
                        for (int kk = 0; kk < DH / 16; ++kk)
                            umma_ss(rb + F::R_DP, desc_plus(dV0, kdesc_off<DH>(kk)),
                                    desc_plus(dO0, kdesc64_off<DH>(kk)), idS, kk > 0);
                        umma_commit(&dp_full[b]);
                    }
                }
            }
        } else {
            constexpr uint32_t idG = idesc_f16(128, DH, false, true);
            constexpr uint32_t idQ = idesc_f16(DH, 64, true, true);
            // A of dQ^T = K^T: the K tile read MN-major (rows = keys, head dims
            // contiguous in two 128-byte atoms); K steps of 16 keys advance 2 KB
            const uint64_t dKt0 = sdesc(smem_u32(smem + F::OFF_K), C::ATOM_BYTES, 8 * C::SWB, C::LAYOUT);
            for (int it = blockIdx.x; it < fp.num_items && ok; it += gridDim.x, ++item_iter) {
                const int kv0 = (a.kv_order[it] / a.H) * 128;
                if (!lead_wait(leader, leader_lane, kv_full, item_iter & 1, abort_flag, err)) break;
                bool first = true;
                DescWalk w;
                for (w.seek(vis, kv0); w.q < nq64; w.next(vis, kv0), ++g) {
                    const int s = g % F::QST, b = g & 1, n = g >> 1;
                    if (!lead_wait(leader, leader_lane, &p_full[b], n & 1, abort_flag, err)) {
                        ok = false;
                        break;
                    }
                    // the first dV / dK MMA of an item overwrites the accumulators
                    // that the previous item's epilogue reads
                    if (first && item_iter > 0 &&
                        !lead_wait(leader, leader_lane, acc_empty, (item_iter - 1) & 1, abort_flag, err)) {
                        ok = false;
                        break;
                    }
                    if (leader) {
                        tc_fence_after();
                        const uint32_t rb = tmem + F::T_R + b * F::R_COLS;
                        const uint64_t gQ0 = mndesc64<DH>(smem_u32(smem + F::OFF_Q + s * F::QTILE), 0);
                        const uint64_t gO0 = mndesc64<DH>(smem_u32(smem + F::OFF_DO + s * F::QTILE), 0);
                        // B of dQ^T = dS^T [128 keys][64 queries]: MN-major, one atom wide
                        const uint64_t dSt0 = sdesc(smem_u32(smem + F::OFF_DST + b * F::DST_BYTES), 8192, 1024,
                                                    kSwizzle128);
                        // A operands from TMEM: queries 16 kk .. 16 kk + 15 packed at column 8 kk
#pragma unroll
                        for (int kk = 0; kk < F::BQ / 16; ++kk)
                            umma_ts(tmem + F::T_DV, rb + F::R_PP + kk * 8, desc_plus(gO0, mndesc64_off<DH>(kk)), idG,
                                    (!first || kk > 0) ? 1u : 0u);
#pragma unroll
                        for (int kk = 0; kk < F::BQ / 16; ++kk)
                            umma_ts(tmem + F::T_DK, rb + F::R_PDS + kk * 8, desc_plus(gQ0, mndesc64_off<DH>(kk)), idG,
                                    (!first || kk > 0) ? 1u : 0u);
                        // dQ^T [dh][64] = K^T dS^T over the 128 keys, 16 at a time,
                        // over dP^T's columns (read by every element-wise thread
                        // before p_full)
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            umma_ss(rb + F::R_DQ, desc_plus(dKt0, kk * 16 * C::SWB), desc_plus(dSt0, kk * 2048), idQ,
                                    kk > 0);
                        // this step's S^T / dP^T completed before its p_full, so
                        // the Q / dO stage is free once these MMAs are
                        umma_commit(&mma_done[b]);
                        umma_commit(&q_empty[s]);
                    }
                    first = false;
                }
                // likewise every S^T / dP^T of the item has read the K / V tile
                // before the item's last p_full
                if (leader && ok) umma_commit(kv_empty);
            }
        }
        uint64_t *my_drain = warp == 1 ? drain : drain2;
        const bool bad = __any_sync(0xffffffffu, !ok || *abort_flag);
        if (bad && leader) {
            umma_commit(my_drain);
            spin_drain(my_drain, 0, err.wait_limit);
        }
        __syncwarp();
    } else if (warp < kDrainWarp) {
        // ------------------------------------------------------------ element-wise groups
        const int grp = (warp - 2) / 4;         // query columns [16 grp, 16 grp + 16) of a step
        const int quarter = warp & 3;
        const int trow = quarter * 32 + lane;   // key row of the tile = TMEM lane (head dim for dQ^T)
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        int g = 0;
        for (int it = blockIdx.x; it < fp.num_items; it += gridDim.x) {
            const int kt = a.kv_order[it] / a.H, head = a.kv_order[it] % a.H;
            const int kv0 = kt * 128;
            const int key = kv0 + trow;
            bool ok = true, any = false;
            DescWalk w;
            for (w.seek(vis, kv0); w.q < nq64; w.next(vis, kv0), ++g) {
                const int s = g % F::QST, b = g & 1, n = g >> 1;
                const uint32_t rb = tmem + lane_off + F::T_R + b * F::R_COLS;
                if (!warp_wait(&s_full[b], n & 1, abort_flag, err)) { ok = false; break; }
                tc_fence_after();
                if (!warp_converged("S^T TMEM load")) { ok = false; break; }
                float sv[16], dp[16];
                tmem_ld16(rb + F::R_S + 16 * grp, sv);
                tmem_ld_wait();
                tc_fence_before();
                const float *vec = reinterpret_cast<const float *>(smem + F::OFF_VEC + s * F::VEC_BYTES);
                const int *pos = reinterpret_cast<const int *>(vec + 128);
                // the 64 query rows of a step lie in one zigzag chunk, so their
                // positions are consecutive: this key is visible to column e of
                // the group iff e >= key - pos0
                const int first_vis = key - pos[16 * grp];
                const float4 *lse4 = reinterpret_cast<const float4 *>(vec + 16 * grp);
                const float4 *dl4 = reinterpret_cast<const float4 *>(vec + 64 + 16 * grp);
                uint32_t pk[8], dk[8];
#pragma unroll
                for (int e4 = 0; e4 < 4; ++e4) {
                    const float4 l = lse4[e4];
                    const int e = 4 * e4;
                    // p = 2^kPOff P (the offset rides in the exponent)
                    float p0 = ex2b(fmaf(sv[e], sl2, kPOff - l.x)), p1 = ex2b(fmaf(sv[e + 1], sl2, kPOff - l.y));
                    float p2 = ex2b(fmaf(sv[e + 2], sl2, kPOff - l.z)), p3 = ex2b(fmaf(sv[e + 3], sl2, kPOff - l.w));
                    if (first_vis > 0) {
                        p0 = e >= first_vis ? p0 : 0.f;
                        p1 = e + 1 >= first_vis ? p1 : 0.f;
                        p2 = e + 2 >= first_vis ? p2 : 0.f;
                        p3 = e + 3 >= first_vis ? p3 : 0.f;
                    }
                    pk[2 * e4] = pack_f16(p0, p1);
                    pk[2 * e4 + 1] = pack_f16(p2, p3);
                    // P without the offset, kept for dS
                    sv[e] = p0 * kPOffInv;
                    sv[e + 1] = p1 * kPOffInv;
                    sv[e + 2] = p2 * kPOffInv;
                    sv[e + 3] = p3 * kPOffInv;
                }
                // dP^T of the step (issued once the drain freed its columns)
                if (!warp_wait(&dp_full[b], n & 1, abort_flag, err)) { ok = false; break; }
                tc_fence_after();
                if (!warp_converged("dP^T TMEM load")) { ok = false; break; }
                tmem_ld16(rb + F::R_DP + 16 * grp, dp);
                tmem_ld_wait();
                tc_fence_before();
#pragma unroll
                for (int e4 = 0; e4 < 4; ++e4) {
                    const float4 d = dl4[e4];
                    const int e = 4 * e4;
                    // dS = P (dP - Delta)
                    dk[2 * e4] = pack_f16(sv[e] * (dp[e] - d.x), sv[e + 1] * (dp[e + 1] - d.y));
                    dk[2 * e4 + 1] = pack_f16(sv[e + 2] * (dp[e + 2] - d.z), sv[e + 3] * (dp[e + 3] - d.w));
                }
                // P^T / dS^T go over the S^T columns that the four groups of this
                // lane quarter read: all four must have read them first
                asm volatile("bar.sync %0, 128;" ::"r"(3 + quarter) : "memory");
                tc_fence_after();
                any = true;
                if (!warp_converged("P^T/dS^T TMEM store")) { ok = false; break; }
                tmem_st8u(rb + F::R_PP + 8 * grp, pk);
                tmem_st8u(rb + F::R_PDS + 8 * grp, dk);
                // this key's row of dS^T: its 16 queries are the 16-byte chunks
                // 2 grp and 2 grp + 1 of the 128-byte row, 128-byte swizzled
                uint4 *row = reinterpret_cast<uint4 *>(smem + F::OFF_DST + b * F::DST_BYTES + trow * 128);
                row[(2 * grp) ^ (trow & 7)] = make_uint4(dk[0], dk[1], dk[2], dk[3]);
                row[(2 * grp + 1) ^ (trow & 7)] = make_uint4(dk[4], dk[5], dk[6], dk[7]);
                tmem_st_wait();
                fence_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[b]);
            }
            if (!ok) break;
            if (!any) continue;
            // the item's last step: its MMAs complete means dV and dK are too
            if (!warp_wait(&mma_done[(g - 1) & 1], ((g - 1) >> 1) & 1, abort_flag, err)) break;
            tc_fence_after();
            // groups 0, 1 write dV (offset removed) and groups 2, 3 write dK
            // (scaled), at the key owner's local row; each pair splits the
            // 32-column chunks.  One rank's share goes out as fp32 partial
            // sums, also times *dkv_mul.
            const int lrow = a.inv_map[key];
            const int which = grp >> 1;
            const float f = (which == 0 ? kPOffInv : scale) * (PART ? *a.dkv_mul : 1.0f);
            void *dstp = which == 0 ? a.dv : a.dk;
            __half *orow = PART ? nullptr : static_cast<__half *>(dstp) + static_cast<int64_t>(lrow) * a.ldd + head * DH;
            float *frow = PART ? (which == 0 ? a.dv_part : a.dk_part) + static_cast<int64_t>(lrow) * (a.H * DH) + head * DH
                               : nullptr;
            if (!warp_converged("dV/dK TMEM load")) break;
#pragma unroll 1
            for (int c = grp & 1; c < DH / 32; c += 2) {
                float v[32];
                tmem_ld32(tmem + lane_off + (which == 0 ? F::T_DV : F::T_DK) + c * 32, v);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] *= f;
                if (PART) {
                    float4 *d4 = reinterpret_cast<float4 *>(frow + c * 32);
#pragma unroll
                    for (int qq = 0; qq < 8; ++qq)
                        d4[qq] = make_float4(v[4 * qq], v[4 * qq + 1], v[4 * qq + 2], v[4 * qq + 3]);
                    continue;
                }
                flag_range(maxabs32(v), a.err);
                uint4 *d4 = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
                for (int qq = 0; qq < 4; ++qq)
                    d4[qq] = make_uint4(pack_f16(v[8 * qq], v[8 * qq + 1]), pack_f16(v[8 * qq + 2], v[8 * qq + 3]),
                                        pack_f16(v[8 * qq + 4], v[8 * qq + 5]), pack_f16(v[8 * qq + 6], v[8 * qq + 7]));
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty);
        }
    } else if (warp < kMmaGWarp) {
        // ------------------------------------------------------------ drain warps
        // dQ^T of every step out of TMEM (thread = head dim), which frees the
        // buffer, then added to the integer dQ sum in global memory with one
        // reduction per element.  Measured against staging the integers in
        // shared memory for TMA reduce-adds, this is faster: the drain's time
        // per step no longer delays the buffer's next use.
        const int quarter = warp & 3;
        const int d = quarter * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const int hh = a.H * DH;
        int g = 0;
        bool ok = true;
        for (int it = blockIdx.x; it < fp.num_items && ok; it += gridDim.x) {
            const int head = a.kv_order[it] % a.H, kv0 = (a.kv_order[it] / a.H) * 128;
            const float dq_scale = ldexpf(1.0f, dq_frac_bits(a.dq_bound + 3 * head, DH));
            DescWalk w;
            for (w.seek(vis, kv0); w.q < nq64; w.next(vis, kv0), ++g) {
                const int b = g & 1, n = g >> 1;
                if (!warp_wait(&mma_done[b], n & 1, abort_flag, err)) { ok = false; break; }
                tc_fence_after();
                if (!warp_converged("dQ^T TMEM load")) { ok = false; break; }
                float v[64];
                const uint32_t rb = tmem + lane_off + F::T_R + b * F::R_COLS;
                tmem_ld32(rb + F::R_DQ, *reinterpret_cast<float(*)[32]>(v));
                tmem_ld32(rb + F::R_DQ + 32, *reinterpret_cast<float(*)[32]>(v + 32));
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&buf_free[b]);
                // one global reduction per element: a warp's 32 head dims of one
                // query row are one 128-byte line
                int *col = a.dq_acc + (static_cast<int64_t>(w.q) * 64 - q_row0) * hh + head * DH + d;
#pragma unroll
                for (int j = 0; j < 64; ++j) atomicAdd(col + j * hh, __float2int_rn(v[j] * dq_scale));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// dQ = (fixed-point sum) 2^-F_head / sqrt(dh) as fp16, 8 elements per thread.
__global__ void dq_convert_kernel(const int *acc, const unsigned int *bound, __half *dq, int64_t ldd, int S, int h,
                                  int dh, unsigned int *err) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= static_cast<int64_t>(S) * h / 8) return;
    const int64_t e = i * 8;
    const int64_t row = e / h;
    const int col = static_cast<int>(e - row * h);
    const float f = ldexpf(rsqrtf(static_cast<float>(dh)), -dq_frac_bits(bound + 3 * (col / dh), dh));
    const int4 t0 = *reinterpret_cast<const int4 *>(acc + e);
    const int4 t1 = *reinterpret_cast<const int4 *>(acc + e + 4);
    const float v[8] = {t0.x * f, t0.y * f, t0.z * f, t0.w * f, t1.x * f, t1.y * f, t1.z * f, t1.w * f};
    float m = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[j]));
    flag_range(m, err);
    *reinterpret_cast<uint4 *>(dq + row * ldd + col) =
        make_uint4(pack_f16(v[0], v[1]), pack_f16(v[2], v[3]), pack_f16(v[4], v[5]), pack_f16(v[6], v[7]));
}

template <int DH>
struct BwdMaps {
    CUtensorMap q, k, v, dout;
    bool make(const AttnBwdDesc &a) {
        using C = BCfg<DH>;
        const int h = a.H * DH;
        const auto swz = swz_of<DH>();
        bool ok = encode_tensor_map_2d(&q, a.q, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, h, a.q_rows, int64_t(h) * 2, C::ATOM_COLS, 128, swz);
        ok = ok && encode_tensor_map_2d(&k, a.k, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, h, a.S, int64_t(h) * 2, C::ATOM_COLS, 128, swz);
        ok = ok && encode_tensor_map_2d(&v, a.v, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, h, a.S, int64_t(h) * 2, C::ATOM_COLS, 128, swz);
        ok = ok && encode_tensor_map_2d(&dout, a.dout, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, h, a.q_rows, int64_t(h) * 2, C::ATOM_COLS, 128, swz);
        return ok;
    }
};

BwdParams make_params(const AttnBwdDesc &a, const int *zig, const int *qtile_maxpos) {
    BwdParams bp;
    bp.d = a;
    bp.zig = zig;
    bp.qtile_maxpos = qtile_maxpos;
    bp.num_items = (a.S / 128) * a.H;
    return bp;
}

template <int DH>
cudaError_t launch_dkdv_impl(const AttnBwdDesc &a, const DevErr &err, int num_sms, cudaStream_t st, const int *zig) {
    using C = BCfg<DH>;
    BwdMaps<DH> m;
    if (!m.make(a)) return cudaErrorInvalidValue;
    // Q and dO sub-tiles of 64 rows
    const int h = a.H * DH;
    const auto swz = swz_of<DH>();
    bool ok = encode_tensor_map_2d(&m.q, a.q, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, h, a.S, int64_t(h) * 2, C::ATOM_COLS, 64, swz);
    ok = ok && encode_tensor_map_2d(&m.dout, a.dout, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, h, a.S, int64_t(h) * 2, C::ATOM_COLS, 64, swz);
    if (!ok) return cudaErrorInvalidValue;
    KvParams kp;
    kp.d = a;
    kp.zig = zig;
    kp.num_items = (a.S / 128) * a.H;
    const int grid = kp.num_items < num_sms ? kp.num_items : num_sms;
    auto k1 = attn_dkdv2_kernel<DH>;
    cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, KvCfg<DH>::SMEM);
    if (e != cudaSuccess) return e;
    k1<<<grid, kBwdThreads2, KvCfg<DH>::SMEM, st>>>(m.q, m.k, m.v, m.dout, kp, err);
    return cudaGetLastError();
}

template <int DH>
cudaError_t launch_dq_impl(const AttnBwdDesc &a, const DevErr &err, int num_sms, cudaStream_t st, const int *zig,
                           const int *qtile_maxpos) {
    using C = BCfg<DH>;
    BwdMaps<DH> m;
    if (!m.make(a)) return cudaErrorInvalidValue;
    // K and V sub-tiles of 64 keys
    const int h = a.H * DH;
    const auto swz = swz_of<DH>();
    bool ok = encode_tensor_map_2d(&m.k, a.k, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, h, a.S, int64_t(h) * 2, C::ATOM_COLS, 64, swz);
    ok = ok && encode_tensor_map_2d(&m.v, a.v, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, h, a.S, int64_t(h) * 2, C::ATOM_COLS, 64, swz);
    if (!ok) return cudaErrorInvalidValue;
    const BwdParams bp = make_params(a, zig, qtile_maxpos);
    const int grid = bp.num_items < num_sms ? bp.num_items : num_sms;
    auto k2 = attn_dq2_kernel<DH>;
    cudaError_t e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, Dq2Cfg<DH>::SMEM);
    if (e != cudaSuccess) return e;
    k2<<<grid, kBwdThreads2, Dq2Cfg<DH>::SMEM, st>>>(m.q, m.k, m.v, m.dout, bp, err);
    return cudaGetLastError();
}



template <int DH>
cudaError_t launch_fused_impl(const AttnBwdDesc &a, const DevErr &err, int num_sms, cudaStream_t st, const int *zig) {
    using C = BCfg<DH>;
    BwdMaps<DH> m;
    if (!m.make(a)) return cudaErrorInvalidValue;
    // Q and dO sub-tiles of 64 rows
    const int h = a.H * DH;
    const auto swz = swz_of<DH>();
    bool ok = encode_tensor_map_2d(&m.q, a.q, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, h, a.q_rows, int64_t(h) * 2, C::ATOM_COLS, 64, swz);
    ok = ok && encode_tensor_map_2d(&m.dout, a.dout, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, h, a.q_rows, int64_t(h) * 2, C::ATOM_COLS, 64, swz);
    if (!ok) return cudaErrorInvalidValue;
    FusedParams fp;
    fp.d = a;
    fp.zig = zig;
    fp.num_items = a.rank < 0 ? (a.S / 128) * a.H : a.kv_items;
    if (fp.num_items <= 0) return cudaSuccess;
    // at most one CTA per SM, so every CTA is resident (the dQ order waits need it)
    const int grid = fp.num_items < num_sms ? fp.num_items : num_sms;
    auto k = a.rank < 0 ? attn_bwd_fused_kernel<DH, false> : attn_bwd_fused_kernel<DH, true>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, FusedCfg<DH>::SMEM);
    if (e != cudaSuccess) return e;
    k<<<grid, kFusedThreads, FusedCfg<DH>::SMEM, st>>>(m.q, m.k, m.v, m.dout, fp, err);
    return cudaGetLastError();
}

}  // namespace

bool attn_bwd_fused_supported(int dh) { return dh == 128; }

cudaError_t launch_attn_bwd_fused(const AttnBwdDesc &a, const DevErr &err, int num_sms, cudaStream_t st,
                                  const int *zig) {
    if (a.dh != 128 || !a.dq_acc || !a.dq_bound) return cudaErrorInvalidValue;
    if (a.q_row0 < 0 || a.q_row0 % 64 || a.q_rows % 64 || a.q_row0 + a.q_rows > a.S) return cudaErrorInvalidValue;
    if (a.rank >= 0) {
        const size_t bytes = static_cast<size_t>(a.S) * a.H * a.dh * sizeof(float);
        if (a.rank >= a.D || !a.dk_part || !a.dv_part || !a.dkv_mul) return cudaErrorInvalidValue;
        cudaError_t e = cudaMemsetAsync(a.dk_part, 0, bytes, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(a.dv_part, 0, bytes, st);
        if (e != cudaSuccess) return e;
    }
    return launch_fused_impl<128>(a, err, num_sms, st, zig);
}

cudaError_t launch_dq_convert(const AttnBwdDesc &a, cudaStream_t st) {
    const int h = a.H * a.dh;
    const int64_t n8 = static_cast<int64_t>(a.q_rows) * h / 8;
    if (n8 == 0) return cudaSuccess;
    const int threads = 256;
    const int64_t blocks = (n8 + threads - 1) / threads;
    dq_convert_kernel<<<static_cast<unsigned int>(blocks), threads, 0, st>>>(
        a.dq_acc, a.dq_bound, static_cast<__half *>(a.dq), a.ldd, a.q_rows, h, a.dh, a.err);
    return cudaGetLastError();
}

cudaError_t launch_attn_delta(const AttnBwdDesc &a, int num_sms, cudaStream_t st) {
    if (a.dq_acc) {
        cudaError_t e = cudaMemsetAsync(a.dq_bound, 0, static_cast<size_t>(3) * a.H * sizeof(unsigned int), st);
        if (e != cudaSuccess) return e;
    }
    if (a.dh % 8 || a.dh < 8 || a.dh > 256 || 32 % (a.dh / 8)) return cudaErrorInvalidValue;
    if (a.q_row0 < 0 || a.q_rows < 0 || a.q_row0 + a.q_rows > a.S) return cudaErrorInvalidValue;
    // without the fused kernel's sums only the O / dO rows are read
    const int64_t rows = a.dq_acc ? (a.q_rows > a.S ? a.q_rows : a.S) : a.q_rows;
    if (rows == 0) return cudaSuccess;
    const int hpw = 256 / a.dh;
    const int64_t warps = rows * ((a.H + hpw - 1) / hpw);
    const int64_t want = (warps * 32 + 255) / 256;
    const int blocks = static_cast<int>(want < 8LL * num_sms ? want : 8LL * num_sms);
    attn_delta_kernel<<<blocks, 256, static_cast<size_t>(3) * a.H * sizeof(unsigned int), st>>>(
        static_cast<const __half *>(a.o), static_cast<const __half *>(a.dout), static_cast<const __half *>(a.k),
        static_cast<const __half *>(a.v), a.delta, a.dq_acc, a.dq_bound, a.S, a.H, a.dh, a.q_row0, a.q_rows,
        a.dq_acc ? a.S : 0);
    return cudaGetLastError();
}

cudaError_t launch_attn_dkdv(const AttnBwdDesc &a, const DevErr &err, int num_sms, cudaStream_t st, const int *zig) {
    if (a.rank >= 0 || a.q_row0 != 0 || a.q_rows != a.S) return cudaErrorInvalidValue;
    switch (a.dh) {
        case 32: return launch_dkdv_impl<32>(a, err, num_sms, st, zig);
        case 64: return launch_dkdv_impl<64>(a, err, num_sms, st, zig);
        case 128: return launch_dkdv_impl<128>(a, err, num_sms, st, zig);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_attn_dq(const AttnBwdDesc &a, const DevErr &err, int num_sms, cudaStream_t st, const int *zig,
                           const int *qtile_maxpos) {
    if (a.rank >= 0 || a.q_row0 != 0 || a.q_rows != a.S) return cudaErrorInvalidValue;
    switch (a.dh) {
        case 32: return launch_dq_impl<32>(a, err, num_sms, st, zig, qtile_maxpos);
        case 64: return launch_dq_impl<64>(a, err, num_sms, st, zig, qtile_maxpos);
        case 128: return launch_dq_impl<128>(a, err, num_sms, st, zig, qtile_maxpos);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace tsp
