// Host side of the C ABI: the plan (shape checks, zigzag map, shard schedules,
// workspace layout, device tables, work orders) and the forward / backward
// launch sequences.  Every step of the layer runs in the kernels of this
// library; this file only validates arguments and enqueues launches.
#include <algorithm>
#include <chrono>
#include <cstdio>
#include <thread>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <climits>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/tsp.h"
#include "../../include/tsp_testing.h"
#include "common.cuh"
#include "internal.h"

#define TSP_API extern "C" __attribute__((visibility("default")))

struct tsp_plan_s {
    int h, H, F, D, dh;
    int64_t S, L, c;
    std::vector<int32_t> zig;  // local row -> global position
    // device state, created on first use on the then-current device
    bool dev_ready = false;
    int device = -1;
    int num_sms = 0;
    int32_t *d_zig = nullptr, *d_inv = nullptr, *d_qmax = nullptr;
    int32_t *d_fwd_order = nullptr, *d_kv_order = nullptr, *d_q_order = nullptr;
    // per-rank forward orders (one rank's query blocks, paired in waves), concatenated
    int32_t *d_rank_fwd_order = nullptr;
    std::vector<int> rank_fwd_off, rank_fwd_items;
    // per-rank backward orders (the key tiles one rank's rows see, paired in waves), concatenated
    int32_t *d_rank_bwd_order = nullptr;
    std::vector<int> rank_bwd_off, rank_bwd_items;
    unsigned int *d_err = nullptr;
    int fwd_items = 0;
    long long wait_limit = 0;
    std::mutex mu;
    // profiling: per stage, the (start, stop) events recorded since enable
    bool profiling = false;
    std::vector<std::pair<cudaEvent_t, cudaEvent_t>> prof[TSP_NUM_STAGES];
    int64_t prof_launches[TSP_NUM_STAGES] = {};
    int64_t launches = 0;
};

namespace {

using namespace tsp;

constexpr size_t kAlign = 256;
size_t up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

// Byte layout of the saved-activation buffer and of the backward scratch.
// fp16: a, q, k, v, o, b, g, the weight copies, du, dyh, dO, dqkv, dy16;
// bf16: u; fp32: the rest.  `scales` holds the weight conversion scales
// (kScaleInv + i = 2^-e_i, kScale + i = 2^e_i for wqkv, wo, w1, w2);
// `gscales` the gradient scale of a backward call (2^-k, 2^k).
struct Layout {
    size_t rstd1, a, q, k, v, o, lse, y, rstd2, b, u, g, wqkv_h, wo_h, w1_h, w2_h, scales, cpart, saved_total;
    size_t du, db, dy, dyh, dO, delta, dqkv, da, dgp, dy16, gscales, gpart, dq_acc, dq_bound, bwd_total;
};
constexpr int kScaleInv = 0, kScale = 8;
constexpr int kTargetWeights = 12;  // largest |w| * 2^e in [2^11, 2^12)
constexpr int kTargetGrad = 4;      // largest |dY| * 2^k in [2^3, 2^4)

Layout layout_of(const tsp_plan_s *p) {
    Layout l{};
    const size_t S = p->S, h = p->h, F = p->F, H = p->H;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off += up(bytes);
        return o;
    };
    l.rstd1 = take(S * 4);
    l.a = take(S * h * 2);
    l.q = take(S * h * 2);
    l.k = take(S * h * 2);
    l.v = take(S * h * 2);
    l.o = take(S * h * 2);
    l.lse = take(H * S * 4);
    l.y = take(S * h * 4);
    l.rstd2 = take(S * 4);
    l.b = take(S * h * 2);
    l.u = take(S * F * 2);
    l.g = take(S * F * 2);
    l.wqkv_h = take(3 * h * h * 2);
    l.wo_h = take(h * h * 2);
    l.w1_h = take(F * h * 2);
    l.w2_h = take(h * F * 2);
    l.scales = take(64 * 4);
    l.cpart = take(static_cast<size_t>(kMaxConv) * kConvBlocks * 4);
    l.saved_total = off;
    off = 0;
    l.du = take(S * F * 2);
    l.db = take(S * h * 4);
    l.dy = take(S * h * 4);
    l.dyh = take(S * h * 2);
    l.dO = take(S * h * 2);
    l.delta = take(H * S * 4);
    l.dqkv = take(S * 3 * h * 2);
    l.da = take(S * h * 4);
    l.dgp = take(static_cast<size_t>(rmsnorm_bwd_partial_blocks(static_cast<int>(S))) * h * 4);
    l.dy16 = take(S * h * 2);
    l.gscales = take(64 * 4);
    l.gpart = take(static_cast<size_t>(kMaxConv) * kConvBlocks * 4);
    l.dq_acc = p->dh == 128 ? take(S * h * 4) : 0;
    l.dq_bound = take(3 * H * 4);
    l.bwd_total = off;
    return l;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

using EncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                              const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn get_encode() {
    static EncodeFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeFn>(f);
    });
    return fn;
}

tsp_status cuda_status(cudaError_t e) { return e == cudaSuccess ? TSP_OK : TSP_ERR_CUDA; }

// Host copies of the kernels' tables: inverse map, largest position of each
// 128-row local query tile, and the work orders of the attention kernels
// (head-major, longest item first per head; the forward and dK/dV orders are
// paired in waves before upload, device_orders).  Needs no GPU.
struct HostTables {
    std::vector<int32_t> inv, qmax, forder, korder, qorder;
};

HostTables host_tables(const tsp_plan_s *p) {
    HostTables t;
    const int64_t S = p->S;
    const int H = p->H;
    std::vector<int32_t> &inv = t.inv, &qmax = t.qmax;
    inv.resize(S);
    qmax.resize(S / 128);
    for (int64_t i = 0; i < S; ++i) inv[p->zig[i]] = static_cast<int32_t>(i);
    for (int64_t t = 0; t < S / 128; ++t) {
        int32_t m = 0;
        for (int64_t i = t * 128; i < t * 128 + 128; ++i) m = std::max(m, p->zig[i]);
        qmax[t] = m;
    }
    // forward items: (256-row query block, head), cost = key tiles
    std::vector<std::pair<int, int>> fitems;
    for (int64_t qb = 0; qb < S / 256; ++qb) {
        int32_t m = std::max(qmax[2 * qb], qmax[2 * qb + 1]);
        for (int hd = 0; hd < H; ++hd) fitems.push_back({static_cast<int>(qb * H + hd), m / 128 + 1});
    }
    // Head-major, longest first within a head (then paired in waves for the
    // device, pair_waves): the CTAs running at the same time share one head's
    // K/V (64 MiB at S = 128K) in L2 instead of streaming every head's K/V
    // from HBM.
    std::stable_sort(fitems.begin(), fitems.end(), [H](auto &x, auto &y) {
        const int hx = x.first % H, hy = y.first % H;
        return hx != hy ? hx < hy : x.second > y.second;
    });
    std::vector<int32_t> &forder = t.forder;
    for (auto &it : fitems) {
        forder.push_back(it.first);
        forder.push_back(it.second);
    }
    // backward items: key tiles (cost = query tiles that see them) and query tiles (cost = key tiles)
    std::vector<std::pair<int, int64_t>> kitems, qitems;
    for (int64_t kt = 0; kt < S / 128; ++kt) {
        int64_t cost = 0;
        for (int64_t t = 0; t < S / 128; ++t) cost += qmax[t] >= kt * 128;
        for (int hd = 0; hd < H; ++hd) kitems.push_back({static_cast<int>(kt * H + hd), cost});
    }
    for (int64_t qt = 0; qt < S / 128; ++qt)
        for (int hd = 0; hd < H; ++hd) qitems.push_back({static_cast<int>(qt * H + hd), qmax[qt] / 128 + 1});
    auto by_cost = [H](auto &x, auto &y) {
        const int hx = x.first % H, hy = y.first % H;
        return hx != hy ? hx < hy : x.second > y.second;
    };
    std::stable_sort(kitems.begin(), kitems.end(), by_cost);
    std::stable_sort(qitems.begin(), qitems.end(), by_cost);
    std::vector<int32_t> &korder = t.korder, &qorder = t.qorder;
    for (auto &it : kitems) korder.push_back(it.first);
    for (auto &it : qitems) qorder.push_back(it.first);
    return t;
}

// Pairs every head's j-th longest item with its j-th shortest and deals the
// pairs in waves: the attention kernels hand items round-robin to G
// persistent CTAs (CTA i takes items i, i + G, ...), so a wave of G pairs is
// laid out as the G long items, then the G short ones in the same CTA order.
// Under causality the two items of a pair add up to the same length for every
// pair (key tile kt and key tile N-1-kt together see S/64 + 2 query steps),
// so every CTA finishes a wave at about the same time and the next wave starts
// in step, without a barrier.  Together with walks that start from a common
// end (the backward walks query steps from the top position down, the forward
// walks key tiles from 0 up) the rows that the CTAs touch at one time stay
// within one wave's length differences, a few MB, instead of spreading over
// the whole head (128 MB at S = 128K), which is more than L2 holds.
// `order` is head-major with the longest items of a head first (host_tables);
// `width` table entries per item.
void pair_waves(std::vector<int32_t> &order, int width, int H, int G) {
    const int64_t n = static_cast<int64_t>(order.size()) / width;
    std::vector<int64_t> longs, shorts;  // item indices into `order`
    int64_t start = 0;
    while (start < n) {
        const int head = order[start * width] % H;
        int64_t end = start;
        while (end < n && order[end * width] % H == head) ++end;
        const int64_t m = end - start;
        for (int64_t j = 0; j < m / 2; ++j) {
            longs.push_back(start + j);
            shorts.push_back(end - 1 - j);
        }
        if (m & 1) {  // the middle item pairs with nothing
            longs.push_back(start + m / 2);
            shorts.push_back(-1);
        }
        start = end;
    }
    std::vector<int32_t> out;
    out.reserve(order.size());
    const int64_t np = static_cast<int64_t>(longs.size());
    auto emit = [&](int64_t idx) {
        if (idx >= 0)
            for (int k = 0; k < width; ++k) out.push_back(order[idx * width + k]);
    };
    for (int64_t w0 = 0; w0 < np; w0 += G) {
        const int64_t w1 = std::min<int64_t>(w0 + G, np);
        for (int64_t j = w0; j < w1; ++j) emit(longs[j]);
        for (int64_t j = w0; j < w1; ++j) emit(shorts[j]);
    }
    order.swap(out);
}

// The work orders as uploaded for a device with G SMs.  The dQ kernel's
// order (head sizes 32 and 64) keeps the host order.
void device_orders(HostTables &t, int H, int G) {
    pair_waves(t.forder, 2, H, G);
    pair_waves(t.korder, 1, H, G);
}

// Largest gap, over the rounds of G items, between the earliest and the
// latest start of a round's items when CTA i runs items i, i + G, ... and an
// item takes `cost` units.
int64_t start_spread(const std::vector<int64_t> &cost, int G) {
    std::vector<int64_t> t(G, 0);
    int64_t worst = 0;
    for (size_t r0 = 0; r0 < cost.size(); r0 += G) {
        const size_t n = std::min<size_t>(G, cost.size() - r0);
        const auto [lo, hi] = std::minmax_element(t.begin(), t.begin() + n);
        worst = std::max(worst, *hi - *lo);
        for (size_t i = 0; i < n; ++i) t[i] += cost[r0 + i];
    }
    return worst;
}

// The backward work order of rank r for G SMs: the key tiles that its rows
// see (its highest chunk, 2D-1-r, ends at position (2D-r) c - 1), taken from
// the host order before pairing (a head's tiles in ascending order there, so
// also longest first for one rank's rows).  Paired in waves, unless the
// head-major order keeps the CTAs' start times closer together: for the
// rank that holds the two middle chunks most key tiles cost the same, and
// long-with-short pairs then differ in length.  The order does not change the
// results.
std::vector<int32_t> rank_kv_order(const tsp_plan_s *p, const HostTables &t, int r, int G) {
    const int64_t last = (2 * p->D - r) * p->c - 1;
    std::vector<int32_t> sub;
    for (int32_t it : t.korder)
        if (static_cast<int64_t>(it / p->H) * 128 <= last) sub.push_back(it);
    // cost of key tile kt: the rank's 64-row steps that reach position 128 kt
    const int64_t L = p->L, steps = L / 64, ntiles = p->S / 128;
    std::vector<int64_t> tile_cost(ntiles, 0);
    for (int64_t q = 0; q < steps; ++q) {
        int32_t mx = 0;
        for (int64_t i = 0; i < 64; ++i) mx = std::max(mx, p->zig[r * L + q * 64 + i]);
        for (int64_t kt = 0; kt <= mx / 128 && kt < ntiles; ++kt) ++tile_cost[kt];
    }
    auto costs = [&](const std::vector<int32_t> &order) {
        std::vector<int64_t> c(order.size());
        for (size_t i = 0; i < order.size(); ++i) c[i] = tile_cost[order[i] / p->H];
        return c;
    };
    std::vector<int32_t> paired = sub;
    pair_waves(paired, 1, p->H, G);
    return start_spread(costs(paired), G) <= start_spread(costs(sub), G) ? paired : sub;
}

// Device tables: map, inverse map, per-query-tile max position and the work
// orders of the attention kernels (paired in waves, pair_waves).
tsp_status ensure_device(tsp_plan_s *p) {
    std::lock_guard<std::mutex> g(p->mu);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return TSP_ERR_CUDA;
    if (p->dev_ready) return dev == p->device ? TSP_OK : TSP_ERR_INVALID_ARG;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return TSP_ERR_CUDA;
    if (prop.major != 10) return TSP_ERR_UNSUPPORTED;
    if (!get_encode()) return TSP_ERR_CUDA;
    HostTables t = host_tables(p);
    // per-rank forward orders: the 256-row query blocks of rank r, taken from
    // the host order before pairing, then paired in waves by themselves
    std::vector<int32_t> rank_orders;
    p->rank_fwd_off.assign(p->D, 0);
    p->rank_fwd_items.assign(p->D, 0);
    if (p->L % 256 == 0) {
        const int64_t blocks = p->L / 256;
        for (int r = 0; r < p->D; ++r) {
            std::vector<int32_t> sub;
            for (size_t i = 0; i + 1 < t.forder.size(); i += 2) {
                const int64_t qb = t.forder[i] / p->H;
                if (qb >= r * blocks && qb < (r + 1) * blocks) {
                    sub.push_back(t.forder[i]);
                    sub.push_back(t.forder[i + 1]);
                }
            }
            pair_waves(sub, 2, p->H, prop.multiProcessorCount);
            p->rank_fwd_off[r] = static_cast<int>(rank_orders.size());
            p->rank_fwd_items[r] = static_cast<int>(sub.size() / 2);
            rank_orders.insert(rank_orders.end(), sub.begin(), sub.end());
        }
    }
    // per-rank backward orders (rank_kv_order)
    std::vector<int32_t> rank_korders;
    p->rank_bwd_off.assign(p->D, 0);
    p->rank_bwd_items.assign(p->D, 0);
    for (int r = 0; r < p->D; ++r) {
        const std::vector<int32_t> sub = rank_kv_order(p, t, r, prop.multiProcessorCount);
        p->rank_bwd_off[r] = static_cast<int>(rank_korders.size());
        p->rank_bwd_items[r] = static_cast<int>(sub.size());
        rank_korders.insert(rank_korders.end(), sub.begin(), sub.end());
    }
    device_orders(t, p->H, prop.multiProcessorCount);

    auto upload = [](int32_t **dst, const std::vector<int32_t> &v) {
        if (cudaMalloc(dst, v.size() * 4) != cudaSuccess) return false;
        return cudaMemcpy(*dst, v.data(), v.size() * 4, cudaMemcpyHostToDevice) == cudaSuccess;
    };
    if (!upload(&p->d_zig, p->zig) || !upload(&p->d_inv, t.inv) || !upload(&p->d_qmax, t.qmax) ||
        !upload(&p->d_fwd_order, t.forder) || !upload(&p->d_kv_order, t.korder) || !upload(&p->d_q_order, t.qorder))
        return TSP_ERR_CUDA;
    if (!rank_orders.empty() && !upload(&p->d_rank_fwd_order, rank_orders)) return TSP_ERR_CUDA;
    if (!upload(&p->d_rank_bwd_order, rank_korders)) return TSP_ERR_CUDA;
    if (cudaMalloc(&p->d_err, sizeof(unsigned int)) != cudaSuccess) return TSP_ERR_CUDA;
    if (cudaMemset(p->d_err, 0, sizeof(unsigned int)) != cudaSuccess) return TSP_ERR_CUDA;
    p->fwd_items = static_cast<int>(t.forder.size() / 2);
    p->num_sms = prop.multiProcessorCount;
    // A single device-side wait may spin for about 2 s at the boost clock.
    p->wait_limit = 4000000000LL;
    p->device = dev;
    p->dev_ready = true;
    return TSP_OK;
}

tsp_status check_pending_error(tsp_plan_s *p) {
    unsigned int e = 0;
    if (cudaMemcpy(&e, p->d_err, sizeof(e), cudaMemcpyDeviceToHost) != cudaSuccess) return TSP_ERR_CUDA;
    if (e) {
        cudaMemset(p->d_err, 0, sizeof(unsigned int));
        return (e & kErrTimeout) ? TSP_ERR_TIMEOUT : TSP_ERR_RANGE;
    }
    return TSP_OK;
}

DevErr dev_err(const tsp_plan_s *p) { return DevErr{p->d_err, p->wait_limit}; }

// Enqueue one stage (nk kernel launches); with profiling on, bracket it with
// a pair of CUDA events on the same stream.
extern const char *kStageNames[TSP_NUM_STAGES];

// TSP_DEBUG_SYNC=1: after every stage, poll the stream for up to 30 s and log
// the stage's completion (or that it is still running) to stderr.  For
// localising a stuck or faulting kernel; off by default.
bool debug_sync() {
    static int v = -1;
    if (v < 0) {
        const char *e = std::getenv("TSP_DEBUG_SYNC");
        v = (e && e[0] == '1') ? 1 : 0;
    }
    return v == 1;
}

cudaError_t debug_wait(int id, cudaStream_t s) {
    const auto t0 = std::chrono::steady_clock::now();
    while (true) {
        cudaError_t q = cudaStreamQuery(s);
        double ms = std::chrono::duration<double, std::milli>(std::chrono::steady_clock::now() - t0).count();
        if (q == cudaSuccess) {
            std::fprintf(stderr, "[tsp] stage %-20s done (%.3f ms after launch)\n", kStageNames[id], ms);
            return cudaSuccess;
        }
        if (q != cudaErrorNotReady) {
            std::fprintf(stderr, "[tsp] stage %-20s failed: %s\n", kStageNames[id], cudaGetErrorString(q));
            return q;
        }
        if (ms > 30000.0) {
            std::fprintf(stderr, "[tsp] stage %-20s still running after 30 s\n", kStageNames[id]);
            return cudaErrorLaunchTimeout;
        }
        std::this_thread::sleep_for(std::chrono::milliseconds(1));
    }
}

template <class F>
cudaError_t stage(tsp_plan_s *p, int id, int nk, cudaStream_t s, F &&launch) {
    cudaEvent_t a = nullptr, b = nullptr;
    if (p->profiling) {
        if (cudaEventCreate(&a) != cudaSuccess || cudaEventCreate(&b) != cudaSuccess) return cudaErrorUnknown;
        cudaEventRecord(a, s);
    }
    cudaError_t e = launch();
    if (p->profiling) {
        cudaEventRecord(b, s);
        p->prof[id].push_back({a, b});
        p->prof_launches[id] += nk;
    }
    if (e == cudaSuccess) p->launches += nk;
    if (e == cudaSuccess && debug_sync()) e = debug_wait(id, s);
    return e;
}

void profile_clear(tsp_plan_s *p) {
    for (auto &v : p->prof) {
        for (auto &ev : v) {
            cudaEventDestroy(ev.first);
            cudaEventDestroy(ev.second);
        }
        v.clear();
    }
    for (auto &n : p->prof_launches) n = 0;
}

const char *kStageNames[TSP_NUM_STAGES] = {
    "fwd_rmsnorm1", "fwd_qkv_gemm", "fwd_attention", "fwd_out_proj_gemm", "fwd_rmsnorm2", "fwd_w1_gelu_gemm",
    "fwd_w2_ring_gemm", "bwd_dgelu_gemm", "bwd_dw2_gemm", "bwd_dw1_gemm", "bwd_db_ring_gemm", "bwd_rmsnorm2",
    "bwd_do_gemm", "bwd_dwo_gemm", "bwd_attn_delta", "bwd_attn_dkdv", "bwd_attn_dq", "bwd_dwqkv_gemm",
    "bwd_da_gemm", "bwd_rmsnorm1", "fwd_convert_weights", "bwd_convert_dy", "bwd_attn_fused",
    "bwd_attn_dq_convert", "bwd_convert_dkdv"};

GemmDesc gemm(const void *A, int64_t lda, bool a_mn, const void *B, int64_t ldb, bool b_mn, int M, int N, int K,
              int epi, void *out, int64_t ldo, const float *alpha = nullptr) {
    GemmDesc g{};
    g.f16 = true;
    g.alpha = alpha;
    g.A = A;
    g.lda = lda;
    g.a_mn = a_mn;
    g.B = B;
    g.ldb = ldb;
    g.b_mn = b_mn;
    g.M = M;
    g.N = N;
    g.K = K;
    g.epi = epi;
    g.out = out;
    g.ldo = ldo;
    return g;
}

}  // namespace

namespace tsp {
bool encode_tensor_map_2d(CUtensorMap *m, const void *base, CUtensorMapDataType dtype, int elem_bytes, int64_t inner,
                          int64_t outer, int64_t outer_stride_bytes, int box_inner, int box_outer,
                          CUtensorMapSwizzle swz) {
    EncodeFn fn = get_encode();
    if (!fn) return false;
    (void)elem_bytes;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(outer_stride_bytes)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_outer)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, dtype, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}
}  // namespace tsp

// ===========================================================================
// C ABI
// ===========================================================================

TSP_API tsp_status tsp_plan(int h, int heads, int ffn, int64_t S, int D, tsp_plan_t *out) {
    if (!out) return TSP_ERR_INVALID_ARG;
    *out = nullptr;
    if (h <= 0 || heads <= 0 || ffn <= 0 || S <= 0 || D <= 0) return TSP_ERR_INVALID_ARG;
    if (S % (2 * D) || heads % D || ffn % D || h % heads) return TSP_ERR_INDIVISIBLE;
    const int dh = h / heads;
    if (dh != 32 && dh != 64 && dh != 128) return TSP_ERR_UNSUPPORTED;
    if (h % 128 || S % 256 || (S / D) % 128 || ffn % 128 || (ffn / D) % 64) return TSP_ERR_UNSUPPORTED;
    // The RMSNorm kernels number one warp per row in 32 bits (S * 32 < 2^31);
    // every other global index is 64-bit.  The bound below, heads * S * 32
    // (+ one block) below 2^31, covers that with a margin.
    if (S > (int64_t(1) << 28) || static_cast<int64_t>(heads) * S * 32 + 255 > INT32_MAX) return TSP_ERR_UNSUPPORTED;
    tsp_plan_s *p = new (std::nothrow) tsp_plan_s();
    if (!p) return TSP_ERR_INVALID_ARG;
    p->h = h;
    p->H = heads;
    p->F = ffn;
    p->D = D;
    p->dh = dh;
    p->S = S;
    p->L = S / D;
    p->c = S / (2 * D);
    p->zig.resize(S);
    for (int r = 0; r < D; ++r)
        for (int64_t i = 0; i < p->L; ++i)
            p->zig[r * p->L + i] = static_cast<int32_t>(i < p->c ? r * p->c + i : (2 * D - 1 - r) * p->c + (i - p->c));
    *out = p;
    return TSP_OK;
}

TSP_API void tsp_plan_destroy(tsp_plan_t p) {
    if (!p) return;
    if (p->dev_ready) {
        int cur = 0;
        cudaGetDevice(&cur);
        cudaSetDevice(p->device);
        cudaFree(p->d_zig);
        cudaFree(p->d_inv);
        cudaFree(p->d_qmax);
        cudaFree(p->d_fwd_order);
        cudaFree(p->d_kv_order);
        cudaFree(p->d_q_order);
        cudaFree(p->d_rank_fwd_order);
        cudaFree(p->d_rank_bwd_order);
        cudaFree(p->d_err);
        cudaSetDevice(cur);
    }
    delete p;
}

TSP_API tsp_status tsp_zigzag_map(tsp_plan_t p, int32_t *map_host) {
    if (!p || !map_host) return TSP_ERR_INVALID_ARG;
    std::memcpy(map_host, p->zig.data(), p->zig.size() * sizeof(int32_t));
    return TSP_OK;
}

TSP_API tsp_status tsp_shard_schedule(tsp_plan_t p, int phase, int32_t *sched) {
    if (!p || !sched || (phase != 0 && phase != 1)) return TSP_ERR_INVALID_ARG;
    const int D = p->D;
    for (int t = 0; t < D; ++t)
        for (int r = 0; r < D; ++r) sched[t * D + r] = phase == 0 ? t : (r + t) % D;
    return TSP_OK;
}

TSP_API tsp_status tsp_workspace_size(tsp_plan_t p, int training, size_t *ws, size_t *saved) {
    if (!p) return TSP_ERR_INVALID_ARG;
    Layout l = layout_of(p);
    if (training) {
        if (saved) *saved = l.saved_total;
        if (ws) *ws = l.bwd_total;
    } else {
        if (saved) *saved = 0;
        if (ws) *ws = l.saved_total;
    }
    return TSP_OK;
}

TSP_API double tsp_layer_flops(tsp_plan_t p, int backward) {
    if (!p) return 0.0;
    const double S = static_cast<double>(p->S), h = p->h, F = p->F;
    const double fwd = 2.0 * S * (4.0 * h * h + 2.0 * h * F) + 2.0 * h * S * (S + 1.0);
    return backward ? 2.0 * fwd : fwd;
}

TSP_API const char *tsp_status_string(tsp_status s) {
    switch (s) {
        case TSP_OK: return "TSP_OK";
        case TSP_ERR_INVALID_ARG: return "TSP_ERR_INVALID_ARG";
        case TSP_ERR_INDIVISIBLE: return "TSP_ERR_INDIVISIBLE";
        case TSP_ERR_UNSUPPORTED: return "TSP_ERR_UNSUPPORTED";
        case TSP_ERR_ALIGNMENT: return "TSP_ERR_ALIGNMENT";
        case TSP_ERR_CUDA: return "TSP_ERR_CUDA";
        case TSP_ERR_TIMEOUT: return "TSP_ERR_TIMEOUT";
        case TSP_ERR_RANGE: return "TSP_ERR_RANGE";
    }
    return "TSP_ERR_UNKNOWN";
}

TSP_API tsp_status tsp_sync_status(tsp_plan_t p, void *stream) {
    if (!p) return TSP_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return TSP_ERR_CUDA;
    if (!p->dev_ready) return TSP_OK;
    return check_pending_error(p);
}

namespace {

// The forward's launch sequence.  Intermediates live in `base` (the saved
// buffer, or the workspace of an inference call) with the layout of
// layout_of(); K and V, in global row order, go to `k` and `v`, which are
// base's K/V slots unless a caller-owned cache takes their place.
tsp_status forward_impl(tsp_plan_s *p, const void *x, const float *g1, const void *wqkv, const void *wo,
                        const float *g2, const void *w1, const void *w2, void *y, uint8_t *base, void *k, void *v,
                        cudaStream_t s) {
    const Layout l = layout_of(p);
    const int S = static_cast<int>(p->S), h = p->h, F = p->F, L = static_cast<int>(p->L);
    const DevErr err = dev_err(p);
    auto *rstd1 = reinterpret_cast<float *>(base + l.rstd1);
    void *a = base + l.a, *q = base + l.q, *o = base + l.o;
    auto *lse = reinterpret_cast<float *>(base + l.lse);
    auto *yres = reinterpret_cast<float *>(base + l.y);
    auto *rstd2 = reinterpret_cast<float *>(base + l.rstd2);
    void *b = base + l.b, *u = base + l.u, *g = base + l.g;
    void *wqkv_h = base + l.wqkv_h, *wo_h = base + l.wo_h, *w1_h = base + l.w1_h, *w2_h = base + l.w2_h;
    auto *scales = reinterpret_cast<float *>(base + l.scales);

#define TSP_STAGE(id, nk, call)                                                  \
    do {                                                                         \
        if (stage(p, id, nk, s, [&] { return (call); }) != cudaSuccess)          \
            return TSP_ERR_CUDA;                                                 \
    } while (0)
    // fp16 copies of the weights, each with its own power-of-two scale
    ConvBatch cb{};
    const void *wsrc[4] = {wqkv, wo, w1, w2};
    void *wdst[4] = {wqkv_h, wo_h, w1_h, w2_h};
    const int64_t wn[4] = {int64_t(3) * h * h, int64_t(h) * h, int64_t(F) * h, int64_t(h) * F};
    for (int i = 0; i < 4; ++i)
        cb.t[i] = ConvTensor{wsrc[i], wdst[i], wn[i], kTargetWeights, scales + kScaleInv + i, scales + kScale + i};
    cb.count = 4;
    cb.partial = reinterpret_cast<float *>(base + l.cpart);
    cb.err = p->d_err;
    TSP_STAGE(20, 2, launch_convert_f16(cb, s));
    TSP_STAGE(0, 1, launch_rmsnorm_fwd(x, nullptr, g1, a, true, rstd1, S, h, p->d_err, s));
    // QKV projection over the broadcast attention shards; K/V land at global rows.
    GemmDesc gq = gemm(a, h, false, wqkv_h, h, false, S, 3 * h, h, EPI_QKV, q, h, scales + kScaleInv + 0);
    gq.rowmap = p->d_zig;
    gq.hsplit = h;
    gq.out_k = k;
    gq.out_v = v;
    TSP_STAGE(1, 1, launch_gemm(gq, err, p->num_sms, s));
    AttnDesc ad{};
    ad.S = S;
    ad.L = L;
    ad.D = p->D;
    ad.H = p->H;
    ad.dh = p->dh;
    ad.chunk = static_cast<int>(p->c);
    ad.q = q;
    ad.k = k;
    ad.v = v;
    ad.o = o;
    ad.lse = lse;
    ad.order = p->d_fwd_order;
    ad.num_items = p->fwd_items;
    ad.q_row0 = 0;
    ad.q_rows = S;
    TSP_STAGE(2, 1, launch_attn_fwd(ad, err, p->num_sms, s));
    // out-projection (head-group partial sums in broadcast order) + residual, fp32 residual stream
    GemmDesc go = gemm(o, h, false, wo_h, h, false, S, h, h, EPI_RESID_F32, yres, h, scales + kScaleInv + 1);
    go.aux = x;
    go.ldaux = h;
    TSP_STAGE(3, 1, launch_gemm(go, err, p->num_sms, s));
    TSP_STAGE(4, 1, launch_rmsnorm_fwd(nullptr, yres, g2, b, true, rstd2, S, h, p->d_err, s));
    GemmDesc g1d = gemm(b, h, false, w1_h, h, false, S, F, h, EPI_GELU, u, F, scales + kScaleInv + 2);
    g1d.out2 = g;
    g1d.ldo2 = F;
    TSP_STAGE(5, 1, launch_gemm(g1d, err, p->num_sms, s));
    // W2 with the K loop over FFN shards in ring order (r + t) mod D, + residual
    GemmDesc g2d = gemm(g, F, false, w2_h, F, false, S, h, F, EPI_RESID_BF16, y, h, scales + kScaleInv + 3);
    g2d.aux = yres;
    g2d.ldaux = h;
    g2d.ring_rows = L;
    g2d.ring_kblocks = (F / p->D) / 64;
    TSP_STAGE(6, 1, launch_gemm(g2d, err, p->num_sms, s));
#undef TSP_STAGE
    return TSP_OK;
}

}  // namespace

TSP_API tsp_status tsp_layer_forward(tsp_plan_t p, const void *x, const float *g1, const void *wqkv, const void *wo,
                                     const float *g2, const void *w1, const void *w2, void *y, void *saved, void *ws,
                                     void *stream) {
    if (!p || !x || !g1 || !wqkv || !wo || !g2 || !w1 || !w2 || !y || !ws) return TSP_ERR_INVALID_ARG;
    for (const void *q : {x, (const void *)g1, wqkv, wo, (const void *)g2, w1, w2, (const void *)y, (const void *)ws})
        if (!aligned16(q)) return TSP_ERR_ALIGNMENT;
    if (saved && !aligned16(saved)) return TSP_ERR_ALIGNMENT;
    tsp_status st = ensure_device(p);
    if (st != TSP_OK) return st;
    const Layout l = layout_of(p);
    uint8_t *base = static_cast<uint8_t *>(saved ? saved : ws);
    return forward_impl(p, x, g1, wqkv, wo, g2, w1, w2, y, base, base + l.k, base + l.v,
                        static_cast<cudaStream_t>(stream));
}

TSP_API tsp_status tsp_layer_prefill(tsp_plan_t p, const void *x, const float *g1, const void *wqkv, const void *wo,
                                     const float *g2, const void *w1, const void *w2, void *y, void *k_cache,
                                     void *v_cache, void *ws, void *stream) {
    if (!p || !x || !g1 || !wqkv || !wo || !g2 || !w1 || !w2 || !y || !k_cache || !v_cache || !ws)
        return TSP_ERR_INVALID_ARG;
    for (const void *q : {x, (const void *)g1, wqkv, wo, (const void *)g2, w1, w2, (const void *)y, (const void *)k_cache,
                          (const void *)v_cache, (const void *)ws})
        if (!aligned16(q)) return TSP_ERR_ALIGNMENT;
    tsp_status st = ensure_device(p);
    if (st != TSP_OK) return st;
    return forward_impl(p, x, g1, wqkv, wo, g2, w1, w2, y, static_cast<uint8_t *>(ws), k_cache, v_cache,
                        static_cast<cudaStream_t>(stream));
}

// Scratch of the standalone ring MLP: U (bf16) and G (fp16) [S][F], the fp16
// copies of b, W1 and W2, their scales and the conversion partials.
struct RingLayout {
    size_t u, g, b_h, w1_h, w2_h, scales, cpart, total;
};
RingLayout ring_layout(const tsp_plan_s *p) {
    RingLayout r{};
    const size_t S = p->S, h = p->h, F = p->F;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off += up(bytes);
        return o;
    };
    r.u = take(S * F * 2);
    r.g = take(S * F * 2);
    r.b_h = take(S * h * 2);
    r.w1_h = take(F * h * 2);
    r.w2_h = take(h * F * 2);
    r.scales = take(64 * 4);
    r.cpart = take(static_cast<size_t>(kMaxConv) * kConvBlocks * 4);
    r.total = off;
    return r;
}

TSP_API tsp_status tsp_ring_mlp_workspace_size(tsp_plan_t p, size_t *ws_bytes) {
    if (!p || !ws_bytes) return TSP_ERR_INVALID_ARG;
    *ws_bytes = ring_layout(p).total;
    return TSP_OK;
}

// The layer's W1 + GELU and W2 ring steps, launched as the forward launches
// them, on caller buffers: b is copied to fp16 unscaled (like the layer's own
// RMSNorm output), the weights with their power-of-two scales.
TSP_API tsp_status tsp_ring_mlp_forward(tsp_plan_t p, const void *b, const void *w1, const void *w2, const float *resid,
                                        void *out, void *ws, void *stream) {
    if (!p || !b || !w1 || !w2 || !resid || !out || !ws) return TSP_ERR_INVALID_ARG;
    for (const void *q : {b, w1, w2, (const void *)resid, (const void *)out, (const void *)ws})
        if (!aligned16(q)) return TSP_ERR_ALIGNMENT;
    tsp_status st = ensure_device(p);
    if (st != TSP_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int S = static_cast<int>(p->S), h = p->h, F = p->F, L = static_cast<int>(p->L);
    const DevErr err = dev_err(p);
    const RingLayout rl = ring_layout(p);
    uint8_t *base = static_cast<uint8_t *>(ws);
    void *u = base + rl.u, *g = base + rl.g, *b_h = base + rl.b_h, *w1_h = base + rl.w1_h, *w2_h = base + rl.w2_h;
    auto *scales = reinterpret_cast<float *>(base + rl.scales);
#define TSP_STAGE(id, nk, call)                                                  \
    do {                                                                         \
        if (stage(p, id, nk, s, [&] { return (call); }) != cudaSuccess)          \
            return TSP_ERR_CUDA;                                                 \
    } while (0)
    ConvBatch cb{};
    cb.t[0] = ConvTensor{b, b_h, int64_t(S) * h, kNoScale, nullptr, nullptr};
    cb.t[1] = ConvTensor{w1, w1_h, int64_t(F) * h, kTargetWeights, scales + kScaleInv + 2, scales + kScale + 2};
    cb.t[2] = ConvTensor{w2, w2_h, int64_t(h) * F, kTargetWeights, scales + kScaleInv + 3, scales + kScale + 3};
    cb.count = 3;
    cb.partial = reinterpret_cast<float *>(base + rl.cpart);
    cb.err = p->d_err;
    TSP_STAGE(20, 2, launch_convert_f16(cb, s));
    GemmDesc g1d = gemm(b_h, h, false, w1_h, h, false, S, F, h, EPI_GELU, u, F, scales + kScaleInv + 2);
    g1d.out2 = g;
    g1d.ldo2 = F;
    TSP_STAGE(5, 1, launch_gemm(g1d, err, p->num_sms, s));
    // K loop over FFN shards in ring order (r + t) mod D for rank r's rows, + residual
    GemmDesc g2d = gemm(g, F, false, w2_h, F, false, S, h, F, EPI_RESID_BF16, out, h, scales + kScaleInv + 3);
    g2d.aux = resid;
    g2d.ldaux = h;
    g2d.ring_rows = L;
    g2d.ring_kblocks = (F / p->D) / 64;
    TSP_STAGE(6, 1, launch_gemm(g2d, err, p->num_sms, s));
#undef TSP_STAGE
    return TSP_OK;
}

TSP_API tsp_status tsp_layer_backward(tsp_plan_t p, const void *dy, const void *x, const float *g1, const void *wqkv,
                                      const void *wo, const float *g2, const void *w1, const void *w2,
                                      const void *saved, void *ws, void *dx, float *dg1, float *dwqkv, float *dwo,
                                      float *dg2, float *dw1, float *dw2, void *stream) {
    if (!p || !dy || !x || !g1 || !wqkv || !wo || !g2 || !w1 || !w2 || !saved || !ws || !dx || !dg1 || !dwqkv ||
        !dwo || !dg2 || !dw1 || !dw2)
        return TSP_ERR_INVALID_ARG;
    for (const void *q : {dy, x, (const void *)g1, wqkv, wo, (const void *)g2, w1, w2, saved, (const void *)ws,
                          (const void *)dx, (const void *)dg1, (const void *)dwqkv, (const void *)dwo,
                          (const void *)dg2, (const void *)dw1, (const void *)dw2})
        if (!aligned16(q)) return TSP_ERR_ALIGNMENT;
    tsp_status st = ensure_device(p);
    if (st != TSP_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const Layout l = layout_of(p);
    const uint8_t *sv = static_cast<const uint8_t *>(saved);
    uint8_t *w = static_cast<uint8_t *>(ws);
    const int S = static_cast<int>(p->S), h = p->h, F = p->F, L = static_cast<int>(p->L);
    const DevErr err = dev_err(p);
    (void)wqkv;
    (void)wo;
    (void)w1;
    (void)w2;
    const float *rstd1 = reinterpret_cast<const float *>(sv + l.rstd1);
    const void *a = sv + l.a, *q = sv + l.q, *k = sv + l.k, *v = sv + l.v, *o = sv + l.o;
    const float *lse = reinterpret_cast<const float *>(sv + l.lse);
    const float *yres = reinterpret_cast<const float *>(sv + l.y);
    const float *rstd2 = reinterpret_cast<const float *>(sv + l.rstd2);
    const void *b = sv + l.b, *u = sv + l.u, *g = sv + l.g;
    const void *wqkv_h = sv + l.wqkv_h, *wo_h = sv + l.wo_h, *w1_h = sv + l.w1_h, *w2_h = sv + l.w2_h;
    const float *winv = reinterpret_cast<const float *>(sv + l.scales) + kScaleInv;
    void *du = w + l.du;
    float *db = reinterpret_cast<float *>(w + l.db);
    float *dyf = reinterpret_cast<float *>(w + l.dy);
    void *dyh = w + l.dyh, *dO = w + l.dO, *dqkv = w + l.dqkv, *dy16 = w + l.dy16;
    float *delta = reinterpret_cast<float *>(w + l.delta);
    float *da = reinterpret_cast<float *>(w + l.da);
    float *dgp = reinterpret_cast<float *>(w + l.dgp);
    float *gsc = reinterpret_cast<float *>(w + l.gscales);
    const float *ginv = gsc + 0;  // 2^-k: leaves the scaled gradient domain
    const float *gmul = gsc + 1;  // 2^k: enters it
#define TSP_STAGE(id, nk, call)                                                  \
    do {                                                                         \
        if (stage(p, id, nk, s, [&] { return (call); }) != cudaSuccess)          \
            return TSP_ERR_CUDA;                                                 \
    } while (0)
    // The backward is linear in dY: it runs on dY * 2^k, with 2^k taken from
    // max|dY|, so gradients of any magnitude sit well inside fp16's range;
    // the outputs leave the scaled domain exactly (times 2^-k).
    ConvBatch cb{};
    cb.t[0] = ConvTensor{dy, dy16, int64_t(S) * h, kTargetGrad, gsc + 0, gsc + 1};
    cb.count = 1;
    cb.partial = reinterpret_cast<float *>(w + l.gpart);
    cb.err = p->d_err;
    TSP_STAGE(21, 2, launch_convert_f16(cb, s));
    // MLP ring backward: dU = (dY W2) * GELU'(U); dW2 = dY^T G; dW1 = dU^T b; db = dU W1 (ring K order)
    GemmDesc gdu = gemm(dy16, h, false, w2_h, F, true, S, F, h, EPI_DGELU, du, F, winv + 3);
    gdu.aux = u;
    gdu.ldaux = F;
    TSP_STAGE(7, 1, launch_gemm(gdu, err, p->num_sms, s));
    TSP_STAGE(8, 1, launch_gemm(gemm(dy16, h, true, g, F, true, h, F, S, EPI_F32, dw2, F, ginv), err, p->num_sms, s));
    TSP_STAGE(9, 1, launch_gemm(gemm(du, F, true, b, h, true, F, h, S, EPI_F32, dw1, h, ginv), err, p->num_sms, s));
    GemmDesc gdb = gemm(du, F, false, w1_h, h, true, S, h, F, EPI_F32, db, h, winv + 2);
    gdb.ring_rows = L;
    gdb.ring_kblocks = (F / p->D) / 64;
    TSP_STAGE(10, 1, launch_gemm(gdb, err, p->num_sms, s));
    // RMSNorm2 backward + residual: dy = dY 2^k + RMSNorm2^T(db), fp32 and fp16 copies
    NormBwd n2{};
    n2.dout = db;
    n2.x_f32 = yres;
    n2.rstd = rstd2;
    n2.g = g2;
    n2.resid_bf16 = dy;
    n2.dx_f32 = dyf;
    n2.dx_low = dyh;
    n2.low_f16 = true;
    n2.dg_partial = dgp;
    n2.dg = dg2;
    n2.resid_mul = gmul;
    n2.dg_mul = ginv;
    n2.err = p->d_err;
    n2.rows = S;
    n2.h = h;
    TSP_STAGE(11, 2, launch_rmsnorm_bwd(n2, s));
    // out-projection backward: dO = dy Wo, dWo = dy^T O
    TSP_STAGE(12, 1, launch_gemm(gemm(dyh, h, false, wo_h, h, true, S, h, h, EPI_F16, dO, h, winv + 1), err, p->num_sms, s));
    TSP_STAGE(13, 1, launch_gemm(gemm(dyh, h, true, o, h, true, h, h, S, EPI_F32, dwo, h, ginv), err, p->num_sms, s));
    // attention backward; dK/dV reduced to the keys' owners
    AttnBwdDesc ab{};
    ab.S = S;
    ab.L = L;
    ab.D = p->D;
    ab.H = p->H;
    ab.dh = p->dh;
    ab.chunk = static_cast<int>(p->c);
    ab.q = q;
    ab.k = k;
    ab.v = v;
    ab.o = o;
    ab.dout = dO;
    ab.lse = lse;
    ab.delta = delta;
    ab.dq = dqkv;
    ab.dk = static_cast<uint8_t *>(dqkv) + static_cast<size_t>(h) * 2;
    ab.dv = static_cast<uint8_t *>(dqkv) + static_cast<size_t>(2 * h) * 2;
    ab.ldd = 3 * h;
    ab.err = p->d_err;
    ab.inv_map = p->d_inv;
    ab.kv_order = p->d_kv_order;
    ab.q_order = p->d_q_order;
    ab.dq_acc = attn_bwd_fused_supported(p->dh) ? reinterpret_cast<int *>(w + l.dq_acc) : nullptr;
    ab.dq_bound = reinterpret_cast<unsigned int *>(w + l.dq_bound);
    ab.q_row0 = 0;
    ab.q_rows = S;
    ab.rank = -1;
    TSP_STAGE(14, 1, launch_attn_delta(ab, p->num_sms, s));
    if (attn_bwd_fused_supported(p->dh)) {
        // one pass: dK, dV and the fixed-point dQ sum; then dQ to fp16
        TSP_STAGE(22, 1, launch_attn_bwd_fused(ab, err, p->num_sms, s, p->d_zig));
        TSP_STAGE(23, 1, launch_dq_convert(ab, s));
    } else {
        TSP_STAGE(15, 1, launch_attn_dkdv(ab, err, p->num_sms, s, p->d_zig));
        TSP_STAGE(16, 1, launch_attn_dq(ab, err, p->num_sms, s, p->d_zig, p->d_qmax));
    }
    // projection backward: dWqkv = [dQ|dK|dV]^T a, da = [dQ|dK|dV] Wqkv
    TSP_STAGE(17, 1, launch_gemm(gemm(dqkv, 3 * h, true, a, h, true, 3 * h, h, S, EPI_F32, dwqkv, h, ginv), err, p->num_sms, s));
    TSP_STAGE(18, 1, launch_gemm(gemm(dqkv, 3 * h, false, wqkv_h, h, true, S, h, 3 * h, EPI_F32, da, h, winv + 0), err, p->num_sms, s));
    // RMSNorm1 backward + residual: dx = (dy + RMSNorm1^T(da)) 2^-k
    NormBwd n1{};
    n1.dout = da;
    n1.x_bf16 = x;
    n1.rstd = rstd1;
    n1.g = g1;
    n1.resid_f32 = dyf;
    n1.dx_low = dx;
    n1.low_f16 = false;
    n1.dg_partial = dgp;
    n1.dg = dg1;
    n1.dx_mul = ginv;
    n1.dg_mul = ginv;
    n1.err = p->d_err;
    n1.rows = S;
    n1.h = h;
    TSP_STAGE(19, 2, launch_rmsnorm_bwd(n1, s));
#undef TSP_STAGE
    return TSP_OK;
}

// ===========================================================================
// Test hooks (tsp_testing.h)
// ===========================================================================

// ===========================================================================
// Stack of layers with activation recompute (tsp.h)
// ===========================================================================

namespace {
// The part of a stack's workspace that one layer call uses: the backward's
// scratch, or the intermediates of an inference forward, whichever is larger.
size_t stack_layer_ws(const tsp_plan_s *p) {
    const Layout l = layout_of(p);
    return std::max(l.bwd_total, l.saved_total);
}
bool all_set(int n, const void *const *v) {
    if (!v) return false;
    for (int i = 0; i < n; ++i)
        if (!v[i] || !aligned16(v[i])) return false;
    return true;
}
}  // namespace

TSP_API tsp_status tsp_stack_workspace_size(tsp_plan_t p, int layers, size_t *ws_bytes, size_t *saved_bytes,
                                            size_t *inputs_bytes) {
    if (!p || layers < 1) return TSP_ERR_INVALID_ARG;
    const size_t act = static_cast<size_t>(p->S) * p->h * 2;  // one bf16 [S][h] tensor
    if (ws_bytes) *ws_bytes = stack_layer_ws(p) + 3 * act;
    if (saved_bytes) *saved_bytes = layout_of(p).saved_total;
    if (inputs_bytes) *inputs_bytes = static_cast<size_t>(layers - 1) * act;
    return TSP_OK;
}



TSP_API tsp_status tsp_stack_forward(tsp_plan_t p, int layers, const void *x, const float *const *g1,
                                     const void *const *wqkv, const void *const *wo, const float *const *g2,
                                     const void *const *w1, const void *const *w2, void *z, void *inputs,
                                     void *saved, void *ws, void *stream) {
    if (!p || layers < 1 || !x || !z || !ws || !g1 || !wqkv || !wo || !g2 || !w1 || !w2) return TSP_ERR_INVALID_ARG;
    if (saved && layers > 1 && !inputs) return TSP_ERR_INVALID_ARG;
    if (!all_set(layers, reinterpret_cast<const void *const *>(g1)) || !all_set(layers, wqkv) ||
        !all_set(layers, wo) || !all_set(layers, reinterpret_cast<const void *const *>(g2)) ||
        !all_set(layers, w1) || !all_set(layers, w2))
        return TSP_ERR_INVALID_ARG;
    for (const void *q : {x, (const void *)z, (const void *)ws})
        if (!aligned16(q)) return TSP_ERR_ALIGNMENT;
    if ((saved && !aligned16(saved)) || (inputs && !aligned16(inputs))) return TSP_ERR_ALIGNMENT;
    const size_t act = static_cast<size_t>(p->S) * p->h * 2;
    // inference: layer outputs alternate between two scratch tensors after the layer workspace
    uint8_t *scratch = static_cast<uint8_t *>(ws) + stack_layer_ws(p);
    const void *in = x;
    for (int i = 0; i < layers; ++i) {
        void *out = i == layers - 1 ? z
                    : saved         ? static_cast<void *>(static_cast<uint8_t *>(inputs) + static_cast<size_t>(i) * act)
                                    : static_cast<void *>(scratch + static_cast<size_t>(i & 1) * act);
        const tsp_status st =
            tsp_layer_forward(p, in, g1[i], wqkv[i], wo[i], g2[i], w1[i], w2[i], out, saved, ws, stream);
        if (st != TSP_OK) return st;
        in = out;
    }
    return TSP_OK;
}

TSP_API tsp_status tsp_stack_backward(tsp_plan_t p, int layers, const void *dz, const void *x,
                                      const float *const *g1, const void *const *wqkv, const void *const *wo,
                                      const float *const *g2, const void *const *w1, const void *const *w2,
                                      const void *inputs, void *saved, void *ws, void *dx, float *const *dg1,
                                      float *const *dwqkv, float *const *dwo, float *const *dg2, float *const *dw1,
                                      float *const *dw2, void *stream) {
    if (!p || layers < 1 || !dz || !x || !saved || !ws || !dx || (layers > 1 && !inputs) || !g1 || !wqkv || !wo ||
        !g2 || !w1 || !w2 || !dg1 || !dwqkv || !dwo || !dg2 || !dw1 || !dw2)
        return TSP_ERR_INVALID_ARG;
    auto cv = [](const auto *const *v) { return reinterpret_cast<const void *const *>(v); };
    if (!all_set(layers, cv(g1)) || !all_set(layers, wqkv) || !all_set(layers, wo) || !all_set(layers, cv(g2)) ||
        !all_set(layers, w1) || !all_set(layers, w2) || !all_set(layers, cv(dg1)) || !all_set(layers, cv(dwqkv)) ||
        !all_set(layers, cv(dwo)) || !all_set(layers, cv(dg2)) || !all_set(layers, cv(dw1)) ||
        !all_set(layers, cv(dw2)))
        return TSP_ERR_INVALID_ARG;
    for (const void *q : {dz, x, (const void *)saved, (const void *)ws, (const void *)dx})
        if (!aligned16(q)) return TSP_ERR_ALIGNMENT;
    if (inputs && !aligned16(inputs)) return TSP_ERR_ALIGNMENT;
    const size_t act = static_cast<size_t>(p->S) * p->h * 2;
    uint8_t *scratch = static_cast<uint8_t *>(ws) + stack_layer_ws(p);
    void *grad[2] = {scratch, scratch + act};  // gradients between layers, in turn
    void *znew = scratch + 2 * act;            // output of a recomputed forward (not used)
    const void *g = dz;
    for (int i = layers - 1; i >= 0; --i) {
        const void *in = i == 0 ? x : static_cast<const uint8_t *>(inputs) + static_cast<size_t>(i - 1) * act;
        // the top layer's intermediates are still in `saved` from the forward
        if (i != layers - 1) {
            const tsp_status st =
                tsp_layer_forward(p, in, g1[i], wqkv[i], wo[i], g2[i], w1[i], w2[i], znew, saved, ws, stream);
            if (st != TSP_OK) return st;
        }
        void *out = i == 0 ? dx : grad[i & 1];
        const tsp_status st = tsp_layer_backward(p, g, in, g1[i], wqkv[i], wo[i], g2[i], w1[i], w2[i], saved, ws,
                                                 out, dg1[i], dwqkv[i], dwo[i], dg2[i], dw1[i], dw2[i], stream);
        if (st != TSP_OK) return st;
        g = out;
    }
    return TSP_OK;
}

// ===========================================================================
// One rank's share of the forward, for D devices (tsp.h)
// ===========================================================================

namespace {
// Workspace of one rank: its own L rows of every activation, the LSE of all
// local rows (the kernel indexes it by local row; only this rank's are
// written), and the fp16 weight copies.
struct RankLayout {
    size_t rstd1, a, q, o, lse, y, rstd2, b, u, g, wqkv_h, wo_h, w1_h, w2_h, scales, cpart, total;
};
RankLayout rank_layout_of(const tsp_plan_s *p) {
    RankLayout l{};
    const size_t L = p->L, S = p->S, h = p->h, F = p->F, H = p->H;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off += up(bytes);
        return o;
    };
    l.rstd1 = take(L * 4);
    l.a = take(L * h * 2);
    l.q = take(L * h * 2);
    l.o = take(L * h * 2);
    l.lse = take(H * S * 4);
    l.y = take(L * h * 4);
    l.rstd2 = take(L * 4);
    l.b = take(L * h * 2);
    l.u = take(L * F * 2);
    l.g = take(L * F * 2);
    l.wqkv_h = take(3 * h * h * 2);
    l.wo_h = take(h * h * 2);
    l.w1_h = take(F * h * 2);
    l.w2_h = take(h * F * 2);
    l.scales = take(64 * 4);
    l.cpart = take(static_cast<size_t>(kMaxConv) * kConvBlocks * 4);
    l.total = off;
    return l;
}

tsp_status rank_checks(tsp_plan_s *p, int rank, std::initializer_list<const void *> ptrs) {
    if (rank < 0 || rank >= p->D) return TSP_ERR_INVALID_ARG;
    for (const void *q : ptrs)
        if (!q) return TSP_ERR_INVALID_ARG;
    for (const void *q : ptrs)
        if (!aligned16(q)) return TSP_ERR_ALIGNMENT;
    if (p->L % 256) return TSP_ERR_UNSUPPORTED;  // the forward's query items are 256-row blocks
    return ensure_device(p);
}
}  // namespace

TSP_API tsp_status tsp_rank_workspace_size(tsp_plan_t p, size_t *ws_bytes) {
    if (!p || !ws_bytes) return TSP_ERR_INVALID_ARG;
    *ws_bytes = rank_layout_of(p).total;
    return TSP_OK;
}

#define TSP_RSTAGE(id, nk, call)                                                 \
    do {                                                                         \
        if (stage(p, id, nk, s, [&] { return (call); }) != cudaSuccess)          \
            return TSP_ERR_CUDA;                                                 \
    } while (0)

TSP_API tsp_status tsp_rank_forward_qkv(tsp_plan_t p, int rank, const void *x, const float *g1, const void *wqkv,
                                        void *k, void *v, void *ws, void *stream) {
    if (!p) return TSP_ERR_INVALID_ARG;
    tsp_status st = rank_checks(p, rank, {x, (const void *)g1, wqkv, (const void *)k, (const void *)v,
                                          (const void *)ws});
    if (st != TSP_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const RankLayout l = rank_layout_of(p);
    uint8_t *w = static_cast<uint8_t *>(ws);
    const int L = static_cast<int>(p->L), h = p->h;
    const DevErr err = dev_err(p);
    auto *scales = reinterpret_cast<float *>(w + l.scales);
    ConvBatch cb{};
    cb.t[0] = ConvTensor{wqkv, w + l.wqkv_h, int64_t(3) * h * h, kTargetWeights, scales + kScaleInv + 0,
                         scales + kScale + 0};
    cb.count = 1;
    cb.partial = reinterpret_cast<float *>(w + l.cpart);
    cb.err = p->d_err;
    TSP_RSTAGE(20, 2, launch_convert_f16(cb, s));
    TSP_RSTAGE(0, 1, launch_rmsnorm_fwd(x, nullptr, g1, w + l.a, true, reinterpret_cast<float *>(w + l.rstd1), L, h,
                                        p->d_err, s));
    // this rank's rows against every attention shard; K/V land at the rows'
    // global positions, the rank's part of the all-gather
    GemmDesc gq = gemm(w + l.a, h, false, w + l.wqkv_h, h, false, L, 3 * h, h, EPI_QKV, w + l.q, h,
                       scales + kScaleInv + 0);
    gq.rowmap = p->d_zig + static_cast<int64_t>(rank) * L;
    gq.hsplit = h;
    gq.out_k = k;
    gq.out_v = v;
    TSP_RSTAGE(1, 1, launch_gemm(gq, err, p->num_sms, s));
    return TSP_OK;
}

TSP_API tsp_status tsp_rank_forward_out(tsp_plan_t p, int rank, const void *x, const void *k, const void *v,
                                        const void *wo, const float *g2, const void *w1, const void *w2, void *z,
                                        void *ws, void *stream) {
    if (!p) return TSP_ERR_INVALID_ARG;
    tsp_status st = rank_checks(p, rank, {x, k, v, wo, (const void *)g2, w1, w2, (const void *)z, (const void *)ws});
    if (st != TSP_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const RankLayout l = rank_layout_of(p);
    uint8_t *w = static_cast<uint8_t *>(ws);
    const int S = static_cast<int>(p->S), L = static_cast<int>(p->L), h = p->h, F = p->F;
    const DevErr err = dev_err(p);
    auto *scales = reinterpret_cast<float *>(w + l.scales);
    ConvBatch cb{};
    const void *wsrc[3] = {wo, w1, w2};
    void *wdst[3] = {w + l.wo_h, w + l.w1_h, w + l.w2_h};
    const int64_t wn[3] = {int64_t(h) * h, int64_t(F) * h, int64_t(h) * F};
    for (int i = 0; i < 3; ++i)
        cb.t[i] = ConvTensor{wsrc[i], wdst[i], wn[i], kTargetWeights, scales + kScaleInv + 1 + i,
                             scales + kScale + 1 + i};
    cb.count = 3;
    cb.partial = reinterpret_cast<float *>(w + l.cpart);
    cb.err = p->d_err;
    TSP_RSTAGE(20, 2, launch_convert_f16(cb, s));
    // attention of this rank's queries over the gathered K/V
    AttnDesc ad{};
    ad.S = S;
    ad.L = L;
    ad.D = p->D;
    ad.H = p->H;
    ad.dh = p->dh;
    ad.chunk = static_cast<int>(p->c);
    ad.q = w + l.q;
    ad.k = k;
    ad.v = v;
    ad.o = w + l.o;
    ad.lse = reinterpret_cast<float *>(w + l.lse);
    ad.order = p->d_rank_fwd_order + p->rank_fwd_off[rank];
    ad.num_items = p->rank_fwd_items[rank];
    ad.q_row0 = rank * L;
    ad.q_rows = L;
    TSP_RSTAGE(2, 1, launch_attn_fwd(ad, err, p->num_sms, s));
    auto *yres = reinterpret_cast<float *>(w + l.y);
    GemmDesc go = gemm(w + l.o, h, false, w + l.wo_h, h, false, L, h, h, EPI_RESID_F32, yres, h,
                       scales + kScaleInv + 1);
    go.aux = x;
    go.ldaux = h;
    TSP_RSTAGE(3, 1, launch_gemm(go, err, p->num_sms, s));
    TSP_RSTAGE(4, 1, launch_rmsnorm_fwd(nullptr, yres, g2, w + l.b, true, reinterpret_cast<float *>(w + l.rstd2), L,
                                        h, p->d_err, s));
    GemmDesc g1d = gemm(w + l.b, h, false, w + l.w1_h, h, false, L, F, h, EPI_GELU, w + l.u, F,
                        scales + kScaleInv + 2);
    g1d.out2 = w + l.g;
    g1d.ldo2 = F;
    TSP_RSTAGE(5, 1, launch_gemm(g1d, err, p->num_sms, s));
    // W2 with the K loop over FFN shards in this rank's ring order (rank + t) mod D
    GemmDesc g2d = gemm(w + l.g, F, false, w + l.w2_h, F, false, L, h, F, EPI_RESID_BF16, z, h,
                        scales + kScaleInv + 3);
    g2d.aux = yres;
    g2d.ldaux = h;
    g2d.ring_rows = L;
    g2d.ring_kblocks = (F / p->D) / 64;
    g2d.ring_rank0 = rank;
    TSP_RSTAGE(6, 1, launch_gemm(g2d, err, p->num_sms, s));
    return TSP_OK;
}

namespace {
// Byte layout of one rank's backward scratch: the layer backward's buffers
// over the rank's L rows (delta stays [H][S], indexed by local row like lse).
struct RankBwdLayout {
    size_t dy16, du, db, dy, dyh, dO, delta, dqkv, da, dgp, gscales, gpart, dq_acc, dq_bound, total;
};
RankBwdLayout rank_bwd_layout_of(const tsp_plan_s *p) {
    RankBwdLayout l{};
    const size_t L = p->L, S = p->S, h = p->h, F = p->F, H = p->H;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off += up(bytes);
        return o;
    };
    l.dy16 = take(L * h * 2);
    l.du = take(L * F * 2);
    l.db = take(L * h * 4);
    l.dy = take(L * h * 4);
    l.dyh = take(L * h * 2);
    l.dO = take(L * h * 2);
    l.delta = take(H * S * 4);
    l.dqkv = take(L * 3 * h * 2);
    l.da = take(L * h * 4);
    l.dgp = take(static_cast<size_t>(rmsnorm_bwd_partial_blocks(static_cast<int>(L))) * h * 4);
    l.gscales = take(64 * 4);
    l.gpart = take(static_cast<size_t>(kMaxConv) * kConvBlocks * 4);
    l.dq_acc = take(L * h * 4);
    l.dq_bound = take(3 * H * 4);
    l.total = off;
    return l;
}
}  // namespace

TSP_API tsp_status tsp_rank_backward_workspace_size(tsp_plan_t p, size_t *bws_bytes) {
    if (!p || !bws_bytes) return TSP_ERR_INVALID_ARG;
    *bws_bytes = rank_bwd_layout_of(p).total;
    return TSP_OK;
}

TSP_API tsp_status tsp_rank_backward_attn(tsp_plan_t p, int rank, const void *dz, const void *k, const void *v,
                                          const float *g2, void *ws, void *bws, float *dk_part, float *dv_part,
                                          float *dwo, float *dg2, float *dw1, float *dw2, void *stream) {
    if (!p) return TSP_ERR_INVALID_ARG;
    if (!attn_bwd_fused_supported(p->dh)) return TSP_ERR_UNSUPPORTED;  // the single-pass kernel's rank mode
    tsp_status st = rank_checks(p, rank, {dz, k, v, (const void *)g2, (const void *)ws, (const void *)bws,
                                          (const void *)dk_part, (const void *)dv_part, (const void *)dwo,
                                          (const void *)dg2, (const void *)dw1, (const void *)dw2});
    if (st != TSP_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const RankLayout fl = rank_layout_of(p);
    const RankBwdLayout l = rank_bwd_layout_of(p);
    const uint8_t *sv = static_cast<const uint8_t *>(ws);
    uint8_t *w = static_cast<uint8_t *>(bws);
    const int S = static_cast<int>(p->S), L = static_cast<int>(p->L), h = p->h, F = p->F;
    const DevErr err = dev_err(p);
    const float *winv = reinterpret_cast<const float *>(sv + fl.scales) + kScaleInv;
    const void *u = sv + fl.u, *g = sv + fl.g, *b = sv + fl.b, *o = sv + fl.o;
    void *dy16 = w + l.dy16, *du = w + l.du, *dyh = w + l.dyh, *dO = w + l.dO, *dqkv = w + l.dqkv;
    float *db = reinterpret_cast<float *>(w + l.db);
    float *gsc = reinterpret_cast<float *>(w + l.gscales);
    const float *ginv = gsc + 0, *gmul = gsc + 1;
    // dZ of this rank's rows into the scaled fp16 domain (2^k from this rank's max|dZ|)
    ConvBatch cb{};
    cb.t[0] = ConvTensor{dz, dy16, int64_t(L) * h, kTargetGrad, gsc + 0, gsc + 1};
    cb.count = 1;
    cb.partial = reinterpret_cast<float *>(w + l.gpart);
    cb.err = p->d_err;
    TSP_RSTAGE(21, 2, launch_convert_f16(cb, s));
    // MLP backward over the rank's rows; dW2, dW1 are this rank's partial sums
    GemmDesc gdu = gemm(dy16, h, false, sv + fl.w2_h, F, true, L, F, h, EPI_DGELU, du, F, winv + 3);
    gdu.aux = u;
    gdu.ldaux = F;
    TSP_RSTAGE(7, 1, launch_gemm(gdu, err, p->num_sms, s));
    TSP_RSTAGE(8, 1, launch_gemm(gemm(dy16, h, true, g, F, true, h, F, L, EPI_F32, dw2, F, ginv), err, p->num_sms, s));
    TSP_RSTAGE(9, 1, launch_gemm(gemm(du, F, true, b, h, true, F, h, L, EPI_F32, dw1, h, ginv), err, p->num_sms, s));
    GemmDesc gdb = gemm(du, F, false, sv + fl.w1_h, h, true, L, h, F, EPI_F32, db, h, winv + 2);
    gdb.ring_rows = L;
    gdb.ring_kblocks = (F / p->D) / 64;
    gdb.ring_rank0 = rank;
    TSP_RSTAGE(10, 1, launch_gemm(gdb, err, p->num_sms, s));
    NormBwd n2{};
    n2.dout = db;
    n2.x_f32 = reinterpret_cast<const float *>(sv + fl.y);
    n2.rstd = reinterpret_cast<const float *>(sv + fl.rstd2);
    n2.g = g2;
    n2.resid_bf16 = dz;
    n2.dx_f32 = reinterpret_cast<float *>(w + l.dy);
    n2.dx_low = dyh;
    n2.low_f16 = true;
    n2.dg_partial = reinterpret_cast<float *>(w + l.dgp);
    n2.dg = dg2;
    n2.resid_mul = gmul;
    n2.dg_mul = ginv;
    n2.err = p->d_err;
    n2.rows = L;
    n2.h = h;
    TSP_RSTAGE(11, 2, launch_rmsnorm_bwd(n2, s));
    TSP_RSTAGE(12, 1, launch_gemm(gemm(dyh, h, false, sv + fl.wo_h, h, true, L, h, h, EPI_F16, dO, h, winv + 1), err,
                                  p->num_sms, s));
    TSP_RSTAGE(13, 1, launch_gemm(gemm(dyh, h, true, o, h, true, h, h, L, EPI_F32, dwo, h, ginv), err, p->num_sms, s));
    // attention backward of the rank's query rows over the gathered K / V:
    // dQ of its rows, and its share of every visible key's dK / dV (fp32,
    // out of the scaled domain) for the caller to reduce to the keys' owners
    AttnBwdDesc ab{};
    ab.S = S;
    ab.L = L;
    ab.D = p->D;
    ab.H = p->H;
    ab.dh = p->dh;
    ab.chunk = static_cast<int>(p->c);
    ab.q = sv + fl.q;
    ab.k = k;
    ab.v = v;
    ab.o = o;
    ab.dout = dO;
    ab.lse = reinterpret_cast<const float *>(sv + fl.lse);
    ab.delta = reinterpret_cast<float *>(w + l.delta);
    ab.dq = dqkv;
    ab.ldd = 3 * h;
    ab.err = p->d_err;
    ab.inv_map = p->d_inv;
    ab.kv_order = p->d_rank_bwd_order + p->rank_bwd_off[rank];
    ab.kv_items = p->rank_bwd_items[rank];
    ab.dq_acc = reinterpret_cast<int *>(w + l.dq_acc);
    ab.dq_bound = reinterpret_cast<unsigned int *>(w + l.dq_bound);
    ab.q_row0 = rank * L;
    ab.q_rows = L;
    ab.rank = rank;
    ab.dk_part = dk_part;
    ab.dv_part = dv_part;
    ab.dkv_mul = ginv;
    TSP_RSTAGE(14, 1, launch_attn_delta(ab, p->num_sms, s));
    TSP_RSTAGE(22, 1, launch_attn_bwd_fused(ab, err, p->num_sms, s, p->d_zig));
    TSP_RSTAGE(23, 1, launch_dq_convert(ab, s));
    return TSP_OK;
}

TSP_API tsp_status tsp_rank_backward_qkv(tsp_plan_t p, int rank, const void *x, const float *g1, const float *dk,
                                         const float *dv, void *ws, void *bws, void *dx, float *dg1, float *dwqkv,
                                         void *stream) {
    if (!p) return TSP_ERR_INVALID_ARG;
    if (!attn_bwd_fused_supported(p->dh)) return TSP_ERR_UNSUPPORTED;  // the single-pass kernel's rank mode
    tsp_status st = rank_checks(p, rank, {x, (const void *)g1, (const void *)dk, (const void *)dv,
                                          (const void *)ws, (const void *)bws, dx, (const void *)dg1,
                                          (const void *)dwqkv});
    if (st != TSP_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const RankLayout fl = rank_layout_of(p);
    const RankBwdLayout l = rank_bwd_layout_of(p);
    const uint8_t *sv = static_cast<const uint8_t *>(ws);
    uint8_t *w = static_cast<uint8_t *>(bws);
    const int L = static_cast<int>(p->L), h = p->h;
    const DevErr err = dev_err(p);
    const float *winv = reinterpret_cast<const float *>(sv + fl.scales) + kScaleInv;
    uint8_t *dqkv = w + l.dqkv;
    const float *gsc = reinterpret_cast<const float *>(w + l.gscales);
    const float *ginv = gsc + 0, *gmul = gsc + 1;
    float *da = reinterpret_cast<float *>(w + l.da);
    // the reduced dK / dV of this rank's rows back into its scaled fp16 domain
    TSP_RSTAGE(24, 1, launch_scale_to_f16(dk, L, h, dqkv + static_cast<size_t>(h) * 2, 3 * h, gmul, p->d_err, s));
    TSP_RSTAGE(24, 1, launch_scale_to_f16(dv, L, h, dqkv + static_cast<size_t>(2 * h) * 2, 3 * h, gmul, p->d_err, s));
    TSP_RSTAGE(17, 1, launch_gemm(gemm(dqkv, 3 * h, true, sv + fl.a, h, true, 3 * h, h, L, EPI_F32, dwqkv, h, ginv),
                                  err, p->num_sms, s));
    TSP_RSTAGE(18, 1, launch_gemm(gemm(dqkv, 3 * h, false, sv + fl.wqkv_h, h, true, L, h, 3 * h, EPI_F32, da, h,
                                       winv + 0), err, p->num_sms, s));
    NormBwd n1{};
    n1.dout = da;
    n1.x_bf16 = x;
    n1.rstd = reinterpret_cast<const float *>(sv + fl.rstd1);
    n1.g = g1;
    n1.resid_f32 = reinterpret_cast<const float *>(w + l.dy);
    n1.dx_low = dx;
    n1.low_f16 = false;
    n1.dg_partial = reinterpret_cast<float *>(w + l.dgp);
    n1.dg = dg1;
    n1.dx_mul = ginv;
    n1.dg_mul = ginv;
    n1.err = p->d_err;
    n1.rows = L;
    n1.h = h;
    TSP_RSTAGE(19, 2, launch_rmsnorm_bwd(n1, s));
    return TSP_OK;
}
#undef TSP_RSTAGE

TSP_API tsp_status tsp_test_gemm(int a_mn, int b_mn, int M, int N, int K, const void *A, int64_t lda, const void *B,
                                 int64_t ldb, float *C, int64_t ldc, int force_bn128, int f16, void *stream) {
    if (!A || !B || !C || M <= 0 || N <= 0 || K <= 0) return TSP_ERR_INVALID_ARG;
    if (M % 128 || N % 128 || K % 64) return TSP_ERR_UNSUPPORTED;
    if (!aligned16(A) || !aligned16(B) || !aligned16(C)) return TSP_ERR_ALIGNMENT;
    static unsigned int *d_err = nullptr;
    static int sms = 0;
    if (!d_err) {
        if (cudaMalloc(&d_err, 4) != cudaSuccess || cudaMemset(d_err, 0, 4) != cudaSuccess) return TSP_ERR_CUDA;
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    }
    GemmDesc g = gemm(A, lda, a_mn != 0, B, ldb, b_mn != 0, M, N, K, EPI_F32, C, ldc);
    g.force_bn128 = force_bn128 != 0;
    g.f16 = f16 != 0;
    return cuda_status(launch_gemm(g, DevErr{d_err, 4000000000LL}, sms, static_cast<cudaStream_t>(stream)));
}

TSP_API tsp_status tsp_test_buffer_offset(tsp_plan_t p, const char *name, size_t *offset) {
    if (!p || !name || !offset) return TSP_ERR_INVALID_ARG;
    const Layout l = layout_of(p);
    struct {
        const char *n;
        size_t o;
    } tab[] = {{"rstd1", l.rstd1}, {"a", l.a},   {"q", l.q},         {"k", l.k},     {"v", l.v},
               {"o", l.o},         {"lse", l.lse}, {"y", l.y},       {"rstd2", l.rstd2}, {"b", l.b},
               {"u", l.u},         {"g", l.g},   {"wqkv_h", l.wqkv_h}, {"wo_h", l.wo_h}, {"w1_h", l.w1_h},
               {"w2_h", l.w2_h},   {"scales", l.scales}, {"ws.du", l.du}, {"ws.db", l.db}, {"ws.dy", l.dy},
               {"ws.dyh", l.dyh},  {"ws.dO", l.dO}, {"ws.delta", l.delta}, {"ws.dqkv", l.dqkv}, {"ws.da", l.da},
               {"ws.dy16", l.dy16}, {"ws.gscales", l.gscales}};
    for (auto &t : tab)
        if (std::strcmp(t.n, name) == 0) {
            *offset = t.o;
            return TSP_OK;
        }
    return TSP_ERR_INVALID_ARG;
}

TSP_API tsp_status tsp_test_next_visible(tsp_plan_t p, int from, int kv0, int *out) {
    if (!p || !out) return TSP_ERR_INVALID_ARG;
    const int nq64 = static_cast<int>(p->S / 64);
    if (from < 0 || from > nq64 || kv0 < 0 || kv0 >= p->S) return TSP_ERR_INVALID_ARG;
    *out = zz_next_visible(from, kv0, p->D, static_cast<int>(p->c), nq64);
    return TSP_OK;
}

TSP_API tsp_status tsp_test_tables(tsp_plan_t p, int which, int32_t *out, int64_t capacity, int64_t *count) {
    if (!p || !count || capacity < 0 || (capacity > 0 && !out)) return TSP_ERR_INVALID_ARG;
    const HostTables t = host_tables(p);
    const std::vector<int32_t> *v = nullptr;
    switch (which) {
        case 0: v = &t.inv; break;
        case 1: v = &t.qmax; break;
        case 2: v = &t.forder; break;
        case 3: v = &t.korder; break;
        case 4: v = &t.qorder; break;
        default: return TSP_ERR_INVALID_ARG;
    }
    *count = static_cast<int64_t>(v->size());
    if (*count > capacity) return TSP_ERR_INVALID_ARG;
    std::copy(v->begin(), v->end(), out);
    return TSP_OK;
}

TSP_API tsp_status tsp_test_work_order(tsp_plan_t p, int which, int num_ctas, int32_t *out, int64_t capacity,
                                       int64_t *count) {
    if (!p || !count || capacity < 0 || (capacity > 0 && !out) || num_ctas < 1) return TSP_ERR_INVALID_ARG;
    HostTables t = host_tables(p);
    device_orders(t, p->H, num_ctas);
    const std::vector<int32_t> *v = nullptr;
    switch (which) {
        case 2: v = &t.forder; break;
        case 3: v = &t.korder; break;
        case 4: v = &t.qorder; break;
        default: return TSP_ERR_INVALID_ARG;
    }
    *count = static_cast<int64_t>(v->size());
    if (*count > capacity) return TSP_ERR_INVALID_ARG;
    std::copy(v->begin(), v->end(), out);
    return TSP_OK;
}

TSP_API tsp_status tsp_test_step_walk_desc(tsp_plan_t p, int kv0, int32_t *steps, int capacity, int *count) {
    if (!p || !count || capacity < 0 || (capacity > 0 && !steps)) return TSP_ERR_INVALID_ARG;
    if (kv0 < 0 || kv0 >= p->S) return TSP_ERR_INVALID_ARG;
    const StepVis vis{p->D, static_cast<int>(p->c), static_cast<int>(p->S / 64)};
    int n = 0;
    DescWalk w;
    for (w.seek(vis, kv0); w.q < vis.nq64; w.next(vis, kv0), ++n)
        if (n < capacity) steps[n] = w.q;
    *count = n;
    return n <= capacity ? TSP_OK : TSP_ERR_INVALID_ARG;
}

TSP_API tsp_status tsp_test_step_walk_rank(tsp_plan_t p, int rank, int kv0, int32_t *steps, int capacity,
                                           int *count) {
    if (!p || !count || capacity < 0 || (capacity > 0 && !steps)) return TSP_ERR_INVALID_ARG;
    if (kv0 < 0 || kv0 >= p->S || rank < 0 || rank >= p->D) return TSP_ERR_INVALID_ARG;
    const StepVis vis{p->D, static_cast<int>(p->c), static_cast<int>(p->S / 64), rank};
    int n = 0;
    DescWalk w;
    for (w.seek(vis, kv0); w.q < vis.nq64; w.next(vis, kv0), ++n)
        if (n < capacity) steps[n] = w.q;
    *count = n;
    return n <= capacity ? TSP_OK : TSP_ERR_INVALID_ARG;
}

TSP_API tsp_status tsp_test_rank_kv_order(tsp_plan_t p, int rank, int num_ctas, int32_t *out, int64_t capacity,
                                          int64_t *count) {
    if (!p || !count || capacity < 0 || (capacity > 0 && !out) || num_ctas < 1) return TSP_ERR_INVALID_ARG;
    if (rank < 0 || rank >= p->D) return TSP_ERR_INVALID_ARG;
    const std::vector<int32_t> v = rank_kv_order(p, host_tables(p), rank, num_ctas);
    *count = static_cast<int64_t>(v.size());
    if (*count > capacity) return TSP_ERR_INVALID_ARG;
    std::copy(v.begin(), v.end(), out);
    return TSP_OK;
}

TSP_API tsp_status tsp_test_step_walk(tsp_plan_t p, int kv0, int32_t *steps, int capacity, int *count) {
    if (!p || !count || capacity < 0 || (capacity > 0 && !steps)) return TSP_ERR_INVALID_ARG;
    if (kv0 < 0 || kv0 >= p->S) return TSP_ERR_INVALID_ARG;
    const StepVis vis{p->D, static_cast<int>(p->c), static_cast<int>(p->S / 64)};
    int n = 0;
    StepWalk w;
    for (w.seek(vis, 0, kv0); w.q < vis.nq64; w.next(vis, kv0), ++n)
        if (n < capacity) steps[n] = w.q;
    *count = n;
    return n <= capacity ? TSP_OK : TSP_ERR_INVALID_ARG;
}

// ===========================================================================
// Profiling (tsp.h)
// ===========================================================================

TSP_API tsp_status tsp_profile_enable(tsp_plan_t p, int enable) {
    if (!p) return TSP_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(p->mu);
    profile_clear(p);
    p->profiling = enable != 0;
    return TSP_OK;
}

TSP_API tsp_status tsp_profile_read(tsp_plan_t p, int stage_id, const char **name, double *total_ms,
                                    int64_t *calls, int64_t *kernel_launches) {
    if (!p || stage_id < 0 || stage_id >= TSP_NUM_STAGES) return TSP_ERR_INVALID_ARG;
    double ms = 0.0;
    for (auto &ev : p->prof[stage_id]) {
        if (cudaEventSynchronize(ev.second) != cudaSuccess) return TSP_ERR_CUDA;
        float t = 0.f;
        if (cudaEventElapsedTime(&t, ev.first, ev.second) != cudaSuccess) return TSP_ERR_CUDA;
        ms += t;
    }
    if (name) *name = kStageNames[stage_id];
    if (total_ms) *total_ms = ms;
    if (calls) *calls = static_cast<int64_t>(p->prof[stage_id].size());
    if (kernel_launches) *kernel_launches = p->prof_launches[stage_id];
    return TSP_OK;
}

TSP_API int64_t tsp_kernel_launches(tsp_plan_t p) { return p ? p->launches : 0; }

// ===========================================================================
// Bounded-wait self test (tsp_testing.h)
// ===========================================================================

namespace {
__global__ void wait_timeout_kernel(DevErr err, int *result) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // nothing ever arrives on it
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    bool ok = mbar_wait(&bar, 0, &abort_flag, err);
    __syncthreads();
    if (threadIdx.x == 0) result[blockIdx.x] = ok ? 1 : 0;
}
}  // namespace

TSP_API tsp_status tsp_test_exp2(const float *x, float *y, int n, int which, void *stream) {
    if (n < 0 || (n > 0 && (!x || !y)) || (which != 0 && which != 1)) return TSP_ERR_INVALID_ARG;
    return cuda_status(launch_exp2_test(x, y, n, which, static_cast<cudaStream_t>(stream)));
}

TSP_API tsp_status tsp_test_wait_timeout(tsp_plan_t p, long long limit_cycles, int *result_dev, void *stream) {
    if (!p || !result_dev || limit_cycles <= 0) return TSP_ERR_INVALID_ARG;
    tsp_status st = ensure_device(p);
    if (st != TSP_OK) return st;
    DevErr e{p->d_err, limit_cycles};
    wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(e, result_dev);
    return cuda_status(cudaGetLastError());
}

