// RMSNorm backward with library-owned scratch, for callers that cannot
// allocate device memory.
//
// The ordinary path takes its scratch (the per-block partial sums of the gain
// gradient) from the caller's workspace.  Some callers have no way to provide
// one: code that runs where cudaMalloc is not allowed or not wanted (inside a
// region that must not allocate, an allocator-less runtime, a host thread
// that owns no memory pool).  This entry point keeps that scratch in a
// file-scope device array instead, so it needs nothing but its inputs and
// outputs.
#include <mutex>

#include "../../include/tsp.h"
#include "common.cuh"
#include "internal.h"

#define TSP_API extern "C" __attribute__((visibility("default")))

namespace {

// Scratch for the per-block partial sums of dg: (rows / 64) x h floats, at
// most 4,194,304 floats (16 MiB).  Every GPU that loads this library holds it
// until the process exits.
constexpr size_t kNoAllocFloats = size_t(1) << 22;
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocFloats];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device with that device current.  In host code the array's name is only
// a host-side stand-in, so the kernel must be given this address instead.
// The address is cached for the life of the process: after cudaDeviceReset
// on a device the cached value is stale, so this entry point must not be used
// on a device that has been reset since its first call.
tsp_status scratch_for_current_device(float **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return TSP_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return TSP_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return TSP_ERR_CUDA;
        g_scratch_ptr[dev] = static_cast<float *>(p);
    }
    *out = g_scratch_ptr[dev];
    return TSP_OK;
}

}  // namespace

TSP_API tsp_status tsp_rmsnorm_backward_noalloc(const float *dout, const void *x, const float *rstd, const float *g,
                                                const float *resid, void *dx, float *dg, int rows, int h,
                                                void *stream) {
    if (!dout || !x || !rstd || !g || !resid || !dx || !dg || rows <= 0 || h <= 0) return TSP_ERR_INVALID_ARG;
    if (h % 128) return TSP_ERR_UNSUPPORTED;
    const size_t need = static_cast<size_t>(tsp::rmsnorm_bwd_partial_blocks(rows)) * static_cast<size_t>(h);
    if (need > kNoAllocFloats) return TSP_ERR_UNSUPPORTED;
    for (const void *q : {(const void *)dout, x, (const void *)rstd, (const void *)g, (const void *)resid,
                          (const void *)dx, (const void *)dg})
        if (reinterpret_cast<uintptr_t>(q) & 15u) return TSP_ERR_ALIGNMENT;
    float *scratch = nullptr;
    tsp_status st = scratch_for_current_device(&scratch);
    if (st != TSP_OK) return st;
    // Every partial-sum slot the kernel reads is written by the same call, so
    // nothing has to be cleared between calls.
    tsp::NormBwd n{};
    n.dout = dout;
    n.x_bf16 = x;
    n.rstd = rstd;
    n.g = g;
    n.resid_f32 = resid;
    n.dx_low = dx;
    n.low_f16 = false;
    n.dg_partial = scratch;
    n.dg = dg;
    n.rows = rows;
    n.h = h;
    cudaError_t e = tsp::launch_rmsnorm_bwd(n, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TSP_OK : TSP_ERR_CUDA;
}
