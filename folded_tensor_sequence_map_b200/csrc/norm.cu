// RMSNorm forward and backward (memory-bound, fp32 arithmetic).
//
//   forward:  rstd = 1/sqrt(mean(x^2) + 1e-5),  out = x * rstd * g   (bf16 out)
//   backward: n = x*rstd, dn = dout*g,
//             dx = resid + rstd * (dn - n * mean(dn*n)),  dg = sum_rows dout*n
//
// The backward adds the residual branch's gradient (resid) so that one pass
// produces the gradient of "x + f(RMSNorm(x))" w.r.t. x.  dg is reduced in two
// deterministic steps: per-block partial sums in fixed row order, then a sum
// over blocks in block order.
#include "common.cuh"
#include "internal.h"

namespace tsp {
namespace {

constexpr float kEps = 1e-5f;
constexpr int kBwdRows = 64;  // rows per backward block

template <bool X_F32>
__device__ __forceinline__ float4 load4(const void *p, int64_t idx) {
    if (X_F32) return *reinterpret_cast<const float4 *>(static_cast<const float *>(p) + idx);
    uint2 w = *reinterpret_cast<const uint2 *>(static_cast<const __nv_bfloat16 *>(p) + idx);
    return make_float4(bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y));
}

// One warp per row.
template <bool X_F32>
__global__ void rmsnorm_fwd_kernel(const void *x, const float *g, __nv_bfloat16 *out, float *rstd_out, int rows,
                                   int h) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) / 32;
    const int lane = threadIdx.x % 32;
    if (warp >= rows) return;
    const int64_t base = static_cast<int64_t>(warp) * h;
    float ss = 0.f;
    for (int c = lane * 4; c < h; c += 128) {
        float4 v = load4<X_F32>(x, base + c);
        ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float r = rsqrtf(ss / static_cast<float>(h) + kEps);
    if (lane == 0) rstd_out[warp] = r;
    for (int c = lane * 4; c < h; c += 128) {
        float4 v = load4<X_F32>(x, base + c);
        float4 gg = *reinterpret_cast<const float4 *>(g + c);
        uint2 w;
        w.x = pack_bf16(v.x * r * gg.x, v.y * r * gg.y);
        w.y = pack_bf16(v.z * r * gg.z, v.w * r * gg.w);
        *reinterpret_cast<uint2 *>(out + base + c) = w;
    }
}

template <bool X_F32, bool R_F32>
__global__ void rmsnorm_bwd_kernel(const float *dout, const void *x, const float *rstd, const float *g,
                                   const void *resid, float *dx_f32, __nv_bfloat16 *dx_bf16, float *dg_partial,
                                   int rows, int h) {
    __shared__ float s_mean[kBwdRows];
    const int row0 = blockIdx.x * kBwdRows;
    const int nrows = min(kBwdRows, rows - row0);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, nwarps = blockDim.x / 32;
    // Phase 1: mean(dn * n) of every row of the block.
    for (int i = warp; i < nrows; i += nwarps) {
        const int64_t base = static_cast<int64_t>(row0 + i) * h;
        const float r = rstd[row0 + i];
        float s = 0.f;
        for (int c = lane * 4; c < h; c += 128) {
            float4 d = *reinterpret_cast<const float4 *>(dout + base + c);
            float4 v = load4<X_F32>(x, base + c);
            float4 gg = *reinterpret_cast<const float4 *>(g + c);
            s += d.x * gg.x * v.x + d.y * gg.y * v.y + d.z * gg.z * v.z + d.w * gg.w * v.w;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) s_mean[i] = s * r / static_cast<float>(h);
    }
    __syncthreads();
    // Phase 2: column-parallel; every thread owns 4-column groups and walks the rows.
    for (int c = threadIdx.x * 4; c < h; c += blockDim.x * 4) {
        float4 gg = *reinterpret_cast<const float4 *>(g + c);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int i = 0; i < nrows; ++i) {
            const int64_t idx = static_cast<int64_t>(row0 + i) * h + c;
            const float r = rstd[row0 + i];
            const float m = s_mean[i];
            float4 d = *reinterpret_cast<const float4 *>(dout + idx);
            float4 v = load4<X_F32>(x, idx);
            float4 rs = load4<R_F32>(resid, idx);
            float4 n = make_float4(v.x * r, v.y * r, v.z * r, v.w * r);
            float4 o;
            o.x = rs.x + r * (d.x * gg.x - n.x * m);
            o.y = rs.y + r * (d.y * gg.y - n.y * m);
            o.z = rs.z + r * (d.z * gg.z - n.z * m);
            o.w = rs.w + r * (d.w * gg.w - n.w * m);
            if (dx_f32) *reinterpret_cast<float4 *>(dx_f32 + idx) = o;
            if (dx_bf16) {
                uint2 w;
                w.x = pack_bf16(o.x, o.y);
                w.y = pack_bf16(o.z, o.w);
                *reinterpret_cast<uint2 *>(dx_bf16 + idx) = w;
            }
            acc.x += d.x * n.x;
            acc.y += d.y * n.y;
            acc.z += d.z * n.z;
            acc.w += d.w * n.w;
        }
        *reinterpret_cast<float4 *>(dg_partial + static_cast<int64_t>(blockIdx.x) * h + c) = acc;
    }
}

__global__ void column_sum_kernel(const float *partial, float *out, int nblocks, int h) {
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= h) return;
    float s = 0.f;
    for (int b = 0; b < nblocks; ++b) s += partial[static_cast<int64_t>(b) * h + c];
    out[c] = s;
}

}  // namespace

int rmsnorm_bwd_partial_blocks(int rows) { return (rows + kBwdRows - 1) / kBwdRows; }

cudaError_t launch_rmsnorm_fwd(const void *x_bf16, const float *x_f32, const float *g, void *out, float *rstd,
                               int rows, int h, cudaStream_t st) {
    const int threads = 256;
    const int blocks = (rows * 32 + threads - 1) / threads;
    if (x_f32)
        rmsnorm_fwd_kernel<true><<<blocks, threads, 0, st>>>(x_f32, g, static_cast<__nv_bfloat16 *>(out), rstd,
                                                             rows, h);
    else
        rmsnorm_fwd_kernel<false><<<blocks, threads, 0, st>>>(x_bf16, g, static_cast<__nv_bfloat16 *>(out), rstd,
                                                              rows, h);
    return cudaGetLastError();
}

cudaError_t launch_rmsnorm_bwd(const float *dout, const void *x_bf16, const float *x_f32, const float *rstd,
                               const float *g, const void *resid_bf16, const float *resid_f32, float *dx_f32,
                               void *dx_bf16, float *dg_partial, float *dg, int rows, int h, cudaStream_t st) {
    const int nb = rmsnorm_bwd_partial_blocks(rows);
    const int threads = 256;
    auto *dxb = static_cast<__nv_bfloat16 *>(dx_bf16);
    if (x_f32 && !resid_f32)
        rmsnorm_bwd_kernel<true, false><<<nb, threads, 0, st>>>(dout, x_f32, rstd, g, resid_bf16, dx_f32, dxb,
                                                                dg_partial, rows, h);
    else if (!x_f32 && resid_f32)
        rmsnorm_bwd_kernel<false, true><<<nb, threads, 0, st>>>(dout, x_bf16, rstd, g, resid_f32, dx_f32, dxb,
                                                                dg_partial, rows, h);
    else if (x_f32 && resid_f32)
        rmsnorm_bwd_kernel<true, true><<<nb, threads, 0, st>>>(dout, x_f32, rstd, g, resid_f32, dx_f32, dxb,
                                                               dg_partial, rows, h);
    else
        rmsnorm_bwd_kernel<false, false><<<nb, threads, 0, st>>>(dout, x_bf16, rstd, g, resid_bf16, dx_f32, dxb,
                                                                 dg_partial, rows, h);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    column_sum_kernel<<<(h + 255) / 256, 256, 0, st>>>(dg_partial, dg, nb, h);
    return cudaGetLastError();
}

}  // namespace tsp
