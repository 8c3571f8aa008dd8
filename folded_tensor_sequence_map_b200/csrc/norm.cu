// RMSNorm forward and backward (memory-bound, fp32 arithmetic).
//
//   forward:  rstd = 1/sqrt(mean(x^2) + 1e-5),  out = x * rstd * g   (fp16 or bf16 out)
//   backward: n = x*rstd, dn = dout*g,
//             dx = resid + rstd * (dn - n * mean(dn*n)),  dg = sum_rows dout*n
//
// The backward takes optional power-of-two multipliers for the residual, for
// dx and for dg: the layer's backward runs in a scaled gradient domain and
// these carry values into and out of it exactly.
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

__device__ __forceinline__ uint2 pack4(bool f16, float a, float b, float c, float d) {
    return f16 ? make_uint2(pack_f16(a, b), pack_f16(c, d)) : make_uint2(pack_bf16(a, b), pack_bf16(c, d));
}

// One warp per row.
template <bool X_F32>
__global__ void rmsnorm_fwd_kernel(const void *x, const float *g, void *out, bool out_f16, float *rstd_out, int rows,
                                   int h, unsigned int *err) {
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
    float mx = 0.f;
    for (int c = lane * 4; c < h; c += 128) {
        float4 v = load4<X_F32>(x, base + c);
        float4 gg = *reinterpret_cast<const float4 *>(g + c);
        const float a0 = v.x * r * gg.x, a1 = v.y * r * gg.y, a2 = v.z * r * gg.z, a3 = v.w * r * gg.w;
        mx = fmaxf(mx, fmaxf(fmaxf(fabsf(a0), fabsf(a1)), fmaxf(fabsf(a2), fabsf(a3))));
        *reinterpret_cast<uint2 *>(static_cast<uint16_t *>(out) + base + c) = pack4(out_f16, a0, a1, a2, a3);
    }
    if (out_f16) flag_range(mx, err);
}

template <bool X_F32, bool R_F32>
__global__ void rmsnorm_bwd_kernel(const NormBwd n) {
    __shared__ float s_mean[kBwdRows];
    const int rows = n.rows, h = n.h;
    const void *x = X_F32 ? static_cast<const void *>(n.x_f32) : n.x_bf16;
    const void *resid = R_F32 ? static_cast<const void *>(n.resid_f32) : n.resid_bf16;
    const float rm = n.resid_mul ? *n.resid_mul : 1.0f;
    const float xm = n.dx_mul ? *n.dx_mul : 1.0f;
    const int row0 = blockIdx.x * kBwdRows;
    const int nrows = min(kBwdRows, rows - row0);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, nwarps = blockDim.x / 32;
    // Phase 1: mean(dn * n) of every row of the block.
    for (int i = warp; i < nrows; i += nwarps) {
        const int64_t base = static_cast<int64_t>(row0 + i) * h;
        const float r = n.rstd[row0 + i];
        float s = 0.f;
        for (int c = lane * 4; c < h; c += 128) {
            float4 d = *reinterpret_cast<const float4 *>(n.dout + base + c);
            float4 v = load4<X_F32>(x, base + c);
            float4 gg = *reinterpret_cast<const float4 *>(n.g + c);
            s += d.x * gg.x * v.x + d.y * gg.y * v.y + d.z * gg.z * v.z + d.w * gg.w * v.w;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) s_mean[i] = s * r / static_cast<float>(h);
    }
    __syncthreads();
    // Phase 2: column-parallel; every thread owns 4-column groups and walks the rows.
    float mx = 0.f;
    for (int c = threadIdx.x * 4; c < h; c += blockDim.x * 4) {
        float4 gg = *reinterpret_cast<const float4 *>(n.g + c);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int i = 0; i < nrows; ++i) {
            const int64_t idx = static_cast<int64_t>(row0 + i) * h + c;
            const float r = n.rstd[row0 + i];
            const float m = s_mean[i];
            float4 d = *reinterpret_cast<const float4 *>(n.dout + idx);
            float4 v = load4<X_F32>(x, idx);
            float4 rs = load4<R_F32>(resid, idx);
            float4 nn = make_float4(v.x * r, v.y * r, v.z * r, v.w * r);
            float4 o;
            o.x = (rs.x * rm + r * (d.x * gg.x - nn.x * m)) * xm;
            o.y = (rs.y * rm + r * (d.y * gg.y - nn.y * m)) * xm;
            o.z = (rs.z * rm + r * (d.z * gg.z - nn.z * m)) * xm;
            o.w = (rs.w * rm + r * (d.w * gg.w - nn.w * m)) * xm;
            if (n.dx_f32) *reinterpret_cast<float4 *>(n.dx_f32 + idx) = o;
            if (n.dx_low) {
                if (n.low_f16) mx = fmaxf(mx, fmaxf(fmaxf(fabsf(o.x), fabsf(o.y)), fmaxf(fabsf(o.z), fabsf(o.w))));
                *reinterpret_cast<uint2 *>(static_cast<uint16_t *>(n.dx_low) + idx) = pack4(n.low_f16, o.x, o.y, o.z, o.w);
            }
            acc.x += d.x * nn.x;
            acc.y += d.y * nn.y;
            acc.z += d.z * nn.z;
            acc.w += d.w * nn.w;
        }
        *reinterpret_cast<float4 *>(n.dg_partial + static_cast<int64_t>(blockIdx.x) * h + c) = acc;
    }
    if (n.dx_low && n.low_f16) flag_range(mx, n.err);
}

// Backward with each row read once: a block of 128 threads takes kBwdRows
// rows in turn and holds a row's dout, x and residual in registers (EPT = h /
// 128 values per thread, 16-byte column groups interleaved across threads),
// so the row's reduction and its dx come from one read.  dg sums each
// thread's columns over the block's rows in row order, as the kernel above
// does, so the partial sums are the same.
template <bool X_F32, bool R_F32, int EPT>
__global__ void __launch_bounds__(128) rmsnorm_bwd_reg_kernel(const NormBwd n) {
    constexpr int V = EPT / 4;  // 4-column groups per thread
    __shared__ float red[4];
    const int rows = n.rows, h = n.h;
    const void *x = X_F32 ? static_cast<const void *>(n.x_f32) : n.x_bf16;
    const void *resid = R_F32 ? static_cast<const void *>(n.resid_f32) : n.resid_bf16;
    const float rm = n.resid_mul ? *n.resid_mul : 1.0f;
    const float xm = n.dx_mul ? *n.dx_mul : 1.0f;
    const int row0 = blockIdx.x * kBwdRows;
    const int nrows = min(kBwdRows, rows - row0);
    const int t = threadIdx.x, warp = t / 32, lane = t % 32;
    float4 acc[V];
#pragma unroll
    for (int j = 0; j < V; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    float mx = 0.f;
    for (int i = 0; i < nrows; ++i) {
        const int64_t base = static_cast<int64_t>(row0 + i) * h;
        const float r = n.rstd[row0 + i];
        float4 d[V], v[V], rs[V];
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const int c = (j * 128 + t) * 4;
            d[j] = *reinterpret_cast<const float4 *>(n.dout + base + c);
            v[j] = load4<X_F32>(x, base + c);
            rs[j] = load4<R_F32>(resid, base + c);
        }
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const float4 gg = *reinterpret_cast<const float4 *>(n.g + (j * 128 + t) * 4);
            s += d[j].x * gg.x * v[j].x + d[j].y * gg.y * v[j].y + d[j].z * gg.z * v[j].z + d[j].w * gg.w * v[j].w;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) red[warp] = s;
        __syncthreads();
        const float m = ((red[0] + red[1]) + (red[2] + red[3])) * r / static_cast<float>(h);
        __syncthreads();  // red is written again for the next row
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const int c = (j * 128 + t) * 4;
            const int64_t idx = base + c;
            const float4 gg = *reinterpret_cast<const float4 *>(n.g + c);
            const float4 nn = make_float4(v[j].x * r, v[j].y * r, v[j].z * r, v[j].w * r);
            float4 o;
            o.x = (rs[j].x * rm + r * (d[j].x * gg.x - nn.x * m)) * xm;
            o.y = (rs[j].y * rm + r * (d[j].y * gg.y - nn.y * m)) * xm;
            o.z = (rs[j].z * rm + r * (d[j].z * gg.z - nn.z * m)) * xm;
            o.w = (rs[j].w * rm + r * (d[j].w * gg.w - nn.w * m)) * xm;
            if (n.dx_f32) *reinterpret_cast<float4 *>(n.dx_f32 + idx) = o;
            if (n.dx_low) {
                if (n.low_f16) mx = fmaxf(mx, fmaxf(fmaxf(fabsf(o.x), fabsf(o.y)), fmaxf(fabsf(o.z), fabsf(o.w))));
                *reinterpret_cast<uint2 *>(static_cast<uint16_t *>(n.dx_low) + idx) = pack4(n.low_f16, o.x, o.y, o.z, o.w);
            }
            acc[j].x += d[j].x * nn.x;
            acc[j].y += d[j].y * nn.y;
            acc[j].z += d[j].z * nn.z;
            acc[j].w += d[j].w * nn.w;
        }
    }
#pragma unroll
    for (int j = 0; j < V; ++j)
        *reinterpret_cast<float4 *>(n.dg_partial + static_cast<int64_t>(blockIdx.x) * h + (j * 128 + t) * 4) = acc[j];
    if (n.dx_low && n.low_f16) flag_range(mx, n.err);
}

template <bool X_F32, bool R_F32>
cudaError_t launch_bwd_reg(const NormBwd &n, int nb, cudaStream_t st) {
    switch (n.h) {
        case 512: rmsnorm_bwd_reg_kernel<X_F32, R_F32, 4><<<nb, 128, 0, st>>>(n); break;
        case 1024: rmsnorm_bwd_reg_kernel<X_F32, R_F32, 8><<<nb, 128, 0, st>>>(n); break;
        case 2048: rmsnorm_bwd_reg_kernel<X_F32, R_F32, 16><<<nb, 128, 0, st>>>(n); break;
        default: rmsnorm_bwd_reg_kernel<X_F32, R_F32, 32><<<nb, 128, 0, st>>>(n); break;
    }
    return cudaGetLastError();
}

__global__ void column_sum_kernel(const float *partial, float *out, const float *mul, int nblocks, int h) {
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= h) return;
    float s = 0.f;
    for (int b = 0; b < nblocks; ++b) s += partial[static_cast<int64_t>(b) * h + c];
    out[c] = mul ? s * *mul : s;
}

}  // namespace

int rmsnorm_bwd_partial_blocks(int rows) { return (rows + kBwdRows - 1) / kBwdRows; }

cudaError_t launch_rmsnorm_fwd(const void *x_bf16, const float *x_f32, const float *g, void *out, bool out_f16,
                               float *rstd, int rows, int h, unsigned int *err, cudaStream_t st) {
    const int threads = 256;
    const int blocks = (rows * 32 + threads - 1) / threads;
    if (x_f32)
        rmsnorm_fwd_kernel<true><<<blocks, threads, 0, st>>>(x_f32, g, out, out_f16, rstd, rows, h, err);
    else
        rmsnorm_fwd_kernel<false><<<blocks, threads, 0, st>>>(x_bf16, g, out, out_f16, rstd, rows, h, err);
    return cudaGetLastError();
}

cudaError_t launch_rmsnorm_bwd(const NormBwd &n, cudaStream_t st) {
    const int nb = rmsnorm_bwd_partial_blocks(n.rows);
    const int threads = 256;
    const bool xf = n.x_f32 != nullptr, rf = n.resid_f32 != nullptr;
    // rows held in registers for h = 512 .. 4096 (powers of two); else the
    // two-read kernel
    const bool reg = n.h == 512 || n.h == 1024 || n.h == 2048 || n.h == 4096;
    cudaError_t e = cudaSuccess;
    if (reg) {
        if (xf && !rf) e = launch_bwd_reg<true, false>(n, nb, st);
        else if (!xf && rf) e = launch_bwd_reg<false, true>(n, nb, st);
        else if (xf && rf) e = launch_bwd_reg<true, true>(n, nb, st);
        else e = launch_bwd_reg<false, false>(n, nb, st);
    } else if (xf && !rf)
        rmsnorm_bwd_kernel<true, false><<<nb, threads, 0, st>>>(n);
    else if (!xf && rf)
        rmsnorm_bwd_kernel<false, true><<<nb, threads, 0, st>>>(n);
    else if (xf && rf)
        rmsnorm_bwd_kernel<true, true><<<nb, threads, 0, st>>>(n);
    else
        rmsnorm_bwd_kernel<false, false><<<nb, threads, 0, st>>>(n);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    column_sum_kernel<<<(n.h + 255) / 256, 256, 0, st>>>(n.dg_partial, n.dg, n.dg_mul, nb, n.h);
    return cudaGetLastError();
}

}  // namespace tsp
