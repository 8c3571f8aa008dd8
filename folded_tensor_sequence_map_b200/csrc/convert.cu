// bf16 -> fp16 conversion with a power-of-two scale (memory-bound).
//
// The layer's tensor-core operands are fp16: its 11-bit significand keeps the
// rounding of every stored intermediate 8x finer than bf16's, at the same
// MMA rate.  Caller tensors arrive as bf16; a bf16 value times a power of two
// is exactly an fp16 value as long as it lands in fp16's normal range, so
// each tensor is scaled by 2^e, chosen from its largest magnitude so that the
// largest lands just below 2^target.  A consumer undoes the scale exactly in
// its epilogue with 2^-e.
//
// Two launches for a batch of tensors:
//   absmax_kernel   block b of tensor i writes the largest |x| of its grid
//                   stride to partial[i][b];
//   convert_kernel  every block reduces partial[i][*] itself (296 floats), so
//                   all blocks derive the same exponent without atomics or a
//                   cleared accumulator; block 0 publishes 2^-e and 2^e; then
//                   each block converts its grid stride, 8 elements per load.
#include "common.cuh"
#include "internal.h"

namespace tsp {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float block_max(float v, float *red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < kThreads / 32 ? red[lane] : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0) red[0] = v;
    }
    __syncthreads();
    const float r = red[0];
    __syncthreads();
    return r;
}

__global__ void __launch_bounds__(kThreads) absmax_kernel(const ConvBatch b) {
    __shared__ float red[kThreads / 32];
    const ConvTensor &t = b.t[blockIdx.y];
    const uint4 *src = static_cast<const uint4 *>(t.src);
    const int64_t n8 = t.n / 8;
    float m = 0.f;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < n8;
         i += static_cast<int64_t>(gridDim.x) * kThreads) {
        const uint4 w = src[i];
        m = fmaxf(m, fmaxf(fmaxf(fabsf(bf16_lo(w.x)), fabsf(bf16_hi(w.x))), fmaxf(fabsf(bf16_lo(w.y)), fabsf(bf16_hi(w.y)))));
        m = fmaxf(m, fmaxf(fmaxf(fabsf(bf16_lo(w.z)), fabsf(bf16_hi(w.z))), fmaxf(fabsf(bf16_lo(w.w)), fabsf(bf16_hi(w.w)))));
    }
    m = block_max(m, red);
    if (threadIdx.x == 0) b.partial[blockIdx.y * kConvBlocks + blockIdx.x] = m;
}

__global__ void __launch_bounds__(kThreads) convert_kernel(const ConvBatch b) {
    __shared__ float red[kThreads / 32];
    const ConvTensor &t = b.t[blockIdx.y];
    float m = 0.f;
    for (int i = threadIdx.x; i < kConvBlocks; i += kThreads) m = fmaxf(m, b.partial[blockIdx.y * kConvBlocks + i]);
    m = block_max(m, red);
    int e = 0;
    if (t.target == kNoScale) {
        if (blockIdx.x == 0 && threadIdx.x == 0) flag_range(m, b.err);
    } else if (m > 0.f && m <= 3.0e38f) {
        int E = 0;
        frexpf(m, &E);  // m = f * 2^E, f in [0.5, 1)
        e = min(max(t.target - E, -100), 100);
    }
    const float sc = ldexpf(1.0f, e);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        if (t.scale_inv) *t.scale_inv = ldexpf(1.0f, -e);
        if (t.scale) *t.scale = sc;
    }
    const uint4 *src = static_cast<const uint4 *>(t.src);
    uint4 *dst = static_cast<uint4 *>(t.dst);
    const int64_t n8 = t.n / 8;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < n8;
         i += static_cast<int64_t>(gridDim.x) * kThreads) {
        const uint4 w = src[i];
        uint4 o;
        o.x = pack_f16(bf16_lo(w.x) * sc, bf16_hi(w.x) * sc);
        o.y = pack_f16(bf16_lo(w.y) * sc, bf16_hi(w.y) * sc);
        o.z = pack_f16(bf16_lo(w.z) * sc, bf16_hi(w.z) * sc);
        o.w = pack_f16(bf16_lo(w.w) * sc, bf16_hi(w.w) * sc);
        dst[i] = o;
    }
}

// fp32 rows of `cols` values -> fp16 times *mul into rows of stride ldd,
// 8 elements per thread; values past fp16's range set the range error bit.
__global__ void __launch_bounds__(kThreads) scale_to_f16_kernel(const float *src, int64_t n8, int cols, __half *dst,
                                                                int64_t ldd, const float *mul, unsigned int *err) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
    if (i >= n8) return;
    const int64_t e = i * 8;
    const int64_t row = e / cols;
    const int col = static_cast<int>(e - row * cols);
    const float m = *mul;
    const float4 a = *reinterpret_cast<const float4 *>(src + e);
    const float4 b = *reinterpret_cast<const float4 *>(src + e + 4);
    const float v[8] = {a.x * m, a.y * m, a.z * m, a.w * m, b.x * m, b.y * m, b.z * m, b.w * m};
    float mx = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) mx = fmaxf(mx, fabsf(v[j]));
    flag_range(mx, err);
    *reinterpret_cast<uint4 *>(dst + row * ldd + col) =
        make_uint4(pack_f16(v[0], v[1]), pack_f16(v[2], v[3]), pack_f16(v[4], v[5]), pack_f16(v[6], v[7]));
}

}  // namespace

cudaError_t launch_scale_to_f16(const float *src, int64_t rows, int cols, void *dst, int64_t ldd, const float *mul,
                                unsigned int *err, cudaStream_t st) {
    if (cols % 8 || ldd % 8 || (reinterpret_cast<uintptr_t>(src) & 15u) || (reinterpret_cast<uintptr_t>(dst) & 15u))
        return cudaErrorInvalidValue;
    const int64_t n8 = rows * cols / 8;
    if (n8 == 0) return cudaSuccess;
    scale_to_f16_kernel<<<static_cast<unsigned int>((n8 + kThreads - 1) / kThreads), kThreads, 0, st>>>(
        src, n8, cols, static_cast<__half *>(dst), ldd, mul, err);
    return cudaGetLastError();
}

cudaError_t launch_convert_f16(const ConvBatch &b, cudaStream_t st) {
    if (b.count <= 0 || b.count > kMaxConv) return cudaErrorInvalidValue;
    for (int i = 0; i < b.count; ++i)
        if (b.t[i].n % 8 || (reinterpret_cast<uintptr_t>(b.t[i].src) & 15u) ||
            (reinterpret_cast<uintptr_t>(b.t[i].dst) & 15u))
            return cudaErrorInvalidValue;
    const dim3 grid(kConvBlocks, b.count);
    absmax_kernel<<<grid, kThreads, 0, st>>>(b);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    convert_kernel<<<grid, kThreads, 0, st>>>(b);
    return cudaGetLastError();
}

}  // namespace tsp
