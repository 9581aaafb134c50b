// norm.cu - RMSNorm between stacked layers: xn = bf16(x / sqrt(mean(x^2) + eps)).
#include "common.cuh"

namespace moeq {
namespace {

// Any alignment and row length: one CTA of 256 threads per token, one value per step.
__global__ void rmsnorm_scalar_kernel(const uint16_t* __restrict__ x, int H, float eps, uint16_t* __restrict__ xn) {
    __shared__ float red[32];
    const int t = blockIdx.x;
    const uint16_t* xr = x + (int64_t)t * H;
    float ss = 0.0f;
    for (int j = threadIdx.x; j < H; j += blockDim.x) {
        const float v = bf16f(xr[j]);
        ss = fmaf(v, v, ss);
    }
    ss = warp_sum(ss);
    if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = ss;
    __syncthreads();
    if (threadIdx.x < 32) {
        float v = threadIdx.x < blockDim.x / 32 ? red[threadIdx.x] : 0.0f;
        v = warp_sum(v);
        if (threadIdx.x == 0) red[0] = v;
    }
    __syncthreads();
    const float inv = 1.0f / sqrtf(red[0] / (float)H + eps);
    for (int j = threadIdx.x; j < H; j += blockDim.x) xn[(int64_t)t * H + j] = f2bf16(bf16f(xr[j]) * inv);
}

// 16-byte aligned rows, H % 8 == 0: one warp per token (8 per CTA); the row comes in 16-byte pieces (8 values), kept in
// registers between the sum of squares and the scaling (rows up to 2048 values; longer
// rows re-read the rest).
__global__ void __launch_bounds__(256) rmsnorm_kernel(const uint16_t* __restrict__ x, int T, int H, float eps,
                                                     uint16_t* __restrict__ xn) {
    const int t = blockIdx.x * 8 + threadIdx.x / 32, lane = threadIdx.x % 32, nv = H / 8;
    if (t >= T) return;
    const uint4* xr = reinterpret_cast<const uint4*>(x + (int64_t)t * H);
    uint4* yr = reinterpret_cast<uint4*>(xn + (int64_t)t * H);
    auto sumsq = [](const uint4& u) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        float ss = 0.0f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float lo = __uint_as_float(w[k] << 16), hi = __uint_as_float(w[k] & 0xFFFF0000u);
            ss = fmaf(lo, lo, fmaf(hi, hi, ss));
        }
        return ss;
    };
    auto scaled = [](const uint4& u, float inv) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint32_t lo = f2bf16(__uint_as_float(w[k] << 16) * inv);
            const uint32_t hi = f2bf16(__uint_as_float(w[k] & 0xFFFF0000u) * inv);
            o[k] = lo | (hi << 16);
        }
        return make_uint4(o[0], o[1], o[2], o[3]);
    };
    constexpr int kKeep = 8;  // pieces kept per lane: 8 x 32 x 8 = 2048 values
    uint4 keep[kKeep];
#pragma unroll
    for (int j = 0; j < kKeep; ++j) {
        const int v = lane + 32 * j;
        keep[j] = v < nv ? xr[v] : make_uint4(0u, 0u, 0u, 0u);
    }
    float ss = 0.0f;
#pragma unroll
    for (int j = 0; j < kKeep; ++j) ss += sumsq(keep[j]);
    for (int v = lane + 32 * kKeep; v < nv; v += 32) ss += sumsq(xr[v]);
    ss = warp_sum(ss);
    const float inv = 1.0f / sqrtf(ss / (float)H + eps);
#pragma unroll
    for (int j = 0; j < kKeep; ++j) {
        const int v = lane + 32 * j;
        if (v < nv) yr[v] = scaled(keep[j], inv);
    }
    for (int v = lane + 32 * kKeep; v < nv; v += 32) yr[v] = scaled(xr[v], inv);
}

}  // namespace

cudaError_t launch_rmsnorm(const uint16_t* x, int T, int H, float eps, uint16_t* xn, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    if (((uintptr_t)x & 15) || ((uintptr_t)xn & 15) || H % 8)
        rmsnorm_scalar_kernel<<<T, 256, 0, s>>>(x, H, eps, xn);
    else
        rmsnorm_kernel<<<(T + 7) / 8, 256, 0, s>>>(x, T, H, eps, xn);
    return cudaGetLastError();
}

}  // namespace moeq
