// norm.cu - RMSNorm between stacked layers: xn = bf16(x / sqrt(mean(x^2) + eps)).
#include "common.cuh"

namespace moeq {
namespace {

// One CTA of 256 threads per token; the row comes in 16-byte pieces (8 values), kept in
// registers between the sum of squares and the scaling (rows up to 8192 values; longer
// rows re-read the rest).
__global__ void __launch_bounds__(256) rmsnorm_kernel(const uint16_t* __restrict__ x, int H, float eps,
                                                     uint16_t* __restrict__ xn) {
    __shared__ float red[8];
    const int t = blockIdx.x, nv = H / 8;
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
    uint4 keep[4];
    float ss = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int v = threadIdx.x + 256 * j;
        keep[j] = v < nv ? xr[v] : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) ss += sumsq(keep[j]);
    for (int v = threadIdx.x + 1024; v < nv; v += 256) ss += sumsq(xr[v]);
    ss = warp_sum(ss);
    if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = ss;
    __syncthreads();
    float tot = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) tot += red[w];
    const float inv = 1.0f / sqrtf(tot / (float)H + eps);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int v = threadIdx.x + 256 * j;
        if (v < nv) yr[v] = scaled(keep[j], inv);
    }
    for (int v = threadIdx.x + 1024; v < nv; v += 256) yr[v] = scaled(xr[v], inv);
}

}  // namespace

cudaError_t launch_rmsnorm(const uint16_t* x, int T, int H, float eps, uint16_t* xn, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    rmsnorm_kernel<<<T, 256, 0, s>>>(x, H, eps, xn);
    return cudaGetLastError();
}

}  // namespace moeq
