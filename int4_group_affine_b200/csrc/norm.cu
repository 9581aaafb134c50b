// norm.cu - RMSNorm between stacked layers: xn = bf16(x / sqrt(mean(x^2) + eps)).
#include "common.cuh"

namespace moeq {
namespace {

__global__ void rmsnorm_kernel(const uint16_t* __restrict__ x, int H, float eps, uint16_t* __restrict__ xn) {
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

}  // namespace

cudaError_t launch_rmsnorm(const uint16_t* x, int T, int H, float eps, uint16_t* xn, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    rmsnorm_kernel<<<T, 256, 0, s>>>(x, H, eps, xn);
    return cudaGetLastError();
}

}  // namespace moeq
