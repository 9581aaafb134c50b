// mixed.cu - a7: EdgeRazor mixed ternary / 4-bit weight-only GEMV/GEMM on CUDA
// cores.  y_o = s_o * sum_j q_oj x_j: the integer codes are dotted with the
// activations and the per-row scale is applied once at the end (the weight-only
// form of the EdgeRazor matmul decomposition).
//
// Row layout: super-groups of G rows, the first 4-bit (in/8 words, nibble q+8),
// the rest ternary (in/16 words, 2-bit field q+1).  A warp owns one output row
// and streams it with 16-byte loads: a vector is 32 elements of a 4-bit row or
// 64 elements of a ternary row.  Codes are offset (q+8, q+1), so the kernels
// dot the raw field with x and subtract offset * sum(x) per 32-element chunk.
#include "common.cuh"

namespace moeq {
namespace {

constexpr int kMT = 8;      // tokens per shared-memory chunk
constexpr int kMWarps = 8;  // warps (rows) per CTA

__device__ __forceinline__ int mswz(int j) {
    const int c = j >> 5;
    return (c << 5) | (((j & 31) + ((c & 7) << 2)) & 31);
}

template <typename Src>
__device__ void mstage(float* xs, float* xsum, const Src* src, int ld, int t0, int nt, int n) {
    for (int i = threadIdx.x; i < kMT * n; i += blockDim.x) {
        const int tt = i / n, j = i % n;
        float v = 0.0f;
        if (tt < nt) {
            if constexpr (sizeof(Src) == 2) v = bf16f(src[(int64_t)(t0 + tt) * ld + j]);
            else v = src[(int64_t)(t0 + tt) * ld + j];
        }
        xs[tt * n + mswz(j)] = v;
    }
    __syncthreads();
    const int nc = n / 32;
    for (int i = threadIdx.x; i < kMT * nc; i += blockDim.x) {
        const int tt = i / nc, c = i % nc;
        float s = 0.0f;
        for (int f = 0; f < 32; ++f) s += xs[tt * n + (c << 5) + f];
        xsum[i] = s;
    }
    __syncthreads();
}

// Dot of 32 consecutive code fields (bits = 4 or 2, stored in `nw` words) with
// chunk c of every staged token; subtracts offset * chunk sum.
template <int BITS>
__device__ __forceinline__ void code_chunk(const uint32_t* w, int c, float offset, const float* xs, const float* xsum,
                                           int n, float* acc) {
    constexpr int kPer = 32 / BITS;  // fields per word
    constexpr uint32_t kMask = (1u << BITS) - 1u;
    float qf[32];
#pragma unroll
    for (int f = 0; f < 32; ++f) qf[f] = u2f_small((w[f / kPer] >> (BITS * (f % kPer))) & kMask);
    const int rot = (c & 7) << 2;
#pragma unroll
    for (int tt = 0; tt < kMT; ++tt) {
        const float* xr = xs + tt * n + (c << 5);
        float a = 0.0f;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 xv = *reinterpret_cast<const float4*>(xr + ((4 * q + rot) & 31));
            a = fmaf(qf[4 * q + 0], xv.x, a);
            a = fmaf(qf[4 * q + 1], xv.y, a);
            a = fmaf(qf[4 * q + 2], xv.z, a);
            a = fmaf(qf[4 * q + 3], xv.w, a);
        }
        acc[tt] += fmaf(-offset, xsum[tt * (n / 32) + c], a);
    }
}

// sum_j q_oj x[tt][j] for one row, accumulated per lane (caller reduces).
__device__ __forceinline__ void mixed_row(const moe_mixed_tensor& W, int G, int o, const float* xs, const float* xsum,
                                          float* acc, int lane) {
    const int n = W.in;
    const uint32_t* pw = W.packed + mixed_row_offset(o, n, G);
    if (G > 0 && o % G == 0) {
        const uint4* v4 = reinterpret_cast<const uint4*>(pw);
        for (int c = lane; c < n / 32; c += 32) {
            const uint4 q = v4[c];
            const uint32_t w[4] = {q.x, q.y, q.z, q.w};
            code_chunk<4>(w, c, 8.0f, xs, xsum, n, acc);
        }
    } else {
        const uint4* v4 = reinterpret_cast<const uint4*>(pw);
        for (int v = lane; v < n / 64; v += 32) {
            const uint4 q = v4[v];
            const uint32_t w0[2] = {q.x, q.y}, w1[2] = {q.z, q.w};
            code_chunk<2>(w0, 2 * v, 1.0f, xs, xsum, n, acc);
            code_chunk<2>(w1, 2 * v + 1, 1.0f, xs, xsum, n, acc);
        }
    }
}

__global__ void __launch_bounds__(kMWarps * 32)
mixed_linear_kernel(moe_mixed_tensor W, int G, const uint16_t* __restrict__ x, int T, float* __restrict__ y) {
    extern __shared__ float4 smem_f4[];
    float* xs = reinterpret_cast<float*>(smem_f4);
    float* xsum = xs + kMT * W.in;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int o = blockIdx.x * kMWarps + warp;
    for (int t0 = 0; t0 < T; t0 += kMT) {
        const int nt = min(kMT, T - t0);
        __syncthreads();
        mstage(xs, xsum, x, W.in, t0, nt, W.in);
        if (o >= W.out) continue;
        float acc[kMT];
#pragma unroll
        for (int tt = 0; tt < kMT; ++tt) acc[tt] = 0.0f;
        mixed_row(W, G, o, xs, xsum, acc, lane);
        const float s = bf16f(W.scales[o]);
#pragma unroll
        for (int tt = 0; tt < kMT; ++tt) {
            const float v = warp_sum(acc[tt]);
            if (lane == 0 && tt < nt) y[(int64_t)(t0 + tt) * W.out + o] = s * v;
        }
    }
}

__global__ void __launch_bounds__(kMWarps * 32)
mixed_gate_up_kernel(moe_mixed_tensor Wg, moe_mixed_tensor Wu, int G, const uint16_t* __restrict__ x, int T,
                     float* __restrict__ h) {
    extern __shared__ float4 smem_f4[];
    float* xs = reinterpret_cast<float*>(smem_f4);
    float* xsum = xs + kMT * Wg.in;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int o = blockIdx.x * kMWarps + warp;
    for (int t0 = 0; t0 < T; t0 += kMT) {
        const int nt = min(kMT, T - t0);
        __syncthreads();
        mstage(xs, xsum, x, Wg.in, t0, nt, Wg.in);
        if (o >= Wg.out) continue;
        float ag[kMT], au[kMT];
#pragma unroll
        for (int tt = 0; tt < kMT; ++tt) ag[tt] = au[tt] = 0.0f;
        mixed_row(Wg, G, o, xs, xsum, ag, lane);
        mixed_row(Wu, G, o, xs, xsum, au, lane);
        const float sg = bf16f(Wg.scales[o]), su = bf16f(Wu.scales[o]);
#pragma unroll
        for (int tt = 0; tt < kMT; ++tt) {
            const float g = sg * warp_sum(ag[tt]);
            const float u = su * warp_sum(au[tt]);
            if (lane == 0 && tt < nt) h[(int64_t)(t0 + tt) * Wg.out + o] = silu(g) * u;
        }
    }
}

__global__ void __launch_bounds__(kMWarps * 32)
mixed_down_kernel(moe_mixed_tensor Wd, int G, const float* __restrict__ h, int T, const uint16_t* __restrict__ res,
                  uint16_t* __restrict__ y) {
    extern __shared__ float4 smem_f4[];
    float* xs = reinterpret_cast<float*>(smem_f4);
    float* xsum = xs + kMT * Wd.in;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int o = blockIdx.x * kMWarps + warp;
    for (int t0 = 0; t0 < T; t0 += kMT) {
        const int nt = min(kMT, T - t0);
        __syncthreads();
        mstage(xs, xsum, h, Wd.in, t0, nt, Wd.in);
        if (o >= Wd.out) continue;
        float acc[kMT];
#pragma unroll
        for (int tt = 0; tt < kMT; ++tt) acc[tt] = 0.0f;
        mixed_row(Wd, G, o, xs, xsum, acc, lane);
        const float s = bf16f(Wd.scales[o]);
#pragma unroll
        for (int tt = 0; tt < kMT; ++tt) {
            float v = s * warp_sum(acc[tt]);
            if (lane == 0 && tt < nt) {
                const int64_t i = (int64_t)(t0 + tt) * Wd.out + o;
                if (res) v += bf16f(res[i]);
                y[i] = f2bf16(v);
            }
        }
    }
}

cudaError_t set_smem(const void* fn, size_t smem) {
    static int c_lin = 0, c_gu = 0, c_down = 0;
    int& c = fn == (const void*)mixed_linear_kernel ? c_lin : fn == (const void*)mixed_gate_up_kernel ? c_gu : c_down;
    return ensure_smem(fn, smem, c);
}

size_t stage_bytes(int n) { return (size_t)kMT * n * sizeof(float) + (size_t)kMT * (n / 32) * sizeof(float); }

}  // namespace

cudaError_t launch_mixed_linear(const moe_mixed_tensor& W, int G, const uint16_t* x, int T, float* y, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    const size_t smem = stage_bytes(W.in);
    cudaError_t e = set_smem((const void*)mixed_linear_kernel, smem);
    if (e != cudaSuccess) return e;
    mixed_linear_kernel<<<(W.out + kMWarps - 1) / kMWarps, kMWarps * 32, smem, s>>>(W, G, x, T, y);
    return cudaGetLastError();
}

cudaError_t launch_mixed_gate_up(const moe_mixed_tensor& g, const moe_mixed_tensor& u, int G, const uint16_t* x,
                                 int T, float* h, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    const size_t smem = stage_bytes(g.in);
    cudaError_t e = set_smem((const void*)mixed_gate_up_kernel, smem);
    if (e != cudaSuccess) return e;
    mixed_gate_up_kernel<<<(g.out + kMWarps - 1) / kMWarps, kMWarps * 32, smem, s>>>(g, u, G, x, T, h);
    return cudaGetLastError();
}

cudaError_t launch_mixed_down(const moe_mixed_tensor& d, int G, const float* h, int T, const uint16_t* residual,
                              uint16_t* y, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    const size_t smem = stage_bytes(d.in);
    cudaError_t e = set_smem((const void*)mixed_down_kernel, smem);
    if (e != cudaSuccess) return e;
    mixed_down_kernel<<<(d.out + kMWarps - 1) / kMWarps, kMWarps * 32, smem, s>>>(d, G, h, T, residual, y);
    return cudaGetLastError();
}

}  // namespace moeq
