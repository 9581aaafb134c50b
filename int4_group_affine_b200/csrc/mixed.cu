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

constexpr int kMT = 8;      // tokens per shared-memory chunk (the largest instantiation)
constexpr int kMWarps = 8;  // warps (rows) per CTA

__device__ __forceinline__ int mswz(int j) {
    const int c = j >> 5;
    return (c << 5) | (((j & 31) + ((c & 7) << 2)) & 31);
}

// Stage the nt live token rows (of at most MT) of length n into swizzled fp32 shared
// memory with 32-element chunk sums.  Rows at 16-byte aligned addresses come in 16-byte
// pieces (8 bf16 or 4 fp32 values, one per thread and step; the lanes of a chunk add
// their sums with shuffles); other rows value by value.
template <int MT, typename Src>
__device__ void mstage(float* xs, float* xsum, const Src* src, int ld, int t0, int nt, int n) {
    constexpr int kE = 16 / (int)sizeof(Src);  // values per 16-byte piece
    constexpr int kL = 32 / kE;                // pieces (lanes) per 32-value chunk
    const Src* base = src + (int64_t)t0 * ld;
    const bool vec = ((((uintptr_t)base) | ((uintptr_t)ld * sizeof(Src))) & 15) == 0;
    if (vec) {
        const int per = n / kE, total = nt * per, lim = (total + 31) / 32 * 32;
        for (int i = threadIdx.x; i < lim; i += blockDim.x) {
            const bool live = i < total;
            const int tt = live ? i / per : 0, q = live ? i % per : 0;
            float f[kE];
            if (live) {
                const uint4 u = reinterpret_cast<const uint4*>(base + (int64_t)tt * ld)[q];
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
                if constexpr (kE == 8) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        f[2 * k] = __uint_as_float(w[k] << 16);
                        f[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < 4; ++k) f[k] = __uint_as_float(w[k]);
                }
            } else {
#pragma unroll
                for (int k = 0; k < kE; ++k) f[k] = 0.0f;
            }
            const int c = q / kL, o = (q % kL) * kE, rot = (c & 7) << 2;
            float sm = 0.0f;
#pragma unroll
            for (int k = 0; k < kE; ++k) sm += f[k];
#pragma unroll
            for (int x = 1; x < kL; x <<= 1) sm += __shfl_xor_sync(0xffffffffu, sm, x);
            if (live) {
                float* d = xs + tt * n + (c << 5);
#pragma unroll
                for (int k = 0; k < kE; k += 4)
                    *reinterpret_cast<float4*>(d + ((o + k + rot) & 31)) = make_float4(f[k], f[k + 1], f[k + 2], f[k + 3]);
                if (q % kL == 0) xsum[tt * (n / 32) + c] = sm;
            }
        }
        __syncthreads();
        return;
    }
    for (int i = threadIdx.x; i < nt * n; i += blockDim.x) {
        const int tt = i / n, j = i % n;
        float v;
        if constexpr (sizeof(Src) == 2) v = bf16f(base[(int64_t)tt * ld + j]);
        else v = base[(int64_t)tt * ld + j];
        xs[tt * n + mswz(j)] = v;
    }
    __syncthreads();
    const int nc = n / 32;
    for (int i = threadIdx.x; i < nt * nc; i += blockDim.x) {
        const int tt = i / nc, c = i % nc;
        float sm = 0.0f;
        for (int f = 0; f < 32; ++f) sm += xs[tt * n + (c << 5) + f];
        xsum[i] = sm;
    }
    __syncthreads();
}

// Dot of 32 consecutive code fields (bits = 4 or 2, stored in `nw` words) with
// chunk c of each of the nt staged tokens; subtracts offset * chunk sum.
template <int BITS, int MT>
__device__ __forceinline__ void code_chunk(const uint32_t* w, int c, float offset, const float* xs, const float* xsum,
                                           int n, int nt, float* acc) {
    constexpr int kPer = 32 / BITS;  // fields per word
    constexpr uint32_t kMask = (1u << BITS) - 1u;
    float qf[32];
#pragma unroll
    for (int f = 0; f < 32; ++f) qf[f] = u2f_small((w[f / kPer] >> (BITS * (f % kPer))) & kMask);
    const int rot = (c & 7) << 2;
#pragma unroll
    for (int tt = 0; tt < MT; ++tt) {
        if (tt >= nt) break;
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
template <int MT>
__device__ __forceinline__ void mixed_row(const moe_mixed_tensor& W, int G, int o, const float* xs, const float* xsum,
                                          int nt, float* acc, int lane) {
    const int n = W.in;
    const uint32_t* pw = W.packed + mixed_row_offset(o, n, G);
    if (G > 0 && o % G == 0) {
        const uint4* v4 = reinterpret_cast<const uint4*>(pw);
        for (int c = lane; c < n / 32; c += 32) {
            const uint4 q = v4[c];
            const uint32_t w[4] = {q.x, q.y, q.z, q.w};
            code_chunk<4, MT>(w, c, 8.0f, xs, xsum, n, nt, acc);
        }
    } else {
        const uint4* v4 = reinterpret_cast<const uint4*>(pw);
        for (int v = lane; v < n / 64; v += 32) {
            const uint4 q = v4[v];
            const uint32_t w0[2] = {q.x, q.y}, w1[2] = {q.z, q.w};
            code_chunk<2, MT>(w0, 2 * v, 1.0f, xs, xsum, n, nt, acc);
            code_chunk<2, MT>(w1, 2 * v + 1, 1.0f, xs, xsum, n, nt, acc);
        }
    }
}

// MT: tokens per shared-memory chunk of this instantiation (T is walked in chunks of MT).
template <int MT>
__global__ void __launch_bounds__(kMWarps * 32)
mixed_linear_kernel(moe_mixed_tensor W, int G, const uint16_t* __restrict__ x, int T, float* __restrict__ y) {
    extern __shared__ float4 smem_f4[];
    float* xs = reinterpret_cast<float*>(smem_f4);
    float* xsum = xs + MT * W.in;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int o = blockIdx.x * kMWarps + warp;
    for (int t0 = 0; t0 < T; t0 += MT) {
        const int nt = min(MT, T - t0);
        __syncthreads();
        mstage<MT>(xs, xsum, x, W.in, t0, nt, W.in);
        if (o >= W.out) continue;
        float acc[MT];
#pragma unroll
        for (int tt = 0; tt < MT; ++tt) acc[tt] = 0.0f;
        mixed_row<MT>(W, G, o, xs, xsum, nt, acc, lane);
        const float s = bf16f(W.scales[o]);
#pragma unroll
        for (int tt = 0; tt < MT; ++tt) {
            if (tt >= nt) break;
            const float v = warp_sum(acc[tt]);
            if (lane == 0) y[(int64_t)(t0 + tt) * W.out + o] = s * v;
        }
    }
}

template <int MT>
__global__ void __launch_bounds__(kMWarps * 32)
mixed_gate_up_kernel(moe_mixed_tensor Wg, moe_mixed_tensor Wu, int G, const uint16_t* __restrict__ x, int T,
                     float* __restrict__ h) {
    extern __shared__ float4 smem_f4[];
    float* xs = reinterpret_cast<float*>(smem_f4);
    float* xsum = xs + MT * Wg.in;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int o = blockIdx.x * kMWarps + warp;
    for (int t0 = 0; t0 < T; t0 += MT) {
        const int nt = min(MT, T - t0);
        __syncthreads();
        mstage<MT>(xs, xsum, x, Wg.in, t0, nt, Wg.in);
        if (o >= Wg.out) continue;
        float ag[MT], au[MT];
#pragma unroll
        for (int tt = 0; tt < MT; ++tt) ag[tt] = au[tt] = 0.0f;
        mixed_row<MT>(Wg, G, o, xs, xsum, nt, ag, lane);
        mixed_row<MT>(Wu, G, o, xs, xsum, nt, au, lane);
        const float sg = bf16f(Wg.scales[o]), su = bf16f(Wu.scales[o]);
#pragma unroll
        for (int tt = 0; tt < MT; ++tt) {
            if (tt >= nt) break;
            const float g = sg * warp_sum(ag[tt]);
            const float u = su * warp_sum(au[tt]);
            if (lane == 0) h[(int64_t)(t0 + tt) * Wg.out + o] = silu(g) * u;
        }
    }
}

template <int MT>
__global__ void __launch_bounds__(kMWarps * 32)
mixed_down_kernel(moe_mixed_tensor Wd, int G, const float* __restrict__ h, int T, const uint16_t* __restrict__ res,
                  uint16_t* __restrict__ y) {
    extern __shared__ float4 smem_f4[];
    float* xs = reinterpret_cast<float*>(smem_f4);
    float* xsum = xs + MT * Wd.in;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int o = blockIdx.x * kMWarps + warp;
    for (int t0 = 0; t0 < T; t0 += MT) {
        const int nt = min(MT, T - t0);
        __syncthreads();
        mstage<MT>(xs, xsum, h, Wd.in, t0, nt, Wd.in);
        if (o >= Wd.out) continue;
        float acc[MT];
#pragma unroll
        for (int tt = 0; tt < MT; ++tt) acc[tt] = 0.0f;
        mixed_row<MT>(Wd, G, o, xs, xsum, nt, acc, lane);
        const float s = bf16f(Wd.scales[o]);
#pragma unroll
        for (int tt = 0; tt < MT; ++tt) {
            if (tt >= nt) break;
            float v = s * warp_sum(acc[tt]);
            if (lane == 0) {
                const int64_t i = (int64_t)(t0 + tt) * Wd.out + o;
                if (res) v += bf16f(res[i]);
                y[i] = f2bf16(v);
            }
        }
    }
}

size_t stage_bytes(int n, int mt) { return (size_t)mt * n * sizeof(float) + (size_t)mt * (n / 32) * sizeof(float); }

int mt_for(int T) { return T <= 1 ? 1 : T <= 2 ? 2 : T <= 4 ? 4 : kMT; }

}  // namespace

#define MOEQ_MIXED_DISPATCH(MTV, CALL) \
    switch (MTV) {                       \
        case 1: CALL(1); break;          \
        case 2: CALL(2); break;          \
        case 4: CALL(4); break;          \
        default: CALL(8); break;         \
    }

cudaError_t launch_mixed_linear(const moe_mixed_tensor& W, int G, const uint16_t* x, int T, float* y, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    const int mt = mt_for(T);
    const size_t smem = stage_bytes(W.in, mt);
    cudaError_t e = cudaSuccess;
#define MOEQ_CALL(M)                                                                                                 \
    {                                                                                                                \
        e = ensure_smem((const void*)mixed_linear_kernel<M>, smem, cache_lin[M]);                                     \
        if (e == cudaSuccess)                                                                                        \
            mixed_linear_kernel<M><<<(W.out + kMWarps - 1) / kMWarps, kMWarps * 32, smem, s>>>(W, G, x, T, y);       \
    }
    static int cache_lin[kMT + 1] = {0};
    MOEQ_MIXED_DISPATCH(mt, MOEQ_CALL)
#undef MOEQ_CALL
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_mixed_gate_up(const moe_mixed_tensor& g, const moe_mixed_tensor& u, int G, const uint16_t* x,
                                 int T, float* h, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    const int mt = mt_for(T);
    const size_t smem = stage_bytes(g.in, mt);
    cudaError_t e = cudaSuccess;
#define MOEQ_CALL(M)                                                                                                 \
    {                                                                                                                \
        e = ensure_smem((const void*)mixed_gate_up_kernel<M>, smem, cache_gu[M]);                                     \
        if (e == cudaSuccess)                                                                                        \
            mixed_gate_up_kernel<M><<<(g.out + kMWarps - 1) / kMWarps, kMWarps * 32, smem, s>>>(g, u, G, x, T, h);   \
    }
    static int cache_gu[kMT + 1] = {0};
    MOEQ_MIXED_DISPATCH(mt, MOEQ_CALL)
#undef MOEQ_CALL
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_mixed_down(const moe_mixed_tensor& d, int G, const float* h, int T, const uint16_t* residual,
                              uint16_t* y, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    const int mt = mt_for(T);
    const size_t smem = stage_bytes(d.in, mt);
    cudaError_t e = cudaSuccess;
#define MOEQ_CALL(M)                                                                                                 \
    {                                                                                                                \
        e = ensure_smem((const void*)mixed_down_kernel<M>, smem, cache_dn[M]);                                        \
        if (e == cudaSuccess)                                                                                        \
            mixed_down_kernel<M><<<(d.out + kMWarps - 1) / kMWarps, kMWarps * 32, smem, s>>>(d, G, h, T, residual, y); \
    }
    static int cache_dn[kMT + 1] = {0};
    MOEQ_MIXED_DISPATCH(mt, MOEQ_CALL)
#undef MOEQ_CALL
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace moeq
