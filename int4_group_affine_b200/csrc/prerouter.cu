// prerouter.cu - the prerouter head of one layer ("Edge0 项目推荐" review, 亮点一):
//   logits = linear_init(f) + fc2(gelu_erf(fc1(f))),
//   f = [h, onehot(this token's executed top-K), onehot(the previous token's)],
// with fp16 weights and fp32 arithmetic.  Its top-K is the expert set the next
// layer runs for the next token (the double shift on that page).
//
// Each one-hot part of f has K ones among E zeros, so it contributes K columns of
// a weight row: those are gathered and added instead of taking a dot product over
// 2E mostly-zero features.  A GEMV over the head's rows at decode: bound by the
// fp16 weight bytes (the h part of fc1 and linear_init, fc2).
#include <cuda_fp16.h>

#include "common.cuh"

namespace moeq {
namespace {

constexpr int kPT = 8;  // tokens per CTA
constexpr int kPW = 4;  // warps per CTA, one weight row each

__device__ __forceinline__ float gelu_erf(float v) { return 0.5f * v * (1.0f + erff(v * 0.70710678118654752f)); }

// Sum over the distinct experts of one token's list `ids` (K entries) of row[base + e],
// split over the lanes (lane k takes entry k unless an earlier entry repeats it).  An
// entry outside [0, E) adds nothing and raises MOE_ERR_DEVICE_INDEX.
__device__ __forceinline__ float onehot_part(const uint16_t* row, int base, const int32_t* ids, int K, int E,
                                             int lane, int32_t* status) {
    const int e = lane < K ? ids[lane] : -1;
    bool first = lane < K && e >= 0 && e < E;
    if (lane < K && !first) raise_status(status, MOE_ERR_DEVICE_INDEX);
    for (int j = 0; j < K; ++j) {
        const int ej = __shfl_sync(0xffffffffu, e, j);
        if (j < lane && ej == e) first = false;
    }
    return first ? __half2float(__ushort_as_half(row[base + e])) : 0.0f;
}

// Rows [0, D): fc1 then GELU -> hidden [T][D]; rows [D, D + E): linear_init -> lin [T][E]
// (biases included).  One warp per row, kPT tokens per CTA (blockIdx.y).
__global__ void __launch_bounds__(kPW * 32) pr_first_kernel(const moe_prerouter P, const uint16_t* __restrict__ h,
                                                            const int32_t* __restrict__ exec_idx,
                                                            const int32_t* __restrict__ prev_idx, int T,
                                                            float* __restrict__ hidden, float* __restrict__ lin,
                                                            int32_t* status) {
    extern __shared__ __align__(16) unsigned char psm[];
    uint16_t* hs = reinterpret_cast<uint16_t*>(psm);  // [kPT][H] bf16
    const int H = P.hidden, E = P.n_experts, K = P.top_k, D = P.head_dim, F = H + 2 * E;
    const int t0 = blockIdx.y * kPT, nt = min(kPT, T - t0);
    const int per = H / 8;  // 16-byte pieces of a row's h part
    for (int i = threadIdx.x; i < nt * per; i += blockDim.x)
        reinterpret_cast<uint4*>(hs)[i] = reinterpret_cast<const uint4*>(h + (int64_t)t0 * H)[i];
    __syncthreads();
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int row = blockIdx.x * kPW + warp;
    if (row >= D + E) return;
    const bool fc1 = row < D;
    const uint16_t* W = fc1 ? P.w1 + (int64_t)row * F : P.wl + (int64_t)(row - D) * F;
    float acc[kPT];
#pragma unroll
    for (int m = 0; m < kPT; ++m) acc[m] = 0.0f;
#pragma unroll 4
    for (int c = lane; c < per; c += 32) {
        const uint4 wv = reinterpret_cast<const uint4*>(W)[c];
        const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
        float wf[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f2 = __half22float2(*reinterpret_cast<const __half2*>(&ww[j]));
            wf[2 * j] = f2.x;
            wf[2 * j + 1] = f2.y;
        }
#pragma unroll
        for (int m = 0; m < kPT; ++m) {
            if (m >= nt) break;
            const uint4 xv = reinterpret_cast<const uint4*>(hs + m * H)[c];
            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
            float a = acc[m];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                a = fmaf(wf[2 * j], __uint_as_float(xw[j] << 16), a);
                a = fmaf(wf[2 * j + 1], __uint_as_float(xw[j] & 0xFFFF0000u), a);
            }
            acc[m] = a;
        }
    }
#pragma unroll
    for (int m = 0; m < kPT; ++m) {
        if (m >= nt) break;
        const int t = t0 + m;
        float v = acc[m] + onehot_part(W, H, exec_idx + (int64_t)t * K, K, E, lane, status);
        if (prev_idx) v += onehot_part(W, H + E, prev_idx + (int64_t)t * K, K, E, lane, status);
        v = warp_sum(v);
        if (lane == 0) {
            if (fc1) {
                const float b = P.b1 ? __half2float(__ushort_as_half(P.b1[row])) : 0.0f;
                hidden[(int64_t)t * D + row] = gelu_erf(v + b);
            } else {
                const int e = row - D;
                const float b = P.bl ? __half2float(__ushort_as_half(P.bl[e])) : 0.0f;
                lin[(int64_t)t * E + e] = v + b;
            }
        }
    }
}

// logits[t][e] = lin[t][e] + b2[e] + fc2 row e . hidden[t]; one warp per row.
__global__ void __launch_bounds__(kPW * 32) pr_second_kernel(const moe_prerouter P, const float* __restrict__ hidden,
                                                             const float* __restrict__ lin, int T,
                                                             float* __restrict__ logits) {
    extern __shared__ __align__(16) unsigned char psm[];
    float* hd = reinterpret_cast<float*>(psm);  // [kPT][D]
    const int E = P.n_experts, D = P.head_dim;
    const int t0 = blockIdx.y * kPT, nt = min(kPT, T - t0);
    for (int i = threadIdx.x; i < nt * D / 4; i += blockDim.x)
        reinterpret_cast<float4*>(hd)[i] = reinterpret_cast<const float4*>(hidden + (int64_t)t0 * D)[i];
    __syncthreads();
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int e = blockIdx.x * kPW + warp;
    if (e >= E) return;
    const uint16_t* W = P.w2 + (int64_t)e * D;
    float acc[kPT];
#pragma unroll
    for (int m = 0; m < kPT; ++m) acc[m] = 0.0f;
    for (int c = lane; c < D / 8; c += 32) {
        const uint4 wv = reinterpret_cast<const uint4*>(W)[c];
        const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
        float wf[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f2 = __half22float2(*reinterpret_cast<const __half2*>(&ww[j]));
            wf[2 * j] = f2.x;
            wf[2 * j + 1] = f2.y;
        }
#pragma unroll
        for (int m = 0; m < kPT; ++m) {
            if (m >= nt) break;
            const float4 a0 = reinterpret_cast<const float4*>(hd + m * D)[2 * c];
            const float4 a1 = reinterpret_cast<const float4*>(hd + m * D)[2 * c + 1];
            float a = acc[m];
            a = fmaf(wf[0], a0.x, a);
            a = fmaf(wf[1], a0.y, a);
            a = fmaf(wf[2], a0.z, a);
            a = fmaf(wf[3], a0.w, a);
            a = fmaf(wf[4], a1.x, a);
            a = fmaf(wf[5], a1.y, a);
            a = fmaf(wf[6], a1.z, a);
            a = fmaf(wf[7], a1.w, a);
            acc[m] = a;
        }
    }
#pragma unroll
    for (int m = 0; m < kPT; ++m) {
        if (m >= nt) break;
        const float v = warp_sum(acc[m]);
        if (lane == 0) {
            const int t = t0 + m;
            const float b = P.b2 ? __half2float(__ushort_as_half(P.b2[e])) : 0.0f;
            logits[(int64_t)t * E + e] = lin[(int64_t)t * E + e] + b + v;
        }
    }
}

inline size_t al256(size_t v) { return (v + 255) / 256 * 256; }

}  // namespace

// Workspace: the 256-byte status header, hidden [T][D], lin [T][E], top-K weights [T][K].
size_t prerouter_workspace_bytes(const moe_prerouter& P, int T) {
    return 256 + al256((size_t)T * P.head_dim * 4) + al256((size_t)T * P.n_experts * 4) +
           al256((size_t)T * P.top_k * 4);
}

cudaError_t launch_prerouter(const moe_prerouter& P, const uint16_t* h, const int32_t* exec_idx,
                             const int32_t* prev_idx, int T, float* logits, int32_t* pred_idx, void* ws,
                             cudaStream_t s) {
    int32_t* status = (int32_t*)ws;
    char* b = (char*)ws + 256;
    float* hidden = (float*)b;
    float* lin = (float*)(b + al256((size_t)T * P.head_dim * 4));
    float* wtmp = (float*)(b + al256((size_t)T * P.head_dim * 4) + al256((size_t)T * P.n_experts * 4));
    const int chunks = (T + kPT - 1) / kPT;
    const size_t sm1 = (size_t)kPT * P.hidden * 2, sm2 = (size_t)kPT * P.head_dim * 4;
    static int c1 = 0, c2 = 0;
    cudaError_t e = ensure_smem((const void*)pr_first_kernel, sm1, c1);
    if (e != cudaSuccess) return e;
    e = ensure_smem((const void*)pr_second_kernel, sm2, c2);
    if (e != cudaSuccess) return e;
    pr_first_kernel<<<dim3((P.head_dim + P.n_experts + kPW - 1) / kPW, chunks), kPW * 32, sm1, s>>>(
        P, h, exec_idx, prev_idx, T, hidden, lin, status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    timing_mark(kPrerouter, s);
    pr_second_kernel<<<dim3((P.n_experts + kPW - 1) / kPW, chunks), kPW * 32, sm2, s>>>(P, hidden, lin, T, logits);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    timing_mark(kPrerouter, s);
    if (pred_idx) {
        e = launch_topk(logits, nullptr, false, T, P.n_experts, P.top_k, pred_idx, wtmp, nullptr, s);
        if (e != cudaSuccess) return e;
        timing_mark(kTopk, s);
    }
    return cudaSuccess;
}

}  // namespace moeq
