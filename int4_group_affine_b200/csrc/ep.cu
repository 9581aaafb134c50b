// ep.cu - the device pieces of expert parallelism: routed experts run on given rows,
// the stable partition of a batch's routed jobs by owning rank (the dispatch), and the
// fixed-order combine of the rows that come back.
//
// With G ranks each owning E/G consecutive experts, a token's K routed jobs go to the
// ranks owning their experts (one all-to-all), run there, and come back (a second
// all-to-all); the router and the shared expert are replicated on every rank.  The
// collectives themselves are NCCL's (host orchestration in ep.py).
#include "common.cuh"

namespace moeq {
namespace {

constexpr int kPackThreads = 1024;

// Writes idx = expert[n] (K = 1), w = 1 and sg = 1 for the experts-only forward.
__global__ void given_experts_kernel(const int32_t* __restrict__ expert, int N, int32_t* __restrict__ idx,
                                     float* __restrict__ w, float* __restrict__ sg) {
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= N) return;
    idx[n] = expert[n];
    w[n] = 1.0f;
    sg[n] = 1.0f;
}

// Stable partition of the J = T*K routed jobs (j = t*K + k, expert idx[j]) by owner
// rank idx[j] / (E/G): pos[j] = the job's place in the send order (rank-major, job order
// within a rank), counts[g] = jobs for rank g.  One CTA: for each chunk of jobs, each
// warp counts its jobs per rank with ballots, the per-warp counts are scanned in shared
// memory, and a running base per rank carries over between chunks.
__global__ void __launch_bounds__(kPackThreads) ep_partition_kernel(const int32_t* __restrict__ idx, int J, int E,
                                                                    int G, int32_t* __restrict__ pos,
                                                                    int32_t* __restrict__ counts,
                                                                    int32_t* status) {
    __shared__ int s_warp[kPackThreads / 32][MOEQ_EP_MAX_RANKS];
    __shared__ int s_base[MOEQ_EP_MAX_RANKS];
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32, per = E / G;
    if (tid < G) s_base[tid] = 0;
    __syncthreads();
    for (int c0 = 0; c0 < J; c0 += kPackThreads) {
        const int j = c0 + tid;
        int d = -1;
        if (j < J) {
            const int e = idx[j];
            if (e < 0 || e >= E) raise_status(status, MOE_ERR_DEVICE_INDEX);
            d = min(max(e, 0), E - 1) / per;
        }
        int rank_in_warp = 0;
        for (int g = 0; g < G; ++g) {
            const uint32_t m = __ballot_sync(0xffffffffu, d == g);
            if (d == g) rank_in_warp = __popc(m & ((1u << lane) - 1u));
            if (lane == 0) s_warp[warp][g] = __popc(m);
        }
        __syncthreads();
        if (tid < G) {  // exclusive scan over the warps for rank tid, then advance its base
            int run = s_base[tid];
            for (int w = 0; w < kPackThreads / 32; ++w) {
                const int c = s_warp[w][tid];
                s_warp[w][tid] = run;
                run += c;
            }
            s_base[tid] = run;
        }
        __syncthreads();
        if (j < J) pos[j] = s_warp[warp][d] + rank_in_warp;  // (rank-local place for now)
        __syncthreads();
    }
    // rank-local places -> global send positions
    __shared__ int s_off[MOEQ_EP_MAX_RANKS + 1];
    if (tid == 0) {
        int o = 0;
        for (int g = 0; g < G; ++g) {
            s_off[g] = o;
            o += s_base[g];
        }
        s_off[G] = o;
    }
    __syncthreads();
    if (tid < G) counts[tid] = s_base[tid];
    for (int j = tid; j < J; j += kPackThreads) {
        const int e = min(max(idx[j], 0), E - 1);
        pos[j] += s_off[e / per];
    }
}

// send rows: row pos[j] = x[token(j)], meta = {expert, adapter}; one warp per job.
__global__ void ep_pack_rows_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ idx,
                                    const int32_t* __restrict__ adapter_id, int n_adapters, const int32_t* pos, int J,
                                    int K, int H, int E, uint16_t* __restrict__ send_x, int32_t* __restrict__ meta) {
    const int j = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32, lane = threadIdx.x % 32;
    if (j >= J) return;
    const int t = j / K, p = pos[j];
    const uint4* src = reinterpret_cast<const uint4*>(x + (int64_t)t * H);
    uint4* dst = reinterpret_cast<uint4*>(send_x + (int64_t)p * H);
    for (int c = lane; c < H / 8; c += 32) dst[c] = src[c];
    if (lane == 0) {
        meta[2 * p] = min(max(idx[j], 0), E - 1);
        meta[2 * p + 1] = adapter_id ? adapter_id[t] : (n_adapters > 0 ? 0 : -1);
    }
}

// y[t] = bf16(sum_k w[t][k] ret[pos[t k]] + sg[t] shared[t]) in fixed order, 2 outputs a thread.
__global__ void ep_combine_kernel(const uint16_t* __restrict__ ret, const int32_t* __restrict__ pos,
                                  const float* __restrict__ w, const uint16_t* __restrict__ shared,
                                  const float* __restrict__ sg, int T, int K, int H, uint16_t* __restrict__ y) {
    const int t = blockIdx.y, o = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (t >= T || o >= H) return;
    float a0 = 0.0f, a1 = 0.0f;
    for (int k = 0; k < K; ++k) {
        const float wk = w[t * K + k];
        const uint32_t v = *reinterpret_cast<const uint32_t*>(ret + (int64_t)pos[t * K + k] * H + o);
        a0 = fmaf(wk, __uint_as_float(v << 16), a0);
        a1 = fmaf(wk, __uint_as_float(v & 0xFFFF0000u), a1);
    }
    if (shared) {
        const uint32_t v = *reinterpret_cast<const uint32_t*>(shared + (int64_t)t * H + o);
        const float s = sg ? sg[t] : 1.0f;
        a0 = fmaf(s, __uint_as_float(v << 16), a0);
        a1 = fmaf(s, __uint_as_float(v & 0xFFFF0000u), a1);
    }
    *reinterpret_cast<uint32_t*>(y + (int64_t)t * H + o) = (uint32_t)f2bf16(a0) | ((uint32_t)f2bf16(a1) << 16);
}

}  // namespace

cudaError_t launch_given_experts(const int32_t* expert, int N, int32_t* idx, float* w, float* sg, cudaStream_t s) {
    if (N == 0) return cudaSuccess;
    given_experts_kernel<<<(N + 255) / 256, 256, 0, s>>>(expert, N, idx, w, sg);
    return cudaGetLastError();
}

cudaError_t launch_ep_dispatch(const uint16_t* x, const int32_t* idx, const int32_t* adapter_id, int n_adapters, int T,
                               int K, int H, int E, int G, int32_t* pos, int32_t* counts, uint16_t* send_x,
                               int32_t* meta, int32_t* status, cudaStream_t s) {
    const int J = T * K;
    if (J == 0) return cudaSuccess;
    ep_partition_kernel<<<1, kPackThreads, 0, s>>>(idx, J, E, G, pos, counts, status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    ep_pack_rows_kernel<<<(J + 7) / 8, 256, 0, s>>>(x, idx, adapter_id, n_adapters, pos, J, K, H, E, send_x, meta);
    return cudaGetLastError();
}

cudaError_t launch_ep_combine(const uint16_t* ret, const int32_t* pos, const float* w, const uint16_t* shared,
                              const float* sg, int T, int K, int H, uint16_t* y, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    dim3 grid((H / 2 + 127) / 128, T);
    ep_combine_kernel<<<grid, 128, 0, s>>>(ret, pos, w, shared, sg, T, K, H, y);
    return cudaGetLastError();
}

}  // namespace moeq
