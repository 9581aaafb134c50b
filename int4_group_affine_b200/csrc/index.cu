// index.cu - a3: expert-grouped job list built on the device.
//
// Every token owns K routed jobs and one shared-expert job (expert index E).
// Jobs are bucketed by (expert, adapter) with adapter "none" last, and ordered
// by token then k inside a bucket.  Deterministic three-pass counting sort over
// chunks of 32 tokens:
//   count   : per (bucket, chunk) job counts (integer atomics, order free)
//   scan    : exclusive prefix over buckets-major (bucket, chunk) -> bases,
//             per-expert group offsets and the list of non-empty experts
//   scatter : inside a chunk, rank = jobs of earlier tokens (or earlier k of
//             the same token) in the same bucket; position = base + rank.
#include "tc.cuh"

namespace moeq {
namespace {

struct JobKey {
    int expert, adapter, bucket;
    bool bad;         // some index was out of range (flags the status)
    bool bad_expert;  // the job cannot run: its weight becomes 0
};

// Same mapping in count and scatter: an out-of-range expert becomes expert 0
// with weight 0; an out-of-range adapter becomes "none" (the token runs on the
// base weights); both flag the status.
__device__ __forceinline__ JobKey job_key(const Work& wk, const int32_t* adapter_id, int n_adapters, int t, int k) {
    JobKey j;
    j.bad = j.bad_expert = false;
    int e = k < wk.K ? wk.idx[(int64_t)t * wk.K + k] : wk.E;
    if (k < wk.K && (e < 0 || e >= wk.E)) {
        e = 0;
        j.bad = j.bad_expert = true;
    }
    int a = adapter_id ? adapter_id[t] : (n_adapters > 0 ? 0 : -1);
    if (a < -1 || a >= n_adapters) {
        a = -1;
        j.bad = true;
    }
    j.expert = e;
    j.adapter = a;
    j.bucket = e * wk.A1 + (a < 0 ? n_adapters : a);
    return j;
}

// One CTA per chunk of 32 tokens, one thread per job (token c*32 + j / (K+1), k = j % (K+1)).
__global__ void index_count_kernel(Work wk, const int32_t* __restrict__ adapter_id, int n_adapters) {
    const int c = blockIdx.x, nk = wk.K + 1, j = threadIdx.x;
    const int t = c * 32 + j / nk;
    if (j >= 32 * nk || t >= wk.T) return;
    const JobKey key = job_key(wk, adapter_id, n_adapters, t, j % nk);
    if (key.bad) raise_status(wk.status, MOE_ERR_DEVICE_INDEX);
    atomicAdd(&wk.cnt[(int64_t)key.bucket * wk.C + c], 1);
}

// Single CTA, counts in shared memory: they come in by cp.async (every copy in flight at
// once); thread t scans the contiguous run [t per, (t+1) per), the run totals are scanned
// across the CTA, and the results go back with coalesced stores.  Then group offsets and
// the list of non-empty experts.
__global__ void __launch_bounds__(1024) index_scan_smem_kernel(Work wk, int32_t* __restrict__ counts_out) {
    extern __shared__ int32_t sc[];
    __shared__ int32_t warp_tot[32];
    const int n = wk.nb * wk.C;
    const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
    const int n4 = n / 4;
    for (int i = tid; i < n4; i += 1024) tc::cp16(tc::smem_u32(sc + 4 * i), wk.cnt + 4 * i, 16u);
    for (int i = 4 * n4 + tid; i < n; i += 1024) tc::cp4(tc::smem_u32(sc + i), wk.cnt + i, 4u);
    tc::cp_commit();
    tc::cp_wait<0>();
    __syncthreads();
    const int per = (n + 1023) / 1024;
    const int i0 = min(n, tid * per), i1 = min(n, i0 + per);
    int32_t run = 0;
    for (int i = i0; i < i1; ++i) run += sc[i];
    int32_t incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int32_t wv = warp_tot[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t u = __shfl_up_sync(0xffffffffu, wv, o);
            if (lane >= o) wv += u;
        }
        warp_tot[lane] = wv;
    }
    __syncthreads();
    int32_t acc = (warp > 0 ? warp_tot[warp - 1] : 0) + incl - run;
    for (int i = i0; i < i1; ++i) {
        const int32_t v = sc[i];
        sc[i] = acc;
        acc += v;
    }
    __syncthreads();
    for (int i = tid; i < n; i += 1024) wk.cnt[i] = sc[i];
    for (int e = tid; e <= wk.E + 1; e += 1024) wk.goff[e] = e <= wk.E ? sc[e * wk.A1 * wk.C] : wk.J;
    __syncthreads();
    int32_t flag = 0, e = tid;
    if (e <= wk.E) {
        const int32_t c = (e < wk.E ? sc[(e + 1) * wk.A1 * wk.C] : wk.J) - sc[e * wk.A1 * wk.C];
        flag = c > 0;
        if (counts_out) counts_out[e] = c;
    }
    incl = flag;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int32_t wv = warp_tot[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t u = __shfl_up_sync(0xffffffffu, wv, o);
            if (lane >= o) wv += u;
        }
        warp_tot[lane] = wv;
    }
    __syncthreads();
    const int32_t pos = (warp > 0 ? warp_tot[warp - 1] : 0) + incl - flag;
    if (flag && wk.active) wk.active[pos] = e;
    if (tid == 1023 && wk.n_active) *wk.n_active = warp_tot[31];
}

// Single CTA, for counts that do not fit in shared memory: in place, 1024 at a time.
__global__ void __launch_bounds__(1024) index_scan_kernel(Work wk, int32_t* __restrict__ counts_out) {
    __shared__ int32_t warp_tot[32];
    __shared__ int32_t carry;
    const int64_t n = (int64_t)wk.nb * wk.C;
    const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int64_t base = 0; base < n; base += 1024) {
        const int64_t i = base + tid;
        const int32_t v = i < n ? wk.cnt[i] : 0;
        int32_t incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t u = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += u;
        }
        if (lane == 31) warp_tot[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            int32_t wv = warp_tot[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int32_t u = __shfl_up_sync(0xffffffffu, wv, o);
                if (lane >= o) wv += u;
            }
            warp_tot[lane] = wv;  // inclusive prefix of warp totals
        }
        __syncthreads();
        const int32_t excl = carry + (warp > 0 ? warp_tot[warp - 1] : 0) + incl - v;
        if (i < n) wk.cnt[i] = excl;
        __syncthreads();
        if (tid == 1023) carry = excl + v;
        __syncthreads();
    }
    // group offsets: the first (expert, adapter 0, chunk 0) base of each expert
    for (int e = tid; e <= wk.E + 1; e += 1024)
        wk.goff[e] = e <= wk.E ? wk.cnt[(int64_t)e * wk.A1 * wk.C] : wk.J;
    __syncthreads();
    // compact list of non-empty experts (E + 1 <= 513 entries, one pass)
    int32_t flag = 0, e = tid;
    if (e <= wk.E) {
        const int32_t c = wk.goff[e + 1] - wk.goff[e];
        flag = c > 0;
        if (counts_out) counts_out[e] = c;
    }
    int32_t incl = flag;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int32_t wv = warp_tot[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t u = __shfl_up_sync(0xffffffffu, wv, o);
            if (lane >= o) wv += u;
        }
        warp_tot[lane] = wv;
    }
    __syncthreads();
    const int32_t pos = (warp > 0 ? warp_tot[warp - 1] : 0) + incl - flag;
    if (flag && wk.active) wk.active[pos] = e;
    if (tid == 1023 && wk.n_active) *wk.n_active = warp_tot[31];
}

// One CTA per chunk of 32 tokens, one thread per job j (token c*32 + j / (K+1), k = j %
// (K+1)): its rank in its bucket is the number of the chunk's earlier jobs (earlier token,
// or same token and earlier k) in the same bucket.
__global__ void index_scatter_kernel(Work wk, const int32_t* __restrict__ adapter_id, int n_adapters) {
    __shared__ int32_t keys[32 * (MOEQ_MAX_TOPK + 1)];
    const int c = blockIdx.x, nk = wk.K + 1, j = threadIdx.x;
    const int t = c * 32 + j / nk, k = j % nk;
    const bool live = j < 32 * nk && t < wk.T;
    JobKey key;
    key.bucket = -1;
    if (live) key = job_key(wk, adapter_id, n_adapters, t, k);
    if (j < 32 * nk) keys[j] = key.bucket;
    __syncthreads();
    if (!live) return;
    int rank = 0;
    for (int u = 0; u < j; ++u) rank += keys[u] == key.bucket;
    const int pos = wk.cnt[(int64_t)key.bucket * wk.C + c] + rank;
    wk.perm[pos] = make_int4(t, k, key.adapter, key.expert);
    if (wk.wperm) {
        const float wt = k < wk.K ? wk.w[(int64_t)t * wk.K + k] : wk.sg[t];
        wk.wperm[pos] = key.bad_expert ? 0.0f : wt;
    }
    if (wk.inv) wk.inv[(int64_t)t * (wk.K + 1) + k] = pos;
}

}  // namespace

cudaError_t launch_index_build_counts(const Work& wk, const int32_t* adapter_id, int n_adapters,
                                      int32_t* counts_out, cudaStream_t s) {
    if (wk.T == 0) return cudaSuccess;
    cudaError_t e = cudaMemsetAsync(wk.cnt, 0, (size_t)wk.nb * wk.C * sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
    const int jobs = (32 * (wk.K + 1) + 31) / 32 * 32;  // threads per chunk: one per job
    index_count_kernel<<<wk.C, jobs, 0, s>>>(wk, adapter_id, n_adapters);
    timing_mark(kIndexCount, s);
    const size_t scan_smem = (size_t)wk.nb * wk.C * sizeof(int32_t);
    static int cached = 0;
    if (scan_smem <= 200 * 1024 && ensure_smem((const void*)index_scan_smem_kernel, scan_smem, cached) == cudaSuccess) {
        index_scan_smem_kernel<<<1, 1024, scan_smem, s>>>(wk, counts_out);
    } else {
        (void)cudaGetLastError();
        index_scan_kernel<<<1, 1024, 0, s>>>(wk, counts_out);
    }
    timing_mark(kIndexScan, s);
    index_scatter_kernel<<<wk.C, jobs, 0, s>>>(wk, adapter_id, n_adapters);
    timing_mark(kIndexScatter, s);
    return cudaGetLastError();
}

cudaError_t launch_index_build(const Work& wk, const int32_t* adapter_id, int n_adapters, cudaStream_t s) {
    return launch_index_build_counts(wk, adapter_id, n_adapters, nullptr, s);
}

}  // namespace moeq
