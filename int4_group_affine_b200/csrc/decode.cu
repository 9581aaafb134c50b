// decode.cu - the whole MoE layer for a handful of tokens in one persistent,
// cooperative kernel (one CTA per SM).
//
// At decode the layer is a chain of small dependent steps (router -> top-K ->
// expert rows -> down rows), each far too small to fill the GPU on its own; run
// as separate kernels the chain is bound by launch and memory latency.  Here the
// steps are phases of one kernel separated by grid barriers (bounded spins), and
// the code is arranged so that each phase pays about one memory round trip:
// every CTA asks for the weight rows of its later phases (bulk L2 prefetch) as
// soon as routing names them, and each warp issues all the loads of its tasks
// before it computes.
//
//  A  (no routing needed) router + shared-gate rows, shared-expert LoRA-A dots,
//     shared-expert gate/up rows (pre-activation, kept in scratch).
//  -- barrier --
//  B  every CTA: top-K of every token and the expert-grouped job list (a3) in
//     shared memory; L2 prefetch of this CTA's phase-C and phase-D rows; routed
//     LoRA-A dots; shared-expert SwiGLU with its LoRA-B delta and its partial
//     down LoRA-A sums.
//  -- barrier --
//  C  routed gate/up rows (a CTA owns a contiguous range of (expert, row) pairs),
//     LoRA-B delta, SwiGLU, partial down LoRA-A sums.
//  -- barrier --
//  D  down rows: a CTA owns a range of output rows for every job, adds the LoRA-B
//     delta, and combines the jobs of each token in fixed order (k = 0..K-1, then
//     the shared expert), optionally adding the residual.
#include "common.cuh"
#include "warp_topk.cuh"

namespace moeq {
namespace {

constexpr int kW = 16;  // warps per CTA
constexpr int kThreads = kW * 32;
constexpr int kMaxT = MOEQ_DECODE_MAX_TOKENS;
constexpr int kMaxJ = MOEQ_DECODE_MAX_JOBS;
constexpr int kMaxR = 32;                  // LoRA rank handled by the fused path (one lane per k)
constexpr unsigned kSpinLimit = 1u << 21;  // about a second of polling
constexpr int kMaxOut = 32;                // output rows per CTA in phase D
constexpr int kSplit = 8;                  // chunk split of the down LoRA-A dots in phase D

struct DArgs {
    LayerArgs L;
    const uint16_t* x;
    const int32_t* adapter_id;
    uint16_t* y;
    int T, block;
    float eps;
    float* logits;  // [T][E]
    float* gsl;     // [T]
    float* ts;      // [T][2r]   shared-expert LoRA-A products (gate | up)
    float* tg;      // [T*K][2r] routed LoRA-A products, by routed slot t*K+k
    float* gus;     // [T][Is][2] shared gate/up pre-activations
    float* h;       // [J][Imax] SwiGLU outputs, slot t*K+k (routed), T*K+t (shared)
    float* tdp;     // (unused)
    unsigned long long* bar;  // monotonic arrival counter
    int32_t* status;
};

__device__ __forceinline__ unsigned long long ld_acquire(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// Grid-wide barrier on a monotonic 64-bit arrival counter: barrier k of a launch
// is complete when the counter reaches base + (k + 1) * gridDim.x, where base (a
// multiple of gridDim.x) is learnt from this CTA's first arrival.  One atomic per
// CTA, nothing to reset.  Returns false (raising MOE_ERR_TIMEOUT) if the bounded
// wait gave up; the counter is then out of step and the workspace must be
// re-initialised.
__device__ bool grid_sync(unsigned long long* bar, unsigned long long& target, int32_t* status) {
    __shared__ int ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        ok = 1;
        const unsigned long long nb = gridDim.x;
        __threadfence();
        if (target == 0) {
            const unsigned long long prev = atomicAdd(bar, 1ull);
            target = (prev / nb + 1) * nb;
        } else {
            atomicAdd(bar, 1ull);
            target += nb;
        }
        unsigned spins = 0;
        while (ld_acquire(bar) < target) {
            if (++spins > kSpinLimit) {
                raise_status(status, MOE_ERR_TIMEOUT);
                ok = 0;
                break;
            }
            if (spins > 32) __nanosleep(32);
        }
        __threadfence();
    }
    __syncthreads();
    return ok != 0;
}

__device__ __forceinline__ void prefetch_l2(const void* p, size_t bytes) {
    if (bytes == 0 || (bytes & 15) || ((uintptr_t)p & 15)) return;
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"((unsigned)bytes) : "memory");
}

__device__ __forceinline__ void prefetch_qrow(const moe_qtensor& q, int64_t row) {
    const int64_t wpr = (int64_t)q.in * q.bits / 32;
    const int ng = q.in / q.group;
    prefetch_l2(q.packed + row * wpr, (size_t)wpr * 4);
    prefetch_l2(q.scales + row * ng, (size_t)ng * 2);
    prefetch_l2(q.biases + row * ng, (size_t)ng * 2);
}

// Stage nv bf16 rows of length n (n % 32 == 0) into swizzled fp32 shared memory
// with 32-element chunk sums; one 16-byte load per thread and step.  With
// `scale`, each value becomes bf16(x * scale[v]) (the normalised block input).
__device__ void stage_bf16(float* dst, float* dsum, const uint16_t* src, int nv, int n, const float* scale) {
    const int per = n / 8, total = nv * per;
    const int lim = (total + 31) / 32 * 32;
    for (int i = threadIdx.x; i < lim; i += kThreads) {
        const bool live = i < total;
        const int v = live ? i / per : 0, q = live ? i % per : 0;
        float f[8];
        if (live) {
            const uint4 u = reinterpret_cast<const uint4*>(src + (int64_t)v * n)[q];
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                f[2 * k] = __uint_as_float(w[k] << 16);
                f[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
            }
            if (scale)
#pragma unroll
                for (int k = 0; k < 8; ++k) f[k] = bf16f(f2bf16(f[k] * scale[v]));
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) f[k] = 0.0f;
        }
        const int c = q / 4, o = (q % 4) * 8, rot = (c & 7) << 2;
        float s = 0.0f;
#pragma unroll
        for (int k = 0; k < 8; ++k) s += f[k];
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        if (live) {
            float* d = dst + v * n + (c << 5);
            *reinterpret_cast<float4*>(d + ((o + rot) & 31)) = make_float4(f[0], f[1], f[2], f[3]);
            *reinterpret_cast<float4*>(d + ((o + 4 + rot) & 31)) = make_float4(f[4], f[5], f[6], f[7]);
            if ((q % 4) == 0) dsum[v * (n / 32) + c] = s;
        }
    }
}

// Same for fp32 rows written by other CTAs (read from L2), row stride `ld`.
__device__ void stage_f32(float* dst, float* dsum, const float* src, int ld, int nv, int n) {
    const int per = n / 4, total = nv * per;
    const int lim = (total + 31) / 32 * 32;
    for (int i = threadIdx.x; i < lim; i += kThreads) {
        const bool live = i < total;
        const int v = live ? i / per : 0, q = live ? i % per : 0;
        float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
        if (live) f = __ldcg(reinterpret_cast<const float4*>(src + (int64_t)v * ld) + q);
        const int c = q / 8, o = (q % 8) * 4, rot = (c & 7) << 2;
        float s = f.x + f.y + f.z + f.w;
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        s += __shfl_xor_sync(0xffffffffu, s, 4);
        if (live) {
            *reinterpret_cast<float4*>(dst + v * n + (c << 5) + ((o + rot) & 31)) = f;
            if ((q % 8) == 0) dsum[v * (n / 32) + c] = s;
        }
    }
}

// 32 nibbles -> 32 floats.
__device__ __forceinline__ void unpack4(const uint4 q4, float* qf) {
    const uint32_t qw[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
    for (int w = 0; w < 4; ++w)
#pragma unroll
        for (int f = 0; f < 8; ++f) qf[w * 8 + f] = u2f_small((qw[w] >> (4 * f)) & 15u);
}

// sum over chunk c of q[j] * v[j] for a staged (swizzled) vector row v.
__device__ __forceinline__ float chunk_qdot(const float* qf, const float* vrow, int c) {
    const float* vr = vrow + (c << 5);
    const int rot = (c & 7) << 2;
    float a = 0.0f;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const float4 xv = *reinterpret_cast<const float4*>(vr + ((4 * u + rot) & 31));
        a = fmaf(qf[4 * u + 0], xv.x, a);
        a = fmaf(qf[4 * u + 1], xv.y, a);
        a = fmaf(qf[4 * u + 2], xv.z, a);
        a = fmaf(qf[4 * u + 3], xv.w, a);
    }
    return a;
}

// acc[m] += sum_j (s q_j + b) v_m[j] over one int4 row of length n (<= 4096), for
// staged vectors v_m = vbase + vid[m] * n (m < nv <= MT), by a group of `lpt`
// lanes (sl = lane index in the group).  All of the row's loads are issued
// before any use.
// (Not inlined: one copy of the code serves every call site, which keeps the
// kernel's instruction footprint small; each launch runs every phase once.)
template <int MT>
__device__ __noinline__ void dot_int4(const uint32_t* __restrict__ prow, const uint16_t* __restrict__ srow,
                                         const uint16_t* __restrict__ brow, int group, int n, const float* vbase,
                                         const float* vsum, const int* vid, int nv, float* acc, int sl, int lpt) {
    constexpr int kIt = 4;
    const uint4* p4 = reinterpret_cast<const uint4*>(prow);
    const int nc = n / 32;
    uint4 q[kIt];
    float s[kIt], b[kIt];
#pragma unroll
    for (int it = 0; it < kIt; ++it) {
        const int c = sl + lpt * it;
        if (c < nc) {
            q[it] = p4[c];
            const int g = (c * 32) / group;
            s[it] = bf16f(srow[g]);
            b[it] = bf16f(brow[g]);
        }
    }
#pragma unroll
    for (int it = 0; it < kIt; ++it) {
        const int c = sl + lpt * it;
        if (c >= nc) break;
        float qf[32];
        unpack4(q[it], qf);
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            if (m >= nv) break;
            const float a = chunk_qdot(qf, vbase + vid[m] * n, c);
            acc[m] = fmaf(s[it], a, fmaf(b[it], vsum[vid[m] * nc + c], acc[m]));
        }
    }
}

// Same for an int8 row (H <= 4096), full warp, vectors v_m = vbase + m * n.
template <int MT>
__device__ __noinline__ void dot_int8(const uint32_t* __restrict__ prow, const uint16_t* __restrict__ srow,
                                         const uint16_t* __restrict__ brow, int group, int n, const float* vbase,
                                         const float* vsum, int nv, float* acc, int lane) {
    constexpr int kIt = 4;
    const uint4* p4 = reinterpret_cast<const uint4*>(prow);
    const int nc = n / 32;
    uint4 q0[kIt], q1[kIt];
    float s[kIt], b[kIt];
#pragma unroll
    for (int it = 0; it < kIt; ++it) {
        const int c = lane + 32 * it;
        if (c < nc) {
            q0[it] = p4[2 * c];
            q1[it] = p4[2 * c + 1];
            const int g = (c * 32) / group;
            s[it] = bf16f(srow[g]);
            b[it] = bf16f(brow[g]);
        }
    }
#pragma unroll
    for (int it = 0; it < kIt; ++it) {
        const int c = lane + 32 * it;
        if (c >= nc) break;
        const uint32_t qw[8] = {q0[it].x, q0[it].y, q0[it].z, q0[it].w, q1[it].x, q1[it].y, q1[it].z, q1[it].w};
        float qf[32];
#pragma unroll
        for (int w = 0; w < 8; ++w)
#pragma unroll
            for (int f = 0; f < 4; ++f) qf[w * 4 + f] = u2f_small((qw[w] >> (8 * f)) & 255u);
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            if (m >= nv) break;
            const float a = chunk_qdot(qf, vbase + m * n, c);
            acc[m] = fmaf(s[it], a, fmaf(b[it], vsum[m * nc + c], acc[m]));
        }
    }
}

// sum_j A[j] v[j] for a bf16 row A of length n (<= 4096) and one staged vector
// (lane partial; the caller reduces).  All loads first.
__device__ __noinline__ float dot_bf16(const uint16_t* __restrict__ arow, int n, const float* v, int lane) {
    constexpr int kIt = 4;
    const uint4* a4 = reinterpret_cast<const uint4*>(arow);
    const int nc = n / 32;
    uint4 q[kIt][4];
#pragma unroll
    for (int it = 0; it < kIt; ++it) {
        const int c = lane + 32 * it;
        if (c < nc)
#pragma unroll
            for (int u = 0; u < 4; ++u) q[it][u] = a4[4 * c + u];
    }
    float acc = 0.0f;
#pragma unroll
    for (int it = 0; it < kIt; ++it) {
        const int c = lane + 32 * it;
        if (c >= nc) break;
        const int rot = (c & 7) << 2;
        const float* vr = v + (c << 5);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const uint32_t aw[4] = {q[it][u].x, q[it][u].y, q[it][u].z, q[it][u].w};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float4 xv = *reinterpret_cast<const float4*>(vr + ((8 * u + 4 * h + rot) & 31));
                acc = fmaf(__uint_as_float(aw[2 * h] << 16), xv.x, acc);
                acc = fmaf(__uint_as_float(aw[2 * h] & 0xFFFF0000u), xv.y, acc);
                acc = fmaf(__uint_as_float(aw[2 * h + 1] << 16), xv.z, acc);
                acc = fmaf(__uint_as_float(aw[2 * h + 1] & 0xFFFF0000u), xv.w, acc);
            }
        }
    }
    return acc;
}

__device__ __forceinline__ float group_sum(float v, int lpt) {
    for (int o = lpt / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ const moe_lora_proj* dlora(const LayerArgs& L, int a, bool shared, int which) {
    if (a < 0 || a >= L.n_adapters) return nullptr;
    const moe_lora_ptrs& p = L.lora[a];
    const moe_lora_proj* q = which == 0 ? (shared ? &p.s_gate : &p.gate)
                           : which == 1 ? (shared ? &p.s_up : &p.up)
                                        : (shared ? &p.s_down : &p.down);
    return (q->A && q->B) ? q : nullptr;
}

__device__ __forceinline__ float ldb(const moe_lora_proj* lp, int64_t idx) { return lp ? bf16f(lp->B[idx]) : 0.0f; }

// MT: token capacity of this instantiation (register arrays), T <= MT.
template <int MT>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ DArgs a) {
    extern __shared__ float4 dsm[];
    const LayerArgs& L = a.L;
    const int T = a.T, H = L.H, E = L.E, K = L.K, r = L.rank, I = L.I, Is = L.Is;
    const int J = T * (K + 1);
    const int Imax = I > Is ? I : Is;
    const int NB = gridDim.x, cta = blockIdx.x;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const bool has_shared = L.has_shared;
    float* xs = reinterpret_cast<float*>(dsm);  // [T][H]
    float* xsum = xs + T * H;                    // [T][H/32]
    float* hs = xsum + T * (H / 32);             // [J][Imax] (phase D)
    float* hsum = hs + J * Imax;                 // [J][Imax/32]
    float* wpart = hsum + J * (Imax / 32);       // [kW][2][kMaxT][kMaxR] per-warp partial sums
    float* tdsplit = wpart;                      // phase D reuses it for [kMaxJ][kMaxR][kSplit] sums

    __shared__ int s_aid[kMaxT];
    __shared__ float s_inv[kMaxT];
    __shared__ int s_idx[kMaxT][MOEQ_MAX_TOPK];
    __shared__ float s_w[kMaxT][MOEQ_MAX_TOPK];
    __shared__ float s_sg[kMaxT];
    __shared__ int s_nu;
    __shared__ int s_uexp[kMaxJ], s_ucnt[kMaxJ], s_uslot[kMaxJ][kMaxT];
    __shared__ float s_td[kMaxJ][kMaxR];
    __shared__ float s_v[kMaxOut][kMaxJ];
    __shared__ int s_tok[kMaxT];
    unsigned long long bar_target = 0;

    const int R = E + (L.has_sgate ? 1 : 0);
    const int per_s = has_shared ? (Is + NB - 1) / NB : 0;
    const int s_lo = has_shared ? min(Is, cta * per_s) : 0, s_hi = has_shared ? min(Is, s_lo + per_s) : 0;

    // ------------------------------------------------------------ phase A
    // rows this CTA reads in phase A start moving now
    for (int q = threadIdx.x; q < (R + NB - 1) / NB + (s_hi - s_lo); q += kThreads) {
        const int nr = (R + NB - 1) / NB;
        if (q < nr) {
            const int tau = cta + NB * q;
            if (tau < E) prefetch_qrow(L.router, tau);
            else if (tau < R) prefetch_qrow(L.shared_gate, 0);
        } else {
            const int i = s_lo + (q - nr);
            prefetch_qrow(L.s_gate, i);
            prefetch_qrow(L.s_up, i);
        }
    }
    if (threadIdx.x < T) {
        const int t = threadIdx.x;
        int ad = a.adapter_id ? a.adapter_id[t] : (L.n_adapters > 0 ? 0 : -1);
        if (ad < -1 || ad >= L.n_adapters) {
            if (cta == 0) raise_status(a.status, MOE_ERR_DEVICE_INDEX);
            ad = -1;
        }
        s_aid[t] = ad;
        s_tok[t] = t;
    }
    if (a.block) {  // RMSNorm: warp t reduces token t
        for (int t = warp; t < T; t += kW) {
            float ss = 0.0f;
            const uint4* xr = reinterpret_cast<const uint4*>(a.x + (int64_t)t * H);
            for (int v = lane; v < H / 8; v += 32) {
                const uint4 u = xr[v];
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float lo = __uint_as_float(w[k] << 16), hi = __uint_as_float(w[k] & 0xFFFF0000u);
                    ss = fmaf(lo, lo, fmaf(hi, hi, ss));
                }
            }
            ss = warp_sum(ss);
            if (lane == 0) s_inv[t] = 1.0f / sqrtf(ss / (float)H + a.eps);
        }
        __syncthreads();
    } else {
        __syncthreads();
    }
    stage_bf16(xs, xsum, a.x, T, H, a.block ? s_inv : nullptr);
    __syncthreads();

    const int nA = R + (has_shared ? T * 2 * r : 0);
    for (int j = warp; cta + NB * j < nA; j += kW) {
        const int tau = cta + NB * j;
        if (tau < R) {  // router / shared-gate row
            const moe_qtensor& q = tau < E ? L.router : L.shared_gate;
            const int64_t row = tau < E ? tau : 0;
            const int ng = H / q.group;
            float acc[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
            dot_int8<MT>(q.packed + row * (H / 4), q.scales + row * ng, q.biases + row * ng, q.group, H, xs, xsum, T,
                     acc, lane);
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[m] = warp_sum(acc[m]);
            if (lane < T) {
                float v = 0.0f;
#pragma unroll
                for (int m = 0; m < MT; ++m)
                    if (m == lane) v = acc[m];
                if (tau < E) a.logits[(int64_t)lane * E + tau] = v + (L.logit_bias ? L.logit_bias[tau] : 0.0f);
                else a.gsl[lane] = v;
            }
        } else {  // shared-expert LoRA-A dot (token t, output d of gate|up)
            const int q = tau - R, t = q / (2 * r), d = q % (2 * r);
            const moe_lora_proj* lp = dlora(L, s_aid[t], true, d < r ? 0 : 1);
            float v = 0.0f;
            if (lp) v = warp_sum(dot_bf16(lp->A + (int64_t)(d % r) * H, H, xs + t * H, lane));
            if (lane == 0) a.ts[t * 2 * r + d] = v;
        }
    }
    // shared-expert gate/up pre-activations over this CTA's row range
    for (int i = s_lo + warp; i < s_hi; i += kW) {
        const int ng = H / L.s_gate.group;
        float ag[MT], au[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) ag[m] = au[m] = 0.0f;
        dot_int4<MT>(L.s_gate.packed + (int64_t)i * (H / 8), L.s_gate.scales + (int64_t)i * ng,
                 L.s_gate.biases + (int64_t)i * ng, L.s_gate.group, H, xs, xsum, s_tok, T, ag, lane, 32);
        dot_int4<MT>(L.s_up.packed + (int64_t)i * (H / 8), L.s_up.scales + (int64_t)i * ng,
                 L.s_up.biases + (int64_t)i * ng, L.s_up.group, H, xs, xsum, s_tok, T, au, lane, 32);
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            if (m >= T) break;
            const float g = warp_sum(ag[m]), u = warp_sum(au[m]);
            if (lane == 0) *reinterpret_cast<float2*>(a.gus + ((int64_t)m * Is + i) * 2) = make_float2(g, u);
        }
    }
    if (!grid_sync(a.bar, bar_target, a.status)) return;

    // ------------------------------------------------------------ phase B
    if (threadIdx.x < T) s_sg[threadIdx.x] = L.has_sgate ? 1.0f / (1.0f + expf(-__ldcg(a.gsl + threadIdx.x))) : 1.0f;
    // softmax, top-K (ties to the lower expert index) and renormalisation: one warp per
    // token over its logits, read from L2
    for (int t = warp; t < T; t += kW) {
        int ki[MOEQ_MAX_TOPK];
        float kw[MOEQ_MAX_TOPK];
        warp_topk<true>(a.logits + (int64_t)t * E, E, K, ki, kw);
        if (lane == 0)
            for (int k = 0; k < K; ++k) {
                s_idx[t][k] = ki[k];
                s_w[t][k] = kw[k];
            }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // routed jobs grouped by expert (ascending), inside by (adapter, token)
        int n = 0;
        for (int t = 0; t < T; ++t)
            for (int k = 0; k < K; ++k) {
                const int e = s_idx[t][k];
                int u = 0;
                while (u < n && s_uexp[u] < e) ++u;
                if (u == n || s_uexp[u] != e) {
                    for (int v = n; v > u; --v) {
                        s_uexp[v] = s_uexp[v - 1];
                        s_ucnt[v] = s_ucnt[v - 1];
                        for (int m = 0; m < MT; ++m) s_uslot[v][m] = s_uslot[v - 1][m];
                    }
                    s_uexp[u] = e;
                    s_ucnt[u] = 0;
                    ++n;
                }
                const int ar = s_aid[t] < 0 ? L.n_adapters : s_aid[t];
                int m = s_ucnt[u];
                while (m > 0) {
                    const int ps = s_uslot[u][m - 1], pt = ps / K;
                    const int par = s_aid[pt] < 0 ? L.n_adapters : s_aid[pt];
                    if (par < ar || (par == ar && pt < t)) break;
                    s_uslot[u][m] = ps;
                    --m;
                }
                s_uslot[u][m] = t * K + k;
                s_ucnt[u]++;
            }
        s_nu = n;
    }
    __syncthreads();
    const int U = s_nu;
    const int nC = U * I;
    const int perC = (nC + NB - 1) / NB;
    const int c_lo = min(nC, cta * perC), c_hi = min(nC, c_lo + perC);
    const int per_o = (H + NB - 1) / NB;
    const int o_lo = min(H, cta * per_o), o_hi = min(H, o_lo + per_o);
    const int UD = U + (has_shared ? 1 : 0);  // phase-D experts (the shared one last)
    for (int q = c_lo + threadIdx.x; q < c_hi; q += kThreads) {
        const int64_t row = (int64_t)s_uexp[q / I] * I + q % I;
        prefetch_qrow(L.gate, row);
        prefetch_qrow(L.up, row);
    }
    for (int q = threadIdx.x; q < (o_hi - o_lo) * UD; q += kThreads) {
        const int o = o_lo + q / UD, u = q % UD;
        if (u < U) prefetch_qrow(L.down, (int64_t)s_uexp[u] * H + o);
        else prefetch_qrow(L.s_down, o);
    }
    // routed LoRA-A dots, spread over the grid
    const int nB = T * K * 2 * r;
    for (int j = warp; cta + NB * j < nB; j += kW) {
        const int tau = cta + NB * j;
        const int slot = tau / (2 * r), d = tau % (2 * r);
        const int t = slot / K, k = slot % K, e = s_idx[t][k];
        const moe_lora_proj* lp = dlora(L, s_aid[t], false, d < r ? 0 : 1);
        float v = 0.0f;
        if (lp) v = warp_sum(dot_bf16(lp->A + ((int64_t)e * r + d % r) * H, H, xs + t * H, lane));
        if (lane == 0) a.tg[slot * 2 * r + d] = v;
    }
    // shared expert: LoRA-B delta and SwiGLU for this CTA's rows (lane k < r holds component k)
    if (has_shared) {
        for (int i = s_lo + warp; i < s_hi; i += kW) {
            float g[MT], u[MT], bg[MT], bu[MT], tgv[MT], tuv[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m >= T) break;
                const float2 gu = __ldcg(reinterpret_cast<const float2*>(a.gus + ((int64_t)m * Is + i) * 2));
                g[m] = gu.x;
                u[m] = gu.y;
                const moe_lora_proj* lg = dlora(L, s_aid[m], true, 0);
                const moe_lora_proj* lu = dlora(L, s_aid[m], true, 1);
                const bool kk = lane < r;
                bg[m] = kk ? ldb(lg, (int64_t)i * r + lane) : 0.0f;
                bu[m] = kk ? ldb(lu, (int64_t)i * r + lane) : 0.0f;
                tgv[m] = kk && lg ? __ldcg(a.ts + m * 2 * r + lane) : 0.0f;
                tuv[m] = kk && lu ? __ldcg(a.ts + m * 2 * r + r + lane) : 0.0f;
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m >= T) break;
                const float gv = g[m] + L.scale * warp_sum(bg[m] * tgv[m]);
                const float uv = u[m] + L.scale * warp_sum(bu[m] * tuv[m]);
                const float hv = silu(gv) * uv;
                if (lane == 0) a.h[(int64_t)(T * K + m) * Imax + i] = hv;
            }
        }
    }
    if (!grid_sync(a.bar, bar_target, a.status)) return;

    // ------------------------------------------------------------ phase C
    {
        for (int q = c_lo + warp; q < c_hi; q += kW) {
            const int u = q / I, i = q % I, e = s_uexp[u], nt = s_ucnt[u];
            const int64_t row = (int64_t)e * I + i;
            const int ng = H / L.gate.group;
            int toks[MT];
            float bg[MT], bu[MT], tgv[MT], tuv[MT];
            const bool kk = lane < r;
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                toks[m] = 0;
                bg[m] = bu[m] = tgv[m] = tuv[m] = 0.0f;
                if (m >= nt) continue;
                const int slot = s_uslot[u][m], t = slot / K;
                toks[m] = t;
                const moe_lora_proj* lg = dlora(L, s_aid[t], false, 0);
                const moe_lora_proj* lu = dlora(L, s_aid[t], false, 1);
                if (kk) {
                    bg[m] = ldb(lg, row * r + lane);
                    bu[m] = ldb(lu, row * r + lane);
                    tgv[m] = lg ? __ldcg(a.tg + slot * 2 * r + lane) : 0.0f;
                    tuv[m] = lu ? __ldcg(a.tg + slot * 2 * r + r + lane) : 0.0f;
                }
            }
            float ag[MT], au[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) ag[m] = au[m] = 0.0f;
            dot_int4<MT>(L.gate.packed + row * (H / 8), L.gate.scales + row * ng, L.gate.biases + row * ng,
                     L.gate.group, H, xs, xsum, toks, nt, ag, lane, 32);
            dot_int4<MT>(L.up.packed + row * (H / 8), L.up.scales + row * ng, L.up.biases + row * ng, L.up.group, H,
                     xs, xsum, toks, nt, au, lane, 32);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m >= nt) break;
                const int slot = s_uslot[u][m];
                const float g = warp_sum(ag[m]) + L.scale * warp_sum(bg[m] * tgv[m]);
                const float uu = warp_sum(au[m]) + L.scale * warp_sum(bu[m] * tuv[m]);
                const float hv = silu(g) * uu;
                if (lane == 0) a.h[(int64_t)slot * Imax + i] = hv;
            }
        }
    }
    if (!grid_sync(a.bar, bar_target, a.status)) return;

    // ------------------------------------------------------------ phase D
    stage_f32(hs, hsum, a.h, Imax, T * K, I);
    if (has_shared) stage_f32(hs + T * K * I, hsum + T * K * (I / 32), a.h + (int64_t)T * K * Imax, Imax, T, Is);
    __syncthreads();
    // t_d = A_d h of every job, from the staged h: each CTA computes all of them (the A_d
    // rows come from L2), so no cross-CTA reduction is needed.  Thread task (slot, k, p)
    // sums the 32-element chunks c = p (mod kSplit); the kSplit partials are then added in
    // order.
    for (int q = threadIdx.x; q < J * r * kSplit; q += kThreads) {
        const int slot = q / (r * kSplit), k = (q / kSplit) % r, p = q % kSplit;
        const bool shared = slot >= T * K;
        const int t = shared ? slot - T * K : slot / K;
        const int n = shared ? Is : I;
        const moe_lora_proj* ld = dlora(L, s_aid[t], shared, 2);
        float v = 0.0f;
        if (ld) {
            const int e = shared ? 0 : s_idx[t][slot % K];
            const uint16_t* arow = ld->A + ((int64_t)e * r + k) * n;
            const float* hrow = shared ? hs + T * K * I + (slot - T * K) * Is : hs + slot * I;
            for (int c = p; c < n / 32; c += kSplit) {  // chunk c: 32 elements, swizzled like stage_f32
                const uint4* a4 = reinterpret_cast<const uint4*>(arow + c * 32);
                const uint4 w4[4] = {a4[0], a4[1], a4[2], a4[3]};
                const int rot = (c & 7) << 2;
                const float* hr = hrow + (c << 5);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const uint32_t ww[4] = {w4[u].x, w4[u].y, w4[u].z, w4[u].w};
#pragma unroll
                    for (int h2 = 0; h2 < 4; ++h2) {
                        const int j0 = 8 * u + 2 * h2;
                        v = fmaf(__uint_as_float(ww[h2] << 16), hr[(j0 + rot) & 31], v);
                        v = fmaf(__uint_as_float(ww[h2] & 0xFFFF0000u), hr[(j0 + 1 + rot) & 31], v);
                    }
                }
            }
        }
        tdsplit[(slot * kMaxR + k) * kSplit + p] = v;
    }
    __syncthreads();
    for (int q = threadIdx.x; q < J * r; q += kThreads) {
        const int slot = q / r, k = q % r;
        float v = 0.0f;
        for (int p = 0; p < kSplit; ++p) v += tdsplit[(slot * kMaxR + k) * kSplit + p];
        s_td[slot][k] = v;
    }
    __syncthreads();
    // (output row, expert) tasks; a task is a group of lpt lanes over one down row
    {
        int lpt = 1;
        while (lpt * 2 <= 32 && lpt * 2 <= Imax / 32) lpt *= 2;
        const int gpw = 32 / lpt, sub = lane / lpt, sl = lane % lpt;
        const int ntask = (o_hi - o_lo) * UD;
        for (int q0 = warp * gpw; q0 < ntask; q0 += kW * gpw) {
            const int q = q0 + sub;
            const bool live = q < ntask;
            const int ol = live ? q / UD : 0, u = live ? q % UD : 0, o = o_lo + ol;
            const bool shared = u == U;
            const int n = shared ? Is : I;
            const moe_qtensor& Wd = shared ? L.s_down : L.down;
            const int64_t row = shared ? (int64_t)o : (int64_t)s_uexp[u] * H + o;
            const int nt = live ? (shared ? T : s_ucnt[u]) : 0;
            int sl_[MT];
            float bd[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                sl_[m] = 0;
                bd[m] = 0.0f;
                if (m >= nt) continue;
                const int slot = shared ? T * K + m : s_uslot[u][m];
                sl_[m] = slot;
                const moe_lora_proj* ld = dlora(L, s_aid[shared ? m : slot / K], shared, 2);
                if (sl < r) bd[m] = ldb(ld, row * r + sl);
            }
            float acc[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
            const int ng = n / Wd.group;
            if (live)
                dot_int4<MT>(Wd.packed + row * (n / 8), Wd.scales + row * ng, Wd.biases + row * ng, Wd.group, n,
                         shared ? hs + T * K * I - T * K * n : hs, shared ? hsum + T * K * (I / 32) - T * K * (n / 32)
                                                                     : hsum,
                         sl_, nt, acc, sl, lpt);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const float d = group_sum(acc[m], lpt);
                float t = (m < nt && sl < r) ? bd[m] * s_td[sl_[m]][sl] : 0.0f;
                if (m < nt && r > lpt) {  // ranks wider than the lane group (small rows)
                    const int slot = sl_[m];
                    const moe_lora_proj* ld = dlora(L, s_aid[shared ? m : slot / K], shared, 2);
                    for (int k = sl + lpt; k < r; k += lpt) t += ldb(ld, row * r + k) * s_td[slot][k];
                }
                t = group_sum(t, lpt);
                if (live && m < nt && sl == 0) s_v[ol][sl_[m]] = d + L.scale * t;
            }
        }
    }
    __syncthreads();
    for (int q = threadIdx.x; q < (o_hi - o_lo) * T; q += kThreads) {
        const int ol = q / T, t = q % T, o = o_lo + ol;
        float acc = 0.0f;
        for (int k = 0; k < K; ++k) acc += s_w[t][k] * s_v[ol][t * K + k];
        if (has_shared) acc += s_sg[t] * s_v[ol][T * K + t];
        if (a.block) acc += bf16f(a.x[(int64_t)t * H + o]);
        a.y[(int64_t)t * H + o] = f2bf16(acc);
    }
}

}  // namespace

// Conditions of the fused path (checked on the host before launch).
bool decode_supported(const LayerArgs& L, int T, size_t* smem_out) {
    if (T < 1 || T > kMaxT) return false;
    const int J = T * (L.K + 1);
    if (J > kMaxJ) return false;
    if (L.rank > kMaxR) return false;
    if (L.H > 4096 || L.I > 4096 || (L.has_shared && L.Is > 4096)) return false;  // 4 chunks per lane
    if (L.I % 32 || (L.has_shared && L.Is % 32)) return false;
    int nsm = 0, dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    if (nsm <= 0 || nsm > MOEQ_DECODE_MAX_CTAS) return false;
    if ((L.H + nsm - 1) / nsm > kMaxOut) return false;
    // a CTA's (expert, row) range must span at most two experts
    if ((T * L.K * L.I + nsm - 1) / nsm > L.I) return false;
    const int Imax = L.I > L.Is ? L.I : L.Is;
    const size_t part = (size_t)kW * 2 * kMaxT * kMaxR;
    const size_t zsz = (size_t)T * L.E;
    const size_t smem = sizeof(float) * ((size_t)T * L.H * 33 / 32 + (size_t)J * Imax * 33 / 32 +
                                         (part > zsz ? part : zsz));
    if (smem > 200 * 1024) return false;
    if (smem_out) *smem_out = smem;
    return true;
}

template <int MT>
cudaError_t launch_mt(const DArgs& a, size_t smem, cudaStream_t s) {
    static int cached = 0;
    cudaError_t e = ensure_smem((const void*)decode_kernel<MT>, smem, cached);
    if (e != cudaSuccess) return e;
    int nsm = 0, dev = 0, occ = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_kernel<MT>, kThreads, smem);
    if (e != cudaSuccess) return e;
    if (occ < 1) return cudaErrorCooperativeLaunchTooLarge;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(nsm);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_kernel<MT>, a);
}

cudaError_t launch_decode(const LayerArgs& L, const uint16_t* x, const int32_t* adapter_id, uint16_t* y, int T,
                          int block, float eps, const DecodeScratch& sc, cudaStream_t s) {
    size_t smem = 0;
    if (!decode_supported(L, T, &smem)) return cudaErrorNotSupported;
    DArgs a;
    a.L = L;
    a.x = x;
    a.adapter_id = adapter_id;
    a.y = y;
    a.T = T;
    a.block = block;
    a.eps = eps;
    a.logits = sc.logits;
    a.gsl = sc.gsl;
    a.ts = sc.ts;
    a.tg = sc.tg;
    a.gus = sc.gus;
    a.h = sc.h;
    a.tdp = sc.tdp;
    a.bar = sc.bar;
    a.status = sc.status;
    if (T <= 1) return launch_mt<1>(a, smem, s);
    if (T <= 2) return launch_mt<2>(a, smem, s);
    if (T <= 4) return launch_mt<4>(a, smem, s);
    return launch_mt<8>(a, smem, s);
}

}  // namespace moeq
