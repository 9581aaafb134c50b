// decode.cu - the whole MoE layer for a handful of tokens in one persistent,
// cooperative kernel (one CTA per SM).
//
// At decode the layer is a chain of small dependent steps (router -> top-K ->
// expert rows -> down rows), each far too small to fill the GPU; its time is
// set by the number of dependent memory round trips and grid-wide waits on the
// chain, not by bandwidth.  The kernel is laid out so that each step costs
// about one round trip:
//  - a CTA's share of a step's weight rows is a contiguous range of each
//    tensor, brought into shared memory by a few bulk copies (cp.async.bulk,
//    completing on an mbarrier) issued as soon as the range is known: the
//    router and shared-expert rows at launch, the routed gate/up and down rows
//    right after routing, so they land while the CTA does other work;
//  - the small LoRA pieces a CTA needs later (B rows, A_down columns) are
//    loaded by all of its threads at once right after routing;
//  - the routed LoRA-A products (A x per job and projection) come from
//    dedicated CTAs, which publish each with a per-launch epoch flag, so the
//    expert rows need no grid barrier before them, only a flag test that has
//    usually passed already;
//  - the down LoRA-A products (A_down h) are sums of per-CTA partials.
//
//  A  router + shared-gate rows, shared-expert gate/up rows (pre-activations
//     kept in shared memory), shared-expert LoRA-A products.
//  -- grid barrier --
//  B  every CTA: top-K of every token and the expert-grouped job list.
//  C  CTAs 0 .. 2TK-1: the routed LoRA-A products, one (job, gate|up) each;
//     the other CTAs: a contiguous range of routed (expert, row) pairs each.
//     Every CTA: its shared-expert rows.  LoRA-B delta, SwiGLU, partial down
//     LoRA-A sums.
//  -- grid barrier --
//  D  down rows: a CTA owns a range of output rows for every job, adds the
//     LoRA-B delta, and combines the jobs of each token in fixed order
//     (k = 0..K-1, then the shared expert), optionally adding the residual.
#include <algorithm>
#include <cstring>

#include "decode_dots.cuh"

namespace moeq {
namespace {

constexpr int kW = 16;  // warps per CTA
constexpr int kThreads = kW * 32;
static_assert(kThreads == kDecThreads, "one block size for the staging helpers");
constexpr int kMaxT = MOEQ_DECODE_MAX_TOKENS;
constexpr int kMaxJ = MOEQ_DECODE_MAX_JOBS;
constexpr int kMaxR = MOEQ_DECODE_MAX_RANK;  // LoRA rank handled by the fused path (one lane per k)
constexpr int kMaxOut = 32;                // output rows per CTA in phase D
constexpr int kMaxUD = kMaxJ + 1;          // phase-D experts: the routed ones and the shared one
constexpr int kFlagOffset = 16;            // byte offset of the LoRA-A ready flags in the workspace header
constexpr int kMaxFlags = (256 - kFlagOffset) / 4;

// Shared-memory plan of a launch: ranges per CTA and byte offsets into the dynamic
// segment, computed on the host from the shape and the largest possible number of
// distinct routed experts.
struct DPlan {
    int perA, per_s, perC, per_o;  // router rows, shared rows, routed (expert, row) pairs, output rows per CTA
    int nLA;                       // CTAs computing routed LoRA-A products (2 T K, or 0 without LoRA)
    int dalias;                    // the down windows reuse the gate/up region (issued after phase C)
    uint32_t xs, xsum;             // staged x
    uint32_t c, c_off[6];          // routed gate/up windows: {gate, up} x {packed, scales, biases}
    uint32_t d, d_off[3], d_stride;  // down windows of phase-D expert u at d + u * d_stride
    uint32_t ha, hsum;             // staged h (phase D); the phase-A windows share its space
    uint32_t a_off[14];            // phase-A windows: router, (shared gate: none), shared gate/up x {p, s, b},
                                   // two shared-expert LoRA-A rows
    uint32_t sgu, sbd, wpart, cand;
    uint32_t total;
};

struct DArgs {
    LayerArgs L;
    const uint16_t* x;
    const int32_t* adapter_id;
    uint16_t* y;
    int T, block;
    float eps;
    float* logits;     // [T][E]
    float* gsl;        // [T]
    float* ts;         // [T][2r]   shared-expert LoRA-A products (gate | up)
    float* tg;         // [T*K][2r] routed LoRA-A products, by routed slot t*K+k
    float* h;          // [J][Imax] SwiGLU outputs, slot t*K+k (routed), T*K+t (shared)
    float* tdp;        // [NB][3][T][r] partial down LoRA-A sums: routed segment 0, 1, shared
    uint32_t* flags;   // [2 T K] launch epoch once tg of (slot, gate|up) is written
    unsigned long long* bar;  // monotonic arrival counter
    int32_t* status;
    uint64_t wait_ns;  // bound of every wait
    int32_t* idx_out;  // [T][K] routing written by CTA 0 (the forward's routing record)
    float* w_out;      // [T][K]
    DPlan P;
};

__device__ __forceinline__ unsigned long long ld_acquire(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t ld_acquire32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release32(uint32_t* p, uint32_t v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Grid-wide barrier on a monotonic 64-bit arrival counter: barrier k of a launch
// is complete when the counter reaches base + (k + 1) * gridDim.x, where base (a
// multiple of gridDim.x) is learnt from this CTA's first arrival.  One release
// atomic per CTA, nothing to reset.  A CTA always arrives, so one that gave up
// earlier does not stall the others; the wait is bounded (MOE_ERR_TIMEOUT and
// *abort set), after which the counter is out of step and the workspace must be
// re-initialised.
__device__ void grid_sync(unsigned long long* bar, unsigned long long& target, int32_t* status,
                          volatile int* abort, uint64_t limit_ns) {
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned long long nb = gridDim.x;
        unsigned long long prev;
        asm volatile("atom.add.release.gpu.global.u64 %0, [%1], 1;" : "=l"(prev) : "l"(bar) : "memory");
        target = target == 0 ? (prev / nb + 1) * nb : target + nb;
        const uint64_t t0 = tc::globaltimer_ns();
        for (uint32_t i = 0; ld_acquire(bar) < target; ++i) {
            if ((i & 255) == 255) {
                if (tc::globaltimer_ns() - t0 > limit_ns) {
                    raise_status(status, MOE_ERR_TIMEOUT);
                    *abort = 1;
                    break;
                }
                __nanosleep(32);
            }
        }
    }
    __syncthreads();
}

// Top-K of the T tokens' logits (global memory, read from L2) by the whole CTA.  Warps
// take (token, 32-logit chunk) pairs, one logit per lane, and keep each chunk's K largest
// (K rounds of a warp max-reduction; equal logits go to the lower expert index, the lower
// lane); one warp per token then merges the chunks' candidates the same way.  The softmax
// over all E logits renormalised over the chosen K is w_k = exp(z_k - z_0) / sum_j
// exp(z_j - z_0) over the chosen K alone (z_0 the largest), which is what is computed.
// `cand` holds T * ceil(E / 32) * K (key, index) pairs; key 0 marks no candidate.
__device__ void cta_topk(const float* logits, int T, int E, int K, uint2* cand, int (*s_idx)[MOEQ_MAX_TOPK],
                         float (*s_w)[MOEQ_MAX_TOPK]) {
    constexpr uint32_t kNone = 0xffffffffu;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int nch = (E + 31) / 32;
    for (int p = warp; p < T * nch; p += kW) {
        const int t = p / nch, ch = p % nch, e = ch * 32 + lane;
        uint32_t key = e < E ? okey(__ldcg(logits + (int64_t)t * E + e)) : 0u;
        for (int k = 0; k < K; ++k) {
            const uint32_t mx = __reduce_max_sync(0xffffffffu, key);
            const int w = __ffs(__ballot_sync(0xffffffffu, key == mx)) - 1;
            if (lane == w) key = 0u;  // taken
            if (lane == 0) cand[(t * nch + ch) * K + k] = make_uint2(mx, mx ? (uint32_t)(ch * 32 + w) : kNone);
        }
    }
    __syncthreads();
    for (int t = warp; t < T; t += kW) {
        const int nc = nch * K;  // <= 256: at most 8 candidates per lane
        uint32_t ck[8], ci[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int c = lane + 32 * j;
            const uint2 v = c < nc ? cand[t * nc + c] : make_uint2(0u, kNone);
            ck[j] = v.x;
            ci[j] = v.y;
        }
        uint32_t myk = 0u, myi = kNone;
        for (int k = 0; k < K; ++k) {
            uint32_t bk = 0u, bi = kNone;
            int bj = -1;
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (ck[j] > bk || (ck[j] == bk && ci[j] < bi)) {
                    bk = ck[j];
                    bi = ci[j];
                    bj = j;
                }
            const uint32_t mk = __reduce_max_sync(0xffffffffu, bk);
            const uint32_t mi = __reduce_min_sync(0xffffffffu, bk == mk ? bi : kNone);
            if (bj >= 0 && bk == mk && bi == mi)
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    if (j == bj) {
                        ck[j] = 0u;
                        ci[j] = kNone;
                    }
            if (lane == k) {
                myk = mk;
                myi = mi;
            }
        }
        const float z = myk ? okey_value(myk) : -INFINITY;
        const float z0 = __shfl_sync(0xffffffffu, z, 0);
        const float ev = lane < K ? (z0 > -INFINITY ? expf(z - z0) : 1.0f) : 0.0f;
        const float sum = warp_sum(ev);
        if (lane < K) {
            s_idx[t][lane] = myi < (uint32_t)E ? (int)myi : 0;
            s_w[t][lane] = ev / sum;
        }
    }
}

// MT: token capacity of this instantiation (register arrays), T <= MT.
template <int MT>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ DArgs a) {
    extern __shared__ __align__(16) unsigned char dsm[];
    const LayerArgs& L = a.L;
    const DPlan& P = a.P;
    const int T = a.T, H = L.H, E = L.E, K = L.K, I = L.I, Is = L.Is;
    const int TK = T * K;
    const int NB = gridDim.x, cta = blockIdx.x;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const bool has_shared = L.has_shared;
    const bool lora = L.n_adapters > 0 && L.rank > 0;
    const int r = lora ? L.rank : 0;
    const int Jd = TK + (has_shared ? T : 0);  // job slots: routed t*K+k, then shared T*K+t
    const int Imax = I > Is ? I : Is;
    float* xs = reinterpret_cast<float*>(dsm + P.xs);              // [T][H] staged (swizzled) x
    float* xsum = reinterpret_cast<float*>(dsm + P.xsum);          // [T][H/32]
    float* hs = reinterpret_cast<float*>(dsm + P.ha);              // [TK][I] then [T][Is] staged h
    float* hsum = reinterpret_cast<float*>(dsm + P.hsum);
    float* sgu = reinterpret_cast<float*>(dsm + P.sgu);            // [per_s][T][2] shared gate/up pre-activations
    uint16_t* sbd = reinterpret_cast<uint16_t*>(dsm + P.sbd);      // [no][Jd][r] down LoRA-B rows
    float* wpart = reinterpret_cast<float*>(dsm + P.wpart);        // [kW][3][T][r] per-warp A_down h partials

    __shared__ __align__(8) uint64_t s_bar[3];  // bulk copies of phases A, C, D
    __shared__ int s_abort;
    __shared__ int s_issued[3];
    __shared__ uint32_t s_epoch;
    __shared__ int s_aid[kMaxT], s_tok[kMaxT];
    __shared__ float s_inv[kMaxT];
    __shared__ int s_idx[kMaxT][MOEQ_MAX_TOPK];
    __shared__ float s_w[kMaxT][MOEQ_MAX_TOPK];
    __shared__ float s_sg[kMaxT];
    __shared__ int s_nu;
    __shared__ int s_uexp[kMaxJ], s_ucnt[kMaxJ], s_uslot[kMaxJ][kMaxT];
    __shared__ int s_sorted[kMaxJ], s_ju[kMaxJ], s_jm[kMaxJ];
    __shared__ float s_td[kMaxJ][kMaxR];
    __shared__ float s_v[kMaxOut][kMaxJ];
    __shared__ const unsigned char* s_aw[14];
    __shared__ const unsigned char* s_cw[2][6];
    __shared__ const unsigned char* s_dw[kMaxUD][3];

    if (tid == 0) {
        s_abort = 0;
        for (int i = 0; i < 3; ++i) {
            tc::mbar_init(&s_bar[i], 1);
            s_issued[i] = 0;
        }
        tc::mbar_init_fence();
    }
    if (tid < T) {
        int ad = a.adapter_id ? a.adapter_id[tid] : (L.n_adapters > 0 ? 0 : -1);
        if (ad < -1 || ad >= L.n_adapters) {
            if (cta == 0) raise_status(a.status, MOE_ERR_DEVICE_INDEX);
            ad = -1;
        }
        s_aid[tid] = ad;
        s_tok[tid] = tid;
    }
    __syncthreads();

    // ------------------------------------------------------------ phase A
    const int R = E + (L.has_sgate ? 1 : 0);
    const int ra0 = min(R, cta * P.perA), ra1 = min(R, ra0 + P.perA), re1 = min(ra1, E);
    const int s_lo = has_shared ? min(Is, cta * P.per_s) : 0, s_hi = has_shared ? min(Is, s_lo + P.per_s) : 0;
    const int nra = ra1 - ra0, nsr = s_hi - s_lo;
    const int nlt = (has_shared && lora) ? T * 2 * r : 0;  // shared-expert LoRA-A dots over the grid
    const int nla = nlt > cta ? (nlt - cta + NB - 1) / NB : 0;
    if (warp == 0) {  // this CTA's router and shared-expert rows start moving now, one window per lane
        uint32_t tx = 0;
        unsigned char* ab = dsm + P.ha;
        if (lane >= 12 && lane < 14) {  // the A rows of this CTA's first two shared LoRA-A dots
            s_aw[lane] = nullptr;
            const int q = cta + NB * (lane - 12), t = q / (2 * (r > 0 ? r : 1)), d = r > 0 ? q % (2 * r) : 0;
            const moe_lora_proj* lp = lane - 12 < nla ? dlora(L, s_aid[t], true, d < r ? 0 : 1) : nullptr;
            if (lp) s_aw[lane] = win_load(ab + P.a_off[lane], lp->A + (int64_t)(d % r) * H, (uint32_t)H * 2, &s_bar[0], &tx);
        }
        if (lane < 12) {
            s_aw[lane] = nullptr;
            const int k = lane % 3;
            if (lane < 3 && re1 > ra0) {
                const moe_qtensor& q = L.router;
                const int ng = H / q.group, n = re1 - ra0;
                const void* src = k == 0 ? (const void*)(q.packed + (int64_t)ra0 * (H / 4))
                                         : (const void*)((k == 1 ? q.scales : q.biases) + (int64_t)ra0 * ng);
                s_aw[lane] = win_load(ab + P.a_off[lane], src, k == 0 ? (uint32_t)n * H : (uint32_t)n * ng * 2,
                                      &s_bar[0], &tx);
            } else if (lane >= 3 && lane < 6 && ra1 > E) {  // the shared-expert gate row: read from global memory
                s_aw[lane] = k == 0 ? reinterpret_cast<const unsigned char*>(L.shared_gate.packed)
                                    : reinterpret_cast<const unsigned char*>(k == 1 ? L.shared_gate.scales
                                                                                    : L.shared_gate.biases);
            } else if (lane >= 6 && nsr > 0) {
                const moe_qtensor& q = lane >= 9 ? L.s_up : L.s_gate;
                const int ng = H / q.group;
                const void* src = k == 0 ? (const void*)(q.packed + (int64_t)s_lo * (H / 8))
                                         : (const void*)((k == 1 ? q.scales : q.biases) + (int64_t)s_lo * ng);
                s_aw[lane] = win_load(ab + P.a_off[lane], src, k == 0 ? (uint32_t)nsr * (H / 2) : (uint32_t)nsr * ng * 2,
                                      &s_bar[0], &tx);
            }
        }
        for (int o = 16; o > 0; o >>= 1) tx += __shfl_xor_sync(0xffffffffu, tx, o);
        if (lane == 0) {
            tc::mbar_arrive_expect_tx(&s_bar[0], tx);
            s_issued[0] = 1;
        }
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
    }
    stage_bf16(xs, xsum, a.x, T, H, a.block ? s_inv : nullptr);
    __syncthreads();

    // one warp per task: router / shared-gate rows, shared-expert rows, shared-expert LoRA-A dots
    {
        bool landed = false;
        for (int j = warp; j < nra + nsr + nla; j += kW) {
            if (j < nra + nsr + 2 && !landed) {
                if (!copies_landed(&s_bar[0], a.status, &s_abort, a.wait_ns)) break;
                landed = true;
            }
            if (j < nra) {
                const int row = ra0 + j;
                const bool sgrow = row >= E;
                const moe_qtensor& q = sgrow ? L.shared_gate : L.router;
                const int ng = H / q.group, jj = sgrow ? 0 : j;
                const unsigned char* const* w = s_aw + (sgrow ? 3 : 0);
                float acc[MT];
#pragma unroll
                for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
                dot_int8<MT>(reinterpret_cast<const uint32_t*>(w[0] + (size_t)jj * H),
                             reinterpret_cast<const uint16_t*>(w[1]) + jj * ng,
                             reinterpret_cast<const uint16_t*>(w[2]) + jj * ng, q.group, H, xs, xsum, T, acc, lane);
#pragma unroll
                for (int m = 0; m < MT; ++m) acc[m] = warp_sum(acc[m]);
                if (lane < T) {
                    float v = 0.0f;
#pragma unroll
                    for (int m = 0; m < MT; ++m)
                        if (m == lane) v = acc[m];
                    if (!sgrow) a.logits[(int64_t)lane * E + row] = v + (L.logit_bias ? L.logit_bias[row] : 0.0f);
                    else a.gsl[lane] = v;
                }
            } else if (j < nra + nsr) {
                const int il = j - nra;
                const int ngg = H / L.s_gate.group, ngu = H / L.s_up.group;
                float ag[MT], au[MT];
#pragma unroll
                for (int m = 0; m < MT; ++m) ag[m] = au[m] = 0.0f;
                dot_int4<MT>(reinterpret_cast<const uint32_t*>(s_aw[6] + (size_t)il * (H / 2)),
                             reinterpret_cast<const uint16_t*>(s_aw[7]) + il * ngg,
                             reinterpret_cast<const uint16_t*>(s_aw[8]) + il * ngg, L.s_gate.group, H, xs, xsum, s_tok,
                             T, ag, lane, 32);
                dot_int4<MT>(reinterpret_cast<const uint32_t*>(s_aw[9] + (size_t)il * (H / 2)),
                             reinterpret_cast<const uint16_t*>(s_aw[10]) + il * ngu,
                             reinterpret_cast<const uint16_t*>(s_aw[11]) + il * ngu, L.s_up.group, H, xs, xsum, s_tok,
                             T, au, lane, 32);
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m >= T) break;
                    const float g = warp_sum(ag[m]), u = warp_sum(au[m]);
                    if (lane == 0) {
                        sgu[(il * T + m) * 2] = g;
                        sgu[(il * T + m) * 2 + 1] = u;
                    }
                }
            } else {  // shared-expert LoRA-A dot (token t, output d of gate | up)
                const int q = cta + NB * (j - nra - nsr), t = q / (2 * r), d = q % (2 * r);
                const moe_lora_proj* lp = dlora(L, s_aid[t], true, d < r ? 0 : 1);
                const int jw = j - nra - nsr;
                const uint16_t* arow = jw < 2 && s_aw[12 + jw] ? reinterpret_cast<const uint16_t*>(s_aw[12 + jw])
                                                               : (lp ? lp->A + (int64_t)(d % r) * H : nullptr);
                float v = 0.0f;
                if (lp) v = warp_sum(dot_bf16(arow, H, xs + t * H, lane));
                if (lane == 0) a.ts[t * 2 * r + d] = v;
            }
        }
    }
    unsigned long long bar_target = 0;
    grid_sync(a.bar, bar_target, a.status, &s_abort, a.wait_ns);

    // ------------------------------------------------------------ phase B
    if (tid == 0) s_epoch = (uint32_t)(bar_target / (unsigned long long)NB);
    if (tid < T) s_sg[tid] = L.has_sgate ? 1.0f / (1.0f + expf(-__ldcg(a.gsl + tid))) : 1.0f;
    cta_topk(a.logits, T, E, K, reinterpret_cast<uint2*>(dsm + P.cand), s_idx, s_w);
    __syncthreads();
    if (cta == 0 && tid < TK) {  // the routing this call used, for the caller's record
        a.idx_out[tid] = s_idx[tid / K][tid % K];
        a.w_out[tid] = s_w[tid / K][tid % K];
    }
    if (warp == 0) {
        // routed jobs (lane = slot t*K+k) sorted by (expert, adapter, slot): the rank of a
        // lane's key among all keys is its position; experts ascending, each expert's jobs
        // by (adapter, token)
        const bool live = lane < TK;
        int je = 0x7fffffff, jar = 0;
        if (live) {
            const int t = lane / K;
            je = s_idx[t][lane % K];
            jar = s_aid[t] < 0 ? L.n_adapters : s_aid[t];
        }
        int rank = 0;
        for (int j = 0; j < TK; ++j) {
            const int ej = __shfl_sync(0xffffffffu, je, j), aj = __shfl_sync(0xffffffffu, jar, j);
            rank += (ej < je || (ej == je && (aj < jar || (aj == jar && j < lane)))) ? 1 : 0;
        }
        if (live) s_sorted[rank] = lane;
        __syncwarp();
        const int jp = live ? s_sorted[lane] : 0;
        const int ep = live ? s_idx[jp / K][jp % K] : -1;
        const int eprev = __shfl_up_sync(0xffffffffu, ep, 1);
        const bool first = live && (lane == 0 || eprev != ep);
        const uint32_t fm = __ballot_sync(0xffffffffu, first);
        if (live) {
            const uint32_t upto = fm & (0xffffffffu >> (31 - lane));  // expert starts at positions <= lane
            const int u = __popc(upto) - 1, start = 31 - __clz(upto);
            s_uslot[u][lane - start] = jp;
            s_ju[jp] = u;
            s_jm[jp] = lane - start;
            if (first) {
                const uint32_t after = fm & ~(0xffffffffu >> (31 - lane));
                s_uexp[u] = ep;
                s_ucnt[u] = (after ? __ffs(after) - 1 : TK) - start;
            }
        }
        if (lane == 0) s_nu = __popc(fm);
    }
    __syncthreads();

    // ------------------------------------------------------------ phase C
    const bool runC = s_abort == 0;
    const uint32_t epoch = s_epoch;
    const int U = s_nu, UD = U + (has_shared ? 1 : 0);
    const int nC = U * I;
    const int rc = cta - P.nLA;  // index among the CTAs that own routed rows
    const int c_lo = rc >= 0 ? min(nC, rc * P.perC) : 0, c_hi = rc >= 0 ? min(nC, c_lo + P.perC) : 0;
    const int nrows = c_hi - c_lo;
    const int u0 = nrows > 0 ? c_lo / I : 0;
    const int cut = nrows > 0 ? min(c_hi, (u0 + 1) * I) : 0;  // first pair of the second expert
    const int o_lo = min(H, cta * P.per_o), o_hi = min(H, o_lo + P.per_o), no = o_hi - o_lo;

    if (warp == 0) {  // the routed gate/up rows of this CTA's range: lane 6 s + 3 p + k issues one window
        uint32_t tx = 0;
        if (lane < 12) {
            const int sgi = lane / 6, pj = (lane / 3) % 2, k = lane % 3, part = 3 * pj + k;
            s_cw[sgi][part] = nullptr;
            const int q0 = sgi == 0 ? c_lo : cut, q1 = sgi == 0 ? cut : c_hi;
            if (nrows > 0 && runC && q1 > q0) {
                const int e = s_uexp[q0 / I], n = q1 - q0;
                const int64_t row = (int64_t)e * I + q0 % I;
                const moe_qtensor& q = pj ? L.up : L.gate;
                const int ng = H / q.group;
                const void* src = k == 0 ? (const void*)(q.packed + row * (H / 8))
                                         : (const void*)((k == 1 ? q.scales : q.biases) + row * ng);
                const uint32_t bytes = k == 0 ? (uint32_t)n * (H / 2) : (uint32_t)n * ng * 2;
                // segment 1's window follows segment 0's in the part's region
                uint32_t off = P.c + P.c_off[part];
                if (sgi == 1 && cut > c_lo) {
                    const int e0 = s_uexp[c_lo / I], n0 = cut - c_lo;
                    const int64_t row0 = (int64_t)e0 * I + c_lo % I;
                    const void* src0 = k == 0 ? (const void*)(q.packed + row0 * (H / 8))
                                              : (const void*)((k == 1 ? q.scales : q.biases) + row0 * ng);
                    off += win_span(src0, k == 0 ? (uint32_t)n0 * (H / 2) : (uint32_t)n0 * ng * 2);
                }
                s_cw[sgi][part] = win_load(dsm + off, src, bytes, &s_bar[1], &tx);
            }
        }
        for (int o = 16; o > 0; o >>= 1) tx += __shfl_xor_sync(0xffffffffu, tx, o);
        if (lane == 0) {
            tc::mbar_arrive_expect_tx(&s_bar[1], tx);
            s_issued[1] = 1;
        }
    }
    // the down rows of this CTA's output range, one lane per phase-D expert
    auto issue_down = [&]() {
        uint32_t tx = 0;
        if (no > 0 && runC)
            for (int u = lane; u < UD; u += 32) {
                const bool sh = u == U;
                const moe_qtensor& q = sh ? L.s_down : L.down;
                const int n = sh ? Is : I, ng = n / q.group;
                const int64_t row = sh ? (int64_t)o_lo : (int64_t)s_uexp[u] * H + o_lo;
                unsigned char* base = dsm + P.d + (uint32_t)u * P.d_stride;
                s_dw[u][0] = win_load(base + P.d_off[0], q.packed + row * (n / 8), (uint32_t)no * (n / 2), &s_bar[2], &tx);
                s_dw[u][1] = win_load(base + P.d_off[1], q.scales + row * ng, (uint32_t)no * ng * 2, &s_bar[2], &tx);
                s_dw[u][2] = win_load(base + P.d_off[2], q.biases + row * ng, (uint32_t)no * ng * 2, &s_bar[2], &tx);
            }
        for (int o = 16; o > 0; o >>= 1) tx += __shfl_xor_sync(0xffffffffu, tx, o);
        if (lane == 0) {
            tc::mbar_arrive_expect_tx(&s_bar[2], tx);
            s_issued[2] = 1;
        }
    };
    const bool la_cta = lora && cta < P.nLA;
    if (!P.dalias && !la_cta && warp == 1) issue_down();

    // routed LoRA-A products: CTA 2j + p computes A_p x_t of routed slot j (p = gate | up)
    if (lora && cta < P.nLA) {
        const int j = cta / 2, pj = cta % 2, t = j / K, e = s_idx[t][j % K];
        const moe_lora_proj* lp = runC ? dlora(L, s_aid[t], false, pj) : nullptr;
        for (int d = warp; d < r; d += kW) {
            float v = 0.0f;
            if (lp) v = warp_sum(dot_bf16(lp->A + ((int64_t)e * r + d) * H, H, xs + t * H, lane));
            if (lane == 0) a.tg[(int64_t)j * 2 * r + pj * r + d] = v;
        }
        __syncthreads();
        if (tid == 0) {
            __threadfence();
            st_release32(a.flags + cta, epoch);
        }
        if (!P.dalias && warp == kW - 1) issue_down();
    }

    // the down LoRA-B rows of this CTA's output range [ol][slot][k]: 16-byte cp.async pieces,
    // waited for in phase D
    if (lora && runC) {
        const int pp = r / 8, n = no * Jd * pp;
        for (int i = tid; i < n; i += kThreads) {
            const int piece = i % pp, pair = i / pp, slot = pair % Jd, ol = pair / Jd;
            const bool sh = slot >= TK;
            const int t = sh ? slot - TK : slot / K;
            const moe_lora_proj* lp = dlora(L, s_aid[t], sh, 2);
            const void* src = a.tg;  // any valid address when the piece is zero-filled
            if (lp) {
                const int64_t row = sh ? (int64_t)(o_lo + ol) : (int64_t)s_idx[t][slot % K] * H + o_lo + ol;
                src = lp->B + row * r + piece * 8;
            }
            tc::cp16(tc::smem_u32(sbd + (size_t)pair * r + piece * 8), src, lp ? 16u : 0u);
        }
        tc::cp_commit();
    }

    // one warp per row: the shared-expert rows (gate/up pre-activations from phase A), then
    // this CTA's routed rows.  Each issues its LoRA loads (lane k < r: component k) before it
    // waits for anything, adds the LoRA-B delta, applies SwiGLU, writes h and accumulates
    // its part of A_down h.
    float wacc[3][MT];  // segment 0, 1 (routed), shared
#pragma unroll
    for (int s2 = 0; s2 < 3; ++s2)
#pragma unroll
        for (int m = 0; m < MT; ++m) wacc[s2][m] = 0.0f;
    const bool kk = lane < r;
    if (runC) {
        bool landed = false;
        for (int j = warp; j < nsr + nrows; j += kW) {
            float bg[MT], bu[MT], ad[MT], tgv[MT], tuv[MT];
            if (j < nsr) {
                const int i = s_lo + j;
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    bg[m] = bu[m] = ad[m] = tgv[m] = tuv[m] = 0.0f;
                    if (m >= T || !lora) continue;
                    const moe_lora_proj* lg = dlora(L, s_aid[m], true, 0);
                    const moe_lora_proj* lu = dlora(L, s_aid[m], true, 1);
                    const moe_lora_proj* ld = dlora(L, s_aid[m], true, 2);
                    if (kk && lg) {
                        bg[m] = bf16f(lg->B[(int64_t)i * r + lane]);
                        tgv[m] = __ldcg(a.ts + m * 2 * r + lane);
                    }
                    if (kk && lu) {
                        bu[m] = bf16f(lu->B[(int64_t)i * r + lane]);
                        tuv[m] = __ldcg(a.ts + m * 2 * r + r + lane);
                    }
                    if (kk && ld) ad[m] = bf16f(ld->A[(int64_t)lane * Is + i]);
                }
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m >= T) break;
                    float g = sgu[(j * T + m) * 2], u = sgu[(j * T + m) * 2 + 1];
                    if (lora) {
                        g += L.scale * warp_sum(bg[m] * tgv[m]);
                        u += L.scale * warp_sum(bu[m] * tuv[m]);
                    }
                    const float hv = silu(g) * u;
                    if (lane == 0) a.h[(int64_t)(TK + m) * Imax + i] = hv;
                    wacc[2][m] += ad[m] * hv;
                }
                continue;
            }
            const int il = j - nsr, q = c_lo + il, u = q / I, i = q % I, sg = q < cut ? 0 : 1;
            const int rs = q - (sg == 0 ? c_lo : cut), e = s_uexp[u], nt = s_ucnt[u];
            int toks[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                bg[m] = bu[m] = ad[m] = tgv[m] = tuv[m] = 0.0f;
                toks[m] = m < nt ? s_uslot[u][m] / K : 0;
                if (m >= nt || !lora) continue;
                const int a_m = s_aid[toks[m]];
                const moe_lora_proj* lg = dlora(L, a_m, false, 0);
                const moe_lora_proj* lu = dlora(L, a_m, false, 1);
                const moe_lora_proj* ld = dlora(L, a_m, false, 2);
                if (kk && lg) bg[m] = bf16f(lg->B[((int64_t)e * I + i) * r + lane]);
                if (kk && lu) bu[m] = bf16f(lu->B[((int64_t)e * I + i) * r + lane]);
                if (kk && ld) ad[m] = bf16f(ld->A[((int64_t)e * r + lane) * I + i]);
            }
            if (!landed) {
                if (!copies_landed(&s_bar[1], a.status, &s_abort, a.wait_ns)) break;
                landed = true;
            }
            float ag[MT], au[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) ag[m] = au[m] = 0.0f;
            const int ngg = H / L.gate.group, ngu = H / L.up.group;
            dot_int4<MT>(reinterpret_cast<const uint32_t*>(s_cw[sg][0] + (size_t)rs * (H / 2)),
                         reinterpret_cast<const uint16_t*>(s_cw[sg][1]) + rs * ngg,
                         reinterpret_cast<const uint16_t*>(s_cw[sg][2]) + rs * ngg, L.gate.group, H, xs, xsum, toks, nt,
                         ag, lane, 32);
            dot_int4<MT>(reinterpret_cast<const uint32_t*>(s_cw[sg][3] + (size_t)rs * (H / 2)),
                         reinterpret_cast<const uint16_t*>(s_cw[sg][4]) + rs * ngu,
                         reinterpret_cast<const uint16_t*>(s_cw[sg][5]) + rs * ngu, L.up.group, H, xs, xsum, toks, nt,
                         au, lane, 32);
            if (lora) {  // this row's LoRA-A products (after the dots, which cover their latency):
                         // lane 2m + p polls the flag of (job m, gate|up)
                bool ready = true;
                if (lane < 2 * nt) {
                    const int slot = s_uslot[u][lane >> 1];
                    if (dlora(L, s_aid[slot / K], false, lane & 1)) {
                        const uint32_t* fp = a.flags + slot * 2 + (lane & 1);
                        const uint64_t t0 = tc::globaltimer_ns();
                        for (uint32_t it = 0; ld_acquire32(fp) != epoch; ++it)
                            if ((it & 63) == 63 && tc::globaltimer_ns() - t0 > a.wait_ns) {
                                raise_status(a.status, MOE_ERR_TIMEOUT);
                                s_abort = 1;
                                ready = false;
                                break;
                            }
                    }
                }
                ready = __all_sync(0xffffffffu, ready);  // also orders the warp's reads after the flags
                if (ready && kk)
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        if (m >= nt) break;
                        const int slot = s_uslot[u][m];
                        tgv[m] = __ldcg(a.tg + (int64_t)slot * 2 * r + lane);
                        tuv[m] = __ldcg(a.tg + (int64_t)slot * 2 * r + r + lane);
                    }
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m >= nt) break;
                float g = warp_sum(ag[m]), uu = warp_sum(au[m]);
                if (lora) {
                    g += L.scale * warp_sum(bg[m] * tgv[m]);
                    uu += L.scale * warp_sum(bu[m] * tuv[m]);
                }
                const float hv = silu(g) * uu;
                if (lane == 0) a.h[(int64_t)s_uslot[u][m] * Imax + i] = hv;
                if (sg == 0) wacc[0][m] += ad[m] * hv;
                else wacc[1][m] += ad[m] * hv;
            }
        }
    }
    __syncthreads();
    if (lora) {  // per-warp partials, then a fixed-order sum over the warps
        if (lane < r)
#pragma unroll
            for (int s = 0; s < 3; ++s)
#pragma unroll
                for (int m = 0; m < MT; ++m)
                    if (m < T) wpart[((warp * 3 + s) * T + m) * r + lane] = wacc[s][m];
        __syncthreads();
        for (int q = tid; q < 3 * T * r; q += kThreads) {
            float v = 0.0f;
            for (int w = 0; w < kW; ++w) v += wpart[w * 3 * T * r + q];
            const int k = q % r, m = (q / r) % T, s = q / (r * T);
            a.tdp[(((int64_t)cta * 3 + s) * T + m) * r + k] = v;
        }
    } else {
        __syncthreads();
    }
    if (P.dalias && warp == 0) issue_down();  // the gate/up windows are no longer read
    grid_sync(a.bar, bar_target, a.status, &s_abort, a.wait_ns);

    // ------------------------------------------------------------ phase D
    const bool runD = s_abort == 0;
    float* tdc = wpart;  // [TK*r][8] routed then [T*r][32] shared chunk sums
    if (runD) {
        // three warp groups at once: the routed h rows (length I), the shared ones (Is), and the
        // down LoRA-A products summed from the per-CTA partials (chunks of the grid, every
        // load of a thread in flight together)
        if (warp < 6) {
            stage_f32(hs, hsum, a.h, Imax, TK, I, 0, 6 * 32);
        } else if (warp < 8) {
            if (has_shared)
                stage_f32(hs + TK * I, hsum + TK * (I / 32), a.h + (int64_t)TK * Imax, Imax, T, Is, 6 * 32, 2 * 32);
        } else if (lora) {
            const int nrp = TK * r, nsp = has_shared ? T * r : 0, nit = nrp * 8 + nsp * 32;
            const int t8 = tid - 8 * 32;
            constexpr int kG = kThreads - 8 * 32;
            // item q: chunk c of the sum of one p = (slot, k): routed q = c nrp + p < 8 nrp (8
            // chunks over the CTAs covering the slot's expert), shared q = 8 nrp + c nsp + p
            // (32 chunks over the grid); consecutive lanes take consecutive k, so a warp's
            // loads are contiguous.  The item's partials sit at base + j * step, j < cnt (plus
            // `extra` for j = 0: the first CTA covering an expert may hold it as its second).
            auto item = [&](int q, const float*& base, int& step, int& cnt, int& extra) {
                base = a.tdp;
                step = 0;
                cnt = 0;
                extra = 0;
                if (q < nrp * 8) {
                    const int p = q % nrp, slot = p / r, k = p % r, u = s_ju[slot];
                    const int rc0 = (u * I) / P.perC, rc1 = ((u + 1) * I - 1) / P.perC, x0 = rc0 + q / nrp;
                    if (x0 > rc1) return;
                    cnt = (rc1 - x0) / 8 + 1;
                    step = 8 * 3 * T * r;
                    base = a.tdp + ((int64_t)(P.nLA + x0) * 3 * T + s_jm[slot]) * r + k;
                    if (x0 == rc0 && rc0 * P.perC < u * I) extra = T * r;
                } else if (q < nit) {
                    const int q2 = q - nrp * 8, p = q2 % nsp, t = p / r, k = p % r, c0 = q2 / nsp;
                    if (c0 >= NB) return;
                    cnt = (NB - 1 - c0) / 32 + 1;
                    step = 32 * 3 * T * r;
                    base = a.tdp + (((int64_t)c0 * 3 + 2) * T + t) * r + k;
                }
            };
            for (int i0 = t8; i0 < nit; i0 += 4 * kG) {
                const float* base[4];
                int step[4], cnt[4], extra[4];
#pragma unroll
                for (int b = 0; b < 4; ++b) item(i0 + b * kG, base[b], step[b], cnt[b], extra[b]);
                float w[4][8];
#pragma unroll
                for (int b = 0; b < 4; ++b)
#pragma unroll
                    for (int jx = 0; jx < 8; ++jx)
                        w[b][jx] = jx < cnt[b] ? __ldcg(base[b] + (int64_t)jx * step[b] + (jx == 0 ? extra[b] : 0)) : 0.0f;
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const int q = i0 + b * kG;
                    if (q >= nit) break;
                    float acc = 0.0f;
#pragma unroll
                    for (int jx = 0; jx < 8; ++jx) acc += w[b][jx];
                    for (int jx = 8; jx < cnt[b]; ++jx) acc += __ldcg(base[b] + (int64_t)jx * step[b]);  // > 64 CTAs
                    tdc[q] = acc;
                }
            }
        }
    }
    tc::cp_wait<0>();  // this thread's down LoRA-B pieces
    __syncthreads();
    if (runD && lora) {
        const int nrp = TK * r;
        for (int q = tid; q < Jd * r; q += kThreads) {
            const int slot = q / r, k = q % r;
            float v = 0.0f;
            if (slot < TK)
                for (int c = 0; c < 8; ++c) v += tdc[c * nrp + q];
            else
                for (int c = 0; c < 32; ++c) v += tdc[nrp * 8 + c * (Jd * r - nrp) + (q - nrp)];
            s_td[slot][k] = v;
        }
    }
    __syncthreads();
    // (output row, expert) tasks from the down windows; a task is a group of lpt lanes over one row
    if (runD && no > 0 && copies_landed(&s_bar[2], a.status, &s_abort, a.wait_ns)) {
        int lpt = 1;
        while (lpt * 2 <= 32 && lpt * 2 <= Imax / 32) lpt *= 2;
        const int gpw = 32 / lpt, sub = lane / lpt, sl = lane % lpt;
        const int ntask = no * UD;
        for (int q0 = warp * gpw; q0 < ntask; q0 += kW * gpw) {
            const int q = q0 + sub;
            const bool live = q < ntask;
            const int ol = live ? q / UD : 0, u = live ? q % UD : 0;
            const bool sh = u == U;
            const int n = sh ? Is : I;
            const moe_qtensor& Wd = sh ? L.s_down : L.down;
            const int ng = n / Wd.group;
            const int nt = live ? (sh ? T : s_ucnt[u]) : 0;
            int sl_[MT];
            float bd[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                sl_[m] = 0;
                bd[m] = 0.0f;
                if (m >= nt) continue;
                sl_[m] = sh ? TK + m : s_uslot[u][m];
                if (lora && sl < r) bd[m] = bf16f(sbd[(ol * Jd + sl_[m]) * r + sl]);
            }
            float acc[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
            if (live)
                dot_int4<MT>(reinterpret_cast<const uint32_t*>(s_dw[u][0] + (size_t)ol * (n / 2)),
                             reinterpret_cast<const uint16_t*>(s_dw[u][1]) + ol * ng,
                             reinterpret_cast<const uint16_t*>(s_dw[u][2]) + ol * ng, Wd.group, n,
                             sh ? hs + TK * I - TK * n : hs, sh ? hsum + TK * (I / 32) - TK * (n / 32) : hsum, sl_, nt,
                             acc, sl, lpt);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const float d = group_sum(acc[m], lpt);
                float t = (lora && m < nt && sl < r) ? bd[m] * s_td[sl_[m]][sl] : 0.0f;
                if (lora && m < nt && r > lpt)  // ranks wider than the lane group
                    for (int k = sl + lpt; k < r; k += lpt) t += bf16f(sbd[(ol * Jd + sl_[m]) * r + k]) * s_td[sl_[m]][k];
                t = group_sum(t, lpt);
                if (live && m < nt && sl == 0) s_v[ol][sl_[m]] = d + L.scale * t;
            }
        }
    }
    __syncthreads();
    if (runD && s_abort == 0)
        for (int q = tid; q < no * T; q += kThreads) {
            const int ol = q / T, t = q % T, o = o_lo + ol;
            float acc = 0.0f;
            for (int k = 0; k < K; ++k) acc += s_w[t][k] * s_v[ol][t * K + k];
            if (has_shared) acc += s_sg[t] * s_v[ol][TK + t];
            if (a.block) acc += bf16f(a.x[(int64_t)t * H + o]);
            a.y[(int64_t)t * H + o] = f2bf16(acc);
        }
    // a CTA that gave up leaves no bulk copy in flight (bounded wait)
    if (tid == 0 && s_abort)
        for (int i = 0; i < 3; ++i)
            if (s_issued[i]) tc::mbar_wait(&s_bar[i], 0, nullptr, a.wait_ns);
}

}  // namespace

namespace {

inline size_t r16(size_t v) { return (v + 15) / 16 * 16; }
inline int cdiv(int a, int b) { return (a + b - 1) / b; }

// Every bulk-copied tensor: 16-byte aligned base and a size that is a multiple of 16
// bytes, so that a window rounded out to 16-byte boundaries stays inside the tensor.
bool windows_ok(const moe_qtensor& q) {
    if (!q.packed) return true;
    const size_t rows = (size_t)q.n * q.out;
    const size_t pb = rows * (size_t)q.in * q.bits / 8, sb = rows * (size_t)(q.in / q.group) * 2;
    return ((uintptr_t)q.packed & 15) == 0 && ((uintptr_t)q.scales & 15) == 0 && ((uintptr_t)q.biases & 15) == 0 &&
           pb % 16 == 0 && sb % 16 == 0 && q.group % 32 == 0;
}

int sm_count() {
    static int n = -1;
    if (n < 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = 0;
    }
    return n;
}

int optin_smem() {
    static int v = -1;
    if (v < 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) v = 0;
    }
    return v;
}

template <int MT>
size_t static_smem() {
    static size_t v = (size_t)-1;
    if (v == (size_t)-1) {
        cudaFuncAttributes at;
        v = cudaFuncGetAttributes(&at, decode_kernel<MT>) == cudaSuccess ? at.sharedSizeBytes : (size_t)1 << 30;
    }
    return v;
}

size_t static_smem_for(int T) {
    return T <= 1 ? static_smem<1>() : T <= 2 ? static_smem<2>() : T <= 4 ? static_smem<4>() : static_smem<8>();
}

// Ranges and the shared-memory layout of a launch on NB CTAs; false when the shape is
// outside the fused path (the caller then runs the multi-kernel path).
bool plan_decode(const LayerArgs& L, int T, int NB, DPlan* P) {
    const bool sh = L.has_shared, lora = L.n_adapters > 0 && L.rank > 0;
    const int H = L.H, E = L.E, K = L.K, I = L.I, Is = sh ? L.Is : 0, r = lora ? L.rank : 0;
    const int TK = T * K, J = TK + (sh ? T : 0);
    if (T < 1 || T > kMaxT || T * (K + 1) > kMaxJ || r > kMaxR || NB < 1 || NB > MOEQ_DECODE_MAX_CTAS) return false;
    if (H % 32 || I % 32 || H > 4096 || I > 4096 || (sh && (Is % 32 || Is > 4096 || Is < 1))) return false;
    if (!windows_ok(L.router) || !windows_ok(L.gate) || !windows_ok(L.up) || !windows_ok(L.down)) return false;
    if (sh && (!windows_ok(L.s_gate) || !windows_ok(L.s_up) || !windows_ok(L.s_down))) return false;
    if (L.router.group % 32 || L.router.bits != 8 || L.gate.bits != 4 || L.up.bits != 4 || L.down.bits != 4) return false;
    const int Umax = std::min(E, TK), Imax = std::max(I, Is);
    P->nLA = lora ? 2 * TK : 0;
    if (P->nLA > kMaxFlags || P->nLA >= NB) return false;
    if (lora) {  // the down LoRA-B rows move in 16-byte pieces
        if (r % 8) return false;
        for (int ad = 0; ad < L.n_adapters; ++ad) {
            const moe_lora_proj* d[2] = {&L.lora[ad].down, &L.lora[ad].s_down};
            for (int k = 0; k < 2; ++k)
                if (d[k]->B && ((uintptr_t)d[k]->B & 15)) return false;
            // the shared-expert LoRA-A rows move as bulk-copy windows
            const moe_lora_proj* sa[2] = {&L.lora[ad].s_gate, &L.lora[ad].s_up};
            for (int k = 0; k < 2; ++k)
                if (sa[k]->A && ((uintptr_t)sa[k]->A & 15)) return false;
        }
    }
    const int nbc = NB - P->nLA;
    P->perA = cdiv(E + (L.has_sgate ? 1 : 0), NB);
    P->per_s = sh ? cdiv(Is, NB) : 0;
    P->perC = cdiv(Umax * I, nbc);
    P->per_o = cdiv(H, NB);
    if (P->perC > I || P->per_o > kMaxOut) return false;  // a range spans at most two experts

    const size_t gp = (size_t)P->perC * (H / 2);
    const size_t gs = (size_t)P->perC * (H / L.gate.group) * 2, us = (size_t)P->perC * (H / L.up.group) * 2;
    const size_t cpart[6] = {gp, gs, gs, gp, us, us};
    size_t csz = 0;
    for (int k = 0; k < 6; ++k) {
        P->c_off[k] = (uint32_t)csz;
        csz += r16(cpart[k]) + 64;  // up to two windows (two experts)
    }
    const int gd = sh ? std::min(L.down.group, L.s_down.group) : L.down.group;
    const size_t dp = (size_t)P->per_o * (Imax / 2), ds = (size_t)P->per_o * (Imax / gd) * 2;
    P->d_off[0] = 0;
    P->d_off[1] = (uint32_t)(r16(dp) + 32);
    P->d_off[2] = (uint32_t)(P->d_off[1] + r16(ds) + 32);
    P->d_stride = (uint32_t)(P->d_off[2] + r16(ds) + 32);
    const size_t dsz = (size_t)(Umax + (sh ? 1 : 0)) * P->d_stride;
    // phase-A windows (they share the staged-h space)
    size_t asz = 0;
    auto awin = [&](int i, size_t bytes) {
        P->a_off[i] = (uint32_t)asz;
        asz += r16(bytes) + 32;
    };
    const int ngr = H / L.router.group;
    awin(0, (size_t)P->perA * H);
    awin(1, (size_t)P->perA * ngr * 2);
    awin(2, (size_t)P->perA * ngr * 2);
    awin(3, 0);  // the shared-expert gate row: no window
    awin(4, 0);
    awin(5, 0);
    for (int pj = 0; pj < 2; ++pj) {
        const moe_qtensor& q = pj ? L.s_up : L.s_gate;
        const int ng = sh ? H / q.group : 0;
        awin(6 + 3 * pj, (size_t)P->per_s * (H / 2));
        awin(7 + 3 * pj, (size_t)P->per_s * ng * 2);
        awin(8 + 3 * pj, (size_t)P->per_s * ng * 2);
    }
    awin(12, sh && lora ? (size_t)H * 2 : 0);
    awin(13, sh && lora ? (size_t)H * 2 : 0);
    const size_t hsz = r16((size_t)J * Imax * 4), hsumsz = r16((size_t)J * (Imax / 32) * 4);
    const size_t tdcsz = (size_t)(TK * r * 8 + (sh ? T * r * 32 : 0)) * 4;
    const size_t limit = (size_t)optin_smem() > static_smem_for(T) ? (size_t)optin_smem() - static_smem_for(T) : 0;
    for (int alias = 0; alias < 2; ++alias) {
        size_t o = 0;
        auto take = [&](size_t bytes) {
            const size_t at = o;
            o = r16(o + bytes);
            return (uint32_t)at;
        };
        P->dalias = alias;
        P->xs = take((size_t)T * H * 4);
        P->xsum = take((size_t)T * (H / 32) * 4);
        P->c = take(alias ? std::max(csz, dsz) : csz);
        P->d = alias ? P->c : take(dsz);
        P->ha = take(std::max(hsz + hsumsz, asz));
        P->hsum = (uint32_t)(P->ha + hsz);
        P->sgu = take((size_t)P->per_s * T * 2 * 4);
        P->sbd = take((size_t)P->per_o * J * r * 2);
        P->wpart = take(std::max((size_t)kW * 3 * T * r * 4, tdcsz));
        P->cand = take((size_t)T * ((E + 31) / 32) * K * 8);
        P->total = (uint32_t)o;
        if (o <= limit) return true;
    }
    return false;
}

template <int MT>
cudaError_t launch_mt(const DArgs& a, cudaStream_t s) {
    static int cached = 0;
    cudaError_t e = ensure_smem((const void*)decode_kernel<MT>, a.P.total, cached);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sm_count());
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = a.P.total;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_kernel<MT>, a);
}

}  // namespace

// Conditions of the fused path (checked on the host before launch).
bool decode_supported(const LayerArgs& L, int T, size_t* smem_out) {
    DPlan P;
    if (!plan_decode(L, T, sm_count(), &P)) return false;
    if (smem_out) *smem_out = P.total;
    return true;
}

cudaError_t launch_decode(const LayerArgs& L, const uint16_t* x, const int32_t* adapter_id, uint16_t* y, int T,
                          int block, float eps, const DecodeScratch& sc, cudaStream_t s) {
    DArgs a;
    memset(&a, 0, sizeof(a));
    if (!plan_decode(L, T, sm_count(), &a.P)) return cudaErrorNotSupported;
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
    a.h = sc.h;
    a.tdp = sc.tdp;
    a.flags = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(sc.status) + kFlagOffset);
    a.bar = sc.bar;
    a.status = sc.status;
    a.wait_ns = wait_limit_ns();
    a.idx_out = sc.idx_out;
    a.w_out = sc.w_out;
    if (T <= 1) return launch_mt<1>(a, s);
    if (T <= 2) return launch_mt<2>(a, s);
    if (T <= 4) return launch_mt<4>(a, s);
    return launch_mt<8>(a, s);
}

}  // namespace moeq
