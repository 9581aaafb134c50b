// decode_cluster.cu - the MoE layer for one token as one persistent, cooperative
// kernel of thread-block clusters.
//
// At decode the layer is a chain of dependent steps (router -> top-K -> expert
// rows -> down rows), each far too small to fill the GPU.  A hand-off between CTAs
// through L2 (a grid barrier, a flag or a tagged word) costs a memory round trip plus
// the wait for the slowest CTA, and the single-kernel decodes of decode.cu and
// decode_chain.cu pay it four or five times per layer.  Here the grid is NC clusters
// of CS CTAs (one CTA per SM) and every step that needs pieces from many CTAs but
// little work is done by each cluster for itself, the pieces exchanged through
// distributed shared memory and the cluster barrier:
//  - the router: CTA q of a cluster computes logits [q perA, (q+1) perA) and stores
//    them into the logit array of every CTA of its cluster; after one cluster barrier
//    every CTA holds all E logits and takes the top-K itself (same inputs, same code:
//    the same experts in every CTA);
//  - the LoRA-A products (shared expert, routed experts after top-K, down after h):
//    split over the CTAs of a cluster the same way.
// The streaming work is split over the whole grid: the shared-expert and routed
// gate/up rows (by h element) and the output rows of down.  The one grid-wide
// exchange is h: each CTA publishes its h elements as epoch-tagged words
// {value, tag} and gathers all of them.
//
//  R  x; the CTA's router rows -> logits to the cluster; the shared-gate row (every
//     CTA); the CTA's shared gate/up rows; shared LoRA-A rows -> products to the cluster.
//  K  top-K in every CTA; the routed rows' bulk copies issued.  With a given expert set
//     (the prerouter's prediction) the copies go out as soon as the CTA's router rows are
//     done, and the cluster's logits give only the weights.
//  G  routed LoRA-A rows -> products to the cluster; routed gate/up dots; LoRA-B
//     deltas and SwiGLU: h elements published (shared and routed).
//  X  every CTA gathers h.
//  D  down LoRA-A rows -> products to the cluster; the CTA's output rows for every
//     expert; combine in fixed order (k = 0..K-1, then the shared expert) and the
//     residual in block mode.
//
// Every CTA passes every cluster barrier exactly once whatever happens (a bounded wait
// that gives up sets an abort flag and the CTA runs on with zeros), so a cluster
// barrier always completes; no CTA exits while a peer may still store into it (the
// last stores precede the last cluster barrier).
#include <algorithm>
#include <cstdlib>
#include <cstring>

#include "decode_cdots.cuh"

namespace moeq {
namespace {

constexpr int kQMaxK = 8;     // routed experts
constexpr int kQMaxE = 256;   // experts
constexpr int kQMaxO = 32;    // output rows per CTA
constexpr int kQMaxSA = 8;    // shared LoRA-A rows per CTA
constexpr int kQMaxRA = 16;   // routed LoRA-A rows per CTA
constexpr int kQMaxDA = 16;   // down LoRA-A rows per CTA
constexpr int kQMaxCS = 16;   // CTAs per cluster
constexpr int kQIssue = 5;    // warps 0..4 take the top-K and issue the routed rows' copies
constexpr int kQMaxGT = 8;    // gate/up tiles (8 h elements each) per CTA
constexpr int kQGW = 12;      // h words per thread in the gather ((K+1) max(I, Is) <= 12 * 512)

struct QPlan {
    int CS, perA, perS, perO, perC, nSA, nRA, nDA, imx_sh, i_sh;
    int gu_ns, gu_spg, gu_gsh;    // routed gate/up tensor-core tiles: K slices, groups per slice, log2(group / 32)
    int lean;                     // 1: the routed LoRA-A rows reuse the phase-R windows (copied once the
                                  // shared-expert rows are read) and the packed down rows reuse the
                                  // gate/up windows (copied once the gate/up dots are done)
    uint32_t dp, dp_stride;       // packed down rows of slot k at dp + k * dp_stride
    uint32_t xraw, xs, xsum, z, sa, ra, da;
    uint32_t wr, r_off[3];        // router rows p/s/b
    uint32_t wsg, sg_off[9];      // shared gate rows p/s/b, shared up rows p/s/b, the shared-gate row p/s/b
    uint32_t wra, ra_stride;      // routed LoRA-A rows
    uint32_t wsd, sd_off[3];      // shared down rows p/s/b
    uint32_t wsa, sa_stride;      // shared LoRA-A rows
    uint32_t wsb, sb_stride;      // shared LoRA-B rows: gate, up, down
    uint32_t wc, c_off[6];        // routed gate/up: rows {gate, up} one per element at stride rrs; {s, b} two segments
    uint32_t rrs;                 // row stride of the routed gate/up rows (H/2 + 16: conflict-free fragment loads)
    uint32_t xp, gpart;           // x in the pair order of the tiles (bf16); tile partial sums
    uint32_t wrb, rb_stride;      // routed LoRA-B gate/up rows [segment][gate, up]
    uint32_t wd, d_off[3], d_stride;  // routed down rows of slot k at wd + k * d_stride
    uint32_t wrbd, rbd_stride;    // routed down LoRA-B rows [slot]
    uint32_t wda, da_stride;      // down LoRA-A rows
    uint32_t sgu, hs, hsum, sv;   // (hs, hsum reuse the routed gate/up windows)
    uint32_t total;
};

struct QArgs {
    LayerArgs L;
    const uint16_t* x;
    const int32_t* adapter_id;
    const int32_t* select;     // [K] caller-given expert set, or NULL: top-K of the logits
    uint16_t* y;
    int block;
    float eps;
    int x_host;                // x (and y) in mapped host memory: x read with plain loads
    unsigned long long* tick;  // ticket counter: a launch adds gridDim.x
    uint64_t* hg;              // [K+1][max(I, Is)] tagged h: routed slot k, then the shared expert
    unsigned long long* ready; // [gridDim.x] per CTA: the tag of the last launch whose h it published
    int32_t* status;
    int32_t* idx_out;          // [K] routing record
    float* w_out;
    uint64_t wait_ns;
    QPlan P;
};

// ------------------------------------------------------------ cluster primitives
// (all threads of the CTA take every cluster barrier, each warp converged)
__device__ __forceinline__ void cl_arrive() {
    __syncwarp();
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cl_arrive_relaxed() {
    __syncwarp();
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cl_wait() {
    __syncwarp();
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ int cl_rank() {
    uint32_t r;
    asm("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return (int)r;
}
// Store v at the place of p (this CTA's shared memory) in the shared memory of CTA
// `rank` of the cluster.
__device__ __forceinline__ void dsm_st(float* p, int rank, float v) {
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(tc::smem_u32(p)), "r"(rank));
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(ra), "f"(v) : "memory");
}

// ------------------------------------------------------------ tensor-core row dots
// A weight word holds 8 nibbles n0..n7 (K order); (w >> 4t) & 0x000F000F puts n_t and
// n_{t+4} in the low bits of two bf16 halves, and or-ing 0x43004300 makes them 128 + n
// exactly (128.0 is 0x4300; its mantissa counts units).  A tile of 16 rows (lane
// group g = lane / 4 holds rows g and g + 8) and one activation vector: lane c = lane % 4
// of a group contributes its word's pairs {n0,n4}, {n1,n5} to one mma.sync m16n8k16 and
// {n2,n6}, {n3,n7} to a second, with the activations of the same word stored in the
// pair order (x0,x4)(x1,x5)(x2,x6)(x3,x7), so every product meets its own activation and
// every column of B is the same vector (each lane group reads the same 16 bytes).  The
// 128 comes back out through the bias: s sum (128 + q) x + (b - 128 s) sum x.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t nib_pair(uint32_t w, int t) { return ((w >> (4 * t)) & 0x000F000Fu) | 0x43004300u; }

// Sum over the GPT groups [g0, g0 + GPT) of two int4 rows (ra: the row of lane group g,
// rb: row g + 8; NULL: a padding row) against the pair-ordered vector xp with 32-element
// chunk sums xc; WPL words of a group per lane (group size 128 WPL).  Every load of the
// task is issued first and every group has its own accumulators, so the task is one
// memory round trip and a few dependent steps.  Returns the lane group's two row partials
// (every lane of the group holds them).
template <int WPL, int GPT>
__device__ __noinline__ float2 tile_dot4(const uint32_t* ra, const uint16_t* sa_, const uint16_t* ba_,
                                         const uint32_t* rb, const uint16_t* sb_, const uint16_t* bb_,
                                         const uint4* __restrict__ xp, const float* __restrict__ xc, int g0,
                                         int c) {
    constexpr int NW = WPL * GPT;
    uint32_t qa[NW], qb[NW];
    uint4 xv[NW];
    float sA[GPT], bA[GPT], sB[GPT], bB[GPT], xs_[GPT];
#pragma unroll
    for (int gg = 0; gg < GPT; ++gg) {
        const int gi = g0 + gg, w0 = gi * 4 * WPL + c * WPL;
#pragma unroll
        for (int j = 0; j < WPL; ++j) {
            qa[gg * WPL + j] = ra ? ra[w0 + j] : 0u;
            qb[gg * WPL + j] = rb ? rb[w0 + j] : 0u;
            xv[gg * WPL + j] = xp[w0 + j];
        }
        sA[gg] = ra ? bf16f(sa_[gi]) : 0.0f;
        bA[gg] = ra ? bf16f(ba_[gi]) : 0.0f;
        sB[gg] = rb ? bf16f(sb_[gi]) : 0.0f;
        bB[gg] = rb ? bf16f(bb_[gi]) : 0.0f;
        float t = 0.0f;
#pragma unroll
        for (int k = 0; k < WPL; ++k) t += xc[gi * WPL + k];
        xs_[gg] = t;
    }
    float accA = 0.0f, accB = 0.0f;
#pragma unroll
    for (int gg = 0; gg < GPT; ++gg) {
        float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int j = 0; j < WPL; ++j) {
            const uint32_t a = qa[gg * WPL + j], b = qb[gg * WPL + j];
            const uint4 x = xv[gg * WPL + j];
            mma_bf16(d, nib_pair(a, 0), nib_pair(b, 0), nib_pair(a, 1), nib_pair(b, 1), x.x, x.y);
            mma_bf16(d, nib_pair(a, 2), nib_pair(b, 2), nib_pair(a, 3), nib_pair(b, 3), x.z, x.w);
        }
        accA = fmaf(sA[gg], d[0], fmaf(fmaf(-128.0f, sA[gg], bA[gg]), xs_[gg], accA));
        accB = fmaf(sB[gg], d[2], fmaf(fmaf(-128.0f, sB[gg], bB[gg]), xs_[gg], accB));
    }
    return make_float2(accA, accB);
}

// The task's groups [g0, g0 + n) in steps of GPT (n a multiple of GPT).
template <int WPL>
__device__ __forceinline__ float2 tile_dot4_run(const uint32_t* ra, const uint16_t* sa_, const uint16_t* ba_,
                                                const uint32_t* rb, const uint16_t* sb_, const uint16_t* bb_,
                                                const uint4* xp, const float* xc, int g0, int n, int c) {
    constexpr int GPT = WPL >= 2 ? 2 : 4;
    float2 acc = make_float2(0.0f, 0.0f);
    for (int g = g0; g < g0 + n; g += GPT) {
        const float2 v = tile_dot4<WPL, GPT>(ra, sa_, ba_, rb, sb_, bb_, xp, xc, g, c);
        acc.x += v.x;
        acc.y += v.y;
    }
    return acc;
}

__global__ void __launch_bounds__(kCT, 1) decode_cluster_kernel(const __grid_constant__ QArgs a_param) {
    extern __shared__ __align__(16) unsigned char sm[];
    // (the arguments are read all over the kernel, most fields once: one copy into
    // shared memory by all threads costs one round trip instead of a constant-cache miss
    // at each first use)
    __shared__ __align__(16) QArgs a_sm;
    static_assert(sizeof(QArgs) % 4 == 0, "argument copy in words");
    for (int i = threadIdx.x; i < (int)(sizeof(QArgs) / 4); i += kCT)
        reinterpret_cast<uint32_t*>(&a_sm)[i] = reinterpret_cast<const uint32_t*>(&a_param)[i];
    // every CTA of the cluster has started before any stores into another: arrive now,
    // wait before the first such store
    cl_arrive_relaxed();
    __syncthreads();
    const QArgs& a = a_sm;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const LayerArgs& L = a.L;
    const QPlan& P = a.P;
    const int H = L.H, E = L.E, K = L.K, I = L.I;
    const bool sh = L.has_shared;
    const int Is = sh ? L.Is : 0, Imx = max(I, Is);
    const int NB = gridDim.x, cta = blockIdx.x, CS = P.CS, q = cl_rank();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool lora = L.n_adapters > 0 && L.rank > 0;
    const int r = lora ? L.rank : 0;
    const uint64_t lim = a.wait_ns;
    const uint64_t pol = l2_stream_policy();

    float* xs = reinterpret_cast<float*>(sm + P.xs);
    float* xsum = reinterpret_cast<float*>(sm + P.xsum);
    float* z = reinterpret_cast<float*>(sm + P.z);      // [E] logits (stored by the cluster)
    float* sa = reinterpret_cast<float*>(sm + P.sa);    // [2r] shared LoRA-A products (cluster)
    float* ra = reinterpret_cast<float*>(sm + P.ra);    // [K][2r] routed LoRA-A products (cluster)
    float* da = reinterpret_cast<float*>(sm + P.da);    // [K+1][r] down LoRA-A products (cluster)
    float* sgu = reinterpret_cast<float*>(sm + P.sgu);  // [perS][2] shared gate/up dots
    float* hs = reinterpret_cast<float*>(sm + P.hs);    // [K+1][Imx] h (swizzled)
    float* hsum = reinterpret_cast<float*>(sm + P.hsum);
    float* sv = reinterpret_cast<float*>(sm + P.sv);    // [perO][K+1] per-expert outputs of the CTA's rows

    __shared__ __align__(8) uint64_t s_bar[6];
    __shared__ int s_abort, s_aid, s_gut;
    __shared__ uint32_t s_tag;
    __shared__ float s_inv, s_sig;
    __shared__ int32_t s_sel[kQMaxK];
    __shared__ int s_idx[kQMaxK];
    __shared__ float s_w[kQMaxK];
    __shared__ const unsigned char* s_rw[3];
    __shared__ const unsigned char* s_gw[3];
    __shared__ const unsigned char* s_sgw[6];
    __shared__ const unsigned char* s_sdw[3];
    __shared__ const unsigned char* s_saw[kQMaxSA];
    __shared__ const unsigned char* s_sbw[3];
    __shared__ const unsigned char* s_raw[kQMaxRA];
    __shared__ const unsigned char* s_cw[2][6];
    __shared__ const unsigned char* s_rbw[2][2];
    __shared__ const unsigned char* s_dw[kQMaxK][3];
    __shared__ const unsigned char* s_rbdw[kQMaxK];
    __shared__ const unsigned char* s_daw[kQMaxDA];

    // barrier 0: x, router rows, shared gate/up rows; 1: shared down rows, shared LoRA
    // rows; 2: routed LoRA-A rows; 3: routed gate/up rows (warp 0) + their LoRA-B rows
    // (warp 1); 4: routed down rows + their LoRA-B rows (warp 2) + down LoRA-A rows (warp 4)
    if (tid == 0) {
        s_abort = 0;
        s_gut = 0;
        s_sig = 1.0f;
        s_inv = 1.0f;
        for (int i = 0; i < 6; ++i) tc::mbar_init(&s_bar[i], (i == 3 || i == 4) ? 2u : 1u);
        tc::mbar_init_fence();
    }
    __syncthreads();

    // cluster split (router rows), grid split (shared h rows, output rows, routed h elements)
    const int ra0 = min(E, q * P.perA), nra = min(E, ra0 + P.perA) - ra0;
    const int s_lo = min(Is, cta * P.perS), nsr = min(Is, s_lo + P.perS) - s_lo;
    const int o_lo = min(H, cta * P.perO), no = min(H, o_lo + P.perO) - o_lo;
    const int nC = K * I, c_lo = min(nC, cta * P.perC), c_hi = min(nC, c_lo + P.perC), nrows = c_hi - c_lo;
    const int Ish_ = P.i_sh;  // I = 1 << i_sh
    const int cut = nrows > 0 ? min(c_hi, ((c_lo >> Ish_) + 1) << Ish_) : c_lo;
    const int nsa_here = (lora && sh) ? max(0, min(P.nSA, 2 * r - q * P.nSA)) : 0;
    const int nra_here = lora ? max(0, min(P.nRA, K * 2 * r - q * P.nRA)) : 0;
    const int nda_here = lora ? max(0, min(P.nDA, (K + (sh ? 1 : 0)) * r - q * P.nDA)) : 0;

    // The routed rows' bulk copies (warps 0..4; the routing in s_idx, the adapter ad):
    // gate/up rows, their scales, biases and LoRA-B rows (warps 0, 1), down rows with theirs
    // (warp 2), routed LoRA-A rows (warp 3), down LoRA-A rows (warp 4).
    auto issue_routed = [&](const int ad) {
        if (warp < 2) {
            // routed gate (warp 0) | up (warp 1) rows: lane j copies the rows of h elements c_lo + j,
            // c_lo + j + 32, .. to their own slots (stride rrs); lanes 0..3 copy the scales and
            // biases of the two segments (rows of one expert each); warp 1 lanes 4..7 the LoRA-B rows
            uint32_t tx = 0;
            const int pj = warp;
            const moe_qtensor& qt = pj ? L.up : L.gate;
            const int ng = H / qt.group;
            for (int j = lane; j < nrows; j += 32) {
                const int qq = c_lo + j;
                const int64_t row = ((int64_t)s_idx[qq >> Ish_] << Ish_) + (qq & (I - 1));
                winp(pol, sm + P.wc + P.c_off[3 * pj] + j * P.rrs, s_abort ? nullptr : qt.packed + row * (H / 8),
                     (uint32_t)(H / 2), &s_bar[3], &tx);
            }
            if (lane < 4) {  // scales | biases of the two segments: lane 2 s + (k - 1)
                const int sgi = lane / 2, k = 1 + lane % 2, part = 3 * pj + k;
                const int q0 = sgi == 0 ? c_lo : cut, q1 = sgi == 0 ? cut : c_hi;
                const void* src = nullptr;
                uint32_t off = P.wc + P.c_off[part];
                if (q1 > q0 && s_abort == 0) {
                    const int64_t row = ((int64_t)s_idx[q0 >> Ish_] << Ish_) + (q0 & (I - 1));
                    src = (k == 1 ? qt.scales : qt.biases) + row * ng;
                    if (sgi == 1 && cut > c_lo) {  // segment 1's window follows segment 0's
                        const int64_t row0 = ((int64_t)s_idx[c_lo >> Ish_] << Ish_) + (c_lo & (I - 1));
                        off += win_span((k == 1 ? qt.scales : qt.biases) + row0 * ng, (uint32_t)(cut - c_lo) * ng * 2);
                    }
                }
                s_cw[sgi][part] = winp(pol, sm + off, src, (uint32_t)(q1 - q0) * ng * 2, &s_bar[3], &tx);
            } else if (pj == 1 && lane < 8) {  // LoRA-B rows of the routed gate/up rows: lane 4 + 2 s + p
                const int sgi = (lane - 4) / 2, pb = (lane - 4) % 2;
                const int q0 = sgi == 0 ? c_lo : cut, q1 = sgi == 0 ? cut : c_hi;
                const moe_lora_proj* lp = (lora && q1 > q0 && s_abort == 0) ? dlora(L, ad, false, pb) : nullptr;
                const int64_t row = q1 > q0 ? ((int64_t)s_idx[q0 >> Ish_] << Ish_) + (q0 & (I - 1)) : 0;
                s_rbw[sgi][pb] = winp(pol, sm + P.wrb + (lane - 4) * P.rb_stride, lp ? lp->B + row * r : nullptr,
                                      (uint32_t)((q1 - q0) * r * 2), &s_bar[3], &tx);
            }
            tx = warp_total(tx);
            if (lane == 0) tc::mbar_arrive_expect_tx(&s_bar[3], tx);
        } else if (warp == 2) {  // routed down rows of the CTA's output range and their LoRA-B rows
            uint32_t tx = 0;
            const int ngd = I / L.down.group;
            if (lane < 3 * K) {
                const int k = lane / 3, part = lane % 3;
                const int64_t row = (int64_t)s_idx[k] * H + o_lo;
                const void* src = nullptr;
                uint32_t bytes = 0;
                if (no > 0 && s_abort == 0) {
                    src = part == 0 ? (const void*)(L.down.packed + row * (I / 8))
                                    : (const void*)((part == 1 ? L.down.scales : L.down.biases) + row * ngd);
                    bytes = part == 0 ? (uint32_t)(no * I / 2) : (uint32_t)(no * ngd * 2);
                }
                if (part > 0 || !P.lean)
                    s_dw[k][part] = winp(pol, sm + (part == 0 ? P.dp + k * P.dp_stride : P.wd + k * P.d_stride + P.d_off[part]),
                                         src, bytes, &s_bar[4], &tx);
            }
            if (lane < K) {
                const moe_lora_proj* lp = (lora && no > 0 && s_abort == 0) ? dlora(L, ad, false, 2) : nullptr;
                const int64_t row = (int64_t)s_idx[lane] * H + o_lo;
                s_rbdw[lane] = winp(pol, sm + P.wrbd + lane * P.rbd_stride, lp ? lp->B + row * r : nullptr,
                                   (uint32_t)(no * r * 2), &s_bar[4], &tx);
            }
            tx = warp_total(tx);
            if (lane == 0) tc::mbar_arrive_expect_tx(&s_bar[4], tx);
        } else if (warp == 3) {  // routed LoRA-A rows: row d = q nRA + lane of [slot k][gate A | up A]
            if (P.lean) {  // (their slots are the phase-R windows: wait for warps kQIssue.. to be done with them)
                asm volatile("bar.sync 2, %0;" ::"n"((kCW - kQIssue + 1) * 32) : "memory");
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            }
            uint32_t tx = 0;
            if (lane < kQMaxRA) {
                const int d = q * P.nRA + lane, k = d / max(2 * r, 1), c = d % max(2 * r, 1);
                const moe_lora_proj* lp = (lane < nra_here && s_abort == 0) ? dlora(L, ad, false, c < r ? 0 : 1) : nullptr;
                const int64_t row = lp ? ((int64_t)s_idx[k] * r + c % r) * H : 0;
                s_raw[lane] = winp(pol, sm + P.wra + lane * P.ra_stride, lp ? lp->A + row : nullptr, (uint32_t)(H * 2),
                                  &s_bar[2], &tx);
            }
            tx = warp_total(tx);
            if (lane == 0) tc::mbar_arrive_expect_tx(&s_bar[2], tx);
        } else if (warp == 4) {  // down LoRA-A rows: row d = q nDA + lane of [slot k][component]; slot K shared
            uint32_t tx = 0;
            if (lane < kQMaxDA) {
                const int d = q * P.nDA + lane, k = d / max(r, 1), c = d % max(r, 1);
                const moe_lora_proj* lp = nullptr;
                const uint16_t* src = nullptr;
                int n = I;
                if (lane < nda_here && s_abort == 0) {
                    lp = dlora(L, ad, k == K, 2);
                    if (lp) {
                        src = k < K ? lp->A + ((int64_t)s_idx[k] * r + c) * I : lp->A + (int64_t)c * Is;
                        n = k < K ? I : Is;
                    }
                }
                s_daw[lane] = winp(pol, sm + P.wda + lane * P.da_stride, src, (uint32_t)(n * 2), &s_bar[4], &tx);
            }
            tx = warp_total(tx);
            if (lane == 0) tc::mbar_arrive_expect_tx(&s_bar[4], tx);
        }
    };
    // A given expert set (the prerouter's prediction) needs no top-K: its rows are copied as
    // soon as the CTA's router rows are done, while the cluster's logits (which give only the
    // weights then) come together.  (Not in the lean layout, whose routed LoRA-A windows are
    // free only after phase R.)
    const bool early = a.select != nullptr && !P.lean;

    // ------------------------------------------------------------ phase R: issue
    // The weight rows of this phase depend on nothing the previous kernel on the stream
    // writes: their copies start before the grid-dependency wait.  Everything that reads
    // x, the adapter id, the expert set or the workspace comes after it.
    if (warp == 0) {
        uint32_t tx = 0;
        if (lane < 3) {  // router rows (int8)
            const int ng = H / L.router.group;
            const void* src = nullptr;
            uint32_t bytes = 0;
            if (nra > 0) {
                src = lane == 0 ? (const void*)(L.router.packed + (int64_t)ra0 * (H / 4))
                                : (const void*)((lane == 1 ? L.router.scales : L.router.biases) + (int64_t)ra0 * ng);
                bytes = lane == 0 ? (uint32_t)(nra * H) : (uint32_t)(nra * ng * 2);
            }
            s_rw[lane] = winp(pol, sm + P.wr + P.r_off[lane], src, bytes, &s_bar[0], &tx);
        } else if (lane < 9) {  // shared gate | up rows (int4)
            const int w = lane - 3, pj = w / 3, k = w % 3;
            const moe_qtensor& qt = pj ? L.s_up : L.s_gate;
            const void* src = nullptr;
            uint32_t bytes = 0;
            if (nsr > 0) {
                const int ng = H / qt.group;
                src = k == 0 ? (const void*)(qt.packed + (int64_t)s_lo * (H / 8))
                             : (const void*)((k == 1 ? qt.scales : qt.biases) + (int64_t)s_lo * ng);
                bytes = k == 0 ? (uint32_t)(nsr * H / 2) : (uint32_t)(nsr * ng * 2);
            }
            s_sgw[w] = winp(pol, sm + P.wsg + P.sg_off[w], src, bytes, &s_bar[0], &tx);
        } else if (lane < 12) {  // the shared-gate row (int8)
            const int k = lane - 9;
            const moe_qtensor& qt = L.shared_gate;
            const void* src = nullptr;
            uint32_t bytes = 0;
            if (L.has_sgate) {
                src = k == 0 ? (const void*)qt.packed : (const void*)(k == 1 ? qt.scales : qt.biases);
                bytes = k == 0 ? (uint32_t)H : (uint32_t)(H / qt.group * 2);
            }
            s_gw[k] = winp(pol, sm + P.wsg + P.sg_off[6 + k], src, bytes, &s_bar[0], &tx);
        }
        asm volatile("griddepcontrol.wait;" ::: "memory");
        if (lane == 0 && !a.x_host) win(sm + P.xraw, a.x, (uint32_t)(H * 2), &s_bar[0], &tx);
        tx = warp_total(tx);
        if (lane == 0) tc::mbar_arrive_expect_tx(&s_bar[0], tx);
    } else if (warp == 1) {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        int ad = a.adapter_id ? a.adapter_id[0] : (L.n_adapters > 0 ? 0 : -1);
        if (ad < -1 || ad >= L.n_adapters) {
            if (cta == 0 && lane == 0) raise_status(a.status, MOE_ERR_DEVICE_INDEX);
            ad = -1;
        }
        if (lane == 0) s_aid = ad;
        if (a.select) {  // the given set, repaired (an entry out of range or repeated: the lowest unused expert)
            if (lane < K) s_sel[lane] = a.select[lane];
            __syncwarp();
            bool bad = false;
            const int e = select_entry(s_sel, K, E, lane, &bad);
            if (bad && lane == 0 && cta == 0) raise_status(a.status, MOE_ERR_DEVICE_INDEX);
            if (lane < K) s_idx[lane] = e;
        }
        uint32_t tx = 0;
        if (lane < 3) {  // shared down rows of the CTA's output range
            const void* src = nullptr;
            uint32_t bytes = 0;
            if (sh && no > 0) {
                const int ngd = Is / L.s_down.group;
                src = lane == 0 ? (const void*)(L.s_down.packed + (int64_t)o_lo * (Is / 8))
                                : (const void*)((lane == 1 ? L.s_down.scales : L.s_down.biases) + (int64_t)o_lo * ngd);
                bytes = lane == 0 ? (uint32_t)(no * Is / 2) : (uint32_t)(no * ngd * 2);
            }
            s_sdw[lane] = winp(pol, sm + P.wsd + P.sd_off[lane], src, bytes, &s_bar[1], &tx);
        } else if (lane < 3 + kQMaxSA) {  // shared LoRA-A rows: row d = q nSA + j of [gate A; up A]
            const int j = lane - 3, d = q * P.nSA + j;
            const moe_lora_proj* lp = j < nsa_here ? dlora(L, ad, true, d < r ? 0 : 1) : nullptr;
            s_saw[j] = winp(pol, sm + P.wsa + j * P.sa_stride, lp ? lp->A + (int64_t)(d % r) * H : nullptr,
                           (uint32_t)(H * 2), &s_bar[1], &tx);
        } else if (lane >= 16 && lane < 19) {  // shared LoRA-B rows: gate, up (h rows), down (output rows)
            const int w = lane - 16;
            const moe_lora_proj* lp = (lora && sh) ? dlora(L, ad, true, w) : nullptr;
            const int row0 = w < 2 ? s_lo : o_lo, n = w < 2 ? nsr : no;
            s_sbw[w] = winp(pol, sm + P.wsb + w * P.sb_stride, lp ? lp->B + (int64_t)row0 * r : nullptr,
                           (uint32_t)(n * r * 2), &s_bar[1], &tx);
        }
        tx = warp_total(tx);
        if (lane == 0) tc::mbar_arrive_expect_tx(&s_bar[1], tx);
    } else {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        if (warp == kCW - 1 && lane == 0) {
            unsigned long long prev;
            asm volatile("atom.add.relaxed.gpu.global.u64 %0, [%1], 1;" : "=l"(prev) : "l"(a.tick) : "memory");
            s_tag = (uint32_t)((prev / (unsigned long long)NB) % 0xffffffffull) + 1u;
        }
    }

    // ------------------------------------------------------------ phase R: compute
    if (a.x_host) {
        // x across the bus once per cluster: CTA q reads its 1/CS of x (16-byte pieces) and
        // stores each piece into every CTA of its cluster; after one cluster barrier every CTA
        // holds all of x.  (A bulk copy does not read host memory here, and a read of all of x
        // by every CTA would cross the bus 112 times.)
        cl_wait();  // (every CTA of the cluster has started)
        const int npc = H / 8, per = (npc + CS - 1) / CS;
        if (tid < per && q * per + tid < npc) {
            const int pi = q * per + tid;
            const uint4 v = reinterpret_cast<const uint4*>(a.x)[pi];
            uint32_t ra;
            for (int rk = 0; rk < CS; ++rk) {
                asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
                             : "=r"(ra)
                             : "r"(tc::smem_u32(sm + P.xraw + 16 * pi)), "r"(rk));
                asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(ra), "r"(v.x), "r"(v.y), "r"(v.z),
                             "r"(v.w)
                             : "memory");
            }
        }
        cl_arrive();
        cl_wait();  // all of x is here
    }
    copies_landed(&s_bar[0], a.status, &s_abort, lim);
    const uint16_t* xr = reinterpret_cast<const uint16_t*>(sm + P.xraw);
    if (a.block) {  // RMSNorm scale of the token
        if (warp == 0) {
            float ss = 0.0f;
            const uint4* xv = reinterpret_cast<const uint4*>(xr);
            for (int v = lane; v < H / 8; v += 32) {
                const uint4 u = xv[v];
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float lo = __uint_as_float(w[k] << 16), hi = __uint_as_float(w[k] & 0xFFFF0000u);
                    ss = fmaf(lo, lo, fmaf(hi, hi, ss));
                }
            }
            ss = warp_sum(ss);
            if (lane == 0) s_inv = 1.0f / sqrtf(ss / (float)H + a.eps);
        }
        __syncthreads();
    }
    cstage_bf16(xs, xsum, xr, 1, H, a.block ? &s_inv : nullptr);
    {  // x in the pair order of the tensor-core tiles (the same bf16 values)
        uint4* xpw = reinterpret_cast<uint4*>(sm + P.xp);
        for (int w = tid; w < H / 8; w += kCT) {
            uint4 u = reinterpret_cast<const uint4*>(xr)[w];
            if (a.block) {
                uint32_t v[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float lo = bf16f(f2bf16(__uint_as_float(v[k] << 16) * s_inv));
                    const float hi = bf16f(f2bf16(__uint_as_float(v[k] & 0xFFFF0000u) * s_inv));
                    v[k] = (__float_as_uint(lo) >> 16) | (__float_as_uint(hi) & 0xFFFF0000u);
                }
                u = make_uint4(v[0], v[1], v[2], v[3]);
            }
            xpw[w] = make_uint4(__byte_perm(u.x, u.z, 0x5410), __byte_perm(u.x, u.z, 0x7632),
                                __byte_perm(u.y, u.w, 0x5410), __byte_perm(u.y, u.w, 0x7632));
        }
    }
    __syncthreads();
    if (!a.x_host) cl_wait();  // (every CTA of the cluster has started; with x from host memory, above)
    // router rows (int8): row j of the CTA's range, or the shared-gate row (j == nra)
    auto row8 = [&](int j) {
        const bool sg = j == nra;
        const unsigned char* const* w = sg ? s_gw : s_rw;
        const int ng = H / (sg ? L.shared_gate.group : L.router.group), jj = sg ? 0 : j;
        float acc[1] = {0.0f};
        if (w[0])
            cdot_int8<1>(reinterpret_cast<const uint32_t*>(w[0] + (size_t)jj * H),
                         reinterpret_cast<const uint16_t*>(w[1]) + jj * ng,
                         reinterpret_cast<const uint16_t*>(w[2]) + jj * ng, sg ? L.shared_gate.group : L.router.group,
                         H, xs, xsum, 1, acc, lane);
        return warp_sum(acc[0]);
    };
    for (int j = warp; j < nra; j += kCW) {
        const float v = row8(j);
        if (lane < CS) {
            const int row = ra0 + j;
            dsm_st(z + row, lane, v + (L.logit_bias ? L.logit_bias[row] : 0.0f));
        }
    }
    cl_arrive();  // this CTA's logits are in every CTA of the cluster
    if (warp >= kQIssue) {
        // the shared-gate row, shared gate/up rows and shared LoRA-A rows (their products
        // reach the cluster by the next cluster barrier), while warps 0..kQIssue-1 route and
        // issue the routed rows' copies
        for (int t = warp - kQIssue; t < 1 + nsr + nsa_here; t += kCW - kQIssue) {
            if (t == 0) {
                if (L.has_sgate) {
                    const float v = row8(nra);
                    if (lane == 0) s_sig = 1.0f / (1.0f + expf(-v));
                }
            } else if (t <= nsr) {
                const int j = t - 1;
                float ag[1] = {0.0f}, au[1] = {0.0f};
                const int vid[1] = {0};
                const int ngg = H / L.s_gate.group, ngu = H / L.s_up.group;
                if (s_sgw[0] && s_sgw[3]) {
                    cdot_int4<1>(reinterpret_cast<const uint32_t*>(s_sgw[0] + (size_t)j * (H / 2)),
                                 reinterpret_cast<const uint16_t*>(s_sgw[1]) + j * ngg,
                                 reinterpret_cast<const uint16_t*>(s_sgw[2]) + j * ngg, L.s_gate.group, H, xs, xsum, vid, 1,
                                 ag, lane, 32);
                    cdot_int4<1>(reinterpret_cast<const uint32_t*>(s_sgw[3] + (size_t)j * (H / 2)),
                                 reinterpret_cast<const uint16_t*>(s_sgw[4]) + j * ngu,
                                 reinterpret_cast<const uint16_t*>(s_sgw[5]) + j * ngu, L.s_up.group, H, xs, xsum, vid, 1,
                                 au, lane, 32);
                }
                const float g = warp_sum(ag[0]), u = warp_sum(au[0]);
                if (lane == 0) {
                    sgu[2 * j] = g;
                    sgu[2 * j + 1] = u;
                }
            } else {
                const int jj = t - 1 - nsr;
                copies_landed(&s_bar[1], a.status, &s_abort, lim);
                float v = 0.0f;
                if (s_saw[jj]) v = warp_sum(sdot_bf16(reinterpret_cast<const uint16_t*>(s_saw[jj]), H, xs, lane));
                if (lane < CS) dsm_st(sa + q * P.nSA + jj, lane, v);
            }
        }
        if (P.lean) asm volatile("bar.arrive 2, %0;" ::"n"((kCW - kQIssue + 1) * 32) : "memory");
        cl_wait();  // the logits of the whole cluster are here
    } else {
        // ---------------------------------------------------------- phase K (issuing warps)
        // Two passes, one copy of the issue code: the routed rows' copies go out in the first
        // pass for a given set (before the cluster's logits, which then give only the
        // weights), in the second after the top-K otherwise.
#pragma unroll 1
        for (int pass = 0; pass < 2; ++pass) {
            if (pass == (early ? 0 : 1)) issue_routed(s_aid);
            if (pass == 0) {
                cl_wait();  // the logits of the whole cluster are here
                if (warp == 0) {
                    if (a.select) {  // a caller-given set (repaired in the prologue): only the weights come from z
                        const int e = lane < K ? s_idx[lane] : -1;
                        const float zk = e >= 0 ? z[e] : -INFINITY;
                        const float m = warp_max(zk);
                        const float ev = e >= 0 ? expf(zk - m) : 0.0f;
                        const float sum = warp_sum(ev);
                        if (lane < K) s_w[lane] = ev / sum;
                    } else {
                        warp_topk<kQMaxE / 32>(z, E, K, lane, s_idx, s_w);
                    }
                    __syncwarp();
                    if (cta == 0 && lane < K) {  // the routing this call used, for the caller's record
                        a.idx_out[lane] = s_idx[lane];
                        a.w_out[lane] = s_w[lane];
                    }
                }
                // the routing is known to the issuing warps (the others learn the window
                // pointers through the copies' mbarriers)
                asm volatile("bar.sync 1, %0;" ::"n"(kQIssue * 32) : "memory");
            }
        }
    }

    // ------------------------------------------------------------ phase G
    // routed LoRA-A rows -> products to the cluster, on the last warps (the first ones have just
    // issued the copies and take gate/up tasks as soon as the rows land)
    for (int j = kCW - 1 - warp; j < nra_here; j += kCW) {
        copies_landed(&s_bar[2], a.status, &s_abort, lim);
        float v = 0.0f;
        if (s_raw[j]) v = warp_sum(sdot_bf16(reinterpret_cast<const uint16_t*>(s_raw[j]), H, xs, lane));
        if (lane < CS) dsm_st(ra + q * P.nRA + j, lane, v);
    }
    cl_arrive();  // this CTA's shared and routed LoRA-A products are in the cluster
    {
        // routed gate/up dots: tile t holds the gate rows of elements 8t..8t+7 (rows g) and
        // their up rows (rows g + 8); a task is (tile, K slice); partial sums per slice
        const int NT = (nrows + 7) / 8, NS = P.gu_ns, spg = P.gu_spg, ngr = H / L.gate.group;
        const int g = lane >> 2, c = lane & 3, gsh = P.gu_gsh;
        float* gpart = reinterpret_cast<float*>(sm + P.gpart);
        // tasks are taken from a counter as warps come free (their partial sums have fixed
        // places, so the result does not depend on which warp took a task)
        auto grab = [&]() {
            int v = 0;
            if (lane == 0) v = atomicAdd(&s_gut, 1);
            return __shfl_sync(0xffffffffu, v, 0);
        };
        for (int t = grab(); t < NT * NS; t = grab()) {
            const int tile = t / NS, sl = t % NS, j = 8 * tile + g;
            copies_landed(&s_bar[3], a.status, &s_abort, lim);
            const bool live = j < nrows && s_cw[0][1];
            const uint32_t *ra = nullptr, *rb = nullptr;
            const uint16_t *sa_ = nullptr, *ba_ = nullptr, *sb_ = nullptr, *bb_ = nullptr;
            if (live) {
                const int qq = c_lo + j, sg = qq < cut ? 0 : 1, rs = qq - (sg == 0 ? c_lo : cut);
                ra = reinterpret_cast<const uint32_t*>(sm + P.wc + P.c_off[0] + j * P.rrs);
                rb = reinterpret_cast<const uint32_t*>(sm + P.wc + P.c_off[3] + j * P.rrs);
                sa_ = reinterpret_cast<const uint16_t*>(s_cw[sg][1]) + rs * ngr;
                ba_ = reinterpret_cast<const uint16_t*>(s_cw[sg][2]) + rs * ngr;
                sb_ = reinterpret_cast<const uint16_t*>(s_cw[sg][4]) + rs * ngr;
                bb_ = reinterpret_cast<const uint16_t*>(s_cw[sg][5]) + rs * ngr;
            }
            const uint4* xpw = reinterpret_cast<const uint4*>(sm + P.xp);
            const int n = min(ngr, (sl + 1) * spg) - sl * spg;
            const float2 v = gsh == 1   ? tile_dot4_run<2>(ra, sa_, ba_, rb, sb_, bb_, xpw, xsum, sl * spg, n, c)
                             : gsh == 0 ? tile_dot4_run<1>(ra, sa_, ba_, rb, sb_, bb_, xpw, xsum, sl * spg, n, c)
                                        : tile_dot4_run<4>(ra, sa_, ba_, rb, sb_, bb_, xpw, xsum, sl * spg, n, c);
            if (c == 0) {
                gpart[(tile * NS + sl) * 16 + g] = v.x;
                gpart[(tile * NS + sl) * 16 + 8 + g] = v.y;
            }
        }
    }
    cl_wait();  // the LoRA-A products of the whole cluster are here
    __syncthreads();
    if (P.lean && warp == 2) {  // the packed down rows into the gate/up windows, read by now
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        uint32_t tx = 0;
        if (lane < K && no > 0 && s_abort == 0)
            s_dw[lane][0] = winp(pol, sm + P.dp + lane * P.dp_stride,
                                 L.down.packed + ((int64_t)s_idx[lane] * H + o_lo) * (I / 8), (uint32_t)(no * I / 2),
                                 &s_bar[5], &tx);
        tx = warp_total(tx);
        if (lane == 0) tc::mbar_arrive_expect_tx(&s_bar[5], tx);
    }
    {
        // LoRA-B deltas, SwiGLU; h published: one element per thread (shared rows first, then
        // routed elements), each LoRA-B dot a thread's own loop over the rank
        const uint32_t tag = s_tag;
        const int j = tid;
        if (j < nsr + nrows) {
            float g, u;
            const uint16_t *bg = nullptr, *bu = nullptr;
            const float *tg = nullptr, *tu = nullptr;
            int br = 0;
            uint64_t* dst;
            if (j < nsr) {
                g = sgu[2 * j];
                u = sgu[2 * j + 1];
                if (lora) {
                    copies_landed(&s_bar[1], a.status, &s_abort, lim);
                    bg = reinterpret_cast<const uint16_t*>(s_sbw[0]);
                    bu = reinterpret_cast<const uint16_t*>(s_sbw[1]);
                    tg = sa;
                    tu = sa + r;
                    br = j;
                }
                dst = a.hg + (int64_t)K * Imx + s_lo + j;
            } else {
                const int jj = j - nsr, qq = c_lo + jj, k = qq >> Ish_, sg = qq < cut ? 0 : 1;
                const float* gp = reinterpret_cast<const float*>(sm + P.gpart) + (jj / 8) * P.gu_ns * 16 + jj % 8;
                g = 0.0f;
                u = 0.0f;
                for (int sl = 0; sl < P.gu_ns; ++sl) {  // the K slices in order
                    g += gp[sl * 16];
                    u += gp[sl * 16 + 8];
                }
                if (lora) {
                    bg = reinterpret_cast<const uint16_t*>(s_rbw[sg][0]);
                    bu = reinterpret_cast<const uint16_t*>(s_rbw[sg][1]);
                    tg = ra + k * 2 * r;
                    tu = tg + r;
                    br = qq - (sg == 0 ? c_lo : cut);
                }
                dst = a.hg + (int64_t)k * Imx + (qq & (I - 1));
            }
            if (lora && bg && bu) {
                float dg = 0.0f, du = 0.0f;
                for (int c0 = 0; c0 < r; c0 += 8) {  // (rows of r bf16, r % 8 == 0: 16-byte pieces)
                    const uint4 wg = *reinterpret_cast<const uint4*>(bg + br * r + c0);
                    const uint4 wu = *reinterpret_cast<const uint4*>(bu + br * r + c0);
                    const uint32_t vg[4] = {wg.x, wg.y, wg.z, wg.w}, vu[4] = {wu.x, wu.y, wu.z, wu.w};
#pragma unroll
                    for (int q2 = 0; q2 < 4; ++q2) {
                        dg = fmaf(__uint_as_float(vg[q2] << 16), tg[c0 + 2 * q2], dg);
                        dg = fmaf(__uint_as_float(vg[q2] & 0xFFFF0000u), tg[c0 + 2 * q2 + 1], dg);
                        du = fmaf(__uint_as_float(vu[q2] << 16), tu[c0 + 2 * q2], du);
                        du = fmaf(__uint_as_float(vu[q2] & 0xFFFF0000u), tu[c0 + 2 * q2 + 1], du);
                    }
                }
                g += L.scale * dg;
                u += L.scale * du;
            }
            publish(dst, silu(g) * u, tag);
        }
    }

    const int KS = K + (sh ? 1 : 0);
    // this CTA's h elements are all published: its ready word carries this launch's tag
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(a.ready + cta), "l"((unsigned long long)s_tag)
                     : "memory");
    }
    // ------------------------------------------------------------ phase X
    // every h element, staged in the swizzled layout (slot k at hs + k Imx; the shared
    // expert at slot K), with 32-element chunk sums.  The routed gate/up windows are read
    // by now (the __syncthreads above): hs and hsum reuse them.
    {
        const uint32_t tag = s_tag;
        // every thread reads its h words once at once (most are published by now), warp 0
        // waits for the ready words of all CTAs (one poll stream per CTA instead of one per h
        // word), then the words that were not yet published are read again.  Element i of the
        // [K+1][Imx] layout: slot i >> imx_sh, place i & (Imx - 1); the places past a slot's
        // length (Is < I or I < Is) are skipped.
        const int nh = KS * Imx, Ish = P.imx_sh;
        unsigned long long w[kQGW];
#pragma unroll
        for (int b = 0; b < kQGW; ++b) {
            const int i = b * kCT + tid, slot = i >> Ish, e = i & (Imx - 1);
            w[b] = (i < nh && e < (slot < K ? I : Is)) ? peek(a.hg + i) : 0ull;
        }
        if (warp == 0) {
            uint32_t pend = 0;  // lane's ready words (CTAs lane + 32 m) without this launch's tag
            for (int m = 0; m < (NB + 31) / 32; ++m)
                if (lane + 32 * m < NB) pend |= 1u << m;
            const uint64_t t0 = tc::globaltimer_ns();
            while (__any_sync(0xffffffffu, pend != 0)) {
                for (int m = 0; m < (NB + 31) / 32; ++m)
                    if ((pend >> m) & 1u) {
                        unsigned long long v;
                        asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(a.ready + lane + 32 * m)
                                     : "memory");
                        if ((uint32_t)v == tag) pend &= ~(1u << m);
                    }
                if (pend && (*(volatile int*)&s_abort || tc::globaltimer_ns() - t0 > lim)) {
                    if (!*(volatile int*)&s_abort) {
                        raise_status(a.status, MOE_ERR_TIMEOUT);
                        s_abort = 1;
                    }
                    pend = 0;
                }
                if (pend) __nanosleep(32);
            }
        }
        __syncthreads();
#pragma unroll
        for (int b = 0; b < kQGW; ++b) {
            const int i = b * kCT + tid, slot = i >> Ish, e = i & (Imx - 1);
            if (i < nh && e < (slot < K ? I : Is) && !fresh(w[b], tag)) w[b] = peek(a.hg + i);
        }
        // (a warp's 32 elements of a pass are one 32-element chunk of one slot: I and Is are
        // multiples of 32, so its chunk sum is one warp reduction).  The passes' values first,
        // then their reductions side by side (one chain of five shuffle steps for all passes,
        // not one chain per pass; the second half only when there are that many words)
        float v[kQGW], cs[kQGW];
#pragma unroll
        for (int b = 0; b < kQGW; ++b) {
            v[b] = fresh(w[b], tag) ? wval(w[b]) : 0.0f;  // (0 past the end: those words read as 0)
            cs[b] = v[b];
        }
        constexpr int kH1 = kQGW / 2;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int b = 0; b < kH1; ++b) cs[b] += __shfl_xor_sync(0xffffffffu, cs[b], o);
        if (nh > kH1 * kCT) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                for (int b = kH1; b < kQGW; ++b) cs[b] += __shfl_xor_sync(0xffffffffu, cs[b], o);
        }
#pragma unroll
        for (int b = 0; b < kQGW; ++b) {
            const int i = b * kCT + tid, slot = i >> Ish, e = i & (Imx - 1);
            if (i - lane < nh && e - lane < (slot < K ? I : Is)) {  // (uniform across the warp)
                hs[slot * Imx + swz(e)] = v[b];
                if (lane == 0) hsum[slot * (Imx / 32) + (e >> 5)] = cs[b];
            }
        }
        __syncthreads();
    }

    // ------------------------------------------------------------ phase D
    for (int j = warp; j < nda_here; j += kCW) {  // down LoRA-A rows -> products to the cluster
        const int d = q * P.nDA + j, k = d / r;
        copies_landed(&s_bar[4], a.status, &s_abort, lim);
        float v = 0.0f;
        if (s_daw[j])
            v = warp_sum(sdot_bf16(reinterpret_cast<const uint16_t*>(s_daw[j]), k < K ? I : Is, hs + k * Imx, lane));
        if (lane < CS) dsm_st(da + d, lane, v);
    }
    cl_arrive();  // (the last stores into other CTAs)
    copies_landed(&s_bar[4], a.status, &s_abort, lim);
    copies_landed(&s_bar[1], a.status, &s_abort, lim);
    if (P.lean) copies_landed(&s_bar[5], a.status, &s_abort, lim);
    if (no > 0 && s_abort == 0) {
        // (output row, expert) tasks: lpt lanes over one row
        int lpt = 1;
        while (lpt * 2 <= 32 && lpt * 2 <= Imx / 32) lpt *= 2;
        const int gpw = 32 / lpt, sub = lane / lpt, sl = lane % lpt;
        const int ntask = no * KS;
        for (int q0 = warp * gpw; q0 < ntask; q0 += kCW * gpw) {
            const int t = q0 + sub;
            const bool live = t < ntask;
            const int ol = live ? t / KS : 0, k = live ? t % KS : 0;
            const bool shu = sh && k == K;
            const int n = shu ? Is : I;
            const moe_qtensor& Wd = shu ? L.s_down : L.down;
            const int ng = n / Wd.group;
            const unsigned char* const* dw = shu ? s_sdw : s_dw[k];
            float acc[1] = {0.0f};
            const int vid[1] = {0};
            if (live && dw[0])
                cdot_int4<1>(reinterpret_cast<const uint32_t*>(dw[0] + (size_t)ol * (n / 2)),
                             reinterpret_cast<const uint16_t*>(dw[1]) + ol * ng,
                             reinterpret_cast<const uint16_t*>(dw[2]) + ol * ng, Wd.group, n, hs + k * Imx,
                             hsum + k * (Imx / 32), vid, 1, acc, sl, lpt);
            const float v = group_sum(acc[0], lpt);
            if (live && sl == 0) sv[ol * KS + k] = v;
        }
    }
    cl_wait();  // the down LoRA-A products of the whole cluster are here
    __syncthreads();
    if (lora && s_abort == 0 && tid < no * KS) {  // per (output row, expert): the LoRA-B delta
        const int ol = tid / KS, k = tid - ol * KS;
        const uint16_t* bd = reinterpret_cast<const uint16_t*>(k < K ? s_rbdw[k] : s_sbw[2]);
        if (bd) {
            float t = 0.0f;
            for (int c0 = 0; c0 < r; c0 += 8) {
                const uint4 wb = *reinterpret_cast<const uint4*>(bd + ol * r + c0);
                const uint32_t vb[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
                for (int q2 = 0; q2 < 4; ++q2) {
                    t = fmaf(__uint_as_float(vb[q2] << 16), da[k * r + c0 + 2 * q2], t);
                    t = fmaf(__uint_as_float(vb[q2] & 0xFFFF0000u), da[k * r + c0 + 2 * q2 + 1], t);
                }
            }
            sv[tid] += L.scale * t;
        }
    }
    __syncthreads();
    if (s_abort == 0 && tid < no) {  // combine in fixed order (k = 0..K-1, then the shared expert)
        const int ol = tid;
        float acc = 0.0f;
        for (int k = 0; k < KS; ++k) acc = fmaf(k < K ? s_w[k] : s_sig, sv[ol * KS + k], acc);
        const int o = o_lo + ol;
        if (a.block) acc += bf16f(xr[o]);
        a.y[o] = f2bf16(acc);
    }
    // no bulk copy may be in flight when the CTA exits (bounded waits)
    if (tid == 0)
        for (int i = 0; i < (P.lean ? 6 : 5); ++i) tc::mbar_wait(&s_bar[i], 0, nullptr, lim);
}

}  // namespace

namespace {

inline size_t r16q(size_t v) { return (v + 15) / 16 * 16; }
inline int cdivq(int a, int b) { return (a + b - 1) / b; }

bool qwin_ok(const moe_qtensor& t) {
    if (!t.packed) return true;
    const size_t rows = (size_t)t.n * t.out;
    const size_t pb = rows * (size_t)t.in * t.bits / 8, sb = rows * (size_t)(t.in / t.group) * 2;
    return ((uintptr_t)t.packed & 15) == 0 && ((uintptr_t)t.scales & 15) == 0 && ((uintptr_t)t.biases & 15) == 0 &&
           pb % 16 == 0 && sb % 16 == 0 && t.group % 32 == 0 &&
           (t.group & (t.group - 1)) == 0;
}

int q_optin_smem() {
    static int v = -1;
    if (v < 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) v = 0;
    }
    return v;
}

size_t q_static_smem() {
    static size_t v = (size_t)-1;
    if (v == (size_t)-1) {
        cudaFuncAttributes at;
        v = cudaFuncGetAttributes(&at, decode_cluster_kernel) == cudaSuccess ? at.sharedSizeBytes : (size_t)1 << 30;
    }
    return v;
}

bool plan_cluster(const LayerArgs& L, int T, int CS, int NB, QPlan* P, bool lean) {
    const bool sh = L.has_shared, lora = L.n_adapters > 0 && L.rank > 0;
    const int H = L.H, E = L.E, K = L.K, I = L.I, Is = sh ? L.Is : 0, r = lora ? L.rank : 0;
    const int Imx = std::max(I, Is), KS = K + (sh ? 1 : 0);
    if (T != 1 || K < 1 || K > kQMaxK || r > 32 || CS < 2 || CS > kQMaxCS || NB < CS || NB % CS ||
        NB > MOEQ_DECODE_MAX_CTAS)
        return false;
    if (E > kQMaxE || H % 32 || H > 4096 || I % 32 || I > 4096 || (sh && (Is % 32 || Is > 4096))) return false;
    if (!qwin_ok(L.router) || !qwin_ok(L.gate) || !qwin_ok(L.up) || !qwin_ok(L.down)) return false;
    if (L.has_sgate && (((uintptr_t)L.shared_gate.packed & 15) || L.shared_gate.bits != 8 ||
                        L.shared_gate.group % 32 || (L.shared_gate.group & (L.shared_gate.group - 1))))
        return false;
    if (sh && (!qwin_ok(L.s_gate) || !qwin_ok(L.s_up) || !qwin_ok(L.s_down))) return false;
    if (L.router.bits != 8 || L.gate.bits != 4 || L.up.bits != 4 || L.down.bits != 4) return false;
    if (sh && (L.s_gate.bits != 4 || L.s_up.bits != 4 || L.s_down.bits != 4)) return false;
    if (lora) {  // LoRA rows move by bulk copies: 16-byte aligned factors, rows of whole 16-byte pieces
        if (r % 8) return false;
        for (int ad = 0; ad < L.n_adapters; ++ad) {
            const moe_lora_proj* p[6] = {&L.lora[ad].gate, &L.lora[ad].up, &L.lora[ad].down,
                                         &L.lora[ad].s_gate, &L.lora[ad].s_up, &L.lora[ad].s_down};
            for (int k = 0; k < 6; ++k)
                if ((p[k]->A && ((uintptr_t)p[k]->A & 15)) || (p[k]->B && ((uintptr_t)p[k]->B & 15))) return false;
        }
    }
    if (Imx & (Imx - 1) || KS * Imx > kQGW * kCT) return false;  // (h gathered over [K+1][Imx] by shifts)
    P->CS = CS;
    P->lean = lean ? 1 : 0;
    P->imx_sh = 0;
    while ((1 << P->imx_sh) < Imx) ++P->imx_sh;
    if (I & (I - 1)) return false;  // (h elements are split into (expert, row) by shifts)
    P->i_sh = 0;
    while ((1 << P->i_sh) < I) ++P->i_sh;
    P->perA = cdivq(E, CS);
    P->perS = sh ? cdivq(Is, NB) : 0;
    P->perO = cdivq(H, NB);
    P->perC = cdivq(K * I, NB);
    P->nSA = (lora && sh) ? cdivq(2 * r, CS) : 0;
    P->nRA = lora ? cdivq(K * 2 * r, CS) : 0;
    P->nDA = lora ? cdivq(KS * r, CS) : 0;
    if (P->perO > kQMaxO || P->perC > I || P->perC > 8 * kQMaxGT || P->nSA > kQMaxSA || P->nRA > kQMaxRA ||
        P->nDA > kQMaxDA)
        return false;
    // the gate/up tiles: one group size for gate and up, 32, 64 or 128
    if (L.gate.group != L.up.group || (L.gate.group != 32 && L.gate.group != 64 && L.gate.group != 128)) return false;
    if ((H / L.gate.group) % 4) return false;  // (whole tasks of four groups)

    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o = r16q(o + bytes);
        return (uint32_t)at;
    };
    auto slack = [](size_t bytes) { return bytes ? r16q(bytes) + 32 : 0; };
    P->xraw = take((size_t)H * 2);
    P->xs = take((size_t)H * 4);
    P->xsum = take((size_t)(H / 32) * 4);
    P->z = take((size_t)E * 4);
    P->sa = take((size_t)2 * std::max(r, 1) * 4);
    P->ra = take((size_t)K * 2 * std::max(r, 1) * 4);
    P->da = take((size_t)KS * std::max(r, 1) * 4);
    {  // phase-R windows
        size_t wsz = 0;
        const int ng = H / L.router.group;
        const size_t rsz[3] = {(size_t)P->perA * H, (size_t)P->perA * ng * 2, (size_t)P->perA * ng * 2};
        for (int k = 0; k < 3; ++k) {
            P->r_off[k] = (uint32_t)wsz;
            wsz += slack(rsz[k]);
        }
        for (int pj = 0; pj < 2; ++pj) {
            const moe_qtensor& qt = pj ? L.s_up : L.s_gate;
            const int ngs = (sh && qt.packed) ? H / qt.group : 0;
            const size_t ssz[3] = {(size_t)P->perS * H / 2, (size_t)P->perS * ngs * 2, (size_t)P->perS * ngs * 2};
            for (int k = 0; k < 3; ++k) {
                P->sg_off[3 * pj + k] = (uint32_t)wsz;
                wsz += sh ? slack(ssz[k]) : 0;
            }
        }
        {
            const int ngg = L.has_sgate ? H / L.shared_gate.group : 0;
            const size_t gsz[3] = {(size_t)H, (size_t)ngg * 2, (size_t)ngg * 2};
            for (int k = 0; k < 3; ++k) {
                P->sg_off[6 + k] = (uint32_t)wsz;
                wsz += L.has_sgate ? slack(gsz[k]) : 0;
            }
        }
        P->ra_stride = (uint32_t)slack((size_t)H * 2);
        const size_t rasz = (size_t)P->nRA * P->ra_stride;
        P->wr = take(lean ? std::max(wsz, rasz) : wsz);
        P->wsg = P->wr;
        P->wra = lean ? P->wr : take(rasz);
    }
    {
        const int ngd = sh ? Is / L.s_down.group : 0;
        const size_t sz[3] = {(size_t)P->perO * Is / 2, (size_t)P->perO * ngd * 2, (size_t)P->perO * ngd * 2};
        size_t wsz = 0;
        for (int k = 0; k < 3; ++k) {
            P->sd_off[k] = (uint32_t)wsz;
            wsz += slack(sz[k]);
        }
        P->wsd = take(wsz);
    }
    P->sa_stride = (uint32_t)slack((size_t)H * 2);
    P->wsa = take((size_t)P->nSA * P->sa_stride);
    P->sb_stride = (uint32_t)slack((size_t)std::max(P->perS, P->perO) * std::max(r, 1) * 2);
    P->wsb = take(lora && sh ? (size_t)3 * P->sb_stride : 0);
    {  // routed gate/up windows: a padded slot per row, two segments per scales/biases part;
        // then h and its chunk sums in the same space
        P->rrs = (uint32_t)(H / 2 + 16);
        const size_t gp = (size_t)P->perC * P->rrs;
        const size_t gs = (size_t)P->perC * (H / L.gate.group) * 2, us = (size_t)P->perC * (H / L.up.group) * 2;
        const size_t cpart[6] = {gp, gs, gs, gp, us, us};
        size_t wsz = 0;
        for (int k = 0; k < 6; ++k) {
            P->c_off[k] = (uint32_t)wsz;
            wsz += r16q(cpart[k]) + 64;
        }
        const size_t hbytes = r16q((size_t)KS * Imx * 4), hsbytes = r16q((size_t)KS * (Imx / 32) * 4);
        P->dp_stride = (uint32_t)slack((size_t)P->perO * I / 2);
        const size_t dpbytes = (size_t)K * P->dp_stride;
        P->wc = take(std::max(wsz, hbytes + hsbytes + (lean ? dpbytes : 0)));
        P->hs = P->wc;
        P->hsum = P->wc + (uint32_t)hbytes;
        P->dp = lean ? P->wc + (uint32_t)(hbytes + hsbytes) : take(dpbytes);
    }
    P->rb_stride = (uint32_t)slack((size_t)P->perC * std::max(r, 1) * 2);
    P->wrb = take(lora ? (size_t)4 * P->rb_stride : 0);
    {
        const int ngd = I / L.down.group;  // (scales and biases of slot k; its packed rows at dp)
        P->d_off[0] = 0;
        P->d_off[1] = 0;
        P->d_off[2] = (uint32_t)slack((size_t)P->perO * ngd * 2);
        P->d_stride = P->d_off[2] + (uint32_t)slack((size_t)P->perO * ngd * 2);
        P->wd = take((size_t)K * P->d_stride);
    }
    P->rbd_stride = (uint32_t)slack((size_t)P->perO * std::max(r, 1) * 2);
    P->wrbd = take(lora ? (size_t)K * P->rbd_stride : 0);
    P->da_stride = (uint32_t)slack((size_t)Imx * 2);
    P->wda = take((size_t)P->nDA * P->da_stride);
    P->xp = take((size_t)H * 2);
    {
        const int ngr = H / L.gate.group, ntm = (P->perC + 7) / 8;
        // one task per slice of the smallest size (2 groups; 4 at group 32)
        P->gu_spg = L.gate.group == 32 ? 4 : 2;
        P->gu_ns = ngr / P->gu_spg;
        P->gu_gsh = L.gate.group == 32 ? 0 : L.gate.group == 64 ? 1 : 2;
        P->gpart = take((size_t)ntm * P->gu_ns * 16 * 4);
    }
    P->sgu = take((size_t)std::max(P->perS, 1) * 2 * 4);
    P->sv = take((size_t)P->perO * KS * 4);
    P->total = (uint32_t)o;
    const size_t limit = (size_t)q_optin_smem() > q_static_smem() ? (size_t)q_optin_smem() - q_static_smem() : 0;
    return o <= limit;
}

// Cluster shapes this device runs with one CTA per SM, larger clusters first: CTAs per
// cluster and clusters resident at once (queried once).  A larger cluster splits the
// per-cluster work (router rows, LoRA-A rows) finer; on a B200 16-CTA clusters leave
// 112 SMs busy, 8-CTA clusters 120.
struct QShape {
    int CS = 0, NC = 0;
};
constexpr int kQShapes = 2;

const QShape* q_shapes() {
    static QShape s[kQShapes];
    static bool done = false;
    if (done) return s;
    done = true;
    const int want = q_optin_smem() - (int)std::min<size_t>(q_static_smem(), 1 << 20);
    if (want <= 0) return s;
    if (cudaFuncSetAttribute(decode_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, want) != cudaSuccess ||
        cudaFuncSetAttribute(decode_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
        (void)cudaGetLastError();
        return s;
    }
    const int sizes[kQShapes] = {16, 8};
    for (int i = 0; i < kQShapes; ++i) {
        const int cs = sizes[i];
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(cs);
        cfg.blockDim = dim3(kCT);
        cfg.dynamicSmemBytes = (size_t)want;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = cs;
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        int nc = 0;
        if (cudaOccupancyMaxActiveClusters(&nc, decode_cluster_kernel, &cfg) != cudaSuccess) {
            (void)cudaGetLastError();
            nc = 0;
        }
        s[i].CS = cs;
        s[i].NC = std::min(nc, MOEQ_DECODE_MAX_CTAS / cs);
    }
    return s;
}

// The first cluster shape whose plan fits this layer, or nullptr.
const QShape* q_pick(const LayerArgs& L, int T, QPlan* P) {
    const QShape* s = q_shapes();
    for (int i = 0; i < kQShapes; ++i)
        if (s[i].NC >= 4 && (plan_cluster(L, T, s[i].CS, s[i].CS * s[i].NC, P, false) ||
                             plan_cluster(L, T, s[i].CS, s[i].CS * s[i].NC, P, true)))
            return &s[i];
    return nullptr;
}

}  // namespace

// Words (8 bytes) of the cluster kernel's workspace region: its ticket counter and
// spares, the tagged h words [K+1][max(I, Is)], and one ready word per CTA.
size_t cluster_slot_words(int K, int I, int Is) {
    return 8 + (size_t)(K + 1) * std::max(I, Is) + MOEQ_DECODE_MAX_CTAS;
}

bool cluster_supported(const LayerArgs& L, int T) {
    QPlan P;
    return T == 1 && q_pick(L, T, &P) != nullptr;
}

cudaError_t launch_cluster(const LayerArgs& L, const uint16_t* x, const int32_t* adapter_id, const int32_t* select,
                           uint16_t* y, int T, int block, float eps, const ClusterScratch& sc, cudaStream_t s) {
    QArgs a;
    memset(&a, 0, sizeof(a));
    const QShape* sp = T == 1 ? q_pick(L, T, &a.P) : nullptr;
    if (!sp) return cudaErrorNotSupported;
    a.L = L;
    a.x = x;
    a.adapter_id = adapter_id;
    a.select = select;
    a.y = y;
    a.block = block;
    a.eps = eps;
    a.x_host = sc.x_host;
    a.tick = reinterpret_cast<unsigned long long*>(sc.slots);
    a.hg = sc.slots + 8;
    a.ready = reinterpret_cast<unsigned long long*>(sc.slots + 8 + (size_t)(L.K + 1) * std::max(L.I, L.has_shared ? L.Is : 0));
    a.status = sc.status;
    a.idx_out = sc.idx_out;
    a.w_out = sc.w_out;
    a.wait_ns = wait_limit_ns();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sp->CS * sp->NC);
    cfg.blockDim = dim3(kCT);
    cfg.dynamicSmemBytes = a.P.total;
    cfg.stream = s;
    cudaLaunchAttribute attr[3];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = sp->CS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeCooperative;
    attr[1].val.cooperative = 1;
    attr[2].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[2].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    // MOEQ_NCU_COMPAT=1 (read once): the cluster attribute alone.  ncu cannot replay the
    // kernel launched as a cooperative programmatic dependent; without those attributes the
    // grid (the device's resident cluster count, one CTA per SM) still runs all at once on
    // an otherwise idle GPU, which is how a profiling run has it.
    static const bool compat = [] {
        const char* e = getenv("MOEQ_NCU_COMPAT");
        return e && e[0] == '1';
    }();
    cfg.numAttrs = compat ? 1 : 3;
    return cudaLaunchKernelEx(&cfg, decode_cluster_kernel, a);
}

}  // namespace moeq
