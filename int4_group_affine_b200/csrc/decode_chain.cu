// decode_chain.cu - the MoE layer for one to four tokens as one persistent,
// cooperative kernel whose hand-offs between CTAs are epoch-tagged words.
//
// At decode the layer is a chain of dependent steps (router -> top-K -> expert
// rows -> down rows), each far too small to fill the GPU, so its time is the
// sum of the steps' latencies.  This kernel keeps every step at one memory
// round trip and puts no grid-wide barrier on the chain:
//  - every value one CTA hands to others (a router logit, a LoRA-A product, an
//    activation h, a partial down LoRA-A sum) is published as one 64-bit word
//    {value, tag} with a single store, and a consumer polls the words it needs
//    until they carry this launch's tag: an exchange costs one store and one
//    L2 round trip, and a CTA moves on as soon as its own inputs are there;
//  - the tag comes from one ticket per CTA on a 64-bit counter in the
//    workspace header (a launch adds gridDim.x), taken at launch and first
//    needed at the first publication;
//  - each CTA's share of a step's weight rows is a contiguous range of each
//    tensor, moved into shared memory by bulk copies completing on an
//    mbarrier, issued as soon as the range is known: the router, shared-expert
//    and shared LoRA rows at launch, the routed rows right after top-K;
//  - the routed LoRA-A products are spread over all CTAs, one or two rows each.
//
//  R  x, the CTA's router rows, the shared-gate row (every CTA), its shared
//     gate/up rows; logits and shared LoRA-A products are published.
//  K  every CTA polls the logits, takes the top-K of each token, groups the
//     routed jobs by expert and issues its routed windows.
//  G  shared-expert h; routed LoRA-A products (published); routed gate/up dots,
//     LoRA-B delta, SwiGLU: h and the partial down LoRA-A sums published.
//  D  every CTA polls h and the partial sums, computes its output rows for
//     every job and combines them in fixed order (k = 0..K-1, then the shared
//     expert), adding the residual in block mode.
#include <algorithm>
#include <cstring>

#include "decode_cdots.cuh"

namespace moeq {
namespace {

constexpr int kCMaxT = 4;     // tokens
constexpr int kCMaxTK = 16;   // routed jobs T*K (so also distinct routed experts)
constexpr int kCMaxR = 32;    // LoRA rank: one lane per component
constexpr int kCMaxO = 32;    // output rows per CTA
constexpr int kCMaxSA = 4;    // shared-expert LoRA-A dots per CTA
constexpr int kCMaxRA = 8;    // routed LoRA-A dots per CTA

// Shared-memory plan and per-CTA ranges (host-computed; the routed row ranges are
// recomputed on the device from the actual number of distinct experts).
struct CPlan {
    int perA, perS, perO, perCmax, nSA, nRA, Umax;
    uint32_t xraw, xs, xsum, z, sax;
    uint32_t wa, a_off[12];      // router p/s/b, shared gate p/s/b, s_gate p/s/b, s_up p/s/b
    uint32_t wsd, sd_off[3];     // shared down rows p/s/b
    uint32_t wsa, sa_stride;     // shared LoRA-A rows
    uint32_t wsb, sb_stride;     // shared LoRA-B rows [T][gate, up, down]
    uint32_t wc, c_off[6];       // routed gate/up rows {gate, up} x {p, s, b}, two segments each
    uint32_t wd, d_off[3], d_stride;  // routed down rows of distinct expert u at wd + u * d_stride
    uint32_t wra, ra_stride;     // routed LoRA-A rows
    uint32_t wrb, rb_stride;     // routed LoRA-B gate/up rows [segment][token slot][gate, up]
    uint32_t wrbd, rbd_stride;   // routed LoRA-B down rows [routed job]
    uint32_t sgu, hs, hsum, td, wpart, sv;
    uint32_t gat, gat_n;         // gather space for the partial sums (aliases the gate/up windows)
    uint32_t total;
};

struct CArgs {
    LayerArgs L;
    const uint16_t* x;
    const int32_t* adapter_id;
    const int32_t* select;     // [T][K] caller-given expert sets, or NULL: top-K of the logits
    uint16_t* y;
    int T, block;
    float eps;
    unsigned long long* tick;  // ticket counter: a launch adds gridDim.x
    unsigned long long* hcnt;  // arrivals after publishing h: a launch adds gridDim.x
    unsigned long long* rflag; // tag of the last routing CTA 0 published
    uint64_t* zs;              // [T][E] tagged logits (polled by CTA 0)
    uint64_t* sax;             // [T][2r] tagged shared LoRA-A products (gate | up)
    uint64_t* rax;             // [TK][2r] tagged routed LoRA-A products, routed slot t*K+k
    uint64_t* route;           // [T][K] {expert, weight} published by CTA 0
    float* hx;                 // [J][Imax] h: routed slot t*K+k, shared T*K+t
    float* part;               // [NB][3][T][r] partial down LoRA-A sums: segment 0, 1, shared
    int32_t* status;
    int32_t* idx_out;          // [T][K] routing record
    float* w_out;
    uint64_t wait_ns;
    CPlan P;
};

template <int MT>
__global__ void __launch_bounds__(kCT, 1) decode_chain_kernel(const __grid_constant__ CArgs a_param) {
    extern __shared__ __align__(16) unsigned char sm[];
    // The arguments (layer descriptor, adapter table, plan: about 2.3 KB) are read all over
    // the kernel, most fields once; copied to shared memory by all threads at once, they
    // cost one round trip here instead of a cold constant-cache miss at each first use.
    __shared__ __align__(16) CArgs a_sm;
    static_assert(sizeof(CArgs) % 4 == 0, "argument copy in words");
    for (int i = threadIdx.x; i < (int)(sizeof(CArgs) / 4); i += kCT)
        reinterpret_cast<uint32_t*>(&a_sm)[i] = reinterpret_cast<const uint32_t*>(&a_param)[i];
    __syncthreads();
    const CArgs& a = a_sm;
    // the next kernel on the stream may launch now; it waits for this grid before it
    // reads anything this grid writes
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const LayerArgs& L = a.L;
    const CPlan& P = a.P;
    const int T = a.T, H = L.H, E = L.E, K = L.K, I = L.I;
    const bool sh = L.has_shared;
    const int Is = sh ? L.Is : 0;
    const int TK = T * K;
    const int NB = gridDim.x, cta = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool lora = L.n_adapters > 0 && L.rank > 0;
    const int r = lora ? L.rank : 0;
    const int J = TK + (sh ? T : 0);
    const uint64_t lim = a.wait_ns;

    float* xs = reinterpret_cast<float*>(sm + P.xs);      // [T][H] staged input (swizzled)
    float* xsum = reinterpret_cast<float*>(sm + P.xsum);  // [T][H/32]
    float* z = reinterpret_cast<float*>(sm + P.z);        // [T][E] logits
    float* sgu = reinterpret_cast<float*>(sm + P.sgu);    // [perS][T][2] shared gate/up pre-activations
    float* hsm = reinterpret_cast<float*>(sm + P.hs);     // routed h [TK][I], then shared [T][Is] (swizzled)
    float* hsum = reinterpret_cast<float*>(sm + P.hsum);
    float* tds = reinterpret_cast<float*>(sm + P.td);     // [J][r] down LoRA-A products
    float* wpart = reinterpret_cast<float*>(sm + P.wpart);  // [kCW][3][MT][r]
    float* sv = reinterpret_cast<float*>(sm + P.sv);      // [perO][J] per-job outputs of this CTA's rows
    float* gat = reinterpret_cast<float*>(sm + P.gat);

    __shared__ __align__(8) uint64_t s_bar[5];
    __shared__ int s_abort;
    __shared__ uint32_t s_tag;
    __shared__ unsigned long long s_hdone;
    __shared__ int s_aid[kCMaxT];
    __shared__ int32_t s_sel[kCMaxTK];
    __shared__ float s_inv[kCMaxT], s_sig[kCMaxT];
    __shared__ int s_idx[kCMaxT][MOEQ_MAX_TOPK];
    __shared__ float s_w[kCMaxT][MOEQ_MAX_TOPK];
    __shared__ int s_nu, s_perC;
    __shared__ int s_uexp[kCMaxTK], s_ucnt[kCMaxTK], s_uslot[kCMaxTK][kCMaxT];
    __shared__ int s_ju[kCMaxTK], s_jm[kCMaxTK], s_sorted[kCMaxTK];
    __shared__ int s_goff[kCMaxTK + kCMaxT + 1];
    __shared__ const unsigned char* s_aw[12];
    __shared__ const unsigned char* s_sdw[3];
    __shared__ const unsigned char* s_saw[kCMaxSA];
    __shared__ const unsigned char* s_sbw[kCMaxT][3];
    __shared__ const unsigned char* s_cw[2][6];
    __shared__ const unsigned char* s_dw[kCMaxTK][3];
    __shared__ const unsigned char* s_raw[kCMaxRA];
    __shared__ const unsigned char* s_rbw[2][MT][2];
    __shared__ const unsigned char* s_rbdw[kCMaxTK];

    // barrier 0: x and the phase-R rows; 1: shared down rows (warp 0) + shared LoRA rows
    // (warp 1); 2: routed LoRA-A rows; 3: routed gate/up rows (warp 0) + their LoRA-B rows
    // (warp 1); 4: routed down rows and their LoRA-B rows
    if (tid == 0) {
        s_abort = 0;
        for (int i = 0; i < 5; ++i) tc::mbar_init(&s_bar[i], (i == 1 || i == 3) ? 2u : 1u);
        tc::mbar_init_fence();
    }
    if (tid < T) s_sig[tid] = 1.0f;
    __syncthreads();

    const int ra0 = min(E, cta * P.perA), ra1 = min(E, ra0 + P.perA), nra = ra1 - ra0;
    const int s_lo = min(Is, cta * P.perS), s_hi = min(Is, s_lo + P.perS), nsr = s_hi - s_lo;
    const int o_lo = min(H, cta * P.perO), o_hi = min(H, o_lo + P.perO), no = o_hi - o_lo;

    // ------------------------------------------------------------ phase R: issue
    // The weight rows of this phase depend on nothing the previous kernel on the stream
    // writes: their copies start before the grid-dependency wait (launched as a
    // programmatic dependent, this kernel's CTAs get here while that kernel finishes).
    // Everything that reads the workspace, x or the adapter ids comes after the wait.
    unsigned long long prev = 0;  // this launch's ticket (first needed after x is staged)
    if (warp == 0) {
        uint32_t tx = 0;
        unsigned char* wa = sm + P.wa;
        if (lane >= 1 && lane < 13) {
            const int w = lane - 1, k = w % 3, g = w / 3;  // g: router, shared gate, s_gate, s_up
            const moe_qtensor& q = g == 0 ? L.router : g == 1 ? L.shared_gate : g == 2 ? L.s_gate : L.s_up;
            if (g == 1) {  // the shared-gate row is read by every CTA straight from global memory (L2)
                s_aw[w] = !L.has_sgate ? nullptr
                          : k == 0     ? reinterpret_cast<const unsigned char*>(q.packed)
                                       : reinterpret_cast<const unsigned char*>(k == 1 ? q.scales : q.biases);
            } else {
                const int bits = g < 2 ? 8 : 4;
                const int row0 = g == 0 ? ra0 : s_lo;
                const int n = g == 0 ? nra : nsr;
                const int ng = q.packed ? H / q.group : 0;
                const void* src = nullptr;
                uint32_t bytes = 0;
                if (n > 0 && q.packed) {
                    src = k == 0 ? (const void*)(q.packed + (int64_t)row0 * (H * bits / 32))
                                 : (const void*)((k == 1 ? q.scales : q.biases) + (int64_t)row0 * ng);
                    bytes = k == 0 ? (uint32_t)(n * H * bits / 8) : (uint32_t)(n * ng * 2);
                }
                s_aw[w] = win(wa + P.a_off[w], src, bytes, &s_bar[0], &tx);
            }
        }
        uint32_t tx1 = 0;
        if (lane < 3) {  // the shared-expert down rows of this CTA's output range
            const int ngd = sh ? Is / L.s_down.group : 0;
            const void* src = nullptr;
            uint32_t bytes = 0;
            if (sh && no > 0) {
                src = lane == 0 ? (const void*)(L.s_down.packed + (int64_t)o_lo * (Is / 8))
                                : (const void*)((lane == 1 ? L.s_down.scales : L.s_down.biases) + (int64_t)o_lo * ngd);
                bytes = lane == 0 ? (uint32_t)(no * Is / 2) : (uint32_t)(no * ngd * 2);
            }
            s_sdw[lane] = win(sm + P.wsd + P.sd_off[lane], src, bytes, &s_bar[1], &tx1);
        }
        tx1 = warp_total(tx1);
        if (lane == 0) tc::mbar_arrive_expect_tx(&s_bar[1], tx1);
        asm volatile("griddepcontrol.wait;" ::: "memory");
        if (lane == 0) win(sm + P.xraw, a.x, (uint32_t)(T * H * 2), &s_bar[0], &tx);
        tx = warp_total(tx);
        if (lane == 0) tc::mbar_arrive_expect_tx(&s_bar[0], tx);
    } else if (warp == 1) {
        // adapter ids, then the shared-expert LoRA rows this CTA needs
        asm volatile("griddepcontrol.wait;" ::: "memory");
        if (lane < T) {
            int ad = a.adapter_id ? a.adapter_id[lane] : (L.n_adapters > 0 ? 0 : -1);
            if (ad < -1 || ad >= L.n_adapters) {
                if (cta == 0) raise_status(a.status, MOE_ERR_DEVICE_INDEX);
                ad = -1;
            }
            s_aid[lane] = ad;
        }
        if (a.select && lane < TK) s_sel[lane] = a.select[lane];
        __syncwarp();
        uint32_t tx = 0;
        if (lane < P.nSA) {  // LoRA-A rows of this CTA's shared LoRA-A dots: dot q = cta + NB * lane
            const int q = cta + NB * lane;
            const moe_lora_proj* lp = nullptr;
            int d = 0;
            if (lora && sh && q < T * 2 * r) {
                d = q % (2 * r);
                lp = dlora(L, s_aid[q / (2 * r)], true, d < r ? 0 : 1);
            }
            s_saw[lane] = win(sm + P.wsa + lane * P.sa_stride, lp ? lp->A + (int64_t)(d % r) * H : nullptr,
                              (uint32_t)(H * 2), &s_bar[1], &tx);
        } else if (lane >= 8 && lane < 8 + 3 * T) {  // LoRA-B rows: [token][gate, up, down]
            const int t = (lane - 8) / 3, w = (lane - 8) % 3;
            const moe_lora_proj* lp = (lora && sh) ? dlora(L, s_aid[t], true, w) : nullptr;
            const int row0 = w < 2 ? s_lo : o_lo, n = w < 2 ? nsr : no;
            s_sbw[t][w] = win(sm + P.wsb + (t * 3 + w) * P.sb_stride, lp ? lp->B + (int64_t)row0 * r : nullptr,
                              (uint32_t)(n * r * 2), &s_bar[1], &tx);
        }
        tx = warp_total(tx);
        if (lane == 0) tc::mbar_arrive_expect_tx(&s_bar[1], tx);
    }

    if (warp >= 2) {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        if (warp == kCW - 1 && lane == 0)
            asm volatile("atom.add.relaxed.gpu.global.u64 %0, [%1], 1;" : "=l"(prev) : "l"(a.tick) : "memory");
    }

    // ------------------------------------------------------------ phase R: compute
    if (!copies_landed(&s_bar[0], a.status, &s_abort, lim)) {
        // the input never arrived: the rest runs on zeros and publishes them
    }
    const uint16_t* xr = reinterpret_cast<const uint16_t*>(sm + P.xraw);
    if (a.block) {  // RMSNorm scale of each token (warp t)
        for (int t = warp; t < T; t += kCW) {
            float ss = 0.0f;
            const uint4* xv = reinterpret_cast<const uint4*>(xr + (int64_t)t * H);
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
            if (lane == 0) s_inv[t] = 1.0f / sqrtf(ss / (float)H + a.eps);
        }
        __syncthreads();
    }
    cstage_bf16(xs, xsum, xr, T, H, a.block ? s_inv : nullptr);
    if (warp == kCW - 1 && lane == 0) {
        s_tag = (uint32_t)((prev / (unsigned long long)NB) % 0xffffffffull) + 1u;
        s_hdone = (prev / (unsigned long long)NB + 1) * (unsigned long long)NB;  // h arrivals complete at this count
    }
    __syncthreads();
    const uint32_t tag = s_tag;

    {
        // router rows first, on warps 2.. (warps 0 and 1 issued the copies, the last warp
        // took the ticket)
        const int nsg = L.has_sgate ? 1 : 0;
        const int ntask = nra + nsg + nsr;
        for (int j = (warp + kCW - 2) % kCW; j < ntask; j += kCW) {
            if (j < nra + nsg) {  // router row or the shared-expert gate row (int8)
                const bool sg = j >= nra;
                const moe_qtensor& q = sg ? L.shared_gate : L.router;
                const int ng = H / q.group, jj = sg ? 0 : j;
                const unsigned char* const* w = s_aw + (sg ? 3 : 0);
                float acc[MT];
#pragma unroll
                for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
                if (w[0])
                    cdot_int8<MT>(reinterpret_cast<const uint32_t*>(w[0] + (size_t)jj * H),
                                 reinterpret_cast<const uint16_t*>(w[1]) + jj * ng,
                                 reinterpret_cast<const uint16_t*>(w[2]) + jj * ng, q.group, H, xs, xsum, T, acc, lane);
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m >= T) break;
                    const float v = warp_sum(acc[m]);
                    if (lane == 0) {
                        if (sg) {
                            s_sig[m] = 1.0f / (1.0f + expf(-v));
                        } else {
                            const int row = ra0 + j;
                            publish(a.zs + (int64_t)m * E + row, v + (L.logit_bias ? L.logit_bias[row] : 0.0f), tag);
                        }
                    }
                }
            } else if (j < nra + nsg + nsr) {  // shared-expert gate and up rows
                const int il = j - nra - nsg;
                const int ngg = H / L.s_gate.group, ngu = H / L.s_up.group;
                float ag[MT], au[MT];
                int vid[MT];
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    ag[m] = au[m] = 0.0f;
                    vid[m] = m;
                }
                cdot_int4<MT>(reinterpret_cast<const uint32_t*>(s_aw[6] + (size_t)il * (H / 2)),
                             reinterpret_cast<const uint16_t*>(s_aw[7]) + il * ngg,
                             reinterpret_cast<const uint16_t*>(s_aw[8]) + il * ngg, L.s_gate.group, H, xs, xsum, vid, T,
                             ag, lane, 32);
                cdot_int4<MT>(reinterpret_cast<const uint32_t*>(s_aw[9] + (size_t)il * (H / 2)),
                             reinterpret_cast<const uint16_t*>(s_aw[10]) + il * ngu,
                             reinterpret_cast<const uint16_t*>(s_aw[11]) + il * ngu, L.s_up.group, H, xs, xsum, vid, T,
                             au, lane, 32);
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m >= T) break;
                    const float g = warp_sum(ag[m]), u = warp_sum(au[m]);
                    if (lane == 0) {
                        sgu[(il * T + m) * 2] = g;
                        sgu[(il * T + m) * 2 + 1] = u;
                    }
                }
            }
        }
    }

    // ------------------------------------------------------------ phase K
    // CTA 0 alone polls the logits, takes the top-K of each token (warp t for token t)
    // and publishes the routing behind one release flag; every other CTA polls that
    // flag with one thread, so no line is polled by the whole grid.
    if (cta == 0) {
        gather_range(a.zs, T * E, z, tag, a.status, &s_abort, lim);
        __syncthreads();
        if (warp < T) {
            const int t = warp;
            if (a.select) {  // caller-given sets (the prerouter's prediction): only the weights come from z
                bool bad = false;
                const int e = select_entry(s_sel + t * K, K, E, lane, &bad);
                if (bad && lane == 0) raise_status(a.status, MOE_ERR_DEVICE_INDEX);
                const float zk = e >= 0 ? z[t * E + e] : -INFINITY;
                const float m = warp_max(zk);
                const float ev = e >= 0 ? expf(zk - m) : 0.0f;
                const float sum = warp_sum(ev);
                if (lane < K) {
                    s_idx[t][lane] = e;
                    s_w[t][lane] = ev / sum;
                }
            } else {
                warp_topk<MOEQ_MAX_EXPERTS / 32>(z + t * E, E, K, lane, s_idx[t], s_w[t]);
            }
        }
        __syncthreads();
        if (warp == 0) {
            if (lane < TK) {
                const int e = s_idx[lane / K][lane % K];
                const float w = s_w[lane / K][lane % K];
                a.route[lane] = ((unsigned long long)__float_as_uint(w) << 32) | (uint32_t)e;
                a.idx_out[lane] = e;  // the routing this call used, for the caller's record
                a.w_out[lane] = w;
            }
            __syncwarp();
            if (lane == 0) {
                __threadfence();
                asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(a.rflag), "l"((unsigned long long)tag)
                             : "memory");
            }
        }
    } else if (warp == 0) {
        if (lane == 0) wait_word(a.rflag, tag, false, a.status, &s_abort, lim);
        __syncwarp();
        if (lane < TK) {
            const unsigned long long v = ld_acq64(reinterpret_cast<const unsigned long long*>(a.route) + lane);
            s_idx[lane / K][lane % K] = (int)min((uint32_t)v, (uint32_t)(E - 1));  // (in range even after a timeout)
            s_w[lane / K][lane % K] = __uint_as_float((uint32_t)(v >> 32));
        }
        __syncwarp();
    }
    if (warp == 0) {
        // routed jobs (lane = slot t*K+k) grouped by expert, ascending, then by slot
        const bool live = lane < TK;
        const int je = live ? s_idx[lane / K][lane % K] : 0x7fffffff;
        int rank = 0;
        for (int j = 0; j < TK; ++j) {
            const int ej = __shfl_sync(0xffffffffu, je, j);
            rank += (ej < je || (ej == je && j < lane)) ? 1 : 0;
        }
        if (live) s_sorted[rank] = lane;
        __syncwarp();
        const int jp = live ? s_sorted[lane] : 0;
        const int ep = live ? s_idx[jp / K][jp % K] : -1;
        const int eprev = __shfl_up_sync(0xffffffffu, ep, 1);
        const bool first = live && (lane == 0 || eprev != ep);
        const uint32_t fm = __ballot_sync(0xffffffffu, first);
        if (live) {
            const uint32_t upto = fm & (0xffffffffu >> (31 - lane));
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
        const int U = __popc(fm);
        const int perC = (U * I + NB - 1) / NB;
        if (lane == 0) {
            s_nu = U;
            s_perC = perC;
        }
        // this CTA's routed gate/up rows: lane 6 s + 3 p + k issues one window (segment s,
        // gate | up, packed | scales | biases)
        const int nC = U * I, c_lo = min(nC, cta * perC), c_hi = min(nC, c_lo + perC);
        const int cut = c_hi > c_lo ? min(c_hi, (c_lo / I + 1) * I) : c_lo;
        uint32_t tx = 0;
        __syncwarp();
        if (lane < 12) {
            const int sgi = lane / 6, pj = (lane / 3) % 2, k = lane % 3, part = 3 * pj + k;
            const int q0 = sgi == 0 ? c_lo : cut, q1 = sgi == 0 ? cut : c_hi;
            const void* src = nullptr;
            uint32_t bytes = 0, off = P.wc + P.c_off[part];
            const moe_qtensor& q = pj ? L.up : L.gate;
            const int ng = H / q.group;
            if (q1 > q0 && s_abort == 0) {
                const int64_t row = (int64_t)s_uexp[q0 / I] * I + q0 % I;
                src = k == 0 ? (const void*)(q.packed + row * (H / 8))
                             : (const void*)((k == 1 ? q.scales : q.biases) + row * ng);
                bytes = k == 0 ? (uint32_t)(q1 - q0) * (H / 2) : (uint32_t)(q1 - q0) * ng * 2;
                if (sgi == 1 && cut > c_lo) {  // segment 1's window follows segment 0's
                    const int64_t row0 = (int64_t)s_uexp[c_lo / I] * I + c_lo % I;
                    const void* src0 = k == 0 ? (const void*)(q.packed + row0 * (H / 8))
                                              : (const void*)((k == 1 ? q.scales : q.biases) + row0 * ng);
                    off += win_span(src0, k == 0 ? (uint32_t)(cut - c_lo) * (H / 2) : (uint32_t)(cut - c_lo) * ng * 2);
                }
            }
            s_cw[sgi][part] = win(sm + off, src, bytes, &s_bar[3], &tx);
        }
        tx = warp_total(tx);
        if (lane == 0) tc::mbar_arrive_expect_tx(&s_bar[3], tx);
    }
    __syncthreads();
    const int U = s_nu, perC = s_perC;
    const int nC = U * I, c_lo = min(nC, cta * perC), c_hi = min(nC, c_lo + perC), nrows = c_hi - c_lo;
    const int cut = nrows > 0 ? min(c_hi, (c_lo / I + 1) * I) : c_lo;
    int nra_here = 0;
    if (lora)
        for (int j = 0; j < P.nRA; ++j) nra_here += (cta + NB * j < TK * 2 * r) ? 1 : 0;

    if (warp == 1) {  // LoRA-B rows of the routed gate/up rows: lane = (segment, token slot, gate | up)
        uint32_t tx = 0;
        if (lane < 4 * MT) {
            const int sgi = lane / (2 * MT), m = (lane / 2) % MT, pj = lane % 2;
            const int q0 = sgi == 0 ? c_lo : cut, q1 = sgi == 0 ? cut : c_hi;
            const moe_lora_proj* lp = nullptr;
            int64_t row = 0;
            if (lora && q1 > q0 && s_abort == 0) {
                const int u = q0 / I;
                if (m < s_ucnt[u]) {
                    lp = dlora(L, s_aid[s_uslot[u][m] / K], false, pj);
                    row = (int64_t)s_uexp[u] * I + q0 % I;
                }
            }
            s_rbw[sgi][m][pj] = win(sm + P.wrb + lane * P.rb_stride, lp ? lp->B + row * r : nullptr,
                                    (uint32_t)((q1 - q0) * r * 2), &s_bar[3], &tx);
        }
        tx = warp_total(tx);
        if (lane == 0) tc::mbar_arrive_expect_tx(&s_bar[3], tx);
    } else if (warp == 2) {  // routed down rows of this CTA's output range, and their LoRA-B rows
        uint32_t tx = 0;
        const int ngd = I / L.down.group;
        for (int w = lane; w < 3 * U; w += 32) {
            const int u = w / 3, k = w % 3;
            const int64_t row = (int64_t)s_uexp[u] * H + o_lo;
            const void* src = nullptr;
            uint32_t bytes = 0;
            if (no > 0 && s_abort == 0) {
                src = k == 0 ? (const void*)(L.down.packed + row * (I / 8))
                             : (const void*)((k == 1 ? L.down.scales : L.down.biases) + row * ngd);
                bytes = k == 0 ? (uint32_t)(no * I / 2) : (uint32_t)(no * ngd * 2);
            }
            s_dw[u][k] = win(sm + P.wd + u * P.d_stride + P.d_off[k], src, bytes, &s_bar[4], &tx);
        }
        if (lane < TK) {
            const moe_lora_proj* lp = (lora && no > 0 && s_abort == 0) ? dlora(L, s_aid[lane / K], false, 2) : nullptr;
            const int64_t row = (int64_t)s_idx[lane / K][lane % K] * H + o_lo;
            s_rbdw[lane] = win(sm + P.wrbd + lane * P.rbd_stride, lp ? lp->B + row * r : nullptr,
                               (uint32_t)(no * r * 2), &s_bar[4], &tx);
        }
        tx = warp_total(tx);
        if (lane == 0) tc::mbar_arrive_expect_tx(&s_bar[4], tx);
    } else if (warp == 3) {  // LoRA-A rows of this CTA's routed LoRA-A dots: dot q = cta + NB * lane
        uint32_t tx = 0;
        if (lane < P.nRA) {
            const int q = cta + NB * lane;
            const moe_lora_proj* lp = nullptr;
            int64_t row = 0;
            if (lora && q < TK * 2 * r && s_abort == 0) {
                const int j = q / (2 * r), d = q % (2 * r);
                lp = dlora(L, s_aid[j / K], false, d < r ? 0 : 1);
                row = (int64_t)s_idx[j / K][j % K] * r + d % r;
            }
            s_raw[lane] = win(sm + P.wra + lane * P.ra_stride, lp ? lp->A + row * H : nullptr, (uint32_t)(H * 2),
                              &s_bar[2], &tx);
        }
        tx = warp_total(tx);
        if (lane == 0) tc::mbar_arrive_expect_tx(&s_bar[2], tx);
    }

    // ------------------------------------------------------------ phase G
    // tasks: routed LoRA-A dots, shared-expert rows, routed rows (one warp each)
    float wacc[3][MT];  // partial down LoRA-A sums (lane = component): segment 0, 1, shared
#pragma unroll
    for (int s = 0; s < 3; ++s)
#pragma unroll
        for (int m = 0; m < MT; ++m) wacc[s][m] = 0.0f;
    const bool kk = lane < r;
    int nsa_here = 0;
    if (lora && sh)
        for (int j = 0; j < P.nSA; ++j) nsa_here += (cta + NB * j < T * 2 * r) ? 1 : 0;
    {
        const int ntask = nra_here + nsa_here + nsr + nrows;
        bool landed[4] = {false, false, false, false};
        auto land = [&](int b) {
            if (!landed[b - 1]) {
                copies_landed(&s_bar[b], a.status, &s_abort, lim);
                landed[b - 1] = true;
            }
        };
        for (int j = warp; j < ntask; j += kCW) {
            if (j < nra_here) {  // routed LoRA-A dot q: job slot js, component d of gate | up
                const int q = cta + NB * j, js = q / (2 * r), d = q % (2 * r);
                land(2);
                float v = 0.0f;
                if (s_raw[j])
                    v = warp_sum(sdot_bf16(reinterpret_cast<const uint16_t*>(s_raw[j]), H, xs + (js / K) * H, lane));
                if (lane == 0) publish(a.rax + (int64_t)js * 2 * r + d, v, tag);
                continue;
            }
            if (j < nra_here + nsa_here) {  // shared LoRA-A dot q: token t, component d of gate | up
                const int jj = j - nra_here, q = cta + NB * jj, t = q / (2 * r), d = q % (2 * r);
                land(1);
                float v = 0.0f;
                if (s_saw[jj]) v = warp_sum(sdot_bf16(reinterpret_cast<const uint16_t*>(s_saw[jj]), H, xs + t * H, lane));
                if (lane == 0) publish(a.sax + (int64_t)t * 2 * r + d, v, tag);
                continue;
            }
            if (j < nra_here + nsa_here + nsr) {  // shared-expert row i: LoRA-B delta, SwiGLU, h, partial A_down h
                const int il = j - nra_here - nsa_here, i = s_lo + il;
                float ad[MT];
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    ad[m] = 0.0f;
                    if (m < T && kk) {
                        const moe_lora_proj* ld = dlora(L, s_aid[m], true, 2);
                        if (ld) ad[m] = bf16f(ld->A[(int64_t)lane * Is + i]);
                    }
                }
                unsigned long long sw[MT][2];  // this token's shared LoRA-A products (lane = component)
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    sw[m][0] = sw[m][1] = 0ull;
                    if (m < T && kk) {
                        sw[m][0] = peek(a.sax + (int64_t)m * 2 * r + lane);
                        sw[m][1] = peek(a.sax + (int64_t)m * 2 * r + r + lane);
                    }
                }
                land(1);
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m >= T) break;
                    float g = sgu[(il * T + m) * 2], u = sgu[(il * T + m) * 2 + 1];
                    if (lora) {
                        const uint16_t* bg = reinterpret_cast<const uint16_t*>(s_sbw[m][0]);
                        const uint16_t* bu = reinterpret_cast<const uint16_t*>(s_sbw[m][1]);
                        float tg = 0.0f, tu = 0.0f;
                        if (kk) {
                            const uint64_t* sp = a.sax + (int64_t)m * 2 * r + lane;
                            tg = fresh(sw[m][0], tag) ? wval(sw[m][0]) : spin(sp, tag, a.status, &s_abort, lim);
                            tu = fresh(sw[m][1], tag) ? wval(sw[m][1]) : spin(sp + r, tag, a.status, &s_abort, lim);
                        }
                        const float dg = (kk && bg) ? bf16f(bg[il * r + lane]) * tg : 0.0f;
                        const float du = (kk && bu) ? bf16f(bu[il * r + lane]) * tu : 0.0f;
                        g += L.scale * warp_sum(dg);
                        u += L.scale * warp_sum(du);
                    }
                    const float hv = silu(g) * u;
                    if (lane == 0) a.hx[(int64_t)(TK + m) * max(I, Is) + i] = hv;
                    wacc[2][m] += ad[m] * hv;
                }
                continue;
            }
            // routed row q: distinct expert u, row i, segment sg
            const int q = c_lo + (j - nra_here - nsa_here - nsr), u = q / I, i = q % I, sg = q < cut ? 0 : 1;
            const int rs = q - (sg == 0 ? c_lo : cut), e = s_uexp[u], nt = s_ucnt[u];
            int toks[MT];
            float ad[MT];
            unsigned long long tw[MT][2];
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                ad[m] = 0.0f;
                tw[m][0] = tw[m][1] = 0ull;
                toks[m] = m < nt ? s_uslot[u][m] / K : 0;
                if (m < nt && kk && lora) {  // A_down column i and this job's LoRA-A products: loads in flight
                    const moe_lora_proj* ld = dlora(L, s_aid[toks[m]], false, 2);
                    if (ld) ad[m] = bf16f(ld->A[((int64_t)e * r + lane) * I + i]);
                    const uint64_t* tp = a.rax + (int64_t)s_uslot[u][m] * 2 * r + lane;
                    tw[m][0] = peek(tp);
                    tw[m][1] = peek(tp + r);
                }
            }
            land(3);
            float ag[MT], au[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) ag[m] = au[m] = 0.0f;
            const int ngg = H / L.gate.group, ngu = H / L.up.group;
            if (s_cw[sg][0] && s_cw[sg][3]) {  // (missing only when the CTA gave up before issuing them)
                cdot_int4<MT>(reinterpret_cast<const uint32_t*>(s_cw[sg][0] + (size_t)rs * (H / 2)),
                             reinterpret_cast<const uint16_t*>(s_cw[sg][1]) + rs * ngg,
                             reinterpret_cast<const uint16_t*>(s_cw[sg][2]) + rs * ngg, L.gate.group, H, xs, xsum, toks,
                             nt, ag, lane, 32);
                cdot_int4<MT>(reinterpret_cast<const uint32_t*>(s_cw[sg][3] + (size_t)rs * (H / 2)),
                             reinterpret_cast<const uint16_t*>(s_cw[sg][4]) + rs * ngu,
                             reinterpret_cast<const uint16_t*>(s_cw[sg][5]) + rs * ngu, L.up.group, H, xs, xsum, toks,
                             nt, au, lane, 32);
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m >= nt) break;
                const int slot = s_uslot[u][m];
                float g = warp_sum(ag[m]), uu = warp_sum(au[m]);
                if (lora) {
                    float tg = 0.0f, tu = 0.0f;
                    if (kk) {
                        const uint64_t* tp = a.rax + (int64_t)slot * 2 * r + lane;
                        tg = fresh(tw[m][0], tag) ? wval(tw[m][0]) : spin(tp, tag, a.status, &s_abort, lim);
                        tu = fresh(tw[m][1], tag) ? wval(tw[m][1]) : spin(tp + r, tag, a.status, &s_abort, lim);
                    }
                    const uint16_t* bg = reinterpret_cast<const uint16_t*>(s_rbw[sg][m][0]);
                    const uint16_t* bu = reinterpret_cast<const uint16_t*>(s_rbw[sg][m][1]);
                    g += L.scale * warp_sum((kk && bg) ? bf16f(bg[rs * r + lane]) * tg : 0.0f);
                    uu += L.scale * warp_sum((kk && bu) ? bf16f(bu[rs * r + lane]) * tu : 0.0f);
                }
                const float hv = silu(g) * uu;
                if (lane == 0) a.hx[(int64_t)slot * max(I, Is) + i] = hv;
                if (sg == 0) wacc[0][m] += ad[m] * hv;
                else wacc[1][m] += ad[m] * hv;
            }
        }
    }
    if (lora) {  // per-warp partials, summed over the warps in fixed order, published
        if (kk)
#pragma unroll
            for (int s = 0; s < 3; ++s)
#pragma unroll
                for (int m = 0; m < MT; ++m) wpart[((warp * 3 + s) * MT + m) * r + lane] = wacc[s][m];
        __syncthreads();
        for (int q = tid; q < 3 * T * r; q += kCT) {
            const int k = q % r, m = (q / r) % T, s = q / (r * T);
            float v = 0.0f;
            for (int w = 0; w < kCW; ++w) v += wpart[((w * 3 + s) * MT + m) * r + k];
            a.part[(((int64_t)cta * 3 + s) * T + m) * r + k] = v;
        }
    }
    // h and the partial sums of this CTA are written: one arrival (every CTA, every launch)
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(a.hcnt) : "memory");
    }

    // ------------------------------------------------------------ phase D
    // every CTA has written its h rows and partial sums once the arrival count is reached
    if (tid == 0) wait_word(a.hcnt, s_hdone, true, a.status, &s_abort, lim);
    __syncthreads();
    // h of every job (routed rows of length I, then the shared ones of length Is), staged in
    // the swizzled layout: 16-byte loads from L2, all of a thread's in flight together
    {
        const int Imx = max(I, Is);
        const int nr4 = TK * (I / 4), nh4 = nr4 + T * (Is / 4);
        for (int base = 0; base < nh4; base += 4 * kCT) {
            float4 v[4];
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int q = base + b * kCT + tid;
                if (q < nh4) {
                    const float* src = q < nr4 ? a.hx + (int64_t)(q / (I / 4)) * Imx + (q % (I / 4)) * 4
                                               : a.hx + (int64_t)(TK + (q - nr4) / (Is / 4)) * Imx +
                                                     ((q - nr4) % (Is / 4)) * 4;
                    v[b] = __ldcg(reinterpret_cast<const float4*>(src));
                }
            }
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int q = base + b * kCT + tid;
                if (q >= nh4) break;
                float* dst = q < nr4 ? hsm + (q / (I / 4)) * I + swz((q % (I / 4)) * 4)
                                     : hsm + TK * I + ((q - nr4) / (Is / 4)) * Is + swz(((q - nr4) % (Is / 4)) * 4);
                *reinterpret_cast<float4*>(dst) = v[b];
            }
        }
    }
    if (lora) {
        // down LoRA-A products: for each job, the sum over the CTAs whose rows cover its
        // expert of their partial sums, in CTA order.  An item is (job, component, a run of
        // up to 8 of those CTAs): its 8 loads are in flight together; the items of a (job,
        // component) are then added in order.
        constexpr int kRun = 8;
        if (tid == 0) {
            int o = 0;
            for (int j = 0; j < J; ++j) {
                s_goff[j] = o;
                int ncta;
                if (j < TK) {
                    const int u = s_ju[j];
                    ncta = (((u + 1) * I - 1) / perC) - (u * I) / perC + 1;
                } else {
                    ncta = (Is + P.perS - 1) / P.perS;
                }
                o += (ncta + kRun - 1) / kRun * r;
            }
            s_goff[J] = o;
        }
        copies_landed(&s_bar[3], a.status, &s_abort, lim);  // the gather space aliases these windows
        __syncthreads();
        for (int q = tid; q < J * r; q += kCT) tds[q] = 0.0f;
        const int total = s_goff[J];
        for (int base = 0; base < total; base += (int)P.gat_n) {
            const int n = min((int)P.gat_n, total - base);
            for (int q = tid; q < n; q += kCT) {
                const int g = base + q;
                int j = 0;
                while (j + 1 < J && s_goff[j + 1] <= g) ++j;
                const int loc = g - s_goff[j], k = loc % r, run = loc / r;
                int c0, cnt, m, s0;  // first CTA of the run, CTAs in it, token slot, segment of the first
                if (j < TK) {
                    const int u = s_ju[j], cf = (u * I) / perC, cl = ((u + 1) * I - 1) / perC;
                    c0 = cf + run * kRun;
                    cnt = min(kRun, cl - c0 + 1);
                    m = s_jm[j];
                    s0 = (run == 0 && cf * perC < u * I) ? 1 : 0;  // only the first covering CTA can hold u second
                } else {
                    c0 = run * kRun;
                    cnt = min(kRun, (Is + P.perS - 1) / P.perS - c0);
                    m = j - TK;
                    s0 = 2;
                }
                const int64_t step = (int64_t)3 * T * r, off = (int64_t)m * r + k;
                float w[kRun];
#pragma unroll
                for (int i = 0; i < kRun; ++i) {
                    const int s = i == 0 ? s0 : (j < TK ? 0 : 2);
                    w[i] = i < cnt ? __ldcg(a.part + (int64_t)(c0 + i) * step + (int64_t)s * T * r + off) : 0.0f;
                }
                float v = 0.0f;
#pragma unroll
                for (int i = 0; i < kRun; ++i) v += w[i];
                gat[q] = v;
            }
            __syncthreads();
            // the runs of each (job, component) in order: entry (j, run, k) at s_goff[j] + run * r + k
            for (int q = tid; q < J * r; q += kCT) {
                const int j = q / r, k = q % r;
                const int g0 = max(s_goff[j], base), g1 = min(s_goff[j + 1], base + n);
                float v = tds[q];
                for (int g = g0 + ((k - (g0 - s_goff[j]) % r) + r) % r; g < g1; g += r) v += gat[g - base];
                tds[q] = v;
            }
            __syncthreads();
        }
    }
    __syncthreads();
    // chunk sums of the staged h rows
    {
        const int nch = TK * (I / 32) + T * (Is / 32);
        for (int c = warp; c < nch; c += kCW) {
            const float* row = c < TK * (I / 32) ? hsm + (c / (I / 32)) * I + (c % (I / 32)) * 32
                                                 : hsm + TK * I + ((c - TK * (I / 32)) / (Is / 32)) * Is +
                                                       ((c - TK * (I / 32)) % (Is / 32)) * 32;
            const float v = warp_sum(row[lane]);
            if (lane == 0) hsum[c] = v;
        }
    }
    __syncthreads();
    copies_landed(&s_bar[4], a.status, &s_abort, lim);
    copies_landed(&s_bar[1], a.status, &s_abort, lim);
    // (output row, expert) tasks from the down windows; a task is a group of lpt lanes over one row
    if (no > 0 && s_abort == 0) {
        const int UD = U + (sh ? 1 : 0);
        const int Imx = max(I, Is);
        int lpt = 1;
        while (lpt * 2 <= 32 && lpt * 2 <= Imx / 32) lpt *= 2;
        const int gpw = 32 / lpt, sub = lane / lpt, sl = lane % lpt;
        const int ntask = no * UD;
        for (int q0 = warp * gpw; q0 < ntask; q0 += kCW * gpw) {
            const int q = q0 + sub;
            const bool live = q < ntask;
            const int ol = live ? q / UD : 0, u = live ? q % UD : 0;
            const bool shu = sh && u == U;
            const int n = shu ? Is : I;
            const moe_qtensor& Wd = shu ? L.s_down : L.down;
            const int ng = n / Wd.group;
            const int nt = live ? (shu ? T : s_ucnt[u]) : 0;
            int sl_[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) sl_[m] = m < nt ? (shu ? TK + m : s_uslot[u][m]) : 0;
            float acc[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
            const unsigned char* const* dw = shu ? s_sdw : s_dw[u];
            if (live && dw[0])
                cdot_int4<MT>(reinterpret_cast<const uint32_t*>(dw[0] + (size_t)ol * (n / 2)),
                             reinterpret_cast<const uint16_t*>(dw[1]) + ol * ng,
                             reinterpret_cast<const uint16_t*>(dw[2]) + ol * ng, Wd.group, n,
                             shu ? hsm + TK * I - TK * n : hsm, shu ? hsum + TK * (I / 32) - TK * (n / 32) : hsum, sl_,
                             nt, acc, sl, lpt);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const float d = group_sum(acc[m], lpt);
                float t = 0.0f;
                if (lora && m < nt) {
                    const uint16_t* bd = reinterpret_cast<const uint16_t*>(shu ? s_sbw[m][2] : s_rbdw[sl_[m]]);
                    if (bd)
                        for (int k = sl; k < r; k += lpt) t += bf16f(bd[ol * r + k]) * tds[sl_[m] * r + k];
                }
                t = group_sum(t, lpt);
                if (live && m < nt && sl == 0) sv[ol * J + sl_[m]] = d + L.scale * t;
            }
        }
    }
    __syncthreads();
    if (s_abort == 0)
        for (int q = tid; q < no * T; q += kCT) {
            const int ol = q / T, t = q % T, o = o_lo + ol;
            float acc = 0.0f;
            for (int k = 0; k < K; ++k) acc += s_w[t][k] * sv[ol * J + t * K + k];
            if (sh) acc += s_sig[t] * sv[ol * J + TK + t];
            if (a.block) acc += bf16f(xr[(int64_t)t * H + o]);
            a.y[(int64_t)t * H + o] = f2bf16(acc);
        }
    // no bulk copy may be in flight when the CTA exits (bounded waits)
    if (tid == 0)
        for (int i = 0; i < 5; ++i) tc::mbar_wait(&s_bar[i], 0, nullptr, lim);
}

}  // namespace

namespace {

inline size_t r16c(size_t v) { return (v + 15) / 16 * 16; }
inline int cdivc(int a, int b) { return (a + b - 1) / b; }

bool cwin_ok(const moe_qtensor& q) {
    if (!q.packed) return true;
    const size_t rows = (size_t)q.n * q.out;
    const size_t pb = rows * (size_t)q.in * q.bits / 8, sb = rows * (size_t)(q.in / q.group) * 2;
    return ((uintptr_t)q.packed & 15) == 0 && ((uintptr_t)q.scales & 15) == 0 && ((uintptr_t)q.biases & 15) == 0 &&
           pb % 16 == 0 && sb % 16 == 0 && q.group % 32 == 0 &&
           (q.group & (q.group - 1)) == 0;
}

int c_sm_count() {
    static int n = -1;
    if (n < 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = 0;
    }
    return n;
}

int c_optin_smem() {
    static int v = -1;
    if (v < 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) v = 0;
    }
    return v;
}

template <int MT>
size_t c_static_smem() {
    static size_t v = (size_t)-1;
    if (v == (size_t)-1) {
        cudaFuncAttributes at;
        v = cudaFuncGetAttributes(&at, decode_chain_kernel<MT>) == cudaSuccess ? at.sharedSizeBytes : (size_t)1 << 30;
    }
    return v;
}

size_t c_static_for(int T) { return T <= 1 ? c_static_smem<1>() : T <= 2 ? c_static_smem<2>() : c_static_smem<4>(); }
int c_mt(int T) { return T <= 1 ? 1 : T <= 2 ? 2 : 4; }

bool plan_chain(const LayerArgs& L, int T, int NB, CPlan* P) {
    const bool sh = L.has_shared, lora = L.n_adapters > 0 && L.rank > 0;
    const int H = L.H, E = L.E, K = L.K, I = L.I, Is = sh ? L.Is : 0, r = lora ? L.rank : 0;
    const int TK = T * K, J = TK + (sh ? T : 0), MT = c_mt(T);
    if (T < 1 || T > kCMaxT || TK > kCMaxTK || r > kCMaxR || NB < 1 || NB > MOEQ_DECODE_MAX_CTAS) return false;
    if (E > MOEQ_MAX_EXPERTS || H % 32 || H > 4096 || I % 32 || I > 4096 || (sh && (Is % 32 || Is > 4096))) return false;
    if (!cwin_ok(L.router) || !cwin_ok(L.gate) || !cwin_ok(L.up) || !cwin_ok(L.down)) return false;
    if (L.has_sgate && (((uintptr_t)L.shared_gate.packed & 15) || L.shared_gate.bits != 8 ||
                        L.shared_gate.group % 32 || (L.shared_gate.group & (L.shared_gate.group - 1))))
        return false;
    if (sh && (!cwin_ok(L.s_gate) || !cwin_ok(L.s_up) || !cwin_ok(L.s_down))) return false;
    if (L.router.bits != 8 || L.gate.bits != 4 || L.up.bits != 4 || L.down.bits != 4) return false;
    if (lora) {  // LoRA rows move by bulk copies: 16-byte aligned factors, rows of whole 16-byte pieces
        if (r % 8) return false;
        for (int ad = 0; ad < L.n_adapters; ++ad) {
            const moe_lora_proj* p[6] = {&L.lora[ad].gate, &L.lora[ad].up, &L.lora[ad].down,
                                         &L.lora[ad].s_gate, &L.lora[ad].s_up, &L.lora[ad].s_down};
            for (int k = 0; k < 6; ++k)
                if ((p[k]->A && ((uintptr_t)p[k]->A & 15)) || (p[k]->B && ((uintptr_t)p[k]->B & 15))) return false;
        }
    }
    const int Umax = std::min(E, TK), Imx = std::max(I, Is);
    P->Umax = Umax;
    P->perA = cdivc(E, NB);
    P->perS = sh ? cdivc(Is, NB) : 0;
    P->perO = cdivc(H, NB);
    P->perCmax = cdivc(Umax * I, NB);
    P->nSA = (lora && sh) ? cdivc(T * 2 * r, NB) : 0;
    P->nRA = lora ? cdivc(TK * 2 * r, NB) : 0;
    if (P->perO > kCMaxO || P->perCmax > I || P->nSA > kCMaxSA || P->nRA > kCMaxRA || P->perA * NB < E) return false;

    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o = r16c(o + bytes);
        return (uint32_t)at;
    };
    auto slack = [](size_t bytes) { return bytes ? r16c(bytes) + 32 : 0; };
    P->xraw = take((size_t)T * H * 2);
    P->xs = take((size_t)T * H * 4);
    P->xsum = take((size_t)T * (H / 32) * 4);
    P->z = take((size_t)T * E * 4);
    P->sax = take((size_t)T * 2 * std::max(r, 1) * 4);
    {  // phase-R windows
        size_t wsz = 0;
        const moe_qtensor* qs[4] = {&L.router, &L.shared_gate, &L.s_gate, &L.s_up};
        const int rows[4] = {P->perA, 0, P->perS, P->perS};  // (the shared-gate row needs no window)
        for (int g = 0; g < 4; ++g) {
            const moe_qtensor& q = *qs[g];
            const int bits = g < 2 ? 8 : 4, ng = q.packed ? H / q.group : 0;
            const size_t sz[3] = {(size_t)rows[g] * H * bits / 8, (size_t)rows[g] * ng * 2, (size_t)rows[g] * ng * 2};
            for (int k = 0; k < 3; ++k) {
                P->a_off[g * 3 + k] = (uint32_t)wsz;
                wsz += q.packed ? slack(sz[k]) : 0;
            }
        }
        P->wa = take(wsz);
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
    P->wsb = take(lora && sh ? (size_t)T * 3 * P->sb_stride : 0);
    {  // routed gate/up windows: two segments per part
        const size_t gp = (size_t)P->perCmax * (H / 2);
        const size_t gs = (size_t)P->perCmax * (H / L.gate.group) * 2, us = (size_t)P->perCmax * (H / L.up.group) * 2;
        const size_t cpart[6] = {gp, gs, gs, gp, us, us};
        size_t wsz = 0;
        for (int k = 0; k < 6; ++k) {
            P->c_off[k] = (uint32_t)wsz;
            wsz += r16c(cpart[k]) + 64;
        }
        // the gather space of the partial sums reuses these windows in phase D
        const size_t gat_bytes = std::max(wsz, (size_t)4096 * 4);
        P->wc = take(gat_bytes);
        P->gat = P->wc;
        P->gat_n = (uint32_t)std::min<size_t>(gat_bytes / 4, (size_t)kGB * kCT);
    }
    {
        const int ngd = I / L.down.group;
        P->d_off[0] = 0;
        P->d_off[1] = (uint32_t)slack((size_t)P->perO * I / 2);
        P->d_off[2] = P->d_off[1] + (uint32_t)slack((size_t)P->perO * ngd * 2);
        P->d_stride = P->d_off[2] + (uint32_t)slack((size_t)P->perO * ngd * 2);
        P->wd = take((size_t)Umax * P->d_stride);
    }
    P->ra_stride = (uint32_t)slack((size_t)H * 2);
    P->wra = take((size_t)P->nRA * P->ra_stride);
    P->rb_stride = (uint32_t)slack((size_t)P->perCmax * std::max(r, 1) * 2);
    P->wrb = take(lora ? (size_t)4 * MT * P->rb_stride : 0);
    P->rbd_stride = (uint32_t)slack((size_t)P->perO * std::max(r, 1) * 2);
    P->wrbd = take(lora ? (size_t)TK * P->rbd_stride : 0);
    P->sgu = take((size_t)std::max(P->perS, 1) * T * 2 * 4);
    P->hs = take(((size_t)TK * I + (size_t)T * Is) * 4);
    P->hsum = take(((size_t)TK * (I / 32) + (size_t)T * (Is / 32)) * 4);
    P->td = take((size_t)J * std::max(r, 1) * 4);
    P->wpart = take(lora ? (size_t)kCW * 3 * MT * r * 4 : 0);
    P->sv = take((size_t)P->perO * J * 4);
    P->total = (uint32_t)o;
    (void)Imx;
    const size_t limit = (size_t)c_optin_smem() > c_static_for(T) ? (size_t)c_optin_smem() - c_static_for(T) : 0;
    return o <= limit;
}

template <int MT>
cudaError_t launch_chain_mt(const CArgs& a, cudaStream_t s) {
    static int cached = 0;
    cudaError_t e = ensure_smem((const void*)decode_chain_kernel<MT>, a.P.total, cached);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(c_sm_count());
    cfg.blockDim = dim3(kCT);
    cfg.dynamicSmemBytes = a.P.total;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, decode_chain_kernel<MT>, a);
}

}  // namespace

// Words (8 bytes) of the chain kernel's region a layer shape needs: its ticket and
// counters, the tagged words (logits, LoRA-A products), the routing CTA 0 publishes, h
// and the partial down LoRA-A sums; sized for the largest token count the kernel takes
// with this top-K, so that its place and size do not depend on T.
size_t chain_slot_words(int E, int K, int I, int Is, int r) {
    const int Tm = std::min(kCMaxT, kCMaxTK / std::max(K, 1));
    if (Tm < 1) return 0;
    const size_t rr = std::max(r, 1), Jm = (size_t)Tm * (K + 1), Imx = std::max(I, Is);
    return 8 + (size_t)Tm * E + (size_t)Tm * 2 * rr + (size_t)Tm * K * 2 * rr + (size_t)Tm * K +
           (Jm * Imx + 1) / 2 + ((size_t)MOEQ_DECODE_MAX_CTAS * 3 * Tm * rr + 1) / 2 + 2;
}

bool chain_supported(const LayerArgs& L, int T) {
    CPlan P;
    return plan_chain(L, T, c_sm_count(), &P);
}

cudaError_t launch_chain(const LayerArgs& L, const uint16_t* x, const int32_t* adapter_id, const int32_t* select,
                         uint16_t* y, int T, int block, float eps, const ChainScratch& sc, cudaStream_t s) {
    CArgs a;
    memset(&a, 0, sizeof(a));
    if (!plan_chain(L, T, c_sm_count(), &a.P)) return cudaErrorNotSupported;
    a.L = L;
    a.x = x;
    a.adapter_id = adapter_id;
    a.select = select;
    a.y = y;
    a.T = T;
    a.block = block;
    a.eps = eps;
    const int K = L.K, I = L.I, Is = L.has_shared ? L.Is : 0;
    const size_t r = std::max(L.n_adapters > 0 ? L.rank : 0, 1);
    const size_t Tm = std::min(kCMaxT, kCMaxTK / K), Jm = Tm * (K + 1), Imx = std::max(I, Is);
    uint64_t* p = sc.slots;
    a.tick = reinterpret_cast<unsigned long long*>(p);
    a.hcnt = reinterpret_cast<unsigned long long*>(p + 1);
    a.rflag = reinterpret_cast<unsigned long long*>(p + 2);
    p += 8;
    a.zs = p;
    p += Tm * L.E;
    a.sax = p;
    p += Tm * 2 * r;
    a.rax = p;
    p += Tm * K * 2 * r;
    a.route = p;
    p += Tm * K;
    p += (reinterpret_cast<uintptr_t>(p) & 15) ? 1 : 0;  // 16-byte aligned float rows
    a.hx = reinterpret_cast<float*>(p);
    p += (Jm * Imx + 1) / 2;
    a.part = reinterpret_cast<float*>(p);
    a.status = sc.status;
    a.idx_out = sc.idx_out;
    a.w_out = sc.w_out;
    a.wait_ns = wait_limit_ns();
    switch (c_mt(T)) {
        case 1: return launch_chain_mt<1>(a, s);
        case 2: return launch_chain_mt<2>(a, s);
        default: return launch_chain_mt<4>(a, s);
    }
}

}  // namespace moeq
