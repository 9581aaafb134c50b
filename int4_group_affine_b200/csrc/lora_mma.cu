// lora_mma.cu - the LoRA-A products of the expert-grouped jobs on warp-level tensor-core
// tiles (unmerged adapters over a read-only base: "LoRA on MoE experts", the low-rank
// branch B(Ax) of every projection; the A x half is computed here).
//
// Every job j (token t, adapter a, expert e) needs, before its gate/up rows, the 2r values
// A_gate x_t | A_up x_t of its own adapter, and before its down rows the r values A_down h_j.
// The index build orders each expert's jobs by (adapter, token) with "no adapter" last, so
// the jobs of one expert group mostly share one adapter's A rows.  A CTA takes one item =
// (expert group, tile of up to 64 consecutive jobs) and runs it as a small GEMM on
// mma.sync m16n8k16 (bf16 operands, fp32 accumulation):
//   M = the jobs (m16 tiles), N = the adapter's A rows (n8 tiles; 32 rows per warp),
//   K = H (gate/up, activations = x by token) or I / Is (down, activations = h by job).
// The 16 warps split the (m tile, 32-row group, K part) triples of the m16 tiles that hold
// the current adapter's jobs; the K parts add in shared memory in a fixed order.  Every
// operand is read straight from global memory with 16-byte loads (the item's job offsets,
// tokens and adapters go through shared memory first): a lane's 8 consecutive K elements
// of a row feed the k-pairs {2c, 2c+1} and {2c+8, 2c+9} of two consecutive MMAs - the same
// reordering of K for both operands, so the dot products are unchanged.  The down activations h are stored with every 8-group of
// K in the order 0 4 1 5 2 6 3 7 (the int4 tiles' order); the A_down chunks are put in the
// same order with four byte permutes.  A tile whose jobs span several adapters is run once
// per adapter, each run writing only its own jobs; jobs without an adapter get zeros.
//
// Output: [J][2r] (gate rows 0..r-1, up rows r..2r-1) or [J][r] fp32, unscaled (alpha / r is
// applied with the LoRA-B product).
#include "common.cuh"

namespace moeq {
namespace {

constexpr int kLWarps = 16;      // warps per CTA
constexpr int kLJobs = 64;       // jobs per item: up to four m16 tiles
constexpr int kLCols = 32;       // A rows (output columns) per warp: four n8 tiles
constexpr int kLUnroll = 2;      // 32-wide K chunks loaded together by a warp
constexpr int kLMaxGroups = 513; // E + 1 expert groups at most (E <= 512)

struct LoraMmaArgs {
    LayerArgs L;
    const uint16_t* act;  // gate/up: x [T][ld] by token; down: h [J][ld] by job (tile K order)
    int ld;               // elements per activation row
    const int4* perm;     // [J] jobs {token, k, adapter, expert}
    const int32_t* goff;  // [E+2] job offsets of the expert groups (group E = shared expert)
    float* out;           // [J][R]
    int down;             // 0: gate/up (R = 2r), 1: down (R = r)
};

__device__ __forceinline__ const moe_lora_proj* lora_rows(const LayerArgs& L, int ad, bool shared, int which) {
    if (ad < 0 || ad >= L.n_adapters) return nullptr;
    const moe_lora_ptrs& p = L.lora[ad];
    const moe_lora_proj* q = which == 0 ? (shared ? &p.s_gate : &p.gate)
                           : which == 1 ? (shared ? &p.s_up : &p.up)
                                        : (shared ? &p.s_down : &p.down);
    return (q->A && q->B) ? q : nullptr;
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 8 bf16 of natural K order -> the order 0 4 1 5 2 6 3 7 of the int4 tiles
__device__ __forceinline__ uint4 to_tile_order(uint4 u) {
    return make_uint4(__byte_perm(u.x, u.z, 0x5410), __byte_perm(u.x, u.z, 0x7632), __byte_perm(u.y, u.w, 0x5410),
                      __byte_perm(u.y, u.w, 0x7632));
}

__device__ __forceinline__ uint4 ld16(const uint16_t* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

// Bring [p, p + bytes) into L2 without waiting (bulk prefetch; p and bytes multiples of 16)
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    for (uint32_t o = 0; o < bytes; o += 65536u) {
        const uint32_t n = bytes - o < 65536u ? bytes - o : 65536u;
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<const char*>(p) + o), "r"(n)
                     : "memory");
    }
}

__device__ __forceinline__ int pow2_ceil4(int v) { return v <= 1 ? 1 : v <= 2 ? 2 : 4; }

__global__ void __launch_bounds__(kLWarps * 32, 1) lora_a_mma_kernel(const __grid_constant__ LoraMmaArgs a) {
    const LayerArgs& L = a.L;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, g = lane / 4, c = lane % 4;
    const int E = L.E, r = L.rank, R = a.down ? r : 2 * r;
    __shared__ int s_goff[kLMaxGroups + 1];              // job offsets of the groups
    __shared__ int s_pre[kLMaxGroups + 1];               // items before each group
    __shared__ int s_tok[kLJobs], s_z[kLJobs];           // tokens and adapters of the item's jobs
    __shared__ float s_part[kLWarps][16][kLCols];         // each warp's partial tile

    // items per group (empty groups and a missing shared expert: none), scanned by warp 0
    for (int i = threadIdx.x; i <= E + 1; i += blockDim.x) s_goff[i] = a.goff[i];
    __syncthreads();
    if (warp == 0) {
        int carry = 0;
        for (int g0 = 0; g0 <= E; g0 += 32) {
            const int gg = g0 + lane;
            int n = 0;
            if (gg <= E) {
                const int cnt = s_goff[gg + 1] - s_goff[gg];
                n = (gg == E && !L.has_shared) ? 0 : (cnt + kLJobs - 1) / kLJobs;
            }
            int incl = n;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            if (gg <= E) s_pre[gg + 1] = carry + incl;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) s_pre[0] = 0;
    }
    __syncthreads();
    const int total = s_pre[E + 1];
    const int ng = (R + kLCols - 1) / kLCols, ngp = pow2_ceil4(ng);  // 32-row groups (R <= 128)

    for (int it = blockIdx.x; it < total; it += gridDim.x) {
        int lo = 0, hi = E;  // the group: the last g with s_pre[g] <= it
        while (lo < hi) {
            const int mid = (lo + hi + 1) / 2;
            if (s_pre[mid] <= it) lo = mid;
            else hi = mid - 1;
        }
        const int grp = lo;
        const bool shared = grp == E;
        const int j0 = s_goff[grp] + (it - s_pre[grp]) * kLJobs;
        const int nj = min(kLJobs, s_goff[grp + 1] - j0);
        const int K = a.down ? (shared ? L.Is : L.I) : L.H;
        const int nch = K / 32;
        if (!a.down && L.n_adapters == 1 && (threadIdx.x == 32 || threadIdx.x == 33)) {
            // one adapter: the A blocks of this item and of this CTA's next item start towards L2
            // before the job list is read (the down products read h, which is still in L2)
            int g2 = grp;
            if (threadIdx.x == 33) {
                const int nx = it + (int)gridDim.x;
                g2 = -1;
                if (nx < total) {
                    int l2 = 0, h2 = E;
                    while (l2 < h2) {
                        const int mid = (l2 + h2 + 1) / 2;
                        if (s_pre[mid] <= nx) l2 = mid;
                        else h2 = mid - 1;
                    }
                    g2 = l2;
                    const int jn = s_goff[g2] + (nx - s_pre[g2]) * kLJobs;
                    prefetch_l2(a.perm + jn, (uint32_t)min(kLJobs, s_goff[g2 + 1] - jn) * 16u);
                }
            }
            if (g2 >= 0)
                for (int which = 0; which < 2; ++which) {
                    const moe_lora_proj* lp = lora_rows(L, 0, g2 == E, which);
                    if (lp) prefetch_l2(lp->A + (int64_t)(g2 == E ? 0 : g2) * r * L.H, (uint32_t)r * L.H * 2);
                }
        }
        __syncthreads();  // the previous item is done with s_z and s_part
        if (threadIdx.x < kLJobs) {
            int tok = 0, z = -1;
            if (threadIdx.x < nj) {
                const int4 pj = a.perm[j0 + threadIdx.x];
                tok = pj.x;
                z = pj.z;
            }
            s_tok[threadIdx.x] = tok;
            s_z[threadIdx.x] = z;
        }
        __syncthreads();
        for (int q = threadIdx.x; q < nj * R; q += blockDim.x) {
            const int zj = s_z[q / R];
            if (zj < 0 || zj >= L.n_adapters) a.out[(int64_t)j0 * R + q] = 0.0f;
        }
        const int zf = s_z[0], zl = s_z[nj - 1];
        const int ad_lo = (zf < 0 || zf >= L.n_adapters) ? L.n_adapters : zf;
        const int ad_hi = (zl < 0 || zl >= L.n_adapters) ? L.n_adapters - 1 : zl;
        if (!a.down) {
            // gate/up: the x rows of the jobs and (several adapters) every present adapter's A
            // blocks start towards L2 together, so the K loops below mostly wait on L2, not HBM
            const int t = threadIdx.x;
            const int npf = L.n_adapters > 1 ? 2 * (ad_hi - ad_lo + 1) : 0;
            if (t < npf) {
                const moe_lora_proj* lp = lora_rows(L, ad_lo + t / 2, shared, t % 2);
                if (lp) prefetch_l2(lp->A + (int64_t)(shared ? 0 : grp) * r * K, (uint32_t)r * K * 2);
            } else if (t >= 64 && t < 64 + nj) {
                prefetch_l2(a.act + (int64_t)s_tok[t - 64] * a.ld, (uint32_t)K * 2);
            }
        }

        for (int ad = ad_lo; ad <= ad_hi; ++ad) {
            // this adapter's jobs: a contiguous run [jlo, jlo + na) of the item ("none" sorts last)
            const int zt = threadIdx.x < nj ? s_z[threadIdx.x] : -1;
            const int na = __syncthreads_count(threadIdx.x < nj && zt == ad);
            if (na == 0) continue;
            const int jlo = __syncthreads_count(threadIdx.x < nj && zt >= 0 && zt < ad);
            // warp roles for this run: m tile (of the run's m16 tiles), 32-row group, K part
            const int mlo = jlo / 16, mta = (jlo + na - 1) / 16 - mlo + 1, mtp = pow2_ceil4(mta);
            const int kp = kLWarps / (mtp * ngp);
            const int mi = warp % mtp, ngi = (warp / mtp) % ngp, kpi = warp / (mtp * ngp);
            const bool busy = mi < mta && ngi < ng;
            const int jr0 = 16 * (mlo + mi) + g, jr1 = jr0 + 8;
            const bool v0 = busy && jr0 < nj, v1 = busy && jr1 < nj;
            const uint16_t* x0 = a.act;
            const uint16_t* x1 = a.act;
            if (v0) x0 += (int64_t)(a.down ? j0 + jr0 : s_tok[jr0]) * a.ld;
            if (v1) x1 += (int64_t)(a.down ? j0 + jr1 : s_tok[jr1]) * a.ld;
            // row g of each of this warp's n8 tiles
            const uint16_t* wr[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int n = kLCols * ngi + 8 * t + g;
                wr[t] = nullptr;
                if (busy && n < R) {
                    const moe_lora_proj* lp = lora_rows(L, ad, shared, a.down ? 2 : (n < r ? 0 : 1));
                    if (lp) wr[t] = lp->A + ((int64_t)(shared ? 0 : grp) * r + (a.down ? n : n % r)) * K;
                }
            }
            float acc[4][4];
#pragma unroll
            for (int t = 0; t < 4; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[t][e] = 0.0f;
            if (busy) {
                const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
                for (int ch0 = kpi; ch0 < nch; ch0 += kLUnroll * kp) {
                    uint4 xa[kLUnroll], xb[kLUnroll], wv[kLUnroll][4];
#pragma unroll
                    for (int u = 0; u < kLUnroll; ++u) {
                        const int ch = ch0 + u * kp;
                        const bool live = ch < nch;
                        const int off = 32 * ch + 8 * c;
                        xa[u] = live && v0 ? ld16(x0 + off) : z4;
                        xb[u] = live && v1 ? ld16(x1 + off) : z4;
#pragma unroll
                        for (int t = 0; t < 4; ++t) wv[u][t] = live && wr[t] ? ld16(wr[t] + off) : z4;
                    }
                    if (a.down)
#pragma unroll
                        for (int u = 0; u < kLUnroll; ++u)
#pragma unroll
                            for (int t = 0; t < 4; ++t) wv[u][t] = to_tile_order(wv[u][t]);
                    // consecutive MMAs go to different accumulators
#pragma unroll
                    for (int u = 0; u < kLUnroll; ++u) {
#pragma unroll
                        for (int t = 0; t < 4; ++t)
                            if (kLCols * ngi + 8 * t < R)  // n8 tile inside the rows (warp-uniform)
                                mma16816(acc[t], xa[u].x, xb[u].x, xa[u].y, xb[u].y, wv[u][t].x, wv[u][t].y);
#pragma unroll
                        for (int t = 0; t < 4; ++t)
                            if (kLCols * ngi + 8 * t < R)
                                mma16816(acc[t], xa[u].z, xb[u].z, xa[u].w, xb[u].w, wv[u][t].z, wv[u][t].w);
                    }
                }
                // partial tile: rows g and g + 8 of the m tile, columns 8 t + 2 c (+1) of the row group
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    float* p0 = &s_part[warp][g][8 * t + 2 * c];
                    float* p1 = &s_part[warp][g + 8][8 * t + 2 * c];
                    p0[0] = acc[t][0];
                    p0[1] = acc[t][1];
                    p1[0] = acc[t][2];
                    p1[1] = acc[t][3];
                }
            }
            __syncthreads();
            // the K parts in a fixed order; one thread per (job, column)
            for (int q = threadIdx.x; q < nj * R; q += blockDim.x) {
                const int jj = q / R, n = q % R;
                if (s_z[jj] != ad) continue;
                const int m = jj / 16 - mlo, row = jj % 16, gi = n / kLCols, col = n % kLCols;
                float v = 0.0f;
                for (int k = 0; k < kp; ++k) v += s_part[m + mtp * (gi + ngp * k)][row][col];
                a.out[(int64_t)j0 * R + q] = v;
            }
            __syncthreads();  // s_part is rewritten by the next adapter's run
        }
    }
}

}  // namespace

cudaError_t launch_lora_a_mma(const LayerArgs& L, int down, const uint16_t* act, int ld, const Work& wk,
                              cudaStream_t s) {
    if (wk.T == 0 || wk.J == 0 || L.n_adapters == 0 || L.rank == 0) return cudaSuccess;
    if (L.E + 1 > kLMaxGroups || (down ? L.rank : 2 * L.rank) > kLCols * 4) return cudaErrorInvalidValue;
    LoraMmaArgs a;
    memset(&a, 0, sizeof(a));
    a.L = L;
    a.act = act;
    a.ld = ld;
    a.perm = wk.perm;
    a.goff = wk.goff;
    a.out = down ? wk.td : wk.tgu;
    a.down = down;
    int dev = 0, nsm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const int64_t items = (int64_t)wk.J / kLJobs + L.E + 1;  // upper bound on the items
    const int grid = (int)(items < nsm ? items : nsm);
    lora_a_mma_kernel<<<grid, kLWarps * 32, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace moeq
