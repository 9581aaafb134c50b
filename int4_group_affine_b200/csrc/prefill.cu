// prefill.cu - expert-grouped GEMMs on the tcgen05 tensor cores (sm_100a) for
// the many-token case: gate/up with fused SwiGLU, down with the routing weight,
// and the two LoRA-A products.
//
// Swap-AB: a tile is 128 weight rows (M, one TMEM lane each) by up to 64 jobs of
// one expert group (N), over K in steps of 64 (= one quantisation group of 64).
// Tiles live in shared memory K-major with the 128-byte swizzle.  Per K-step of
// 64 every thread of the CTA
//   - issues cp.async for later tiles: raw int4 words + scales/biases (or bf16
//     LoRA-A rows) 6 tiles ahead, gathered activation rows 2 tiles ahead;
//   - dequantises its share of this tile's int4 words into bf16 (one 32-bit word
//     = 8 weights = one 16-byte chunk, w = fma(q, s, b) rounded once to bf16);
// then one elected thread issues the tcgen05.mma instructions (4 per 64 of K and
// matrix) into TMEM and commits them to an mbarrier.  After the last K-step of
// a tile the CTA reads the accumulators back with tcgen05.ld and runs the
// mode's epilogue.  Persistent grid: CTA c takes items c, c + grid, ...
#include "tc.cuh"

namespace moeq {
namespace {

constexpr int kTcThreads = 256;
constexpr int kBM = 128;   // rows per MMA tile
constexpr int kNT = 64;    // jobs per tile (MMA N <= 64)
constexpr int kRA = 8;     // raw A ring slots
constexpr int kLA = 6;     // raw A lookahead (tiles)
constexpr int kRB = 4;     // activation ring slots
constexpr int kLB = 2;     // activation lookahead
constexpr int kRawBytes = 10 * 1024;      // int4: 2 x 128 x 32 B words + 2 x 2 x 128 x 4 B scale/bias pairs
constexpr int kBBytes = kNT * 128;        // 64 rows x 128 B
constexpr int kAStage = 2 * kBM * 128;    // gate + up bf16 tiles (32 KB)
constexpr int kLoraRows = 64;             // real LoRA-A rows per M tile
constexpr int kMaxGroups = MOEQ_MAX_EXPERTS + 1;
constexpr int kTBuf = kNT * 64;           // staged LoRA products (floats): 64 jobs x up to 2r = 64

enum Mode { kGU = 0, kDown = 1, kLoraGU = 2, kLoraDown = 3 };

struct TcArgs {
    LayerArgs L;
    int mode;
    const uint16_t* act;  // bf16 activation rows: x (GU, LoraGU: row = token) or h (Down, LoraDown: row = job)
    int ld_act;           // elements per activation row
    const int4* perm;     // [J] jobs {token, k, adapter, expert}
    const float* wperm;   // [J] combine weights
    const int32_t* goff;  // [E+2] job offsets of the expert groups (group E = shared expert)
    uint16_t* h_out;      // GU: [J][ldh] bf16
    int ldh;
    float* ypart;         // Down: [J][H]
    float* t_out;         // LoraGU: [J][2r], LoraDown: [J][r]
    const float* t_in;    // GU: [J][2r], Down: [J][r]
    int32_t* status;
};

struct Geo {  // one expert group's geometry in the current mode
    int M, K, mtiles, ntiles, mat;
    bool shared, skip;
};

__device__ __forceinline__ Geo geo_of(const TcArgs& a, int g, int count) {
    const LayerArgs& L = a.L;
    Geo q;
    q.shared = g == L.E;
    q.skip = count == 0 || (q.shared && !L.has_shared);
    q.mat = q.shared ? 0 : g;
    const int I = q.shared ? L.Is : L.I;
    const int r = L.rank;
    switch (a.mode) {
        case kGU: q.M = I; q.K = L.H; break;
        case kDown: q.M = L.H; q.K = I; break;
        case kLoraGU: q.M = L.n_adapters * 2 * r; q.K = L.H; break;
        default: q.M = L.n_adapters * r; q.K = I; break;
    }
    if (q.M <= 0) q.skip = true;
    const int rows_per_tile = (a.mode == kGU || a.mode == kDown) ? kBM : kLoraRows;
    q.mtiles = q.skip ? 0 : (q.M + rows_per_tile - 1) / rows_per_tile;
    q.ntiles = q.skip ? 0 : (count + kNT - 1) / kNT;
    return q;
}

// Position in this CTA's stream of (item, k-step) tiles.
struct Pos {
    int item;  // global item index (>= nitems: past the end)
    int kt;    // k-step inside the item
    int g, mt, nt, KT;
};

__device__ __forceinline__ const moe_qtensor& wmat(const LayerArgs& L, int mode, bool shared, int which) {
    if (mode == kGU) return which == 0 ? (shared ? L.s_gate : L.gate) : (shared ? L.s_up : L.up);
    return shared ? L.s_down : L.down;
}

__device__ __forceinline__ const moe_lora_proj* tlora(const LayerArgs& L, int a, bool shared, int which) {
    if (a < 0 || a >= L.n_adapters) return nullptr;
    const moe_lora_ptrs& p = L.lora[a];
    const moe_lora_proj* q = which == 0 ? (shared ? &p.s_gate : &p.gate)
                           : which == 1 ? (shared ? &p.s_up : &p.up)
                                        : (shared ? &p.s_down : &p.down);
    return (q->A && q->B) ? q : nullptr;
}

// 8 nibbles of one word -> 8 bf16 (s*q + b, one rounding), in element order.
__device__ __forceinline__ uint4 dequant8(uint32_t w, __nv_bfloat162 s2, __nv_bfloat162 b2) {
    const __nv_bfloat162 k128 = __float2bfloat162_rn(128.0f);
    uint32_t r[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t v = ((w >> (4 * j)) & 0x000F000Fu) | 0x43004300u;  // {128 + q_j, 128 + q_{j+4}}
        __nv_bfloat162 q = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&v), k128);
        __nv_bfloat162 d = __hfma2(q, s2, b2);
        r[j] = *reinterpret_cast<uint32_t*>(&d);
    }
    uint4 o;
    o.x = __byte_perm(r[0], r[1], 0x5410);  // e0 e1
    o.y = __byte_perm(r[2], r[3], 0x5410);  // e2 e3
    o.z = __byte_perm(r[0], r[1], 0x7632);  // e4 e5
    o.w = __byte_perm(r[2], r[3], 0x7632);  // e6 e7
    return o;
}

__global__ void __launch_bounds__(kTcThreads, 1) tc_gemm_kernel(const __grid_constant__ TcArgs a) {
    extern __shared__ __align__(1024) unsigned char tsm_raw[];
    // 128-byte-swizzled tiles need 1024-byte aligned bases: align by hand (the
    // launch requests 1 KB of slack).
    unsigned char* tsm = tsm_raw + ((1024u - (tc::smem_u32(tsm_raw) & 1023u)) & 1023u);
    const LayerArgs& L = a.L;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int mode = a.mode;
    const bool int4_mode = mode == kGU || mode == kDown;
    const int nmat = mode == kGU ? 2 : 1;
    const int r = L.rank;

    // shared memory: [A stages 2 x 32 KB][activation ring 4 x 8 KB][raw ring 8 x 10 KB]
    unsigned char* sA = tsm;
    unsigned char* sB = sA + 2 * kAStage;
    unsigned char* sR = sB + kRB * kBBytes;
    __shared__ uint64_t bar_tile[4];
    __shared__ uint64_t bar_acc;
    __shared__ uint32_t s_tmem;
    __shared__ int s_items[kMaxGroups + 1];
    __shared__ int s_goff[kMaxGroups + 1];
    __shared__ int4 s_job[3][kNT];      // job entries of the three most recent loader items
    __shared__ float s_wt[3][kNT];
    __shared__ float s_t[kTBuf];        // staged LoRA products for the epilogue
    __shared__ int s_ok;

    // ---------------------------------------------------------- set-up
    const int ngroups = L.E + 1;
    for (int g = tid; g <= ngroups; g += kTcThreads) s_goff[g] = a.goff[g];
    if (warp == 0) {
        tc::tmem_alloc(&s_tmem, 512);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 4; ++i) tc::mbar_init(&bar_tile[i], 1);
        tc::mbar_init(&bar_acc, 1);
        tc::mbar_init_fence();
        s_ok = 1;
    }
    // zero both A stages once (LoRA modes never write rows 64..127)
    for (int i = tid; i < 2 * kAStage / 16; i += kTcThreads) reinterpret_cast<uint4*>(sA)[i] = make_uint4(0, 0, 0, 0);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = s_tmem;
    // item prefix over groups (every CTA computes the same table)
    if (tid == 0) {
        int acc = 0;
        for (int g = 0; g < ngroups; ++g) {
            s_items[g] = acc;
            const Geo q = geo_of(a, g, s_goff[g + 1] - s_goff[g]);
            acc += q.mtiles * q.ntiles;
        }
        s_items[ngroups] = acc;
    }
    __syncthreads();
    const int nitems = s_items[ngroups];
    const int NB = gridDim.x;

    auto decode = [&](int item, Pos& p) {
        p.item = item;
        p.kt = 0;
        if (item >= nitems) {
            p.g = p.mt = p.nt = 0;
            p.KT = 1;
            return;
        }
        int lo = 0, hi = ngroups - 1;  // last group with s_items[g] <= item
        while (lo < hi) {
            const int mid = (lo + hi + 1) / 2;
            if (s_items[mid] <= item) lo = mid;
            else hi = mid - 1;
        }
        const Geo q = geo_of(a, lo, s_goff[lo + 1] - s_goff[lo]);
        const int rem = item - s_items[lo];
        p.g = lo;
        p.mt = rem / q.ntiles;
        p.nt = rem % q.ntiles;
        p.KT = q.K / 64;
    };
    auto advance = [&](Pos& p) {
        if (p.item >= nitems) return;
        if (++p.kt == p.KT) decode(p.item + NB, p);
    };

    // ---------------------------------------------------------- loaders
    // raw A of tile position p into raw slot `slot`
    auto load_raw = [&](const Pos& p, int slot) {
        if (p.item >= nitems) return;
        unsigned char* raw = sR + slot * kRawBytes;
        const Geo q = geo_of(a, p.g, s_goff[p.g + 1] - s_goff[p.g]);
        if (int4_mode) {
            const int ng = q.K / wmat(L, mode, q.shared, 0).group;
            const int group = wmat(L, mode, q.shared, 0).group;
            const int gidx = (p.kt * 64) / group;
            const int pair = gidx & ~1;
            for (int u = tid; u < nmat * kBM * 4; u += kTcThreads) {  // 2 x 16 B of words, s pair, b pair
                const int mat = u / (kBM * 4), row = (u / 4) % kBM, part = u % 4;
                const moe_qtensor& W = wmat(L, mode, q.shared, mat);
                const int R = p.mt * kBM + row;
                const bool live = R < q.M;
                const int64_t grow = (int64_t)q.mat * q.M + (live ? R : 0);
                if (part < 2) {
                    const uint32_t* src = W.packed + grow * (q.K / 8) + p.kt * 8 + part * 4;
                    tc::cp16(tc::smem_u32(raw + (mat * kBM + row) * 32 + part * 16), src, live ? 16u : 0u);
                } else {
                    const uint16_t* base = part == 2 ? W.scales : W.biases;
                    unsigned char* dst = raw + 8192 + ((part - 2) * 2 * kBM + mat * kBM + row) * 4;
                    if (live) tc::cp4(tc::smem_u32(dst), base + grow * ng + pair);
                    else *reinterpret_cast<uint32_t*>(dst) = 0u;
                }
            }
        } else {
            // LoRA-A rows (bf16): tile rows 0..63 of M tile mt
            const int rpa = mode == kLoraGU ? 2 * r : r;
            for (int u = tid; u < kLoraRows * 8; u += kTcThreads) {
                const int row = u / 8, c = u % 8;
                const int R = p.mt * kLoraRows + row;
                const int ad = R / rpa, d = R % rpa;
                const uint16_t* src = nullptr;
                if (R < q.M) {
                    const int which = mode == kLoraGU ? (d < r ? 0 : 1) : 2;
                    const moe_lora_proj* lp = tlora(L, ad, q.shared, which);
                    if (lp) src = lp->A + ((int64_t)q.mat * r + (mode == kLoraGU ? d % r : d)) * q.K + p.kt * 64 + c * 8;
                }
                tc::cp16(tc::smem_u32(raw + row * 128 + c * 16), src ? src : a.act, src ? 16u : 0u);
            }
        }
    };
    // activation rows of tile position p into activation slot `slot`; `tab` is the
    // job table of p's item (filled when the loader enters the item)
    auto load_b = [&](const Pos& p, int slot, int tab) {
        if (p.item >= nitems) return;
        unsigned char* dst = sB + slot * kBBytes;
        const int base = s_goff[p.g] + p.nt * kNT, end = s_goff[p.g + 1];
        const bool by_token = mode == kGU || mode == kLoraGU;
        for (int u = tid; u < kNT * 8; u += kTcThreads) {
            const int n = u / 8, c = u % 8;
            const int job = base + n;
            const bool live = job < end;
            const int64_t rowi = live ? (by_token ? s_job[tab][n].x : job) : 0;
            const uint16_t* src = a.act + rowi * a.ld_act + p.kt * 64 + c * 8;
            tc::cp16(tc::smem_u32(dst + tc::sw128_off(n, c)), src, live ? 16u : 0u);
        }
    };
    auto fill_table = [&](const Pos& p, int tab) {
        if (p.item >= nitems) return;
        const int base = s_goff[p.g] + p.nt * kNT, end = s_goff[p.g + 1];
        if (tid < kNT) {
            const int job = base + tid;
            s_job[tab][tid] = job < end ? a.perm[job] : make_int4(0, 0, -1, 0);
            s_wt[tab][tid] = (job < end && a.wperm) ? a.wperm[job] : 0.0f;
        }
    };

    // ---------------------------------------------------------- stream
    Pos pc, pa, pb;  // consumer, raw-A loader, activation loader
    decode(blockIdx.x, pc);
    pa = pc;
    pb = pc;
    int tab_b = 0;  // job-table slot of the activation loader's item (items cycle through 3 slots)
    int seq_b = 0;  // items entered by the activation loader
    int seq_c = 0;  // items entered by the consumer
    // prologue: raw tiles 0..kLA-1 and activation tiles 0..kLB-1
    fill_table(pb, 0);
    __syncthreads();
    for (int i = 0; i < kLA; ++i) {
        load_raw(pa, i % kRA);
        if (i < kLB) {
            load_b(pb, i % kRB, tab_b);
            const int prev = pb.item;
            advance(pb);
            if (pb.item != prev) {
                ++seq_b;
                tab_b = seq_b % 3;
                __syncthreads();
                fill_table(pb, tab_b);
                __syncthreads();
            }
        }
        tc::cp_commit();
        advance(pa);
    }

    uint32_t t = 0;        // tiles consumed by this CTA
    uint32_t n_items = 0;  // items finished by this CTA
    while (pc.item < nitems) {
        // the MMAs of tile t-2 must be done before stage t%2 and activation slot (t+2)%4 are rewritten
        if (t >= 2) {
            const uint32_t tp = t - 2;
            if (!tc::mbar_wait(&bar_tile[tp % 4], (tp / 4) & 1u, a.status)) s_ok = 0;
        }
        // issue loads for raw tile t+kLA and activation tile t+kLB
        load_raw(pa, (t + kLA) % kRA);
        advance(pa);
        load_b(pb, (t + kLB) % kRB, tab_b);
        tc::cp_commit();
        {
            const int prev = pb.item;
            advance(pb);
            if (pb.item != prev) {
                ++seq_b;
                tab_b = seq_b % 3;
                fill_table(pb, tab_b);
            }
        }
        tc::cp_wait<2>();  // this tile's group (issued kLB steps ago) has landed
        __syncthreads();

        const Geo q = geo_of(a, pc.g, s_goff[pc.g + 1] - s_goff[pc.g]);
        const int n_here = min(kNT, s_goff[pc.g + 1] - s_goff[pc.g] - pc.nt * kNT);
        const int Nmma = (n_here + 15) / 16 * 16;
        unsigned char* stA = sA + (t % 2) * kAStage;
        const unsigned char* raw = sR + (t % kRA) * kRawBytes;
        if (int4_mode) {
            const int group = wmat(L, mode, q.shared, 0).group;
            const int gidx0 = (pc.kt * 64) / group, pair = gidx0 & ~1;
            for (int u = tid; u < nmat * kBM * 8; u += kTcThreads) {
                const int mat = u / (kBM * 8), row = (u / 8) % kBM, c = u % 8;
                const uint32_t w = *reinterpret_cast<const uint32_t*>(raw + (mat * kBM + row) * 32 + c * 4);
                const int gsel = (pc.kt * 64 + c * 8) / group - pair;  // 0 or 1 inside the loaded pair
                const __nv_bfloat16* sp =
                    reinterpret_cast<const __nv_bfloat16*>(raw + 8192 + (0 * 2 * kBM + mat * kBM + row) * 4);
                const __nv_bfloat16* bp =
                    reinterpret_cast<const __nv_bfloat16*>(raw + 8192 + (1 * 2 * kBM + mat * kBM + row) * 4);
                const __nv_bfloat162 s2 = __bfloat162bfloat162(sp[gsel]);
                const __nv_bfloat162 b2 = __bfloat162bfloat162(bp[gsel]);
                *reinterpret_cast<uint4*>(stA + mat * (kBM * 128) + tc::sw128_off(row, c)) = dequant8(w, s2, b2);
            }
        } else {
            for (int u = tid; u < kLoraRows * 8; u += kTcThreads) {
                const int row = u / 8, c = u % 8;
                *reinterpret_cast<uint4*>(stA + tc::sw128_off(row, c)) =
                    *reinterpret_cast<const uint4*>(raw + row * 128 + c * 16);
            }
        }
        tc::fence_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        if (!s_ok) break;
        tc::tc_fence_after();
        if (tid == 0) {
            const uint32_t idesc = tc::idesc_bf16(kBM, Nmma);
            const uint32_t bbase = tc::smem_u32(sB + (t % kRB) * kBBytes);
            for (int mat = 0; mat < nmat; ++mat) {
                const uint32_t abase = tc::smem_u32(stA + mat * (kBM * 128));
                const uint64_t ad = tc::sdesc_k_sw128(abase), bd = tc::sdesc_k_sw128(bbase);
                for (int k = 0; k < 4; ++k)  // 4 x K=16 inside the 128-byte swizzle atom: +32 B each
                    tc::mma_bf16(tmem + mat * 256, ad + 2 * k, bd + 2 * k, idesc, (pc.kt > 0 || k > 0) ? 1u : 0u);
            }
            tc::mma_commit(&bar_tile[t % 4]);
            if (pc.kt == pc.KT - 1) tc::mma_commit(&bar_acc);
        }
        ++t;

        if (pc.kt == pc.KT - 1) {
            // ---------------------------------------------------- epilogue
            if (!tc::mbar_wait(&bar_acc, n_items & 1u, a.status)) s_ok = 0;
            ++n_items;
            tc::tc_fence_after();
            const int tab_c = seq_c % 3;
            const int base = s_goff[pc.g] + pc.nt * kNT;
            // LoRA products of this tile's jobs into shared memory
            const int tw = mode == kGU ? 2 * r : (mode == kDown ? r : 0);
            if (tw > 0)
                for (int u = tid; u < kNT * tw; u += kTcThreads) {
                    const int n = u / tw, k = u % tw;
                    s_t[u] = n < n_here ? a.t_in[(int64_t)(base + n) * tw + k] : 0.0f;
                }
            __syncthreads();
            const int quarter = warp % 4, half = warp / 4;
            const int row = quarter * 32 + lane;  // TMEM lane of this thread
            for (int ch = half; ch * 16 < Nmma; ch += 2) {
                uint32_t d0[16], d1[16];
                const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + ch * 16;
                tc::tmem_ld16(taddr, d0);
                if (mode == kGU) tc::tmem_ld16(taddr + 256, d1);
                tc::tmem_wait_ld();
                if (mode == kGU) {
                    const int i = pc.mt * kBM + row;
                    if (i < q.M) {
                        const moe_lora_proj* lg = nullptr;
                        const moe_lora_proj* lu = nullptr;
                        int cur = -2;
                        float bgv[MOEQ_MAX_RANK / 2], buv[MOEQ_MAX_RANK / 2];
                        for (int c = 0; c < 16; ++c) {
                            const int n = ch * 16 + c;
                            if (n >= n_here) break;
                            const int4 job = s_job[tab_c][n];
                            float g = __uint_as_float(d0[c]), u = __uint_as_float(d1[c]);
                            if (job.z != cur) {  // jobs are sorted by adapter: reload B rows per run
                                cur = job.z;
                                lg = tlora(L, cur, q.shared, 0);
                                lu = tlora(L, cur, q.shared, 1);
                                for (int k = 0; k < r && k < MOEQ_MAX_RANK / 2; ++k) {
                                    bgv[k] = lg ? bf16f(lg->B[((int64_t)q.mat * q.M + i) * r + k]) : 0.0f;
                                    buv[k] = lu ? bf16f(lu->B[((int64_t)q.mat * q.M + i) * r + k]) : 0.0f;
                                }
                            }
                            if (lg || lu) {
                                float dg = 0.0f, du = 0.0f;
                                for (int k = 0; k < r && k < MOEQ_MAX_RANK / 2; ++k) {
                                    dg = fmaf(bgv[k], s_t[n * tw + k], dg);
                                    du = fmaf(buv[k], s_t[n * tw + r + k], du);
                                }
                                g += L.scale * dg;
                                u += L.scale * du;
                            }
                            a.h_out[(int64_t)(base + n) * a.ldh + i] = f2bf16(silu(g) * u);
                        }
                    }
                } else if (mode == kDown) {
                    const int o = pc.mt * kBM + row;
                    if (o < q.M) {
                        const moe_lora_proj* ld = nullptr;
                        int cur = -2;
                        float bdv[MOEQ_MAX_RANK / 2];
                        for (int c = 0; c < 16; ++c) {
                            const int n = ch * 16 + c;
                            if (n >= n_here) break;
                            const int4 job = s_job[tab_c][n];
                            float v = __uint_as_float(d0[c]);
                            if (job.z != cur) {
                                cur = job.z;
                                ld = tlora(L, cur, q.shared, 2);
                                for (int k = 0; k < r && k < MOEQ_MAX_RANK / 2; ++k)
                                    bdv[k] = ld ? bf16f(ld->B[((int64_t)q.mat * L.H + o) * r + k]) : 0.0f;
                            }
                            if (ld) {
                                float dd = 0.0f;
                                for (int k = 0; k < r && k < MOEQ_MAX_RANK / 2; ++k) dd = fmaf(bdv[k], s_t[n * tw + k], dd);
                                v += L.scale * dd;
                            }
                            a.ypart[(int64_t)(base + n) * L.H + o] = s_wt[tab_c][n] * v;
                        }
                    }
                } else {
                    const int rpa = mode == kLoraGU ? 2 * r : r;
                    const int R = pc.mt * kLoraRows + row;
                    if (row < kLoraRows && R < q.M) {
                        const int ad = R / rpa, d = R % rpa;
                        for (int c = 0; c < 16; ++c) {
                            const int n = ch * 16 + c;
                            if (n >= n_here) break;
                            if (s_job[tab_c][n].z == ad) a.t_out[(int64_t)(base + n) * rpa + d] = __uint_as_float(d0[c]);
                        }
                    }
                }
            }
            tc::tc_fence_before();
            __syncthreads();
            ++seq_c;
        }
        advance(pc);
    }
    // drain: no cp.async may still target this CTA's shared memory at exit
    tc::cp_wait<0>();
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

}  // namespace

// Host-side conditions of the tensor-core path.
bool tc_supported(const LayerArgs& L) {
    if (L.H % 128 || L.I % 128 || L.H < 128 || L.I < 128) return false;
    if (L.has_shared && (L.Is % 128 || L.Is < 128)) return false;
    if (L.gate.group != 64 && L.gate.group != 32) return false;
    if (L.down.group != L.gate.group || (L.has_shared && (L.s_gate.group != L.gate.group || L.s_down.group != L.gate.group)))
        return false;
    if (L.rank > MOEQ_MAX_RANK / 2) return false;
    if (L.E + 1 > kMaxGroups) return false;
    // scale/bias pairs are fetched as 4-byte words
    const moe_qtensor* ts[] = {&L.gate, &L.up, &L.down, &L.s_gate, &L.s_up, &L.s_down};
    for (const moe_qtensor* q : ts)
        if (q->packed && (((uintptr_t)q->scales & 3) || ((uintptr_t)q->biases & 3))) return false;
    return true;
}

size_t tc_smem_bytes() { return 2 * kAStage + kRB * kBBytes + kRA * kRawBytes + 1024; }

cudaError_t launch_tc_gemm(const LayerArgs& L, int mode, const uint16_t* act, int ld_act, const Work& wk,
                           const uint16_t* hb_out, int ldh, cudaStream_t s) {
    static int cached = 0;
    const size_t smem = tc_smem_bytes();
    cudaError_t e = ensure_smem((const void*)tc_gemm_kernel, smem, cached);
    if (e != cudaSuccess) return e;
    int nsm = 0, dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    TcArgs a;
    a.L = L;
    a.mode = mode;
    a.act = act;
    a.ld_act = ld_act;
    a.perm = wk.perm;
    a.wperm = wk.wperm;
    a.goff = wk.goff;
    a.h_out = const_cast<uint16_t*>(hb_out);
    a.ldh = ldh;
    a.ypart = wk.ypart;
    a.t_out = mode == kLoraGU ? wk.tgu : wk.td;
    a.t_in = mode == kGU ? wk.tgu : wk.td;
    a.status = wk.status;
    tc_gemm_kernel<<<nsm, kTcThreads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace moeq
