// prefill.cu - expert-grouped GEMMs on the tcgen05 tensor cores (sm_100a) for
// the many-token case: the 8-bit router, gate/up with fused SwiGLU and down with
// the routing weight, each with its LoRA-B term (the LoRA-A products come from
// warp-level tiles, lora_mma.cu).
//
// Swap-AB: a tile is weight rows (M = 128 per block, one TMEM lane each) by up
// to 64 jobs of one expert group (N), over K in steps of 128 (two 64-wide
// operand sub-tiles).
//
// Weights stream through the tensor memory accelerator: for each span of 128
// bytes of packed words per row (K = 256 for int4, 128 for int8) the loader warp
// loads a 128-row box per block with cp.async.bulk.tensor (128-byte swizzle)
// into a ring of four slots, so DRAM sees whole 128-byte lines.  Each
// dequantisation thread owns one weight row and thus one TMEM lane: it keeps the
// row's scales and biases in registers one span ahead, dequantises the row's
// weights of each K-step into bf16 (w = fma(q, s, b), one rounding) and writes
// them with tcgen05.st into one of two TMEM stages, the A operand of the MMA; the
// dequantised tile never touches shared memory.  Within every 8 consecutive K
// the tiles hold the order 0 4 1 5 2 6 3 7, the order in which the nibbles of a
// word come out of two shift-and-mask steps, so no byte permutes are spent; the
// activations carry the same order (x permuted once, h written permuted by the
// gate/up epilogue), and a dot product does not depend on the order of its terms.
//
// Activations (operand B) fill a K-major 128-byte-swizzled ring of four slots,
// two steps ahead of the dequantisation: TMA boxes where the rows are contiguous
// (the h rows of the jobs for down, the tokens for the router), cp.async by the
// loader's lanes where they are scattered (gate/up gathers x by token).  One lane of the MMA warp issues the MMAs (8 x
// K=16 per block per step) and commits them to per-step mbarriers; accumulators
// are double-buffered in TMEM and each item's epilogue runs a few steps after its
// last MMA, so the dequantisation never waits on the tensor core at item ends.
//
// The unmerged LoRA-B term (alpha/r) B (A x) is one more MMA K-step per item
// (per 64 columns of K' = adapters x r per matrix): operand A holds the LoRA-B
// rows of every adapter side by side along K', operand B holds each job's scaled
// LoRA-A products in its own adapter's columns (zero elsewhere), so the product
// adds exactly each job's own adapter term into the accumulator.  Operand A is a
// pseudo-span of the weight ring that the loader fills with cp.async (zero past
// the adapters' columns); operand B is staged by the dequantisation threads from
// registers fetched a step ahead.
//
//   gate/up: block 0 = gate rows, block 1 = up rows, two accumulators; epilogue
//            SiLU(g) * u -> h (bf16).
//   down:    blocks = two consecutive 128-row blocks of down_proj; epilogue
//            scales by the job's combine weight -> ypart.
//   router:  int8 rows; block 0 = bf16(w), block 1 = bf16(w - bf16(w)), both
//            into one accumulator, so the logits carry ~16 bits of each weight;
//            epilogue adds the logit bias -> logits.
//
// Warp roles: 8 dequantisation warps (16 in down mode: TcWarps) (scales, dequant, LoRA-B operand, epilogue),
// one MMA warp and one loader warp (weight spans, activations, LoRA-B rows); they
// hand steps over through mbarriers, so no CTA-wide barrier sits in the K loop.
// Every wait is bounded in time and raises MOE_ERR_TIMEOUT when it gives up.
// Persistent grid: CTA c takes items c, c + grid, ...
#include <cudaTypedefs.h>

#include "tc.cuh"

namespace moeq {
namespace {

constexpr int kBM = 128;                          // rows per MMA block
constexpr int kNT = 64;                           // jobs per tile (MMA N <= 64)
constexpr int kKS = 128;                          // K per pipeline step (two 64-wide operand sub-tiles)
constexpr int kAS = 2;                            // A stages in TMEM (dequantisation runs up to kAS steps ahead)
constexpr int kLB = 2;                            // activation lookahead (steps)
constexpr int kRB = kLB + kAS;                    // activation ring: slot of step t - kAS is free at step t
constexpr int kRS = 4;                            // weight span ring (two spans in flight)
constexpr int kTiles = 16;                        // per-step MMA completion barriers
constexpr int kSpanBytes = kBM * 128;             // one block of one span: 128 rows x 128 B
constexpr int kRawSlot = 2 * kSpanBytes;          // two blocks
constexpr int kSub = kNT * 128;                   // one 64-wide K sub-tile of 64 rows (128 B per row)
constexpr int kBSlot = 2 * kSub;                  // activation ring slot: the step's two sub-tiles
constexpr int kMaxGroups = MOEQ_MAX_EXPERTS + 1;
// TMEM columns: accumulator D(buffer b, block k) at 128 b + 64 k; A stage s, block k at 256 + 128 s + 64 k
constexpr uint32_t kTmemA = 256;
static_assert(kTmemA + kAS * 128 <= 512, "TMEM columns");

enum Mode { kGU = 0, kDown = 1, kRouterMode = 4 };

// Dequantisation warps per mode: 16 for down (two threads per weight row, each half of a
// step's words: measured 174 against 192 us per prefill layer), 8 elsewhere (gate/up ran
// 318 against 268 us with 16: the step's TMEM stores and the per-thread state of the
// LoRA-B operand then outweigh the shorter dequantisation chains).
template <int kMode>
struct TcWarps {
    static constexpr int deq = kMode == kDown ? 16 : 8;
    static constexpr int threads = (deq + 2) * 32;
};

struct TcArgs {
    CUtensorMap tm[4];    // weight words: gate/up {gate, up, s_gate, s_up}; down {down, s_down}; router {router}
    CUtensorMap tmb;      // bf16 activations in 64 x 64 boxes: down the h rows of the jobs, router the
                          // token rows of x
    LayerArgs L;
    int mode;
    const uint16_t* act;  // bf16 activation rows: x (by token) or h (by job)
    int ld_act;           // elements per activation row
    const int4* perm;     // [J] jobs {token, k, adapter, expert}
    const float* wperm;   // [J] combine weights
    const int32_t* goff;  // [E+2] job offsets of the expert groups (group E = shared expert)
    uint16_t* h_out;      // gate/up: [J][ldh] bf16
    int ldh;
    float* ypart;         // down: [J][H]
    const float* t_in;    // gate/up: [J][2r], down: [J][r]
    float* logits;        // router: [T][E]
    int T;                // router: tokens
    int32_t* status;
    uint64_t wait_ns;     // bound of every mbarrier wait
};

struct Geo {  // one expert group's geometry in the current mode
    int M, K, mtiles, ntiles, mat;
    bool shared, skip;
};

__device__ __forceinline__ int rows_per_item(int mode) {
    return mode == kDown ? 2 * kBM : kBM;
}

__device__ __forceinline__ Geo geo_of(const TcArgs& a, int mode, int g, int count) {
    const LayerArgs& L = a.L;
    Geo q;
    q.shared = mode != kRouterMode && g == L.E;
    q.skip = count == 0 || (q.shared && !L.has_shared);
    q.mat = q.shared ? 0 : g;
    const int I = q.shared ? L.Is : L.I;
    const int r = L.rank;
    switch (mode) {
        case kGU: q.M = I; q.K = L.H; break;
        case kDown: q.M = L.H; q.K = I; break;
        default: q.M = L.E; q.K = L.H; q.mat = 0; break;
    }
    if (q.M <= 0) q.skip = true;
    const int rpi = rows_per_item(mode);
    q.mtiles = q.skip ? 0 : (q.M + rpi - 1) / rpi;
    q.ntiles = q.skip ? 0 : (count + kNT - 1) / kNT;
    return q;
}

// Position in this CTA's stream of (item, k-step) tiles.
struct Pos {
    int item;  // global item index (>= nitems: past the end)
    int kt;    // k-step inside the item: [0, KW) weight steps, [KW, KT) LoRA-B steps
    int g, mt, nt, KW, KT;
};

__device__ __forceinline__ const moe_lora_proj* tlora(const LayerArgs& L, int a, bool shared, int which) {
    if (a < 0 || a >= L.n_adapters) return nullptr;
    const moe_lora_ptrs& p = L.lora[a];
    const moe_lora_proj* q = which == 0 ? (shared ? &p.s_gate : &p.gate)
                           : which == 1 ? (shared ? &p.s_up : &p.up)
                                        : (shared ? &p.s_down : &p.down);
    return (q->A && q->B) ? q : nullptr;
}

// 8 nibbles of one word -> 8 bf16 (s*q + b, one rounding) as the pairs
// (q0, q4), (q1, q5), (q2, q6), (q3, q7): the K order of every 8-group is
// permuted to 0 4 1 5 2 6 3 7, and the activations the MMA multiplies them with
// are stored in the same order (permute_k8), so the products are unchanged.
__device__ __forceinline__ uint4 dequant8p(uint32_t w, __nv_bfloat162 s2, __nv_bfloat162 b2) {
    const __nv_bfloat162 k128 = __float2bfloat162_rn(128.0f);
    uint32_t r[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t v = ((w >> (4 * j)) & 0x000F000Fu) | 0x43004300u;  // {128 + q_j, 128 + q_{j+4}}
        __nv_bfloat162 q = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&v), k128);
        __nv_bfloat162 d = __hfma2(q, s2, b2);
        r[j] = *reinterpret_cast<uint32_t*>(&d);
    }
    return make_uint4(r[0], r[1], r[2], r[3]);
}

// The same K permutation applied to 8 bf16 in element order (one 16-byte chunk).
__device__ __forceinline__ uint4 permute_k8(uint4 u) {
    return make_uint4(__byte_perm(u.x, u.z, 0x5410), __byte_perm(u.x, u.z, 0x7632), __byte_perm(u.y, u.w, 0x5410),
                      __byte_perm(u.y, u.w, 0x7632));
}

// Position of K element i in the permuted order.
__device__ __forceinline__ int kperm_pos(int i) { return (i & ~7) | ((i & 3) << 1) | ((i >> 2) & 1); }

// Two int8 words (8 codes) -> hi = bf16(w) and lo = bf16(w - hi) for w = s*q + b in fp32.
__device__ __forceinline__ void dequant8_hilo(uint32_t w0, uint32_t w1, float s, float b, uint32_t* hi, uint32_t* lo) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const uint32_t w = p < 2 ? w0 : w1;
        const int sh = 16 * (p & 1);
        const float v0 = fmaf(s, u2f_small((w >> sh) & 0xFFu), b);
        const float v1 = fmaf(s, u2f_small((w >> (sh + 8)) & 0xFFu), b);
        const __nv_bfloat162 hv = __floats2bfloat162_rn(v0, v1);
        const float2 hf = __bfloat1622float2(hv);
        const __nv_bfloat162 lv = __floats2bfloat162_rn(v0 - hf.x, v1 - hf.y);
        hi[p] = *reinterpret_cast<const uint32_t*>(&hv);
        lo[p] = *reinterpret_cast<const uint32_t*>(&lv);
    }
}

// SiLU with the fast exponential and division (a few ulp; the result is rounded to bf16)
__device__ __forceinline__ float silu_fast(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

__device__ __forceinline__ uint32_t pick4(const uint32_t (&v)[4], int i) {
    return i == 0 ? v[0] : i == 1 ? v[1] : i == 2 ? v[2] : v[3];
}
// bf16 number g (0..7) of four words of bf16 pairs
__device__ __forceinline__ uint32_t bf16_at(const uint32_t (&v)[4], int g) {
    return (pick4(v, g >> 1) >> (16 * (g & 1))) & 0xFFFFu;
}
__device__ __forceinline__ __nv_bfloat162 bf16x2_of(uint32_t h) {
    return __bfloat162bfloat162(__ushort_as_bfloat16((unsigned short)h));
}

// This thread's activation rows (and LoRA-A rows) of one item.
struct BCtx {
    const uint16_t* src[2];
    const uint16_t* la[2];  // LoRA-A modes: bf16 A rows (NULL: zero fill)
    bool live[2];
};

// LoRA-B operand B of one step, fetched a step ahead: the thread's job rows, chunk bch,
// sub-tiles 0, 1
template <int LJ>
struct LoraRegs {
    float4 t[LJ][2][2];  // [row][sub-tile][half], unscaled LoRA-A products
    uint32_t live;       // bit (2 row + sub)
};

template <int kMode>
__global__ void __launch_bounds__(TcWarps<kMode>::threads, 1) tc_gemm_kernel(const __grid_constant__ TcArgs a) {
    // warp roles of this mode: dequantisation warps, then the MMA warp and the loader warp
    constexpr int kDeqW = TcWarps<kMode>::deq, kMmaW = kDeqW, kLoadW = kDeqW + 1, kThreads = TcWarps<kMode>::threads;
    constexpr int NQ = kDeqW / 8;               // threads per (block, weight row)
    constexpr int kLRows = kDeqW * 32 / 8;      // distinct LoRA-B operand job rows over the dequantisation threads
    constexpr int kLJ = kNT / kLRows;           // job rows per thread
    extern __shared__ __align__(1024) unsigned char tsm_raw[];
    // 128-byte-swizzled tiles need 1024-byte aligned bases: align by hand (the
    // launch requests 1 KB of slack).
    unsigned char* tsm = tsm_raw + ((1024u - (tc::smem_u32(tsm_raw) & 1023u)) & 1023u);
    const LayerArgs& L = a.L;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    constexpr int mode = kMode;
    // activation tiles by TMA boxes (rows contiguous in the activation matrix); the gate/up
    // rows are tokens scattered over x and the LoRA-A modes add the adapters' rows: cp.async
    constexpr bool tma_b = mode == kDown || mode == kRouterMode;
    constexpr bool int8_mode = mode == kRouterMode;
    constexpr bool int4_mode = mode == kGU || mode == kDown;
    constexpr int SP = int8_mode ? 1 : 2;  // steps per weight span (128 B of words per row)
    const int r = L.rank;
    const int nar = L.n_adapters * r;   // LoRA-B K' per matrix
    const int NL = (int4_mode && r > 0 && L.n_adapters > 0) ? (nar + 63) / 64 : 0;

    // shared memory: [activation ring kRB x 16 KB][weight ring kRS x 32 KB]
    unsigned char* sB = tsm;
    unsigned char* sR = sB + kRB * kBSlot;
    __shared__ uint64_t bar_full[kAS];     // step's A stage (or LoRA-B operand B) written: one arrival per dequant warp
    __shared__ uint64_t bar_bfull[kRB];    // step's activation slot (and LoRA-A rows) landed: 32 loader lanes
    __shared__ uint64_t bar_tile[kTiles];  // MMAs of a step done (tcgen05.commit)
    __shared__ uint64_t bar_acc[2];        // MMAs of an item done, per accumulator buffer
    __shared__ uint64_t bar_raw[kRS];      // span landed: 32 loader lanes (+ TMA transaction count)
    __shared__ uint64_t bar_rawfree[kRS];  // span consumed: one arrival per dequant warp
    __shared__ uint32_t s_tmem;
    __shared__ int s_items[kMaxGroups + 1];
    __shared__ int s_goff[kMaxGroups + 1];
    __shared__ volatile int s_ok;

    // ---------------------------------------------------------- set-up
    const int ngroups = int8_mode ? 1 : L.E + 1;
    if (int8_mode) {
        if (tid == 0) {
            s_goff[0] = 0;
            s_goff[1] = a.T;
        }
    } else {
        for (int g = tid; g <= ngroups; g += kThreads) s_goff[g] = a.goff[g];
    }
    if (warp == kMmaW) {
        tc::tmem_alloc(&s_tmem, 512);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < kAS; ++i) tc::mbar_init(&bar_full[i], kDeqW);
        for (int i = 0; i < kRB; ++i) tc::mbar_init(&bar_bfull[i], 32);
        for (int i = 0; i < kTiles; ++i) tc::mbar_init(&bar_tile[i], 1);
        for (int i = 0; i < kRS; ++i) {
            tc::mbar_init(&bar_raw[i], 32);
            tc::mbar_init(&bar_rawfree[i], kDeqW);
        }
        tc::mbar_init(&bar_acc[0], 1);
        tc::mbar_init(&bar_acc[1], 1);
        tc::mbar_init_fence();
        s_ok = 1;
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = s_tmem;
    if (tid == 0) {  // item prefix over groups (every CTA computes the same table)
        int acc = 0;
        for (int g = 0; g < ngroups; ++g) {
            s_items[g] = acc;
            const Geo q = geo_of(a, mode, g, s_goff[g + 1] - s_goff[g]);
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
            p.KW = p.KT = 1;
            return;
        }
        int lo = 0, hi = ngroups - 1;  // last group with s_items[g] <= item
        while (lo < hi) {
            const int mid = (lo + hi + 1) / 2;
            if (s_items[mid] <= item) lo = mid;
            else hi = mid - 1;
        }
        const Geo q = geo_of(a, mode, lo, s_goff[lo + 1] - s_goff[lo]);
        const int rem = item - s_items[lo];
        p.g = lo;
        p.mt = rem / q.ntiles;
        p.nt = rem % q.ntiles;
        p.KW = q.K / kKS;
        p.KT = p.KW + NL;
    };
    auto tile_jobs = [&](const Pos& p) { return min(kNT, s_goff[p.g + 1] - s_goff[p.g] - p.nt * kNT); };
    auto geo = [&](const Pos& p) { return geo_of(a, mode, p.g, s_goff[p.g + 1] - s_goff[p.g]); };
    // a step opens a span of the weight ring: every LoRA-B step, and every SP-th weight step
    auto opens = [&](const Pos& p) { return p.kt >= p.KW || p.kt % SP == 0; };
    auto advance = [&](Pos& p) {
        if (++p.kt == p.KT) decode(p.item + NB, p);
    };

    if (warp == kLoadW) {
        // ====================================================== loader warp: TMA spans, activation rows,
        // LoRA-B rows.  It runs ahead of the MMAs by up to kRB steps (activation slots) and of the
        // dequantisation by up to kRS spans (weight ring).
        Pos pl;
        decode(blockIdx.x, pl);
        uint32_t t = 0, cs = 0;  // step and span of pl
        uint32_t issued = 0;     // spans issued
        int slot_mma[kRS];       // step whose MMAs read the slot directly (LoRA-B rows), or -1
        for (int i = 0; i < kRS; ++i) slot_mma[i] = -1;
        bool ok = true;
        // this lane's 16 activation rows of the current item (chunk lane % 8, rows lane / 8 + 4 i)
        const int c8 = lane % 8, r0 = lane / 8;
        int64_t rowoff[16];
        uint32_t rowlive = 0;
        auto item_rows = [&](const Pos& p) {
            if (tma_b) return;
            constexpr bool by_token = mode == kGU;
            const int base = s_goff[p.g] + p.nt * kNT, end = s_goff[p.g + 1];
            const Geo q = geo(p);
            rowlive = 0;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int job = base + r0 + 4 * i;
                const bool live = p.item < nitems && job < end;
                rowoff[i] = live ? (int64_t)(by_token ? a.perm[job].x : job) * a.ld_act + c8 * 8 : 0;
                if (live) rowlive |= 1u << i;
            }
        };
        item_rows(pl);
        while (pl.item < nitems && ok) {
            const bool wstep = pl.kt < pl.KW;
            // ---- the weight-ring span this step opens
            if (opens(pl)) {
                const int slot = cs % kRS;
                if (cs >= (uint32_t)kRS) {
                    if (!tc::mbar_wait_ok(&bar_rawfree[slot], ((cs / kRS) - 1) & 1u, a.status, &s_ok, a.wait_ns)) {
                        ok = false;
                        break;
                    }
                    const int tr = slot_mma[slot];
                    if (tr >= 0 && !tc::mbar_wait_ok(&bar_tile[tr % kTiles], (tr / kTiles) & 1u, a.status, &s_ok, a.wait_ns)) {
                        ok = false;
                        break;
                    }
                    slot_mma[slot] = -1;
                }
                if (wstep) {
                    uint64_t* bar = &bar_raw[slot];
                    if (lane == 0) {
                        const Geo q = geo(pl);
                        const uint32_t dst = tc::smem_u32(sR + slot * kRawSlot);
                        const int x = (pl.kt / SP) * 32;  // 32 words = 128 B per row
                        if (mode == kGU) {
                            const int y = q.mat * q.M + pl.mt * kBM;
                            tc::mbar_arrive_expect_tx(bar, 2 * kSpanBytes);
                            tc::tma_load_2d(dst, &a.tm[q.shared ? 2 : 0], x, y, bar);
                            tc::tma_load_2d(dst + kSpanBytes, &a.tm[q.shared ? 3 : 1], x, y, bar);
                        } else if (mode == kDown) {
                            const int y = q.mat * q.M + pl.mt * 2 * kBM;
                            tc::mbar_arrive_expect_tx(bar, 2 * kSpanBytes);
                            tc::tma_load_2d(dst, &a.tm[q.shared ? 1 : 0], x, y, bar);
                            tc::tma_load_2d(dst + kSpanBytes, &a.tm[q.shared ? 1 : 0], x, y + kBM, bar);
                        } else {
                            tc::mbar_arrive_expect_tx(bar, kSpanBytes);
                            tc::tma_load_2d(dst, &a.tm[0], x, pl.mt * kBM, bar);
                        }
                    } else {
                        tc::mbar_arrive(bar);
                    }
                    ++issued;
                } else {
                    // LoRA-B rows of step s: lane -> chunk c8 of rows r0 + 4 i; K' column 64 s + 8 c of
                    // block k = adapter (.. / r), rank index (.. % r) of block k's matrix
                    const Geo q = geo(pl);
                    const int s = pl.kt - pl.KW, cc = 64 * s + 8 * c8;
                    const uint32_t dst0 = tc::smem_u32(sR + slot * kRawSlot);
                    for (int blk = 0; blk < 2; ++blk) {
                        const int which = mode == kGU ? blk : 2;  // gate rows | up rows; down: two row blocks
                        const moe_lora_proj* lp = cc < nar ? tlora(L, cc / r, q.shared, which) : nullptr;
                        const int row0 = mode == kGU ? pl.mt * kBM : pl.mt * 2 * kBM + blk * kBM;
                        const uint16_t* src = lp ? lp->B + ((int64_t)q.mat * q.M + row0) * r + cc % r : a.act;
                        for (int i = 0; i < kBM / 4; ++i) {
                            const int row = r0 + 4 * i;
                            const bool live = lp && row0 + row < q.M;
                            tc::cp16(dst0 + blk * kSpanBytes + tc::sw128_off(row, c8),
                                     live ? src + (int64_t)row * r : a.act, live ? 16u : 0u);
                        }
                    }
                    tc::cp_commit();
                    tc::cp_arrive_noinc(&bar_raw[slot]);
                    slot_mma[slot] = (int)t;
                    ++issued;
                }
            }
            // ---- the step's activation slot (after the MMAs kRB steps back)
            const int bslot = t % kRB;
            if (t >= (uint32_t)kRB &&
                !tc::mbar_wait_ok(&bar_tile[(t - kRB) % kTiles], ((t - kRB) / kTiles) & 1u, a.status, &s_ok, a.wait_ns)) {
                ok = false;
                break;
            }
            if (wstep && tma_b) {
                // activations by TMA: one 64 x 64 box per sub-tile (the tile's jobs for down, its
                // tokens for the router), landing in the MMA's swizzled layout
                const uint32_t bb = tc::smem_u32(sB + bslot * kBSlot);
                uint64_t* bar = &bar_bfull[bslot];
                if (lane == 0) tc::mbar_arrive_expect_tx(bar, kBSlot);
                if (lane < 2)
                    tc::tma_load_2d(bb + lane * kSub, &a.tmb, pl.kt * kKS + 64 * lane, s_goff[pl.g] + pl.nt * kNT, bar);
                if (lane != 0) tc::mbar_arrive(bar);
            } else if (wstep) {
                const uint32_t bb = tc::smem_u32(sB + bslot * kBSlot);
                const int k0 = pl.kt * kKS;
#pragma unroll
                for (int sub = 0; sub < 2; ++sub)
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const bool live = (rowlive >> i) & 1u;
                        tc::cp16(bb + sub * kSub + tc::sw128_off(r0 + 4 * i, c8),
                                 a.act + (live ? rowoff[i] + k0 + 64 * sub : 0), live ? 16u : 0u);
                    }
                tc::cp_commit();
                tc::cp_arrive_noinc(&bar_bfull[bslot]);
            } else {
                tc::mbar_arrive(&bar_bfull[bslot]);  // LoRA-B step: its operand B is staged by the dequantisation
            }
            ++t;
            const int item0 = pl.item;
            advance(pl);
            if (pl.item < nitems && opens(pl)) ++cs;
            if (pl.item != item0) item_rows(pl);
        }
        // drain (bounded): this warp's copies; the latest span issued into each slot
        tc::cp_wait<0>();
        if (lane == 0) {
            for (uint32_t sq = issued > (uint32_t)kRS ? issued - kRS : 0; sq < issued; ++sq)
                tc::mbar_wait(&bar_raw[sq % kRS], (sq / kRS) & 1u, a.status, a.wait_ns);
            if (tma_b)
                for (uint32_t sq = t > (uint32_t)kRB ? t - kRB : 0; sq < t; ++sq)
                    tc::mbar_wait(&bar_bfull[sq % kRB], (sq / kRB) & 1u, a.status, a.wait_ns);
            if (!ok) s_ok = 0;
        }
        __syncwarp();
    } else if (warp == kMmaW) {
        // ====================================================== MMA warp: lane 0 alone, so that
        // between two steps it does little more than wait and issue
        if (lane == 0) {
            if (mode == kGU) for (int i = 0; i < 4; ++i) tc::tma_prefetch_desc(&a.tm[i]);
            if (mode == kDown) for (int i = 0; i < 2; ++i) tc::tma_prefetch_desc(&a.tm[i]);
            if (mode == kRouterMode) tc::tma_prefetch_desc(&a.tm[0]);
            if (tma_b) tc::tma_prefetch_desc(&a.tmb);
            // descriptors of the activation sub-tiles: the base one plus the start-address offset
            // (16-byte units in the low bits; shared addresses stay below 2^18)
            const uint64_t bdesc0 = tc::sdesc_k_sw128(tc::smem_u32(sB));
            auto bdesc = [&](int b, int sub) { return bdesc0 + (uint64_t)((b * kBSlot + sub * kSub) >> 4); };
            Pos pc;
            decode(blockIdx.x, pc);
            uint32_t t = 0, cs = 0, ib = 0;  // steps, spans and items consumed
            bool ok = true;
            uint32_t idesc = tc::idesc_bf16(kBM, (tile_jobs(pc) + 15) / 16 * 16);
            while (pc.item < nitems) {
                const bool wstep = pc.kt < pc.KW;
                if (!tc::mbar_spin_ok(&bar_full[t % kAS], (t / kAS) & 1u, a.status, &s_ok, a.wait_ns) ||
                    !tc::mbar_spin_ok(&bar_bfull[t % kRB], (t / kRB) & 1u, a.status, &s_ok, a.wait_ns) ||
                    (!wstep && !tc::mbar_spin_ok(&bar_raw[cs % kRS], (cs / kRS) & 1u, a.status, &s_ok, a.wait_ns))) {
                    ok = false;
                    break;
                }
                tc::tc_fence_after();
                const uint32_t dacc = tmem + (ib & 1u) * 128u;
                const int b = t % kRB;
                if (!wstep) {  // LoRA-B step: A = LoRA-B rows of the pseudo-span, one accumulator per block
                    const uint32_t rs = tc::smem_u32(sR + (cs % kRS) * kRawSlot);
#pragma unroll
                    for (int blk = 0; blk < 2; ++blk) {
                        const uint64_t ad = tc::sdesc_k_sw128(rs + blk * kSpanBytes);
                        const uint64_t bd = bdesc(b, mode == kGU ? blk : 0);
#pragma unroll
                        for (int k = 0; k < 4; ++k) tc::mma_bf16(dacc + blk * 64, ad + 2 * k, bd + 2 * k, idesc, 1u);
                    }
                } else {  // weight step: A = the dequantised tile in TMEM
                    const uint32_t astage = tmem + kTmemA + (t % kAS) * 128;
                    const uint32_t first = pc.kt == 0 ? 0u : 1u;
#pragma unroll
                    for (int blk = 0; blk < 2; ++blk) {
                        // router: hi and lo parts into one accumulator; otherwise one accumulator per block
                        const uint32_t d = dacc + (int8_mode ? 0u : (uint32_t)blk * 64u);
#pragma unroll
                        for (int sub = 0; sub < 2; ++sub)
#pragma unroll
                            for (int k = 0; k < 4; ++k)  // K=16 per MMA: 8 TMEM columns, +32 B in the swizzled B tile
                                tc::mma_bf16_ts(d, astage + blk * 64 + sub * 32 + 8 * k, bdesc(b, sub) + 2 * k, idesc,
                                                (sub == 0 && k == 0 && (!int8_mode || blk == 0)) ? first : 1u);
                    }
                }
                tc::mma_commit(&bar_tile[t % kTiles]);
                const bool last = pc.kt == pc.KT - 1;
                if (last) tc::mma_commit(&bar_acc[ib & 1u]);
                ++t;
                if (last) ++ib;
                advance(pc);
                if (last && pc.item < nitems) idesc = tc::idesc_bf16(kBM, (tile_jobs(pc) + 15) / 16 * 16);
                if (pc.item < nitems && opens(pc)) ++cs;
            }
            // drain (bounded): the last MMAs
            if (t > 0) tc::mbar_wait(&bar_tile[(t - 1) % kTiles], ((t - 1) / kTiles) & 1u, a.status, a.wait_ns);
            if (!ok) s_ok = 0;
        }
        __syncwarp();
    } else {
        // ====================================================== dequantisation warps
        // ---- weight rows.  int4: thread -> (block, row): the step's 16 words of the row;
        //      int8: thread -> (row, half of the step's 32 words).  Warp w writes TMEM
        //      lanes 32 (w % 4) .. +31, which are its rows.
        static_assert(NQ == 1 || !int8_mode, "the int8 path takes one thread per (row, half)");
        const int wrow = tid % kBM;
        const int wblk = int8_mode ? 0 : (tid / kBM) % 2;
        const int wh = tid / kBM;       // int8: half
        const int whs = NQ == 1 ? 0 : tid / (2 * kBM);  // int4: part of the step's chunks (of NQ)
        const uint32_t tlane = (uint32_t)((warp % 4) * 32) << 16;
        const int group = int8_mode ? L.router.group : L.gate.group;
        const int gshift = group == 64 ? 6 : 5;
        // scale/bias words (pairs of bf16) of one span of this thread's row
        const int span_groups = (SP * kKS) >> gshift;  // 2, 4 or 8
        const int span_words = span_groups / 2;        // 1, 2 or 4
        auto fetch_sb = [&](const Pos& p, int span, uint32_t (&sv)[4], uint32_t (&bv)[4]) {
            const Geo q = geo(p);
            int row;
            const moe_qtensor* W;
            if (mode == kGU) {
                row = p.mt * kBM + wrow;
                W = wblk == 0 ? (q.shared ? &L.s_gate : &L.gate) : (q.shared ? &L.s_up : &L.up);
            } else if (mode == kDown) {
                row = p.mt * 2 * kBM + wblk * kBM + wrow;
                W = q.shared ? &L.s_down : &L.down;
            } else {
                row = p.mt * kBM + wrow;
                W = &L.router;
            }
            const bool ok = row < q.M;
            const int ng = q.K >> gshift;
            const int g0 = span * span_groups;
            const int64_t off = ((int64_t)q.mat * q.M + (ok ? row : 0)) * ng + g0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const bool in = ok && j < span_words && g0 + 2 * j < ng;
                sv[j] = in ? __ldg(reinterpret_cast<const unsigned int*>(W->scales + off + 2 * j)) : 0u;
                bv[j] = in ? __ldg(reinterpret_cast<const unsigned int*>(W->biases + off + 2 * j)) : 0u;
            }
        };

        // ---- LoRA-B operand B of step s (thread: job rows brow, brow + 32; chunk bch of both
        // sub-tiles): sub-tile k holds, for block k's matrix (gate/up: gate, up; down: down in
        // sub-tile 0), each job's scaled LoRA-A products in its adapter's K' columns
        const int brow = tid / 8, bch = tid % 8;
        const uint32_t boff0 = tc::sw128_off(brow, bch), boff1 = tc::sw128_off(brow + kLRows, bch);
        auto fetch_lora = [&](const Pos& p, int s, LoraRegs<kLJ>& R) {
            const Geo q = geo(p);
            const int base = s_goff[p.g] + p.nt * kNT, end = s_goff[p.g + 1];
            const int cc = 64 * s + 8 * bch;
            const int tw = mode == kGU ? 2 * r : r;
            R.live = 0;
#pragma unroll
            for (int j = 0; j < kLJ; ++j) {
                const int job = base + brow + kLRows * j;
                if (job >= end || cc >= nar) continue;
                const int ad = a.perm[job].z;
                if (ad != cc / r) continue;
#pragma unroll
                for (int sub = 0; sub < 2; ++sub) {
                    if (mode == kDown && sub == 1) continue;
                    if (!tlora(L, ad, q.shared, mode == kGU ? sub : 2)) continue;
                    const float4* tp = reinterpret_cast<const float4*>(a.t_in + (int64_t)job * tw + sub * r + cc % r);
                    R.t[j][sub][0] = tp[0];
                    R.t[j][sub][1] = tp[1];
                    R.live |= 1u << (2 * j + sub);
                }
            }
        };
        auto stage_lora = [&](const LoraRegs<kLJ>& R, unsigned char* bslot) {
            const float sc = L.scale;
#pragma unroll
            for (int j = 0; j < kLJ; ++j)
#pragma unroll
                for (int sub = 0; sub < 2; ++sub) {
                    if (mode == kDown && sub == 1) continue;
                    uint4 o = make_uint4(0, 0, 0, 0);
                    if (R.live & (1u << (2 * j + sub))) {
                        const float4 u = R.t[j][sub][0], v = R.t[j][sub][1];
                        const __nv_bfloat162 p0 = __floats2bfloat162_rn(sc * u.x, sc * u.y);
                        const __nv_bfloat162 p1 = __floats2bfloat162_rn(sc * u.z, sc * u.w);
                        const __nv_bfloat162 p2 = __floats2bfloat162_rn(sc * v.x, sc * v.y);
                        const __nv_bfloat162 p3 = __floats2bfloat162_rn(sc * v.z, sc * v.w);
                        o = make_uint4(*reinterpret_cast<const uint32_t*>(&p0), *reinterpret_cast<const uint32_t*>(&p1),
                                       *reinterpret_cast<const uint32_t*>(&p2), *reinterpret_cast<const uint32_t*>(&p3));
                    }
                    *reinterpret_cast<uint4*>(bslot + sub * kSub + (j ? boff1 : boff0)) = o;
                }
        };

        // ---- epilogue of a finished item (accumulator buffer seq % 2)
        auto epilogue = [&](const Pos& p, uint32_t seq) -> bool {
            if (!tc::mbar_wait_ok(&bar_acc[seq & 1u], (seq >> 1) & 1u, a.status, &s_ok, a.wait_ns)) return false;
            tc::tc_fence_after();
            const Geo q = geo(p);
            const int n_here = tile_jobs(p);
            const int base = s_goff[p.g] + p.nt * kNT;
            const uint32_t dacc = tmem + tlane + (seq & 1u) * 128u;
            const int row = (warp % 4) * 32 + lane;  // TMEM lane of this thread
            for (int ch = warp / 4; ch * 16 < n_here; ch += kDeqW / 4) {  // 16-column chunks
                uint32_t d0[16], d1[16];
                tc::tmem_ld16(dacc + ch * 16, d0);
                if (int4_mode) tc::tmem_ld16(dacc + 64 + ch * 16, d1);
                tc::tmem_wait_ld();
                if (mode == kGU) {
                    const int i = p.mt * kBM + row;
                    const int ip = kperm_pos(i);  // h is the down GEMM's operand: permuted K order
                    if (i < q.M) {
#pragma unroll
                        for (int c = 0; c < 16; ++c) {
                            const int n = ch * 16 + c;
                            if (n < n_here)
                                a.h_out[(int64_t)(base + n) * a.ldh + ip] =
                                    f2bf16(silu_fast(__uint_as_float(d0[c])) * __uint_as_float(d1[c]));
                        }
                    }
                } else if (mode == kDown) {
                    const int o0 = p.mt * 2 * kBM + row;
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const int n = ch * 16 + c;
                        if (n < n_here) {
                            const float wj = a.wperm ? __ldg(a.wperm + base + n) : 0.0f;
                            float* yp = a.ypart + (int64_t)(base + n) * L.H;
                            if (o0 < q.M) yp[o0] = wj * __uint_as_float(d0[c]);
                            if (o0 + kBM < q.M) yp[o0 + kBM] = wj * __uint_as_float(d1[c]);
                        }
                    }
                } else {  // router
                    const int e = p.mt * kBM + row;
                    if (e < q.M) {
                        const float lb = L.logit_bias ? L.logit_bias[e] : 0.0f;
#pragma unroll
                        for (int c = 0; c < 16; ++c) {
                            const int n = ch * 16 + c;
                            if (n < n_here) a.logits[(int64_t)(base + n) * L.E + e] = __uint_as_float(d0[c]) + lb;
                        }
                    }
                }
            }
            // the item two later writes this buffer; its first arrival (after these reads) orders them
            tc::tc_fence_before();
            return true;
        };

        // ------------------------------------------------------ stream
        Pos pc;
        decode(blockIdx.x, pc);
        // scale/bias registers: current span and the next one
        uint32_t s_cur[4] = {0, 0, 0, 0}, b_cur[4] = {0, 0, 0, 0}, s_nxt[4] = {0, 0, 0, 0}, b_nxt[4] = {0, 0, 0, 0};
        Pos pn = pc;  // item of the next span whose scales are fetched
        int pn_span = 0;
        auto sb_next = [&]() {
            if (pn.item >= nitems) return;
            fetch_sb(pn, pn_span, s_nxt, b_nxt);
            if (++pn_span * SP >= pn.KW) {
                decode(pn.item + NB, pn);
                pn_span = 0;
            }
        };
        sb_next();
        uint32_t ss0[4] = {0, 0, 0, 0}, sb0[4] = {0, 0, 0, 0}, ss1[4] = {0, 0, 0, 0}, sb1[4] = {0, 0, 0, 0};
        LoraRegs<kLJ> lr;
        // the epilogue of an item runs kAS steps after its last step, when its MMAs are done
        bool ep_pend = false;
        Pos ep_pos = pc;
        uint32_t ep_seq = 0, ep_t = 0;

        uint32_t t = 0;        // steps consumed by this CTA
        uint32_t sseq = 0;     // weight spans consumed by this CTA
        uint32_t n_items = 0;  // items finished by this CTA
        bool good = true;
        while (pc.item < nitems) {
            const bool wstep = pc.kt < pc.KW;
            const bool span_start = wstep && pc.kt % SP == 0;
            // the MMAs of step t - kAS must be done before TMEM stage t % kAS (and, for a LoRA-B
            // step, activation slot t % kRB) is rewritten
            if (t >= (uint32_t)kAS &&
                !tc::mbar_wait_ok(&bar_tile[(t - kAS) % kTiles], ((t - kAS) / kTiles) & 1u, a.status, &s_ok, a.wait_ns)) {
                good = false;
                break;
            }
            if (span_start) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    s_cur[j] = s_nxt[j];
                    b_cur[j] = b_nxt[j];
                }
                sb_next();
                if (int4_mode) {
                    // bf16 scale and bias of each 32-word chunk of the span's two steps
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int g0 = gshift == 6 ? c >> 1 : c, g1 = gshift == 6 ? 2 + (c >> 1) : 4 + c;
                        ss0[c] = bf16_at(s_cur, g0);
                        sb0[c] = bf16_at(b_cur, g0);
                        ss1[c] = bf16_at(s_cur, g1);
                        sb1[c] = bf16_at(b_cur, g1);
                    }
                }
            }
            // inputs of the first LoRA-B step, fetched during the last weight step so their latency
            // overlaps it (later LoRA-B steps fetch theirs right after staging the previous one)
            if (NL > 0 && pc.kt + 1 == pc.KW) fetch_lora(pc, 0, lr);
            if (span_start && !tc::mbar_wait_ok(&bar_raw[sseq % kRS], (sseq / kRS) & 1u, a.status, &s_ok, a.wait_ns)) {
                good = false;
                break;
            }
            const int kk = pc.kt % SP;  // step inside the span
            const uint32_t astage = tmem + tlane + kTmemA + (t % kAS) * 128;
            if (int4_mode && wstep) {
                // the step's 16 words = 16-byte chunks 4kk .. 4kk+3 of the swizzled 128-byte row;
                // word w = K elements 8w .. 8w+7 = TMEM columns 4w .. 4w+3 of this block
                constexpr int CPT = 4 / NQ;  // chunks of the step's 4 per thread
                const unsigned char* rowp = sR + (sseq % kRS) * kRawSlot + wblk * kSpanBytes + wrow * 128;
                const uint32_t ta = astage + wblk * 64 + whs * 16 * CPT;
                // all the thread's chunks are read before any TMEM store (the stores are compiler
                // barriers), so the dequantisation chains overlap
                uint4 w4[CPT];
#pragma unroll
                for (int c = 0; c < CPT; ++c)
                    w4[c] = *reinterpret_cast<const uint4*>(rowp + (((4 * kk + whs * CPT + c) ^ (wrow & 7)) << 4));
                uint32_t v[16 * CPT];
#pragma unroll
                for (int c = 0; c < CPT; ++c) {
                    const int cc = whs * CPT + c;
                    const __nv_bfloat162 s2 = bf16x2_of(kk ? ss1[cc] : ss0[cc]), b2 = bf16x2_of(kk ? sb1[cc] : sb0[cc]);
                    const uint4 o0 = dequant8p(w4[c].x, s2, b2), o1 = dequant8p(w4[c].y, s2, b2);
                    const uint4 o2 = dequant8p(w4[c].z, s2, b2), o3 = dequant8p(w4[c].w, s2, b2);
                    uint32_t* vc = v + 16 * c;
                    vc[0] = o0.x; vc[1] = o0.y; vc[2] = o0.z; vc[3] = o0.w;
                    vc[4] = o1.x; vc[5] = o1.y; vc[6] = o1.z; vc[7] = o1.w;
                    vc[8] = o2.x; vc[9] = o2.y; vc[10] = o2.z; vc[11] = o2.w;
                    vc[12] = o3.x; vc[13] = o3.y; vc[14] = o3.z; vc[15] = o3.w;
                }
#pragma unroll
                for (int i = 0; i < CPT / 2; ++i) tc::tmem_st32(ta + 32 * i, v + 32 * i);
                tc::tmem_wait_st();
            } else if (int4_mode) {
                stage_lora(lr, sB + (t % kRB) * kBSlot);
                if (pc.kt + 1 < pc.KT) fetch_lora(pc, pc.kt + 1 - pc.KW, lr);
            } else if (int8_mode) {
                // half wh of the step's 32 words: chunks 4wh .. 4wh+3 of the row; K elements 64 wh .. +63
                // = TMEM columns 32 wh .. +31 of the hi and lo blocks
                const unsigned char* rowp = sR + (sseq % kRS) * kRawSlot + wrow * 128;
#pragma unroll
                for (int c2 = 0; c2 < 2; ++c2) {
                    const int g = (64 * wh + 32 * c2) >> gshift;
                    const float s = bf16f((uint16_t)bf16_at(s_cur, g)), b = bf16f((uint16_t)bf16_at(b_cur, g));
                    uint32_t hv[16], lv[16];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint4 w4 = *reinterpret_cast<const uint4*>(rowp + (((4 * wh + 2 * c2 + h) ^ (wrow & 7)) << 4));
                        dequant8_hilo(w4.x, w4.y, s, b, hv + 8 * h, lv + 8 * h);
                        dequant8_hilo(w4.z, w4.w, s, b, hv + 8 * h + 4, lv + 8 * h + 4);
                    }
                    tc::tmem_st16(astage + 32 * wh + 16 * c2, hv);
                    tc::tmem_st16(astage + 64 + 32 * wh + 16 * c2, lv);
                }
                tc::tmem_wait_st();
            }
            // hand the step to the MMA warp: shared-memory operands written here made visible to
            // the tensor core, TMEM stores complete, then one arrival per warp
            tc::fence_async_smem();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bar_full[t % kAS]);
            // A LoRA-B step's span (rows the MMAs read directly) is released only once it has
            // landed: the loader must have seen the slot's previous release complete before this
            // one completes, or its parity wait would alias two phases ahead.
            if (!wstep && !tc::mbar_wait_ok(&bar_raw[sseq % kRS], (sseq / kRS) & 1u, a.status, &s_ok, a.wait_ns)) {
                good = false;
                break;
            }
            if (lane == 0 && (!wstep || kk == SP - 1 || pc.kt == pc.KW - 1))
                tc::mbar_arrive(&bar_rawfree[sseq % kRS]);
            ++t;

            if (pc.kt == pc.KT - 1) {  // this step ends an item: its epilogue is deferred
                if (ep_pend && !epilogue(ep_pos, ep_seq)) {
                    good = false;
                    break;
                }
                ep_pend = true;
                ep_pos = pc;
                ep_seq = n_items++;
                ep_t = t;
            } else if (ep_pend && t >= ep_t + kAS) {
                ep_pend = false;
                if (!epilogue(ep_pos, ep_seq)) {
                    good = false;
                    break;
                }
            }
            advance(pc);
            if (pc.item < nitems && opens(pc)) ++sseq;
        }
        if (good && ep_pend && !epilogue(ep_pos, ep_seq)) good = false;
        if (!good) s_ok = 0;  // left early: let the other warps stop waiting
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == kMmaW) tc::tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// Tensor map over packed words [rows][words_per_row] (uint32), boxes of 32 words x
// 128 rows with the 128-byte swizzle; out-of-range rows and words read as zero.
cudaError_t encode_words(CUtensorMap* m, const void* base, int64_t rows, int64_t words_per_row) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {(cuuint64_t)words_per_row, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)words_per_row * 4};
    const cuuint32_t box[2] = {32, (cuuint32_t)kBM};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Tensor map over bf16 rows [rows][cols] (row pitch ld elements) in boxes of 64 columns x
// box_rows rows, 128-byte swizzled like the MMA's K-major operand; rows past the end read
// as zero.
cudaError_t encode_act(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld, int box_rows) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    if (((uintptr_t)base & 15) || (ld * 2) % 16 || cols > ld) return cudaErrorInvalidValue;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)(rows > 0 ? rows : 1)};
    const cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

bool words_tma_ok(const moe_qtensor& q) {
    const int wpr = q.in * q.bits / 32;
    return q.packed && ((uintptr_t)q.packed & 15) == 0 && (wpr * 4) % 16 == 0 && ((uintptr_t)q.scales & 3) == 0 &&
           ((uintptr_t)q.biases & 3) == 0;
}

template <int kMode>
cudaError_t launch_mode(TcArgs& a, int nsm, cudaStream_t s) {
    static int cached = 0;
    const size_t smem = kRB * kBSlot + kRS * kRawSlot + 1024;
    cudaError_t e = ensure_smem((const void*)tc_gemm_kernel<kMode>, smem, cached);
    if (e != cudaSuccess) return e;
    tc_gemm_kernel<kMode><<<nsm, TcWarps<kMode>::threads, smem, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_kernel(TcArgs& a, cudaStream_t s) {
    int nsm = 0, dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    switch (a.mode) {
        case kGU: return launch_mode<kGU>(a, nsm, s);
        case kDown: return launch_mode<kDown>(a, nsm, s);
        default: return launch_mode<kRouterMode>(a, nsm, s);
    }
}


// Activations into the permuted K order of the int4 tiles, one 16-byte chunk per thread.
__global__ void kperm_kernel(const uint4* __restrict__ x, int64_t n, uint4* __restrict__ xp) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        xp[i] = permute_k8(x[i]);
}

}  // namespace

// K-order permutation of bf16 activations (see permute_k8).
cudaError_t launch_kperm(const uint16_t* x, int64_t elems, uint16_t* xp, cudaStream_t s) {
    const int64_t n = elems / 8;
    if (n == 0) return cudaSuccess;
    int nsm = 0, dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (n + 255) / 256;
    const int blocks = (int)(want < 8LL * nsm ? want : 8LL * nsm);
    kperm_kernel<<<blocks, 256, 0, s>>>(reinterpret_cast<const uint4*>(x), n, reinterpret_cast<uint4*>(xp));
    return cudaGetLastError();
}


// Host-side conditions of the tensor-core expert path.
bool tc_supported(const LayerArgs& L) {
    if (L.H % 128 || L.I % 128 || L.H < 128 || L.I < 128) return false;
    if (L.has_shared && (L.Is % 128 || L.Is < 128)) return false;
    if (L.gate.group != 64 && L.gate.group != 32) return false;
    if (L.gate.bits != 4 || L.up.bits != 4 || L.down.bits != 4) return false;
    if (L.up.group != L.gate.group || L.down.group != L.gate.group) return false;
    if (L.has_shared && (L.s_gate.group != L.gate.group || L.s_up.group != L.gate.group ||
                         L.s_down.group != L.gate.group || L.s_gate.bits != 4 || L.s_up.bits != 4 ||
                         L.s_down.bits != 4))
        return false;
    if (L.E + 1 > kMaxGroups) return false;
    // LoRA-B rows and LoRA-A products are moved in 8-element chunks that never
    // straddle two adapters: rank a multiple of 8, B rows 16-byte aligned
    if (L.n_adapters > 0 && L.rank > 0) {
        if (L.rank % 8) return false;
        for (int ad = 0; ad < L.n_adapters; ++ad) {
            const moe_lora_proj* ps[] = {&L.lora[ad].gate, &L.lora[ad].up, &L.lora[ad].down,
                                         &L.lora[ad].s_gate, &L.lora[ad].s_up, &L.lora[ad].s_down};
            for (const moe_lora_proj* p : ps)
                if (p->B && ((uintptr_t)p->B & 15)) return false;
        }
    }
    if (!words_tma_ok(L.gate) || !words_tma_ok(L.up) || !words_tma_ok(L.down)) return false;
    if (L.has_shared && (!words_tma_ok(L.s_gate) || !words_tma_ok(L.s_up) || !words_tma_ok(L.s_down))) return false;
    return encode_fn() != nullptr;
}

bool tc_router_supported(const moe_qtensor& router, int H, int E) {
    return H % 128 == 0 && H >= 128 && E >= 1 && router.bits == 8 && (router.group == 64 || router.group == 32) &&
           router.in == H && words_tma_ok(router) && encode_fn() != nullptr;
}

cudaError_t launch_tc_gemm(const LayerArgs& L, int mode, const uint16_t* act, int ld_act, const Work& wk,
                           const uint16_t* hb_out, int ldh, cudaStream_t s) {
    TcArgs a;
    memset(&a, 0, sizeof(a));
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
    a.t_in = mode == kTcGU ? wk.tgu : wk.td;
    a.status = wk.status;
    a.wait_ns = wait_limit_ns();
    cudaError_t e = cudaSuccess;
    if (mode == kTcDown) e = encode_act(&a.tmb, act, wk.J, ld_act, ld_act, kNT);
    if (e != cudaSuccess) return e;
    if (mode == kTcGU) {
        e = encode_words(&a.tm[0], L.gate.packed, (int64_t)L.E * L.I, L.H / 8);
        if (e == cudaSuccess) e = encode_words(&a.tm[1], L.up.packed, (int64_t)L.E * L.I, L.H / 8);
        if (e == cudaSuccess && L.has_shared) e = encode_words(&a.tm[2], L.s_gate.packed, L.Is, L.H / 8);
        if (e == cudaSuccess && L.has_shared) e = encode_words(&a.tm[3], L.s_up.packed, L.Is, L.H / 8);
    } else if (mode == kTcDown) {
        e = encode_words(&a.tm[0], L.down.packed, (int64_t)L.E * L.H, L.I / 8);
        if (e == cudaSuccess && L.has_shared) e = encode_words(&a.tm[1], L.s_down.packed, L.H, L.Is / 8);
    }
    if (e != cudaSuccess) return e;
    return launch_kernel(a, s);
}

cudaError_t launch_tc_router(const moe_qtensor& router, const float* logit_bias, const uint16_t* x, int T, int H,
                             int E, float* logits, int32_t* status, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    TcArgs a;
    memset(&a, 0, sizeof(a));
    a.L.router = router;
    a.L.logit_bias = logit_bias;
    a.L.H = H;
    a.L.E = E;
    a.mode = kRouterMode;
    a.act = x;
    a.ld_act = H;
    a.logits = logits;
    a.T = T;
    a.status = status;
    a.wait_ns = wait_limit_ns();
    cudaError_t e = encode_words(&a.tm[0], router.packed, E, H / 4);
    if (e == cudaSuccess) e = encode_act(&a.tmb, x, T, H, H, kNT);
    if (e != cudaSuccess) return e;
    return launch_kernel(a, s);
}

}  // namespace moeq
