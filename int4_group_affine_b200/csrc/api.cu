// api.cu - the extern "C" entry points of libmoeq: argument validation on the
// host, workspace layout, and the launch sequence of each call.
#include <string.h>

#include <algorithm>

#include "common.cuh"

namespace moeq {

namespace {
constexpr uint64_t kDefaultWaitNs = 1000000000ull;  // 1 s
uint64_t g_wait_ns = kDefaultWaitNs;
int g_decode_path = MOE_DECODE_AUTO;
}  // namespace
uint64_t wait_limit_ns() { return g_wait_ns; }

cudaError_t launch_index_build_counts(const Work& wk, const int32_t* adapter_id, int n_adapters, int32_t* counts_out,
                                      cudaStream_t s);
}

using namespace moeq;

namespace {

constexpr size_t kAlign = 256;
constexpr int kTcMinTokens = 9;  // from this many tokens on, the expert GEMMs use the tensor cores
inline size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }
inline bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

#define CHECK_ARG(cond) \
    do {                \
        if (!(cond)) return MOE_ERR_INVALID_ARG; \
    } while (0)
#define CHECK_CUDA(expr)                              \
    do {                                              \
        if ((expr) != cudaSuccess) return MOE_ERR_CUDA; \
    } while (0)
// A launch on stream `s` followed by its timing mark.
#define LAUNCH(kind, expr)                            \
    do {                                              \
        if ((expr) != cudaSuccess) return MOE_ERR_CUDA; \
        timing_mark(kind, s);                         \
    } while (0)

// Shape check of an affine tensor: group a multiple of 32 that divides `in`,
// 16-byte aligned packed rows.
bool qtensor_ok(const moe_qtensor& t, int n, int out, int in, int bits) {
    if (!t.packed || !t.scales || !t.biases) return false;
    if (t.n != n || t.out != out || t.in != in || t.bits != bits) return false;
    if (t.group <= 0 || t.group % 32 != 0 || in % t.group != 0) return false;
    if (!aligned(t.packed, 16) || !aligned(t.scales, 2) || !aligned(t.biases, 2)) return false;
    return true;
}

bool lora_proj_ok(const moe_lora_proj& p, int in) {
    if (!p.A && !p.B) return true;
    if (!p.A || !p.B) return false;
    return aligned(p.A, 16) && aligned(p.B, 2) && in % 8 == 0;
}

moe_status validate_layer(const moe_layer* L) {
    if (!L) return MOE_ERR_INVALID_ARG;
    const int H = L->hidden, E = L->n_experts, K = L->top_k, I = L->inter, Is = L->shared_inter;
    if (H <= 0 || E <= 0 || K <= 0 || I <= 0) return MOE_ERR_INVALID_ARG;
    if (E > MOEQ_MAX_EXPERTS || K > MOEQ_MAX_TOPK || K > E || H > MOEQ_MAX_HIDDEN || I > MOEQ_MAX_INTER)
        return MOE_ERR_UNSUPPORTED;
    if (H % 32 || I % 32) return MOE_ERR_INVALID_ARG;
    if (!qtensor_ok(L->router, 1, E, H, 8)) return MOE_ERR_INVALID_ARG;
    if (L->shared_gate.packed && !qtensor_ok(L->shared_gate, 1, 1, H, 8)) return MOE_ERR_INVALID_ARG;
    if (!qtensor_ok(L->gate, E, I, H, 4) || !qtensor_ok(L->up, E, I, H, 4) || !qtensor_ok(L->down, E, H, I, 4))
        return MOE_ERR_INVALID_ARG;
    if (L->gate.group != L->up.group) return MOE_ERR_UNSUPPORTED;
    if (L->s_gate.packed) {
        if (Is <= 0 || Is % 32 || Is > MOEQ_MAX_INTER) return MOE_ERR_INVALID_ARG;
        if (!qtensor_ok(L->s_gate, 1, Is, H, 4) || !qtensor_ok(L->s_up, 1, Is, H, 4) ||
            !qtensor_ok(L->s_down, 1, H, Is, 4))
            return MOE_ERR_INVALID_ARG;
        if (L->s_gate.group != L->s_up.group) return MOE_ERR_UNSUPPORTED;
    }
    if (L->n_adapters < 0 || L->n_adapters > MOEQ_MAX_ADAPTERS) return MOE_ERR_INVALID_ARG;
    if (L->n_adapters > 0) {
        if (L->rank <= 0 || L->rank > MOEQ_MAX_RANK) return MOE_ERR_INVALID_ARG;
        for (int a = 0; a < L->n_adapters; ++a) {
            const moe_lora_ptrs& p = L->lora[a];
            if (!lora_proj_ok(p.gate, H) || !lora_proj_ok(p.up, H) || !lora_proj_ok(p.down, I) ||
                !lora_proj_ok(p.s_gate, H) || !lora_proj_ok(p.s_up, H) || !lora_proj_ok(p.s_down, Is > 0 ? Is : 8))
                return MOE_ERR_INVALID_ARG;
        }
    }
    return MOE_OK;
}

struct Dims {
    int T, K, E, H, I, Is, Imax, A1, C, nb, J, r;
};

Dims dims_of(const moe_layer* L, int T) {
    Dims d;
    d.T = T;
    d.K = L->top_k;
    d.E = L->n_experts;
    d.H = L->hidden;
    d.I = L->inter;
    d.Is = L->s_gate.packed ? L->shared_inter : 0;
    d.Imax = std::max(d.I, d.Is);
    d.A1 = L->n_adapters + 1;
    d.C = (T + 31) / 32;
    d.nb = (d.E + 1) * d.A1;
    d.J = T * (d.K + 1);
    d.r = L->n_adapters > 0 ? L->rank : 1;
    return d;
}

WsPlan plan_of(const Dims& d) {
    WsPlan p;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        size_t at = o;
        o = align_up(o + bytes);
        return at;
    };
    p.status = take(16);  // status word, n_active and the decode ticket counter share the first 256 bytes
    p.n_active = p.status + 4;
    p.bar = p.status + 8;
    // the chain decode kernel's tagged words: first after the header and sized for the
    // layer shape alone, so no other region of any T of this shape ever overlaps them
    p.slots = take(chain_slot_words(d.E, d.K, d.I, d.Is, d.r) * 8);
    p.cslots = take(cluster_slot_words(d.K, d.I, d.Is) * 8);
    p.hxin = take(d.T <= MOEQ_DECODE_MAX_TOKENS ? (size_t)d.T * d.H * 2 : 0);
    p.hyout = take(d.T <= MOEQ_DECODE_MAX_TOKENS ? (size_t)d.T * d.H * 2 : 0);
    p.idx = take((size_t)d.T * d.K * 4);
    p.w = take((size_t)d.T * d.K * 4);
    p.sg = take((size_t)d.T * 4);
    p.logits = take((size_t)d.T * d.E * 4);
    p.gs = take((size_t)d.T * 4);
    p.cnt = take((size_t)d.nb * d.C * 4);
    p.goff = take((size_t)(d.E + 2) * 4);
    p.active = take((size_t)(d.E + 1) * 4);
    p.perm = take((size_t)d.J * 16);
    p.wperm = take((size_t)d.J * 4);
    p.inv = take((size_t)d.J * 4);
    p.tgu = take((size_t)d.J * 2 * d.r * 4);
    p.td = take((size_t)d.J * d.r * 4);
    p.h = take((size_t)d.J * d.Imax * 4);
    p.ypart = take((size_t)d.J * d.H * 4);
    p.xn = take((size_t)d.T * d.H * 2);
    p.xp = take(d.T >= kTcMinTokens ? (size_t)d.T * d.H * 2 : 0);
    const bool dec = d.T <= MOEQ_DECODE_MAX_TOKENS && d.J <= MOEQ_DECODE_MAX_JOBS;
    p.dts = take(dec ? (size_t)d.T * 2 * d.r * 4 : 0);
    p.dtg = take(dec ? (size_t)d.T * d.K * 2 * d.r * 4 : 0);
    p.dtdp = take(dec ? (size_t)MOEQ_DECODE_MAX_CTAS * 3 * d.T * d.r * 4 : 0);
    p.total = o;
    return p;
}

Work work_of(const Dims& d, const WsPlan& p, void* ws) {
    char* b = (char*)ws;
    Work w;
    w.status = (int32_t*)(b + p.status);
    w.n_active = (int32_t*)(b + p.n_active);
    w.idx = (int32_t*)(b + p.idx);
    w.w = (float*)(b + p.w);
    w.sg = (float*)(b + p.sg);
    w.logits = (float*)(b + p.logits);
    w.gs = (float*)(b + p.gs);
    w.cnt = (int32_t*)(b + p.cnt);
    w.goff = (int32_t*)(b + p.goff);
    w.active = (int32_t*)(b + p.active);
    w.perm = (int4*)(b + p.perm);
    w.wperm = (float*)(b + p.wperm);
    w.inv = (int32_t*)(b + p.inv);
    w.tgu = (float*)(b + p.tgu);
    w.td = (float*)(b + p.td);
    w.h = (float*)(b + p.h);
    w.ypart = (float*)(b + p.ypart);
    w.xn = (uint16_t*)(b + p.xn);
    w.xp = (uint16_t*)(b + p.xp);
    w.T = d.T;
    w.K = d.K;
    w.E = d.E;
    w.H = d.H;
    w.I = d.I;
    w.Is = d.Is;
    w.Imax = d.Imax;
    w.A1 = d.A1;
    w.C = d.C;
    w.nb = d.nb;
    w.J = d.J;
    w.r = d.r;
    return w;
}

LayerArgs args_of(const moe_layer* L) {
    LayerArgs a;
    memset(&a, 0, sizeof(a));
    a.gate = L->gate;
    a.up = L->up;
    a.down = L->down;
    a.s_gate = L->s_gate;
    a.s_up = L->s_up;
    a.s_down = L->s_down;
    a.router = L->router;
    a.shared_gate = L->shared_gate;
    a.logit_bias = L->logit_bias;
    a.H = L->hidden;
    a.E = L->n_experts;
    a.K = L->top_k;
    a.I = L->inter;
    a.Is = L->s_gate.packed ? L->shared_inter : 0;
    a.n_adapters = L->n_adapters;
    a.rank = L->n_adapters > 0 ? L->rank : 0;
    a.scale = a.rank > 0 ? L->alpha / (float)a.rank : 0.0f;
    a.has_shared = L->s_gate.packed != nullptr;
    a.has_sgate = L->shared_gate.packed != nullptr;
    for (int i = 0; i < L->n_adapters; ++i) a.lora[i] = L->lora[i];
    return a;
}

moe_status ws_check(void* ws, size_t ws_bytes, size_t need) {
    if (!ws || !aligned(ws, kAlign) || ws_bytes < need) return MOE_ERR_WORKSPACE;
    return MOE_OK;
}

// Router logits (and the shared-expert gate logit in gs): on the tensor cores from
// kTcMinTokens tokens on, the gate row then by the CUDA-core kernel alone.
moe_status router_enqueue(const uint16_t* x, const moe_qtensor& router, const moe_qtensor* sg, const float* lb,
                          int T, int H, int E, float* logits, float* gs, int32_t* status, cudaStream_t s) {
    // the tensor-core router reads x through a TMA map: 16-byte aligned rows only
    if (T >= kTcMinTokens && aligned(x, 16) && H % 8 == 0 && tc_router_supported(router, H, E)) {
        LAUNCH(kTcRouterKind, launch_tc_router(router, lb, x, T, H, E, logits, status, s));
        if (sg && aligned(x, 16) && H % 16 == 0) LAUNCH(kRouter, launch_sgate_logits(x, *sg, T, H, gs, s));
        else if (sg) LAUNCH(kRouter, launch_router_logits(x, router, sg, nullptr, T, H, 0, logits, gs, s));
        return MOE_OK;
    }
    LAUNCH(kRouter, launch_router_logits(x, router, sg, lb, T, H, E, logits, gs, s));
    return MOE_OK;
}

moe_status experts_enqueue(const moe_layer* L, const uint16_t* x, const int32_t* adapter_id, int T,
                           const uint16_t* residual, uint16_t* y, const Work& wk, cudaStream_t s);

// The launch sequence shared by moe_ffn_forward and moe_block_forward.
moe_status ffn_enqueue(const moe_layer* L, const uint16_t* x, const int32_t* adapter_id, const int32_t* select, int T,
                       const uint16_t* residual, uint16_t* y, const Work& wk, cudaStream_t s) {
    const LayerArgs la = args_of(L);
    const moe_qtensor* sg = la.has_sgate ? &L->shared_gate : nullptr;
    moe_status rst = router_enqueue(x, L->router, sg, L->logit_bias, T, la.H, la.E, wk.logits, wk.gs, wk.status, s);
    if (rst != MOE_OK) return rst;
    if (select)
        LAUNCH(kTopk, launch_select(wk.logits, wk.gs, la.has_sgate, select, T, la.E, la.K, wk.idx, wk.w, wk.sg,
                                    wk.status, s));
    else
        LAUNCH(kTopk, launch_topk(wk.logits, wk.gs, la.has_sgate, T, la.E, la.K, wk.idx, wk.w, wk.sg, s));
    return experts_enqueue(L, x, adapter_id, T, residual, y, wk, s);
}

// From the routing in the workspace (idx, w, sg) on: index build, the expert GEMMs or
// GEMVs (tensor cores from kTcMinTokens tokens on) and the fixed-order combine.
moe_status experts_enqueue(const moe_layer* L, const uint16_t* x, const int32_t* adapter_id, int T,
                           const uint16_t* residual, uint16_t* y, const Work& wk, cudaStream_t s) {
    const LayerArgs la = args_of(L);
    CHECK_CUDA(launch_index_build(wk, adapter_id, L->n_adapters, s));
    // Jobs of the shared expert stay in its group even without a shared expert:
    // their weights are zero-sized then, so they are skipped by the kernels.
    const int max_groups = std::min(la.E, T * la.K) + 1;
    if (T >= kTcMinTokens && tc_supported(la)) {
        // many tokens: expert-grouped GEMMs on the tcgen05 tensor cores; the SwiGLU
        // activations go to the workspace's h region as bf16 (the down GEMM's operand)
        uint16_t* hb = reinterpret_cast<uint16_t*>(wk.h);
        // the int4 tiles hold each 8-group of K in the order 0 4 1 5 2 6 3 7: the gate/up
        // operand is x in that order, and h is written in it for the down GEMM
        LAUNCH(kKpermKind, launch_kperm(x, (int64_t)T * la.H, wk.xp, s));
        if (la.rank > 0) LAUNCH(kTcLoraGUKind, launch_lora_a_mma(la, 0, x, la.H, wk, s));
        LAUNCH(kTcGUKind, launch_tc_gemm(la, kTcGU, wk.xp, la.H, wk, hb, wk.Imax, s));
        if (la.rank > 0) LAUNCH(kTcLoraDownKind, launch_lora_a_mma(la, 1, hb, wk.Imax, wk, s));
        LAUNCH(kTcDownKind, launch_tc_gemm(la, kTcDown, hb, wk.Imax, wk, nullptr, wk.Imax, s));
        LAUNCH(kCombine, launch_combine(wk, residual, y, s));
        return MOE_OK;
    }
    if (la.rank > 0) LAUNCH(kLoraA, launch_lora_a(wk, la, 0, x, s));
    LAUNCH(kGateUp, launch_gate_up(wk, la, x, max_groups, s));
    if (la.rank > 0) LAUNCH(kLoraA, launch_lora_a(wk, la, 1, x, s));
    LAUNCH(kDown, launch_down(wk, la, max_groups, s));
    LAUNCH(kCombine, launch_combine(wk, residual, y, s));
    return MOE_OK;
}

// The single-kernel decodes for a few tokens: the chain kernel (csrc/decode_chain.cu) and
// the barrier kernel (csrc/decode.cu).  Returns false when neither applies (too many
// tokens or jobs, shapes outside their limits, or the forced one declines), so the
// caller runs the multi-kernel path instead; otherwise *st is the launch result.
bool try_decode(const moe_layer* L, const uint16_t* x, const int32_t* adapter_id, const int32_t* select, int T,
                int block, float eps, uint16_t* y, const Dims& d, const WsPlan& p, void* ws, cudaStream_t s,
                moe_status* st) {
    if (d.T > MOEQ_DECODE_MAX_TOKENS) return false;
    const LayerArgs la = args_of(L);
    char* b = (char*)ws;
    auto finish = [&](cudaError_t e, int kind) {
        if (e == cudaErrorNotSupported || e == cudaErrorCooperativeLaunchTooLarge) {
            (void)cudaGetLastError();
            return false;
        }
        *st = e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
        if (e == cudaSuccess) timing_mark(kind, s);
        return true;
    };
    auto run_chain = [&]() {
        if (!chain_supported(la, T)) return false;
        ChainScratch cs;
        cs.slots = (uint64_t*)(b + p.slots);
        cs.status = (int32_t*)(b + p.status);
        cs.idx_out = (int32_t*)(b + p.idx);
        cs.w_out = (float*)(b + p.w);
        return finish(launch_chain(la, x, adapter_id, select, y, T, block, eps, cs, s), kDecodeChain);
    };
    auto run_cluster = [&]() {
        if (!cluster_supported(la, T)) return false;
        ClusterScratch cs;
        cs.slots = (uint64_t*)(b + p.cslots);
        cs.x_host = 0;
        cs.status = (int32_t*)(b + p.status);
        cs.idx_out = (int32_t*)(b + p.idx);
        cs.w_out = (float*)(b + p.w);
        return finish(launch_cluster(la, x, adapter_id, select, y, T, block, eps, cs, s), kDecodeCluster);
    };
    auto run_barrier = [&]() {  // (routes by top-K only)
        if (d.J > MOEQ_DECODE_MAX_JOBS || select || !decode_supported(la, T, nullptr)) return false;
        DecodeScratch sc;
        sc.logits = (float*)(b + p.logits);
        sc.gsl = (float*)(b + p.gs);
        sc.ts = (float*)(b + p.dts);
        sc.tg = (float*)(b + p.dtg);
        sc.h = (float*)(b + p.h);
        sc.tdp = (float*)(b + p.dtdp);
        sc.bar = (unsigned long long*)(b + p.bar);
        sc.status = (int32_t*)(b + p.status);
        sc.idx_out = (int32_t*)(b + p.idx);
        sc.w_out = (float*)(b + p.w);
        return finish(launch_decode(la, x, adapter_id, y, T, block, eps, sc, s), kDecode);
    };
    if (g_decode_path == MOE_DECODE_CHAIN) return run_chain();
    if (g_decode_path == MOE_DECODE_BARRIER) return run_barrier();
    if (g_decode_path == MOE_DECODE_CLUSTER) return run_cluster();
    // Measured on one B200 (one token, the Edge0 layer): top-4 34.6 us on the barrier
    // kernel against 37.2 on the chain kernel, top-8 48.3 against 45.9.
    if (run_cluster()) return true;
    if (la.K <= 4) return run_barrier() || run_chain();
    return run_chain() || run_barrier();
}

bool mixed_ok(const moe_mixed_tensor* t, int out, int in) {
    if (!t || !t->packed || !t->scales) return false;
    if (t->out != out || t->in != in) return false;
    if (!(t->rho >= 0.0f && t->rho <= 1.0f)) return false;
    return in % 64 == 0 && aligned(t->packed, 16);
}

// Super-group size floor(1/rho); the slack absorbs fp32 rounding of rho = 1/n.
int mixed_G(float rho) { return rho > 0.0f ? (int)floor(1.0 / (double)rho + 1e-6) : 0; }

}  // namespace

namespace moeq {
// Everything moe_ffn_forward checks before it looks at the workspace: the layer, T,
// and (for T > 0) the input and output pointers.
moe_status ffn_precheck(const moe_layer* layer, const uint16_t* x, const uint16_t* y, int32_t T) {
    moe_status st = validate_layer(layer);
    if (st != MOE_OK) return st;
    CHECK_ARG(T >= 0);
    if (T > 0) CHECK_ARG(x && y && x != y && aligned(x, 16) && aligned(y, 2));
    return MOE_OK;
}
}  // namespace moeq

extern "C" {

moe_status moe_set_decode_path(int path) {
    CHECK_ARG(path == MOE_DECODE_AUTO || path == MOE_DECODE_CHAIN || path == MOE_DECODE_BARRIER ||
              path == MOE_DECODE_CLUSTER);
    g_decode_path = path;
    return MOE_OK;
}

int moe_decode_path(void) { return g_decode_path; }

moe_status moe_set_wait_limit_ns(uint64_t ns) {
    g_wait_ns = ns == 0 ? kDefaultWaitNs : ns;
    return MOE_OK;
}

uint64_t moe_wait_limit_ns(void) { return g_wait_ns; }

int moe_version(void) { return MOEQ_VERSION; }

const char* moe_status_string(moe_status st) {
    switch (st) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case MOE_ERR_DEVICE_INDEX: return "device saw an out-of-range expert or adapter index";
        case MOE_ERR_TIMEOUT: return "bounded device wait timed out";
    }
    return "unknown status";
}

int64_t moe_mixed_words(int32_t out, int32_t in, float rho) {
    if (out <= 0 || in <= 0 || in % 16) return -1;
    const int G = mixed_G(rho);
    const int64_t w4 = in / 8, w2 = in / 16;
    if (G == 0) return (int64_t)out * w2;
    const int64_t full = out / G, rem = out % G;
    return full * (w4 + (int64_t)(G - 1) * w2) + (rem ? w4 + (rem - 1) * w2 : 0);
}

moe_status moe_quant_pack(moe_format fmt, const float* W, int64_t rows, int32_t in, int32_t group, float rho,
                          uint32_t* packed, uint16_t* scales, uint16_t* biases, moe_stream stream) {
    cudaStream_t s = (cudaStream_t)stream;
    CHECK_ARG(rows >= 0 && in > 0);
    if (rows == 0) return MOE_OK;
    CHECK_ARG(W && packed && scales);
    if (fmt == MOE_FMT_AFFINE_INT4 || fmt == MOE_FMT_AFFINE_INT8) {
        const int bits = fmt == MOE_FMT_AFFINE_INT4 ? 4 : 8;
        CHECK_ARG(biases && group > 0 && in % group == 0 && group % 8 == 0);
        timing_begin(s);
        LAUNCH(kPack, launch_pack_affine(W, rows, in, group, bits, packed, scales, biases, s));
        return MOE_OK;
    }
    if (fmt == MOE_FMT_MIXED_TERNARY_INT4) {
        CHECK_ARG(biases == nullptr && in % 16 == 0 && rho >= 0.0f && rho <= 1.0f && rows <= INT32_MAX);
        timing_begin(s);
        LAUNCH(kPack, launch_pack_mixed(W, (int)rows, in, mixed_G(rho), packed, scales, s));
        return MOE_OK;
    }
    return MOE_ERR_INVALID_ARG;
}

moe_status moe_dequant(const moe_qtensor* t, float* w_hat, moe_stream stream) {
    CHECK_ARG(t && w_hat && t->packed && t->scales && t->biases);
    CHECK_ARG((t->bits == 4 || t->bits == 8) && t->n >= 0 && t->out >= 0 && t->in > 0);
    CHECK_ARG(t->group > 0 && t->in % t->group == 0 && t->group % 8 == 0);
    cudaStream_t s = (cudaStream_t)stream;
    timing_begin(s);
    LAUNCH(kDequant, launch_dequant_affine(*t, w_hat, s));
    return MOE_OK;
}

moe_status moe_mixed_dequant(const moe_mixed_tensor* t, float* w_hat, moe_stream stream) {
    CHECK_ARG(t && w_hat && t->packed && t->scales && t->out >= 0 && t->in > 0 && t->in % 16 == 0);
    CHECK_ARG(t->rho >= 0.0f && t->rho <= 1.0f);
    cudaStream_t s = (cudaStream_t)stream;
    timing_begin(s);
    LAUNCH(kDequant, launch_dequant_mixed(*t, mixed_G(t->rho), w_hat, s));
    return MOE_OK;
}

moe_status moe_router_topk(const uint16_t* x, const moe_qtensor* router, const moe_qtensor* shared_gate,
                           const float* logit_bias, int32_t T, int32_t H, int32_t E, int32_t K, int32_t* topk_idx,
                           float* topk_w, float* shared_scale, float* logits, moe_stream stream) {
    CHECK_ARG(T >= 0);
    if (T == 0) return MOE_OK;
    CHECK_ARG(x && router && topk_idx && topk_w && logits);
    CHECK_ARG(E > 0 && K > 0 && H > 0 && H % 32 == 0);
    if (E > MOEQ_MAX_EXPERTS || K > MOEQ_MAX_TOPK || K > E || H > MOEQ_MAX_HIDDEN) return MOE_ERR_UNSUPPORTED;
    CHECK_ARG(qtensor_ok(*router, 1, E, H, 8));
    const bool has_sg = shared_gate && shared_gate->packed && shared_scale;
    if (has_sg) CHECK_ARG(qtensor_ok(*shared_gate, 1, 1, H, 8));
    cudaStream_t s = (cudaStream_t)stream;
    timing_begin(s);
    // no workspace here: a tensor-core wait that ran out has no status word to report to
    moe_status rst = router_enqueue(x, *router, has_sg ? shared_gate : nullptr, logit_bias, T, H, E, logits,
                                    shared_scale, nullptr, s);
    if (rst != MOE_OK) return rst;
    LAUNCH(kTopk, launch_topk(logits, shared_scale, has_sg, T, E, K, topk_idx, topk_w, shared_scale, s));
    return MOE_OK;
}

size_t moe_index_workspace_bytes(int32_t T, int32_t K, int32_t E, int32_t n_adapters) {
    if (T < 0 || K <= 0 || E <= 0 || n_adapters < 0) return 0;
    const size_t nb = (size_t)(E + 1) * (n_adapters + 1);
    const size_t C = (size_t)(T + 31) / 32;
    return kAlign + align_up(nb * C * 4 + 4);
}

moe_status moe_index_build(const int32_t* topk_idx, const int32_t* adapter_id, int32_t T, int32_t K, int32_t E,
                           int32_t n_adapters, int32_t* counts, int32_t* offsets, int32_t* perm, void* workspace,
                           size_t ws_bytes, moe_stream stream) {
    CHECK_ARG(T >= 0 && K > 0 && E > 0 && n_adapters >= 0);
    if (E > MOEQ_MAX_EXPERTS || K > MOEQ_MAX_TOPK || n_adapters > MOEQ_MAX_ADAPTERS) return MOE_ERR_UNSUPPORTED;
    moe_status st = ws_check(workspace, ws_bytes, moe_index_workspace_bytes(T, K, E, n_adapters));
    if (st != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    CHECK_ARG(topk_idx && counts && offsets && perm && aligned(perm, 16));
    Work wk;
    memset(&wk, 0, sizeof(wk));
    char* b = (char*)workspace;
    wk.status = (int32_t*)b;
    wk.cnt = (int32_t*)(b + kAlign);
    wk.idx = const_cast<int32_t*>(topk_idx);
    wk.goff = offsets;
    wk.perm = (int4*)perm;
    wk.T = T;
    wk.K = K;
    wk.E = E;
    wk.A1 = n_adapters + 1;
    wk.C = (T + 31) / 32;
    wk.nb = (E + 1) * wk.A1;
    wk.J = T * (K + 1);
    timing_begin((cudaStream_t)stream);
    CHECK_CUDA(launch_index_build_counts(wk, adapter_id, n_adapters, counts, (cudaStream_t)stream));
    return MOE_OK;
}

moe_status lora_set_adapters(moe_layer* layer, int32_t n_adapters, int32_t rank, float alpha,
                             const moe_lora_ptrs* sets) {
    CHECK_ARG(layer && n_adapters >= 0 && n_adapters <= MOEQ_MAX_ADAPTERS);
    if (n_adapters > 0) CHECK_ARG(sets && rank > 0 && rank <= MOEQ_MAX_RANK);
    for (int a = 0; a < n_adapters; ++a) {
        const moe_lora_ptrs& p = sets[a];
        CHECK_ARG(lora_proj_ok(p.gate, 8) && lora_proj_ok(p.up, 8) && lora_proj_ok(p.down, 8) &&
                  lora_proj_ok(p.s_gate, 8) && lora_proj_ok(p.s_up, 8) && lora_proj_ok(p.s_down, 8));
    }
    memset(layer->lora, 0, sizeof(layer->lora));
    for (int a = 0; a < n_adapters; ++a) layer->lora[a] = sets[a];
    layer->n_adapters = n_adapters;
    layer->rank = n_adapters > 0 ? rank : 0;
    layer->alpha = n_adapters > 0 ? alpha : 0.0f;
    return MOE_OK;
}

size_t moe_ffn_workspace_bytes(const moe_layer* layer, int32_t T) {
    if (!layer || T < 0 || validate_layer(layer) != MOE_OK) return 0;
    return plan_of(dims_of(layer, T)).total;
}

moe_status moe_workspace_init(void* workspace, size_t ws_bytes, moe_stream stream) {
    if (!workspace || !aligned(workspace, kAlign) || ws_bytes < kAlign) return MOE_ERR_WORKSPACE;
    CHECK_CUDA(cudaMemsetAsync(workspace, 0, ws_bytes, (cudaStream_t)stream));
    return MOE_OK;
}

moe_status moe_ffn_forward(const moe_layer* layer, const uint16_t* x, const int32_t* adapter_id, int32_t T,
                           uint16_t* y, void* workspace, size_t ws_bytes, moe_stream stream) {
    moe_status st = ffn_precheck(layer, x, y, T);
    if (st != MOE_OK) return st;
    const Dims d = dims_of(layer, T);
    const WsPlan p = plan_of(d);
    st = ws_check(workspace, ws_bytes, p.total);
    if (st != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    cudaStream_t s = (cudaStream_t)stream;
    timing_begin(s);
    if (try_decode(layer, x, adapter_id, nullptr, T, 0, 0.0f, y, d, p, workspace, s, &st)) return st;
    return ffn_enqueue(layer, x, adapter_id, nullptr, T, nullptr, y, work_of(d, p, workspace), s);
}

moe_status moe_ffn_forward_host(const moe_layer* layer, const uint16_t* x_host, const int32_t* adapter_id, int32_t T,
                                uint16_t* y_host, void* workspace, size_t ws_bytes, moe_stream stream) {
    moe_status st = ffn_precheck(layer, x_host, y_host, T);
    if (st != MOE_OK) return st;
    if (T > MOEQ_DECODE_MAX_TOKENS) return MOE_ERR_UNSUPPORTED;
    const Dims d = dims_of(layer, T);
    const WsPlan p = plan_of(d);
    st = ws_check(workspace, ws_bytes, p.total);
    if (st != MOE_OK) return st;
    void *xd = nullptr, *yd = nullptr;
    if (T > 0 && (cudaHostGetDevicePointer(&xd, const_cast<uint16_t*>(x_host), 0) != cudaSuccess ||
                  cudaHostGetDevicePointer(&yd, y_host, 0) != cudaSuccess || !xd || !yd)) {
        (void)cudaGetLastError();
        return MOE_ERR_INVALID_ARG;
    }
    if (T == 0) return MOE_OK;
    cudaStream_t s = (cudaStream_t)stream;
    timing_begin(s);
    const LayerArgs la = args_of(layer);
    char* b = (char*)workspace;
    if (T == 1 && (g_decode_path == MOE_DECODE_AUTO || g_decode_path == MOE_DECODE_CLUSTER) &&
        cluster_supported(la, 1)) {  // the kernel reads x and writes y across the bus itself
        ClusterScratch cs;
        cs.slots = (uint64_t*)(b + p.cslots);
        cs.x_host = 1;
        cs.status = (int32_t*)(b + p.status);
        cs.idx_out = (int32_t*)(b + p.idx);
        cs.w_out = (float*)(b + p.w);
        const cudaError_t e = launch_cluster(la, (const uint16_t*)xd, adapter_id, nullptr, (uint16_t*)yd, 1, 0, 0.0f,
                                             cs, s);
        if (e == cudaSuccess) {
            timing_mark(kDecodeCluster, s);
            return MOE_OK;
        }
        if (e != cudaErrorNotSupported && e != cudaErrorCooperativeLaunchTooLarge) return MOE_ERR_CUDA;
        (void)cudaGetLastError();
    }
    // staged: x into the workspace, the forward there, y back
    uint16_t* xs = (uint16_t*)(b + p.hxin);
    uint16_t* ys = (uint16_t*)(b + p.hyout);
    const size_t nb = (size_t)T * d.H * 2;
    if (cudaMemcpyAsync(xs, xd, nb, cudaMemcpyDefault, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (!try_decode(layer, xs, adapter_id, nullptr, T, 0, 0.0f, ys, d, p, workspace, s, &st))
        st = ffn_enqueue(layer, xs, adapter_id, nullptr, T, nullptr, ys, work_of(d, p, workspace), s);
    if (st != MOE_OK) return st;
    return cudaMemcpyAsync(yd, ys, nb, cudaMemcpyDefault, s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_ffn_forward_select(const moe_layer* layer, const uint16_t* x, const int32_t* adapter_id,
                                  const int32_t* select, int32_t T, uint16_t* y, void* workspace, size_t ws_bytes,
                                  moe_stream stream) {
    moe_status st = ffn_precheck(layer, x, y, T);
    if (st != MOE_OK) return st;
    const Dims d = dims_of(layer, T);
    const WsPlan p = plan_of(d);
    st = ws_check(workspace, ws_bytes, p.total);
    if (st != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    CHECK_ARG(select);
    cudaStream_t s = (cudaStream_t)stream;
    timing_begin(s);
    if (try_decode(layer, x, adapter_id, select, T, 0, 0.0f, y, d, p, workspace, s, &st)) return st;
    return ffn_enqueue(layer, x, adapter_id, select, T, nullptr, y, work_of(d, p, workspace), s);
}

moe_status moe_block_forward(const moe_layer* layer, const uint16_t* x, const int32_t* adapter_id, int32_t T,
                             float eps, uint16_t* x_out, void* workspace, size_t ws_bytes, moe_stream stream) {
    moe_status st = validate_layer(layer);
    if (st != MOE_OK) return st;
    CHECK_ARG(T >= 0 && eps >= 0.0f);
    const Dims d = dims_of(layer, T);
    const WsPlan p = plan_of(d);
    st = ws_check(workspace, ws_bytes, p.total);
    if (st != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    CHECK_ARG(x && x_out && x != x_out && aligned(x, 16) && aligned(x_out, 2));
    const Work wk = work_of(d, p, workspace);
    cudaStream_t s = (cudaStream_t)stream;
    timing_begin(s);
    if (try_decode(layer, x, adapter_id, nullptr, T, 1, eps, x_out, d, p, workspace, s, &st)) return st;
    LAUNCH(kRmsnorm, launch_rmsnorm(x, T, d.H, eps, wk.xn, s));
    return ffn_enqueue(layer, wk.xn, adapter_id, nullptr, T, x, x_out, wk, s);
}

moe_status moe_rmsnorm(const uint16_t* x, int32_t T, int32_t H, float eps, uint16_t* xn, moe_stream stream) {
    CHECK_ARG(T >= 0 && H > 0 && eps >= 0.0f);
    if (T == 0) return MOE_OK;
    CHECK_ARG(x && xn);
    cudaStream_t s = (cudaStream_t)stream;
    timing_begin(s);
    LAUNCH(kRmsnorm, launch_rmsnorm(x, T, H, eps, xn, s));
    return MOE_OK;
}

size_t moe_prerouter_workspace_bytes(const moe_prerouter* head, int32_t T) {
    if (!head || T < 0 || head->head_dim <= 0 || head->n_experts <= 0 || head->top_k <= 0) return 0;
    return prerouter_workspace_bytes(*head, T);
}

moe_status moe_prerouter_forward(const moe_prerouter* head, const uint16_t* h, const int32_t* exec_idx,
                                 const int32_t* prev_idx, int32_t T, float* logits, int32_t* pred_idx,
                                 void* workspace, size_t ws_bytes, moe_stream stream) {
    CHECK_ARG(head && T >= 0);
    const int H = head->hidden, E = head->n_experts, K = head->top_k, D = head->head_dim;
    CHECK_ARG(H > 0 && E > 0 && K > 0 && D > 0);
    if (E > MOEQ_MAX_EXPERTS || K > MOEQ_MAX_TOPK || K > E || H > MOEQ_MAX_HIDDEN || D > 4096)
        return MOE_ERR_UNSUPPORTED;
    CHECK_ARG(H % 8 == 0 && (H + 2 * E) % 8 == 0 && D % 8 == 0);
    CHECK_ARG(head->w1 && head->w2 && head->wl && aligned(head->w1, 16) && aligned(head->w2, 16) &&
              aligned(head->wl, 16));
    moe_status st = ws_check(workspace, ws_bytes, prerouter_workspace_bytes(*head, T));
    if (st != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    CHECK_ARG(h && exec_idx && logits && aligned(h, 16));
    cudaStream_t s = (cudaStream_t)stream;
    timing_begin(s);
    CHECK_CUDA(launch_prerouter(*head, h, exec_idx, prev_idx, T, logits, pred_idx, workspace, s));
    return MOE_OK;
}

moe_status moe_ffn_routing(const moe_layer* layer, int32_t T, const void* workspace, size_t ws_bytes,
                           int32_t* topk_idx, float* topk_w, moe_stream stream) {
    moe_status st = validate_layer(layer);
    if (st != MOE_OK) return st;
    CHECK_ARG(T >= 0);
    const Dims d = dims_of(layer, T);
    const WsPlan p = plan_of(d);
    st = ws_check(const_cast<void*>(workspace), ws_bytes, p.total);
    if (st != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    CHECK_ARG(topk_idx || topk_w);
    cudaStream_t s = (cudaStream_t)stream;
    const char* b = (const char*)workspace;
    const size_t n = (size_t)T * d.K;
    if (topk_idx) CHECK_CUDA(cudaMemcpyAsync(topk_idx, b + p.idx, n * 4, cudaMemcpyDeviceToDevice, s));
    if (topk_w) CHECK_CUDA(cudaMemcpyAsync(topk_w, b + p.w, n * 4, cudaMemcpyDeviceToDevice, s));
    return MOE_OK;
}

moe_status moe_get_device_status(void* workspace, moe_stream stream, int32_t* status) {
    if (!workspace || !aligned(workspace, kAlign)) return MOE_ERR_WORKSPACE;
    CHECK_ARG(status);
    cudaStream_t s = (cudaStream_t)stream;
    int32_t v = 0;
    CHECK_CUDA(cudaMemcpyAsync(&v, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost, s));
    CHECK_CUDA(cudaStreamSynchronize(s));
    CHECK_CUDA(cudaMemsetAsync(workspace, 0, sizeof(int32_t), s));
    CHECK_CUDA(cudaStreamSynchronize(s));
    *status = v;
    return MOE_OK;
}

moe_status moe_mixed_linear(const moe_mixed_tensor* W, const uint16_t* x, int32_t T, float* y, moe_stream stream) {
    CHECK_ARG(T >= 0);
    if (T == 0) return MOE_OK;
    CHECK_ARG(W && x && y && mixed_ok(W, W->out, W->in) && W->out > 0);
    cudaStream_t s = (cudaStream_t)stream;
    timing_begin(s);
    LAUNCH(kMixedLinear, launch_mixed_linear(*W, mixed_G(W->rho), x, T, y, s));
    return MOE_OK;
}

size_t moe_mixed_mlp_workspace_bytes(int32_t H, int32_t I, int32_t T) {
    if (H <= 0 || I <= 0 || T < 0) return 0;
    return align_up((size_t)T * I * 4) + align_up((size_t)T * H * 2) + kAlign;
}

moe_status moe_mixed_mlp_forward(const moe_mixed_tensor* gate, const moe_mixed_tensor* up,
                                 const moe_mixed_tensor* down, const uint16_t* x, int32_t T, int32_t residual,
                                 float eps, uint16_t* y, void* workspace, size_t ws_bytes, moe_stream stream) {
    CHECK_ARG(T >= 0 && gate && up && down && (residual == 0 || residual == 1));
    const int I = gate->out, H = gate->in;
    CHECK_ARG(H > 0 && I > 0 && mixed_ok(gate, I, H) && mixed_ok(up, I, H) && mixed_ok(down, H, I));
    CHECK_ARG(gate->rho == up->rho && gate->rho == down->rho);
    moe_status st = ws_check(workspace, ws_bytes, moe_mixed_mlp_workspace_bytes(H, I, T));
    if (st != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    CHECK_ARG(x && y && x != y);
    cudaStream_t s = (cudaStream_t)stream;
    float* h = (float*)workspace;
    uint16_t* xn = (uint16_t*)((char*)workspace + align_up((size_t)T * I * 4));
    const int G = mixed_G(gate->rho);
    const uint16_t* xin = x;
    timing_begin(s);
    if (residual) {
        LAUNCH(kRmsnorm, launch_rmsnorm(x, T, H, eps, xn, s));
        xin = xn;
    }
    LAUNCH(kMixedGateUp, launch_mixed_gate_up(*gate, *up, G, xin, T, h, s));
    LAUNCH(kMixedDown, launch_mixed_down(*down, G, h, T, residual ? x : nullptr, y, s));
    return MOE_OK;
}

// ------------------------------------------------ weight-activation mixed layer
namespace {
struct A8Ws {
    int8_t *q4, *q2;
    float* s;
    int32_t* qsum;
};
// 8-bit activation buffers of T rows of n: two permuted code copies, scales, code sums.
size_t a8_bytes(int T, int n) { return 2 * align_up((size_t)T * n) + 2 * align_up((size_t)T * 4); }
A8Ws a8_take(char* b, int T, int n) {
    A8Ws w;
    w.q4 = (int8_t*)b;
    w.q2 = (int8_t*)(b + align_up((size_t)T * n));
    w.s = (float*)(b + 2 * align_up((size_t)T * n));
    w.qsum = (int32_t*)(b + 2 * align_up((size_t)T * n) + align_up((size_t)T * 4));
    return w;
}
}  // namespace

size_t moe_mixed_linear_a8_workspace_bytes(int32_t in, int32_t T) {
    if (in <= 0 || T < 0) return 0;
    return a8_bytes(T, in);
}

size_t moe_mixed_mlp_a8_workspace_bytes(int32_t H, int32_t I, int32_t T) {
    if (H <= 0 || I <= 0 || T < 0) return 0;
    return align_up((size_t)T * H * 2) + a8_bytes(T, H) + align_up((size_t)T * I * 4) + a8_bytes(T, I);
}

moe_status moe_act8_quant(const uint16_t* x, int32_t T, int32_t n, int8_t* q, float* s, moe_stream stream) {
    CHECK_ARG(T >= 0 && n > 0);
    if (T == 0) return MOE_OK;
    CHECK_ARG(x && q && s);
    cudaStream_t st = (cudaStream_t)stream;
    timing_begin(st);
    CHECK_CUDA(launch_act8(x, nullptr, T, n, q, nullptr, nullptr, s, nullptr, st));
    timing_mark(kAct8, st);
    return MOE_OK;
}

moe_status moe_mixed_linear_a8(const moe_mixed_tensor* W, const uint16_t* x, int32_t T, float* y, void* workspace,
                               size_t ws_bytes, moe_stream stream) {
    CHECK_ARG(T >= 0 && W);
    CHECK_ARG(mixed_ok(W, W->out, W->in) && W->out > 0);
    moe_status st = ws_check(workspace, ws_bytes, a8_bytes(T, W->in));
    if (st != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    CHECK_ARG(x && y);
    cudaStream_t s = (cudaStream_t)stream;
    const A8Ws a = a8_take((char*)workspace, T, W->in);
    timing_begin(s);
    LAUNCH(kAct8, launch_act8(x, nullptr, T, W->in, nullptr, a.q4, a.q2, a.s, a.qsum, s));
    LAUNCH(kMixedA8, launch_mixed_a8(*W, nullptr, mixed_G(W->rho), a.q4, a.q2, a.s, a.qsum, T, 0, y, nullptr,
                                     nullptr, s));
    return MOE_OK;
}

moe_status moe_mixed_mlp_forward_a8(const moe_mixed_tensor* gate, const moe_mixed_tensor* up,
                                    const moe_mixed_tensor* down, const uint16_t* x, int32_t T, int32_t residual,
                                    float eps, uint16_t* y, void* workspace, size_t ws_bytes, moe_stream stream) {
    CHECK_ARG(T >= 0 && gate && up && down && (residual == 0 || residual == 1) && eps >= 0.0f);
    const int I = gate->out, H = gate->in;
    CHECK_ARG(H > 0 && I > 0 && mixed_ok(gate, I, H) && mixed_ok(up, I, H) && mixed_ok(down, H, I));
    CHECK_ARG(gate->rho == up->rho && gate->rho == down->rho);
    moe_status st = ws_check(workspace, ws_bytes, moe_mixed_mlp_a8_workspace_bytes(H, I, T));
    if (st != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    CHECK_ARG(x && y && x != y);
    cudaStream_t s = (cudaStream_t)stream;
    char* b = (char*)workspace;
    uint16_t* xn = (uint16_t*)b;
    b += align_up((size_t)T * H * 2);
    const A8Ws ax = a8_take(b, T, H);
    b += a8_bytes(T, H);
    float* h = (float*)b;
    b += align_up((size_t)T * I * 4);
    const A8Ws ah = a8_take(b, T, I);
    const int G = mixed_G(gate->rho);
    const uint16_t* xin = x;
    timing_begin(s);
    if (residual) {
        LAUNCH(kRmsnorm, launch_rmsnorm(x, T, H, eps, xn, s));
        xin = xn;
    }
    LAUNCH(kAct8, launch_act8(xin, nullptr, T, H, nullptr, ax.q4, ax.q2, ax.s, ax.qsum, s));
    LAUNCH(kMixedA8, launch_mixed_a8(*gate, up, G, ax.q4, ax.q2, ax.s, ax.qsum, T, 1, h, nullptr, nullptr, s));
    LAUNCH(kAct8, launch_act8(nullptr, h, T, I, nullptr, ah.q4, ah.q2, ah.s, ah.qsum, s));
    LAUNCH(kMixedA8, launch_mixed_a8(*down, nullptr, G, ah.q4, ah.q2, ah.s, ah.qsum, T, 2, nullptr, y,
                                     residual ? x : nullptr, s));
    return MOE_OK;
}

// ------------------------------------------------------------ expert parallelism
namespace {
// The layer as the experts-only forward sees it: one routed expert per row, no shared expert.
moe_layer experts_only(const moe_layer* L) {
    moe_layer c = *L;
    c.top_k = 1;
    memset(&c.s_gate, 0, sizeof(c.s_gate));
    memset(&c.s_up, 0, sizeof(c.s_up));
    memset(&c.s_down, 0, sizeof(c.s_down));
    memset(&c.shared_gate, 0, sizeof(c.shared_gate));
    for (int a = 0; a < MOEQ_MAX_ADAPTERS; ++a) {
        memset(&c.lora[a].s_gate, 0, sizeof(moe_lora_proj));
        memset(&c.lora[a].s_up, 0, sizeof(moe_lora_proj));
        memset(&c.lora[a].s_down, 0, sizeof(moe_lora_proj));
    }
    return c;
}
}  // namespace

size_t moe_experts_workspace_bytes(const moe_layer* layer, int32_t N) {
    if (!layer || N < 0 || validate_layer(layer) != MOE_OK) return 0;
    const moe_layer c = experts_only(layer);
    return plan_of(dims_of(&c, N)).total;
}

moe_status moe_experts_forward(const moe_layer* layer, const uint16_t* x, const int32_t* expert,
                               const int32_t* adapter_id, int32_t N, uint16_t* y, void* workspace, size_t ws_bytes,
                               moe_stream stream) {
    moe_status st = validate_layer(layer);
    if (st != MOE_OK) return st;
    CHECK_ARG(N >= 0);
    const moe_layer c = experts_only(layer);
    const Dims d = dims_of(&c, N);
    const WsPlan p = plan_of(d);
    st = ws_check(workspace, ws_bytes, p.total);
    if (st != MOE_OK) return st;
    if (N == 0) return MOE_OK;
    CHECK_ARG(x && y && expert && x != y && aligned(x, 16) && aligned(y, 2));
    cudaStream_t s = (cudaStream_t)stream;
    const Work wk = work_of(d, p, workspace);
    timing_begin(s);
    LAUNCH(kTopk, launch_given_experts(expert, N, wk.idx, wk.w, wk.sg, s));
    return experts_enqueue(&c, x, adapter_id, N, nullptr, y, wk, s);
}

moe_status moe_ep_dispatch(const uint16_t* x, const int32_t* topk_idx, const int32_t* adapter_id, int32_t n_adapters,
                           int32_t T, int32_t K, int32_t H, int32_t E, int32_t G, int32_t* pos, int32_t* counts,
                           uint16_t* send_x, int32_t* send_meta, int32_t* status, moe_stream stream) {
    CHECK_ARG(T >= 0 && K > 0 && H > 0 && E > 0 && G > 0 && n_adapters >= 0);
    if (G > MOEQ_EP_MAX_RANKS || E > MOEQ_MAX_EXPERTS || K > MOEQ_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
    CHECK_ARG(E % G == 0 && H % 8 == 0);
    if (T == 0) return MOE_OK;
    CHECK_ARG(x && topk_idx && pos && counts && send_x && send_meta && status && aligned(x, 16) &&
              aligned(send_x, 16));
    cudaStream_t s = (cudaStream_t)stream;
    timing_begin(s);
    LAUNCH(kEpDispatch, launch_ep_dispatch(x, topk_idx, adapter_id, n_adapters, T, K, H, E, G, pos, counts, send_x,
                                           send_meta, status, s));
    return MOE_OK;
}

moe_status moe_ep_combine(const uint16_t* ret, const int32_t* pos, const float* topk_w, const uint16_t* shared,
                          const float* shared_scale, int32_t T, int32_t K, int32_t H, uint16_t* y,
                          moe_stream stream) {
    CHECK_ARG(T >= 0 && K > 0 && H > 0 && H % 2 == 0);
    if (T == 0) return MOE_OK;
    CHECK_ARG(ret && pos && topk_w && y && aligned(ret, 4) && aligned(y, 4) && (!shared || aligned(shared, 4)));
    cudaStream_t s = (cudaStream_t)stream;
    timing_begin(s);
    LAUNCH(kEpCombine, launch_ep_combine(ret, pos, topk_w, shared, shared_scale, T, K, H, y, s));
    return MOE_OK;
}

}  // extern "C"
