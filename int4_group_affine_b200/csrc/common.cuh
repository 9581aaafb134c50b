// common.cuh - device helpers and the internal launch interface of libmoeq.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moeq.h"

namespace moeq {

constexpr int kWarp = 32;

// ------------------------------------------------------------------ bf16
__device__ __forceinline__ float bf16f(uint16_t h) { return __uint_as_float(((uint32_t)h) << 16); }
__device__ __forceinline__ uint16_t f2bf16(float f) { return __bfloat16_as_ushort(__float2bfloat16_rn(f)); }

// First error wins; later errors do not overwrite it.
__device__ __forceinline__ void raise_status(int32_t* st, int code) {
    if (st) atomicCAS(st, 0, code);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// One entry of a caller-given expert set (one warp per token, lane k < K takes entry
// k of sel[0..K)): an entry outside [0, E) or repeating an earlier entry of the same
// token is replaced by the lowest expert index the token does not use yet (entries
// fixed in lane order), and *bad is set; returns this lane's expert (lanes >= K: -1).
__device__ __forceinline__ int select_entry(const int32_t* sel, int K, int E, int lane, bool* bad) {
    int e = lane < K ? sel[lane] : -1;
    bool ok = lane < K && e >= 0 && e < E;
    for (int j = 0; j < K; ++j) {
        const int ej = __shfl_sync(0xffffffffu, e, j);
        if (j < lane && ej == e) ok = false;
    }
    uint32_t badm = __ballot_sync(0xffffffffu, lane < K && !ok);
    *bad = badm != 0;
    if (lane < K && !ok) e = -1;
    while (badm) {
        const int k = __ffs(badm) - 1;
        badm &= badm - 1;
        int c = 0;
        while (__any_sync(0xffffffffu, lane < K && e == c)) ++c;
        if (lane == k) e = c;
    }
    return e;
}

// q (0..2^23) as float without an integer-to-float conversion instruction.
__device__ __forceinline__ float u2f_small(uint32_t q) { return __uint_as_float(0x4B000000u | q) - 8388608.0f; }

__device__ __forceinline__ float silu(float g) { return g / (1.0f + expf(-g)); }

// ------------------------------------------------------------ workspace
// Device view of the forward workspace.  Offsets are fixed by ws_plan().
struct Work {
    int32_t* status;     // sticky error word
    int32_t* n_active;   // number of experts with at least one job (incl. shared)
    int32_t* idx;        // [T][K]
    float* w;            // [T][K]
    float* sg;           // [T]
    float* logits;       // [T][E]
    float* gs;           // [T]
    int32_t* cnt;        // [nb][C] counts, scanned in place to bases
    int32_t* goff;       // [E+2] job offset of each expert group (E = shared)
    int32_t* active;     // [E+1] expert ids of non-empty groups, ascending
    int4* perm;          // [J] {token, k, adapter, expert}
    float* wperm;        // [J] combine weight of each job
    int32_t* inv;        // [T][K+1] position of job (t, k)
    float* tgu;          // [J][2r] LoRA A products for gate | up
    float* td;           // [J][r]  LoRA A products for down
    float* h;            // [J][Imax] SwiGLU activations
    float* ypart;        // [J][H] per-job weighted outputs
    uint16_t* xn;        // [T][H] normalised input (block mode)
    uint16_t* xp;        // [T][H] input in the permuted K order of the tensor-core int4 tiles
    int T, K, E, H, I, Is, Imax, A1, C, nb, J, r;
};

struct WsPlan {
    size_t status, n_active, idx, w, sg, logits, gs, cnt, goff, active, perm, wperm, inv, tgu, td, h, ypart, xn, xp;
    size_t bar, dts, dtg, dtdp;  // fused decode scratch (sizes zero when T is too large for it)
    size_t slots;                // chain decode tagged words (right after the header, for every T)
    size_t cslots;               // cluster decode ticket and tagged words (after the chain's)
    size_t hxin, hyout;          // staging of host x and y (moe_ffn_forward_host, T <= 8)
    size_t total;
};

// All the layer fields a kernel needs, passed by value.
struct LayerArgs {
    moe_qtensor gate, up, down, s_gate, s_up, s_down, router, shared_gate;
    const float* logit_bias;
    int H, E, K, I, Is, n_adapters, rank;
    float scale;  // alpha / rank
    bool has_shared, has_sgate;
    moe_lora_ptrs lora[MOEQ_MAX_ADAPTERS];
};

// Bound (ns of device time) of every bounded device-side wait, passed to the kernels
// with their arguments (moe_set_wait_limit_ns; 1 s by default).
uint64_t wait_limit_ns();

// The forward's checks that precede the workspace check (layer, T, x and y).
moe_status ffn_precheck(const moe_layer* layer, const uint16_t* x, const uint16_t* y, int32_t T);

// Raise a kernel's dynamic shared-memory limit to at least `bytes`, calling the
// runtime only when the cached limit is too small (so repeated launches, and
// launches during stream capture, do not call it again).  The cache assumes one
// device per process.
inline cudaError_t ensure_smem(const void* fn, size_t bytes, int& cached) {
    if (bytes <= 48 * 1024 || (int)bytes <= cached) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) cached = (int)bytes;
    return e;
}

// ------------------------------------------------------------- fused decode
#define MOEQ_DECODE_MAX_TOKENS 8
#define MOEQ_DECODE_MAX_JOBS 32
#define MOEQ_DECODE_MAX_CTAS 256

#define MOEQ_DECODE_MAX_RANK 32

// Scratch of the fused decode kernel (all inside the forward workspace).  Besides the
// status word and the arrival counter, bytes 16..255 of the workspace header (zeroed by
// moe_workspace_init) hold the kernel's per-launch ready flags.
struct DecodeScratch {
    float *logits, *gsl, *ts, *tg, *h;
    float* tdp;               // [MOEQ_DECODE_MAX_CTAS][3][T][rank] partial sums
    unsigned long long* bar;  // monotonic arrival counter: starts zeroed (workspace header)
    int32_t* status;          // workspace base (status word)
    int32_t* idx_out;         // [T][K] routing record (the workspace's top-K region)
    float* w_out;             // [T][K]
};

// ------------------------------------------------------------- timing
enum Kind {
    kPack, kDequant, kRouter, kTopk, kIndexCount, kIndexScan, kIndexScatter, kLoraA, kGateUp, kDown,
    kCombine, kRmsnorm, kMixedGateUp, kMixedDown, kMixedLinear, kDecode, kTcLoraGUKind, kTcGUKind,
    kTcLoraDownKind, kTcDownKind, kTcRouterKind, kKpermKind, kDecodeChain, kPrerouter, kAct8, kMixedA8, kEpDispatch, kEpCombine, kDecodeCluster, kKindCount
};
void timing_begin(cudaStream_t s);
void timing_mark(int kind, cudaStream_t s);

// ------------------------------------------------------------- launchers
cudaError_t launch_pack_affine(const float* W, int64_t rows, int in, int group, int bits, uint32_t* packed,
                               uint16_t* scales, uint16_t* biases, cudaStream_t s);
cudaError_t launch_pack_mixed(const float* W, int out, int in, int G, uint32_t* packed, uint16_t* scales,
                              cudaStream_t s);
cudaError_t launch_dequant_affine(const moe_qtensor& t, float* out, cudaStream_t s);
cudaError_t launch_dequant_mixed(const moe_mixed_tensor& t, int G, float* out, cudaStream_t s);

cudaError_t launch_router_logits(const uint16_t* x, const moe_qtensor& router, const moe_qtensor* sgate,
                                 const float* logit_bias, int T, int H, int E, float* logits, float* gs,
                                 cudaStream_t s);
// the shared-expert gate logit of every token alone (x rows 16-byte aligned, H % 16 == 0)
cudaError_t launch_sgate_logits(const uint16_t* x, const moe_qtensor& sgate, int T, int H, float* gs,
                                cudaStream_t s);
cudaError_t launch_topk(const float* logits, const float* gs, bool has_sgate, int T, int E, int K, int32_t* idx,
                        float* w, float* sg, cudaStream_t s);

// The routing of a caller-given expert set (the prerouter's prediction, say): idx from
// sel [T][K] (repaired as in select_entry, MOE_ERR_DEVICE_INDEX raised), weights the
// softmax of the logits renormalised over the set, sg = sigmoid(gs).
cudaError_t launch_select(const float* logits, const float* gs, bool has_sgate, const int32_t* sel, int T, int E,
                          int K, int32_t* idx, float* w, float* sg, int32_t* status, cudaStream_t s);

cudaError_t launch_index_build(const Work& wk, const int32_t* adapter_id, int n_adapters, cudaStream_t s);
cudaError_t launch_index_build_counts(const Work& wk, const int32_t* adapter_id, int n_adapters,
                                      int32_t* counts_out, cudaStream_t s);

cudaError_t launch_lora_a(const Work& wk, const LayerArgs& L, int phase, const uint16_t* x, cudaStream_t s);
// LoRA-A products of the expert-grouped jobs on mma.sync tiles (down = 0: [J][2r] from x
// by token; down = 1: [J][r] from the bf16 h rows of the jobs, stored in the int4 tiles' K order)
cudaError_t launch_lora_a_mma(const LayerArgs& L, int down, const uint16_t* act, int ld, const Work& wk,
                              cudaStream_t s);
cudaError_t launch_gate_up(const Work& wk, const LayerArgs& L, const uint16_t* x, int max_groups, cudaStream_t s);
cudaError_t launch_down(const Work& wk, const LayerArgs& L, int max_groups, cudaStream_t s);
cudaError_t launch_combine(const Work& wk, const uint16_t* residual, uint16_t* y, cudaStream_t s);

cudaError_t launch_rmsnorm(const uint16_t* x, int T, int H, float eps, uint16_t* xn, cudaStream_t s);

// tcgen05 grouped GEMM modes (csrc/prefill.cu)
enum TcMode { kTcGU = 0, kTcDown = 1 };
bool tc_supported(const LayerArgs& L);
cudaError_t launch_tc_gemm(const LayerArgs& L, int mode, const uint16_t* act, int ld_act, const Work& wk,
                           const uint16_t* hb_out, int ldh, cudaStream_t s);
// x [elems] bf16 -> xp: each 8-element group reordered 0 4 1 5 2 6 3 7 (the K order
// of the tensor-core int4 tiles)
cudaError_t launch_kperm(const uint16_t* x, int64_t elems, uint16_t* xp, cudaStream_t s);
// router logits [T][E] on the tensor cores (the shared-expert gate row is not included)
bool tc_router_supported(const moe_qtensor& router, int H, int E);
cudaError_t launch_tc_router(const moe_qtensor& router, const float* logit_bias, const uint16_t* x, int T, int H,
                             int E, float* logits, int32_t* status, cudaStream_t s);

bool decode_supported(const LayerArgs& L, int T, size_t* smem_out);
cudaError_t launch_decode(const LayerArgs& L, const uint16_t* x, const int32_t* adapter_id, uint16_t* y, int T,
                          int block, float eps, const DecodeScratch& sc, cudaStream_t s);

// The chain decode kernel (csrc/decode_chain.cu): one to four tokens, cross-CTA
// hand-offs through epoch-tagged 64-bit words in a workspace region of
// chain_slot_words(...) words that sits at a fixed place for a layer shape.
struct ChainScratch {
    uint64_t* slots;           // the kernel's region: ticket, counters, tagged words (starts zeroed)
    int32_t* status;
    int32_t* idx_out;          // [T][K] routing record
    float* w_out;
};
size_t chain_slot_words(int E, int K, int I, int Is, int r);
bool chain_supported(const LayerArgs& L, int T);
cudaError_t launch_chain(const LayerArgs& L, const uint16_t* x, const int32_t* adapter_id, const int32_t* select,
                         uint16_t* y, int T, int block, float eps, const ChainScratch& sc, cudaStream_t s);

// The cluster decode kernel (csrc/decode_cluster.cu): one token; the per-cluster steps
// exchange through distributed shared memory, h through epoch-tagged words in a
// workspace region of cluster_slot_words(...) words at a fixed place for a layer shape.
struct ClusterScratch {
    uint64_t* slots;           // ticket counter, spares, tagged h words (starts zeroed)
    int x_host;                // x is mapped host memory: read with plain loads, not a bulk copy
    int32_t* status;
    int32_t* idx_out;          // [K] routing record
    float* w_out;
};
size_t cluster_slot_words(int K, int I, int Is);
bool cluster_supported(const LayerArgs& L, int T);
cudaError_t launch_cluster(const LayerArgs& L, const uint16_t* x, const int32_t* adapter_id, const int32_t* select,
                           uint16_t* y, int T, int block, float eps, const ClusterScratch& sc, cudaStream_t s);

// The prerouter head (csrc/prerouter.cu).
size_t prerouter_workspace_bytes(const moe_prerouter& P, int T);
cudaError_t launch_prerouter(const moe_prerouter& P, const uint16_t* h, const int32_t* exec_idx,
                             const int32_t* prev_idx, int T, float* logits, int32_t* pred_idx, void* ws,
                             cudaStream_t s);

cudaError_t launch_mixed_linear(const moe_mixed_tensor& W, int G, const uint16_t* x, int T, float* y,
                                cudaStream_t s);
cudaError_t launch_mixed_gate_up(const moe_mixed_tensor& g, const moe_mixed_tensor& u, int G, const uint16_t* x,
                                 int T, float* h, cudaStream_t s);
cudaError_t launch_mixed_down(const moe_mixed_tensor& d, int G, const float* h, int T, const uint16_t* residual,
                              uint16_t* y, cudaStream_t s);

// Weight-activation form of the mixed layer (csrc/mixed_a8.cu): 8-bit per-token
// activation codes (natural order and the two permuted copies, any may be NULL) from
// bf16 (xb) or fp32 (xf) rows; then the integer dot in one of three modes
// (0: y fp32; 1: h = SiLU(W x) * (U x) fp32; 2: y bf16 plus an optional residual).
cudaError_t launch_act8(const uint16_t* xb, const float* xf, int T, int n, int8_t* qnat, int8_t* q4, int8_t* q2,
                        float* s, int32_t* qsum, cudaStream_t st);
cudaError_t launch_mixed_a8(const moe_mixed_tensor& W, const moe_mixed_tensor* U, int G, const int8_t* q4,
                            const int8_t* q2, const float* sx, const int32_t* qsum, int T, int mode, float* yf,
                            uint16_t* yb, const uint16_t* residual, cudaStream_t s);

// Expert parallelism (csrc/ep.cu); MOEQ_EP_MAX_RANKS comes from moeq.h.
cudaError_t launch_given_experts(const int32_t* expert, int N, int32_t* idx, float* w, float* sg, cudaStream_t s);
cudaError_t launch_ep_dispatch(const uint16_t* x, const int32_t* idx, const int32_t* adapter_id, int n_adapters, int T,
                               int K, int H, int E, int G, int32_t* pos, int32_t* counts, uint16_t* send_x,
                               int32_t* meta, int32_t* status, cudaStream_t s);
cudaError_t launch_ep_combine(const uint16_t* ret, const int32_t* pos, const float* w, const uint16_t* shared,
                              const float* sg, int T, int K, int H, uint16_t* y, cudaStream_t s);

// Device row offset (in words) of row `o` of a mixed matrix with super-group size G.
__host__ __device__ __forceinline__ int64_t mixed_row_offset(int o, int in, int G) {
    const int64_t w4 = in / 8, w2 = in / 16;
    if (G == 0) return (int64_t)o * w2;
    const int64_t sg = o / G, pos = o % G;
    const int64_t base = sg * (w4 + (int64_t)(G - 1) * w2);
    return pos == 0 ? base : base + w4 + (pos - 1) * w2;
}

}  // namespace moeq
