/*
 * moeq.h - C ABI of libmoeq, the B200 (sm_100a) int4 group-affine MoE expert
 * FFN library.
 *
 * Conventions shared by every entry point:
 *  - Pointers marked "device" are CUDA device pointers in the current device's
 *    address space; the caller allocates and owns them.  Pointers marked
 *    "host" are ordinary host memory.  The library never allocates or frees
 *    memory and never keeps a pointer after the call returns (moe_layer is a
 *    caller-owned plain struct; lora_set_adapters only writes into it).
 *  - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is the
 *    legacy default stream) and the call returns without synchronising, except
 *    where a function says otherwise.  Launch sequences contain no host
 *    synchronisation, so they can be recorded into CUDA graphs.
 *  - bf16 values are passed as their uint16 bit patterns.
 *  - Every function returns a moe_status.  Argument errors are detected on the
 *    host before anything is enqueued and return MOE_ERR_INVALID_ARG or
 *    MOE_ERR_UNSUPPORTED; a failed launch returns MOE_ERR_CUDA.  Problems that
 *    only the device can see set a sticky status word inside the workspace
 *    (read with moe_get_device_status): an expert index out of range in
 *    caller-supplied routing makes that job contribute zero; an adapter id out
 *    of range runs that token on the base weights alone.
 *
 * Storage formats:
 *  - Affine (int4 or int8), groups of `group` consecutive input elements
 *    (64 for the Edge0 weights; 32 also accepted): packed uint32
 *    [n][out][in*bits/32], element j of a row in word j/(32/bits), bit field
 *    (j % (32/bits))*bits, lowest field first (8 nibbles or 4 bytes per word);
 *    scales and biases bf16 [n][out][in/group]; w = s*q + b.  Source: the
 *    "Recover-LoRA: 4-bit 压缩掉的精度" page, section 一 (4-bit, group 64,
 *    affine: per-group scale and zero-point; router and shared_expert_gate at
 *    8 bits); the Edge0-35B-A3B guide, sections 三大核心机制 and 量化实现;
 *    the d1a MLX port page, section "4-bit 分组量化" (bf16 scale and bias).
 *  - Mixed ternary/4-bit (EdgeRazor SQMP, "EDGERAZOR 深度解读" section 2.1):
 *    G = floor(1/rho) consecutive output rows form a super-group whose first
 *    row is 4-bit symmetric (in/8 words, nibble = q+8, q in [-7,7]) and whose
 *    other G-1 rows are ternary (in/16 words, 2-bit field = q+1); super-groups
 *    are stored one after another, a trailing partial one keeping its 4-bit
 *    row first; rho = 0 stores every row ternary.  One bf16 scale per row;
 *    w = s*q.
 *  - LoRA factors bf16: A [n][rank][in], B [n][out][rank]; the delta on a
 *    projection is (alpha/rank) * B (A v), never merged into the base weights
 *    ("Recover-LoRA" page section 二; "Edge0 项目推荐" review, 亮点三).
 */
#ifndef MOEQ_H
#define MOEQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOEQ_API __attribute__((visibility("default")))
#else
#define MOEQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define MOEQ_VERSION 1
#define MOEQ_MAX_ADAPTERS 16
#define MOEQ_MAX_RANK 64
#define MOEQ_MAX_EXPERTS 512
#define MOEQ_MAX_TOPK 16
#define MOEQ_MAX_HIDDEN 8192
#define MOEQ_MAX_INTER 8192

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,  /* a pointer, size or shape violates the contract */
    MOE_ERR_UNSUPPORTED = 2,  /* valid but outside what this build implements */
    MOE_ERR_CUDA = 3,         /* a CUDA call or launch failed */
    MOE_ERR_WORKSPACE = 4,    /* workspace missing, misaligned or too small */
    MOE_ERR_DEVICE_INDEX = 5, /* device saw an expert/adapter index out of range */
    MOE_ERR_TIMEOUT = 6       /* a bounded device-side wait gave up */
} moe_status;

typedef enum {
    MOE_FMT_AFFINE_INT4 = 0,
    MOE_FMT_AFFINE_INT8 = 1,
    MOE_FMT_MIXED_TERNARY_INT4 = 2
} moe_format;

typedef void* moe_stream; /* cudaStream_t */

/* An affine-quantised matrix or a stack of n equally shaped matrices (device). */
typedef struct {
    const uint32_t* packed; /* [n][out][in*bits/32] */
    const uint16_t* scales; /* [n][out][in/group] bf16 */
    const uint16_t* biases; /* [n][out][in/group] bf16 */
    int32_t n, out, in, bits, group;
} moe_qtensor;

/* A mixed ternary/4-bit matrix (device). */
typedef struct {
    const uint32_t* packed; /* moe_mixed_words(out, in, rho) words */
    const uint16_t* scales; /* [out] bf16 */
    int32_t out, in;
    float rho;
} moe_mixed_tensor;

typedef struct {
    const uint16_t* A; /* [n][rank][in] bf16, device; NULL: no delta on this projection */
    const uint16_t* B; /* [n][out][rank] bf16, device */
} moe_lora_proj;

/* One adapter set: factors for the routed experts (n = n_experts) and the
 * shared expert (n = 1). */
typedef struct {
    moe_lora_proj gate, up, down;
    moe_lora_proj s_gate, s_up, s_down;
} moe_lora_ptrs;

/* One MoE layer: non-owning views of device tensors (caller-owned POD). */
typedef struct {
    int32_t hidden;       /* H */
    int32_t n_experts;    /* E */
    int32_t top_k;        /* K */
    int32_t inter;        /* I, routed-expert intermediate size */
    int32_t shared_inter; /* Is, shared-expert intermediate size */
    moe_qtensor router;      /* int8 [1][E][H] */
    moe_qtensor shared_gate; /* int8 [1][1][H]; packed NULL: shared output ungated */
    moe_qtensor gate, up;    /* int4 [E][I][H] */
    moe_qtensor down;        /* int4 [E][H][I] */
    moe_qtensor s_gate, s_up; /* int4 [1][Is][H]; packed NULL: no shared expert */
    moe_qtensor s_down;       /* int4 [1][H][Is] */
    const float* logit_bias;  /* [E] fp32 added to the router logits, or NULL */
    int32_t n_adapters;       /* 0: base weights only */
    int32_t rank;
    float alpha;
    moe_lora_ptrs lora[MOEQ_MAX_ADAPTERS];
} moe_layer;

/* Library version (MOEQ_VERSION) and a readable name for a status. */
MOEQ_API int moe_version(void);
MOEQ_API const char* moe_status_string(moe_status status);

/* ------------------------------------------------------------------ a0 pack
 * Quantise fp32 weights W [rows][in] (device) into the given format.
 *  AFFINE_INT4 / AFFINE_INT8: groups of `group` along `in`; b = the group
 *    minimum rounded down to bf16, s = (max - b)/(2^bits - 1) rounded up to
 *    bf16 (s = 0 and q = 0 when max == b), q = clamp(rint((w - b)/s)), all in
 *    fp64, so that |w - (s*q + b)| <= s/2.  Writes packed [rows][in*bits/32],
 *    scales and biases [rows][in/group].  in % group == 0 and group % 8 == 0.
 *  MIXED_TERNARY_INT4: rows are output channels; `rho` in [0, 1] fixes
 *    G = floor(1/rho); 4-bit rows: s = bf16(max(max|w|/7, 1e-5)), ternary rows:
 *    s = bf16(max(2*mean|w|, 1e-5)) (nearest-even bf16, mean summed in fp64
 *    in index order); q = clamp(rint(w/s)).  `biases` must be NULL, `group`
 *    is ignored, in % 16 == 0.  Writes moe_mixed_words(rows, in, rho) words
 *    and rows scales.
 * The pages fix the group size, the bf16 parameters and the mixed quantisers
 * but not how s and b are chosen for the affine format: the rule above is the
 * reading this library adopts. */
MOEQ_API moe_status moe_quant_pack(moe_format fmt, const float* W, int64_t rows, int32_t in, int32_t group,
                          float rho, uint32_t* packed, uint16_t* scales, uint16_t* biases,
                          moe_stream stream);

/* Number of uint32 words of a mixed matrix (host helper, no device work). */
MOEQ_API int64_t moe_mixed_words(int32_t out, int32_t in, float rho);

/* Dequantise to fp32 (device out [n][out][in]): w = fp32(s*q + b), bit-exact
 * with fmaf(s, q, b).  Verbatim copies of packed words, scales and biases
 * dequantise identically (d1a MLX port page, "0.0 反量化误差"). */
MOEQ_API moe_status moe_dequant(const moe_qtensor* t, float* w_hat, moe_stream stream);
MOEQ_API moe_status moe_mixed_dequant(const moe_mixed_tensor* t, float* w_hat, moe_stream stream);

/* ---------------------------------------------------------- a1 + a2 router
 * logits = dequant8(router) x + logit_bias; p = softmax(logits); the K largest
 * logits in descending order, equal logits to the lower expert index;
 * topk_w = p / sum over the chosen K; shared_scale = sigmoid(dequant8(shared_gate) x)
 * (1 when shared_gate is NULL or its packed is NULL).  SOFTMAX_TOPK routing
 * ("Edge0 项目推荐" review, framework paragraph; renormalisation as stated for
 * this method), 8-bit gates ("Recover-LoRA" page, section 一).
 *  x            device bf16 [T][H]
 *  router       int8 tensor [1][E][H]
 *  topk_idx     device int32 [T][K]    topk_w device fp32 [T][K]
 *  shared_scale device fp32 [T] or NULL; logits device fp32 [T][E] or NULL
 * Constraints: H % router->group == 0, 1 <= K <= min(E, 16), E <= 512. */
MOEQ_API moe_status moe_router_topk(const uint16_t* x, const moe_qtensor* router, const moe_qtensor* shared_gate,
                           const float* logit_bias, int32_t T, int32_t H, int32_t E, int32_t K,
                           int32_t* topk_idx, float* topk_w, float* shared_scale, float* logits,
                           moe_stream stream);

/* ------------------------------------------------------------ a3 index build
 * Expert-grouped job list, kept on the device (routing indices never go back
 * to the host; "Edge0 项目推荐" review, 亮点二).  Each token t owns K routed jobs
 * (k = 0..K-1, expert topk_idx[t][k]) and one shared-expert job (k = K, expert
 * index E).  Jobs are sorted by (expert, adapter, token, k), adapter -1 (none)
 * after the real adapters.
 *  adapter_id device int32 [T] or NULL (NULL: adapter 0 when n_adapters > 0,
 *             else none); values in [-1, n_adapters)
 *  counts     device int32 [E+1]; offsets device int32 [E+2] (exclusive prefix)
 *  perm       device int32 [T*(K+1)][4] = {token, k, adapter, expert}
 *  workspace  device scratch of moe_index_workspace_bytes(T, K, E, n_adapters)
 *             bytes, 256-byte aligned; its status word must be initialised once
 *             with moe_workspace_init. */
MOEQ_API size_t moe_index_workspace_bytes(int32_t T, int32_t K, int32_t E, int32_t n_adapters);
MOEQ_API moe_status moe_index_build(const int32_t* topk_idx, const int32_t* adapter_id, int32_t T, int32_t K,
                           int32_t E, int32_t n_adapters, int32_t* counts, int32_t* offsets, int32_t* perm,
                           void* workspace, size_t ws_bytes, moe_stream stream);

/* ------------------------------------------------------------------- LoRA
 * Install n_adapters unmerged adapter sets of the given rank into `layer`
 * (host struct; only the LoRA fields change).  Pointers in `sets` (host array
 * of n_adapters entries) are device pointers; a NULL A or B disables the delta
 * on that projection.  n_adapters = 0 removes all adapters.  Limits:
 * n_adapters <= 16, 1 <= rank <= 64. */
MOEQ_API moe_status lora_set_adapters(moe_layer* layer, int32_t n_adapters, int32_t rank, float alpha,
                             const moe_lora_ptrs* sets);

/* ---------------------------------------------------------- a4-a6 forward
 * y[t] = sum_k w_k E_{idx_k}(x_t) + sigmoid(g_s(x_t)) S(x_t) with
 *   E(x) = W_d h + (alpha/r) B_d A_d h,  h = SiLU(W_g x + (alpha/r) B_g A_g x)
 *          * (W_u x + (alpha/r) B_u A_u x)
 * (SiLU on the gate branch; "Edge0 项目推荐" review, 优点 on the _swiglu(up,
 * gate) order).  Combined in fixed order (k = 0..K-1, then shared), fp32
 * accumulation, bf16 output.
 *  x          device bf16 [T][H]; y device bf16 [T][H] (may not alias x)
 *  adapter_id device int32 [T] or NULL (see moe_index_build)
 *  workspace  device scratch of moe_ffn_workspace_bytes(layer, T) bytes,
 *             256-byte aligned, initialised once with moe_workspace_init.
 * T = 0 is accepted and enqueues nothing.  Calls sharing a workspace must be
 * ordered on one stream. */
MOEQ_API size_t moe_ffn_workspace_bytes(const moe_layer* layer, int32_t T);
MOEQ_API moe_status moe_workspace_init(void* workspace, size_t ws_bytes, moe_stream stream);
MOEQ_API moe_status moe_ffn_forward(const moe_layer* layer, const uint16_t* x, const int32_t* adapter_id, int32_t T,
                           uint16_t* y, void* workspace, size_t ws_bytes, moe_stream stream);

/* The forward of moe_ffn_forward for a decode-sized call (1 to 8 tokens) whose input x and
 * output y ([T][hidden] bf16, 16-byte aligned) are in page-locked host memory mapped into the
 * device's address space (cudaHostAlloc / cudaMallocHost memory on a 64-bit system with
 * unified addressing, or memory registered with cudaHostRegisterMapped).  The transfers are
 * part of the call, on `stream`: with one token the cluster decode kernel reads x and writes y
 * across the bus itself; otherwise x is copied into the workspace, the forward runs there and y
 * is copied back.  adapter_id, if given, is device memory.  The workspace is
 * moe_ffn_workspace_bytes(layer, T) bytes.  Errors: those of moe_ffn_forward;
 * MOE_ERR_UNSUPPORTED for T above 8; MOE_ERR_INVALID_ARG when x or y is not mapped host
 * memory.  Nothing is enqueued on an error. */
MOEQ_API moe_status moe_ffn_forward_host(const moe_layer* layer, const uint16_t* x_host, const int32_t* adapter_id,
                                         int32_t T, uint16_t* y_host, void* workspace, size_t ws_bytes,
                                         moe_stream stream);

/* ------------------------------------------ forward without device allocation
 * No counterpart on the pages: this entry point exists for callers that cannot
 * allocate device memory at the point where they run the layer (an engine's
 * enqueue hook or plugin that must not allocate, a serving runtime that has
 * reserved all device memory up front, or code that cannot afford the implicit
 * synchronisation an allocation may cause).  It computes exactly what
 * moe_ffn_forward computes, on the same kernels, but takes its workspace from
 * a fixed array of MOEQ_STATIC_WS_BYTES compiled into the library; every device
 * that loads the library holds that array until the process exits.  The caller
 * still passes x, adapter_id and y (device pointers, as for moe_ffn_forward).
 *  - The layer, T, x and y are checked first, with moe_ffn_forward's rules and
 *    status codes; then MOE_ERR_WORKSPACE is returned when
 *    moe_ffn_workspace_bytes(layer, T) exceeds MOEQ_STATIC_WS_BYTES (16 MiB: at
 *    least 256 tokens of the 2048-hidden, 256-expert, top-4 layer with four
 *    rank-16 adapter sets).  A rejected call enqueues nothing.
 *  - The first call on a device looks up the array's device address there
 *    (once per device, with that device current); make that first call before
 *    any stream capture.
 *  - All calls share the one array and it keeps the last call's contents: each
 *    call clears the status header it needs zeroed, and calls that overlap on
 *    the GPU (on different streams, or from several host threads) race on it.
 *    Order them on one stream.
 *  - No device memory is allocated or freed. */
#define MOEQ_STATIC_WS_BYTES (16u * 1024u * 1024u)
MOEQ_API moe_status moe_ffn_forward_static(const moe_layer* layer, const uint16_t* x, const int32_t* adapter_id,
                                           int32_t T, uint16_t* y, moe_stream stream);

/* The sticky device status word of the fixed array above (what moe_get_device_status
 * reads for a caller-owned workspace): the first problem the device saw during the
 * most recent moe_ffn_forward_static call on this device (MOE_ERR_DEVICE_INDEX,
 * MOE_ERR_TIMEOUT) or MOE_OK.  Read it after that call and before the next one,
 * which clears it.  Writes the value into *status (host), clears the word, and
 * synchronises `stream`. */
MOEQ_API moe_status moe_ffn_static_device_status(moe_stream stream, int32_t* status);

/* ------------------------------------------------ routing by a given set
 * The forward of moe_ffn_forward with the expert set of each token given by the
 * caller instead of taken as the top-K of the router: select device int32 [T][K].
 * The router still runs; the weights are its softmax renormalised over the given
 * set (w_k = exp(z_k) / sum over the set), the shared-expert scale is unchanged.
 * This is the prerouter's "the prediction is the routing" step ("Edge0 项目推荐"
 * review, 亮点一: the set the next layer runs for the next token is the head's
 * prediction itself, so nothing predicted is ever discarded or re-read).  An entry
 * outside [0, E), or repeating an earlier entry of its token, is replaced by the
 * lowest expert index that token does not use yet and raises MOE_ERR_DEVICE_INDEX.
 * Workspace and other arguments as for moe_ffn_forward. */
MOEQ_API moe_status moe_ffn_forward_select(const moe_layer* layer, const uint16_t* x, const int32_t* adapter_id,
                                           const int32_t* select, int32_t T, uint16_t* y, void* workspace,
                                           size_t ws_bytes, moe_stream stream);

/* ------------------------------------------------------ prerouter head
 * Layer N's prerouter head ("Edge0 项目推荐" review, 亮点一): from the layer's MoE
 * input h, the experts this token was routed to at layer N and those of the
 * previous token, it predicts layer N+1's router logits,
 *   f = [h, onehot(exec_idx[t]), onehot(prev_idx[t])]       (width H + 2E)
 *   logits = linear_init(f) + fc2(gelu(fc1(f))),  gelu(v) = v * Phi(v)  (erf form)
 * with fp16 weights (fp16 in training and production on that page) and fp32
 * arithmetic here; its top-K (ties to the lower index) is the set layer N+1 runs
 * for token t+1 (pass it to moe_ffn_forward_select).
 *  h         device bf16 [T][H] (16-byte aligned)
 *  exec_idx  device int32 [T][K]; prev_idx device int32 [T][K] or NULL (no
 *            previous token: an all-zero one-hot).  An expert listed twice sets one
 *            one; an entry outside [0, E) sets none and raises MOE_ERR_DEVICE_INDEX
 *            in the workspace's status word (moe_get_device_status).
 *  logits    device fp32 [T][E]; pred_idx device int32 [T][K] or NULL
 *  workspace device scratch of moe_prerouter_workspace_bytes(head, T) bytes,
 *            256-byte aligned, initialised once with moe_workspace_init.
 * Limits: H % 8 == 0, (H + 2E) % 8 == 0, D % 8 == 0, E <= 512, 1 <= K <= min(E, 16),
 * weights 16-byte aligned. */
typedef struct {
    int32_t hidden;     /* H */
    int32_t n_experts;  /* E */
    int32_t top_k;      /* K */
    int32_t head_dim;   /* D, the width of fc1's output (512 for the Edge0-35B heads) */
    const uint16_t* w1; /* fc1 fp16 [D][H + 2E] */
    const uint16_t* b1; /* fp16 [D] or NULL */
    const uint16_t* w2; /* fc2 fp16 [E][D] */
    const uint16_t* b2; /* fp16 [E] or NULL */
    const uint16_t* wl; /* linear_init fp16 [E][H + 2E] */
    const uint16_t* bl; /* fp16 [E] or NULL */
} moe_prerouter;
MOEQ_API size_t moe_prerouter_workspace_bytes(const moe_prerouter* head, int32_t T);
MOEQ_API moe_status moe_prerouter_forward(const moe_prerouter* head, const uint16_t* h, const int32_t* exec_idx,
                                          const int32_t* prev_idx, int32_t T, float* logits, int32_t* pred_idx,
                                          void* workspace, size_t ws_bytes, moe_stream stream);

/* Pre-norm residual block for stacked layers:
 *   x_out = bf16(x + FFN(bf16(RMSNorm(x)))), RMSNorm with unit weight and eps.
 * x_out may not alias x.  Same workspace rules as moe_ffn_forward. */
MOEQ_API moe_status moe_block_forward(const moe_layer* layer, const uint16_t* x, const int32_t* adapter_id, int32_t T,
                             float eps, uint16_t* x_out, void* workspace, size_t ws_bytes, moe_stream stream);

/* xn = bf16(x / sqrt(mean(x^2) + eps)) per row; x, xn device bf16 [T][H]. */
MOEQ_API moe_status moe_rmsnorm(const uint16_t* x, int32_t T, int32_t H, float eps, uint16_t* xn, moe_stream stream);

/* Read the sticky device status word of a workspace into *status (host) and
 * clear it.  Synchronises `stream`. */
MOEQ_API moe_status moe_get_device_status(void* workspace, moe_stream stream, int32_t* status);

/* The routing a forward used: copies the expert indices [T][K] (int32) and the
 * renormalised weights [T][K] (fp32) that the last moe_ffn_forward or
 * moe_block_forward with this layer shape, T and workspace selected (whichever
 * kernels ran it) into topk_idx / topk_w (device pointers; either may be NULL).
 * Enqueued on `stream` after that call; the workspace must not have been used
 * by another call in between.  Routing indices stay on the device ("Edge0 项目推荐"
 * review, 亮点二); this is the record a caller or a test reads them from. */
MOEQ_API moe_status moe_ffn_routing(const moe_layer* layer, int32_t T, const void* workspace, size_t ws_bytes,
                                    int32_t* topk_idx, float* topk_w, moe_stream stream);

/* Which single-kernel decode a forward of 1..8 tokens tries first.  AUTO: the cluster
 * kernel for one token (thread-block clusters; router, top-K and LoRA-A products per
 * cluster through distributed shared memory, one grid-wide exchange of h), else the
 * barrier kernel (two grid-wide barriers, every CTA takes the top-K itself) for top-4 or
 * less without a given expert set, else the chain kernel (no grid barrier; CTA 0 routes
 * and publishes, every hand-off an epoch-tagged word or an arrival count); CHAIN,
 * BARRIER or CLUSTER: that kernel whenever it takes the call.  A call no single kernel
 * takes runs on the multi-kernel paths.  Process-wide, read when a call enqueues its
 * kernels, not thread-safe. */
#define MOE_DECODE_AUTO 0
#define MOE_DECODE_CHAIN 1
#define MOE_DECODE_BARRIER 2
#define MOE_DECODE_CLUSTER 3
MOEQ_API moe_status moe_set_decode_path(int path);
MOEQ_API int moe_decode_path(void);

/* Bound of every device-side wait (a grid-wide arrival, a ready flag, a bulk-copy
 * or pipeline barrier), in nanoseconds of device time; 0 restores the default of
 * one second.  A wait that runs out sets MOE_ERR_TIMEOUT in the status word and the
 * kernel returns (its output is then incomplete).  The value is read when a call
 * enqueues its kernels, so a captured CUDA graph keeps the value of its capture.
 * Process-wide, not thread-safe. */
MOEQ_API moe_status moe_set_wait_limit_ns(uint64_t ns);
MOEQ_API uint64_t moe_wait_limit_ns(void);

/* --------------------------------------------------------- a7 mixed layout
 * y[t][o] = s_o * sum_j q_oj x[t][j] (weight-only form of the EdgeRazor
 * decomposition, "EDGERAZOR 深度解读" section 2.1 矩阵乘法分解).
 *  x device bf16 [T][in]; y device fp32 [T][out]. */
MOEQ_API moe_status moe_mixed_linear(const moe_mixed_tensor* W, const uint16_t* x, int32_t T, float* y,
                            moe_stream stream);

/* SwiGLU MLP on mixed-layout weights, gate/up [I][H], down [H][I]:
 *   residual = 0: y = bf16(down(SiLU(gate x) * up x))
 *   residual = 1: y = bf16(x + MLP(bf16(RMSNorm(x))))
 * x, y device bf16 [T][H] (may not alias); workspace of
 * moe_mixed_mlp_workspace_bytes(H, I, T) bytes, 256-byte aligned. */
MOEQ_API size_t moe_mixed_mlp_workspace_bytes(int32_t H, int32_t I, int32_t T);
MOEQ_API moe_status moe_mixed_mlp_forward(const moe_mixed_tensor* gate, const moe_mixed_tensor* up,
                                 const moe_mixed_tensor* down, const uint16_t* x, int32_t T, int32_t residual,
                                 float eps, uint16_t* y, void* workspace, size_t ws_bytes, moe_stream stream);

/* ------------------------------------------------------ expert parallelism
 * Building blocks of the expert-parallel forward over G ranks (one process per GPU),
 * each owning E/G consecutive experts, with the router and the shared expert
 * replicated: route locally (moe_router_topk), moe_ep_dispatch, an all-to-all of the
 * rows (NCCL, by the caller), moe_experts_forward on the rows received, the reverse
 * all-to-all, the shared expert on the local tokens, moe_ep_combine.  The sum over a
 * token's experts is the forward's own sum (fixed order k = 0..K-1, then the shared
 * expert); the expert outputs cross the all-to-all as bf16.
 *
 * moe_experts_forward: y[n] = E_{expert[n]}(x[n]) for N rows (no router, no shared
 * expert, weight 1), adapter_id [N] or NULL as for moe_ffn_forward; an expert index
 * outside [0, E) makes its row zero and raises MOE_ERR_DEVICE_INDEX.  x, y device bf16
 * [N][H]; workspace of moe_experts_workspace_bytes(layer, N) bytes, 256-byte aligned,
 * initialised once.  A layer whose expert tensors are views of E/G experts (n = E/G)
 * is a rank's slice.
 *
 * moe_ep_dispatch: the routed jobs j = t*K + k of T local tokens (topk_idx device int32
 * [T][K], experts of a layer with E experts) in send order: rank-major (owner =
 * expert / (E/G)), job order within a rank.  Writes pos [T][K] (the send row of each
 * job), counts [G] (rows per rank), send_x [T*K][H] bf16 (x[t] of each job) and
 * send_meta [T*K][2] = {expert, adapter id}.  All device pointers; E % G == 0,
 * G <= 64, H % 8 == 0.  An expert index out of range is clamped and raises
 * MOE_ERR_DEVICE_INDEX in *status (a device int32 word).
 *
 * moe_ep_combine: y[t] = bf16(sum_k topk_w[t][k] ret[pos[t][k]] + shared_scale[t]
 * shared[t]) (shared NULL: no shared term; shared_scale NULL: scale 1); ret device
 * bf16 [T*K][H] in send order. */
#define MOEQ_EP_MAX_RANKS 64
MOEQ_API size_t moe_experts_workspace_bytes(const moe_layer* layer, int32_t N);
MOEQ_API moe_status moe_experts_forward(const moe_layer* layer, const uint16_t* x, const int32_t* expert,
                                        const int32_t* adapter_id, int32_t N, uint16_t* y, void* workspace,
                                        size_t ws_bytes, moe_stream stream);
MOEQ_API moe_status moe_ep_dispatch(const uint16_t* x, const int32_t* topk_idx, const int32_t* adapter_id,
                                    int32_t n_adapters, int32_t T, int32_t K, int32_t H, int32_t E, int32_t G,
                                    int32_t* pos, int32_t* counts, uint16_t* send_x, int32_t* send_meta,
                                    int32_t* status, moe_stream stream);
MOEQ_API moe_status moe_ep_combine(const uint16_t* ret, const int32_t* pos, const float* topk_w,
                                   const uint16_t* shared, const float* shared_scale, int32_t T, int32_t K,
                                   int32_t H, uint16_t* y, moe_stream stream);

/* ------------------------------------- a7 in weight-activation form (8-bit A)
 * The mixed layer with 8-bit activations ("EDGERAZOR 深度解读" section 2.1 矩阵乘法
 * 分解, Y = sum (s_W s_X) Q(W)^T Q(X), and the 1.88-8-8 / 1.58-8-8 rows of the
 * weight-activation table in section 3.1).  Each token's activation row is
 * quantised with the page's symmetric rule at n = 8 (reading: one scale per token):
 * s_X = max(max|x| / 127, 1e-5), Q(X) = clip(round(x / s_X), -127, 127), both in
 * fp32 (IEEE division, round half to even); the dot product is exact integer
 * arithmetic and Y = s_W[o] * s_X[t] * sum_j Q(W)[o][j] Q(X)[t][j].
 *  moe_act8_quant: x device bf16 [T][n] -> q device int8 [T][n], s device fp32 [T].
 *  moe_mixed_linear_a8: x device bf16 [T][in] -> y device fp32 [T][out]; workspace of
 *    moe_mixed_linear_a8_workspace_bytes(in, T) bytes, 256-byte aligned.
 *  moe_mixed_mlp_forward_a8: as moe_mixed_mlp_forward, every linear layer in this form
 *    (the intermediate h = SiLU(gate x) * up x is held in fp32 and quantised per
 *    token like x); workspace of moe_mixed_mlp_a8_workspace_bytes(H, I, T) bytes. */
MOEQ_API moe_status moe_act8_quant(const uint16_t* x, int32_t T, int32_t n, int8_t* q, float* s, moe_stream stream);
MOEQ_API size_t moe_mixed_linear_a8_workspace_bytes(int32_t in, int32_t T);
MOEQ_API moe_status moe_mixed_linear_a8(const moe_mixed_tensor* W, const uint16_t* x, int32_t T, float* y,
                                        void* workspace, size_t ws_bytes, moe_stream stream);
MOEQ_API size_t moe_mixed_mlp_a8_workspace_bytes(int32_t H, int32_t I, int32_t T);
MOEQ_API moe_status moe_mixed_mlp_forward_a8(const moe_mixed_tensor* gate, const moe_mixed_tensor* up,
                                             const moe_mixed_tensor* down, const uint16_t* x, int32_t T,
                                             int32_t residual, float eps, uint16_t* y, void* workspace,
                                             size_t ws_bytes, moe_stream stream);

/* ---------------------------------------------------------- kernel timing
 * Opt-in measurement of the library's own kernels with CUDA events (no device
 * memory is allocated; events are created on the first enable).  While
 * enabled, every entry point records an event on its stream before its first
 * launch and after each launch; the time between consecutive events is charged
 * to the kernel just launched (a memset issued by the library is charged to the
 * kernel after it).  moe_timing_collect synchronises on the recorded events,
 * adds each kind's time (ms) and launch count into the host arrays (n_kinds
 * entries, indexed by kind) and clears the record.  At most 1 << 16 launches
 * are recorded between collects; later ones are not timed.  Under stream
 * capture the records become event nodes of the graph; collect after exactly
 * one replay of that graph.  Enabling is not thread-safe. */
MOEQ_API int moe_timing_kinds(void);
MOEQ_API const char* moe_timing_kind_name(int kind);
MOEQ_API moe_status moe_timing_enable(int enable);
MOEQ_API moe_status moe_timing_collect(float* total_ms, int32_t* launches, int32_t n_kinds);

#ifdef __cplusplus
}
#endif
#endif /* MOEQ_H */
