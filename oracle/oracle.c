/*
 * oracle.c - fp64 CPU reference ("the oracle") for the int4 group-affine MoE
 * expert FFN and the EdgeRazor mixed ternary / 4-bit linear layer.
 *
 * TEST INFRASTRUCTURE ONLY: used by the tests, the smoke check and the
 * benchmark's CPU baseline; never by the product library.  Plain loops in the
 * order the method states them, fp64 throughout, one rounding to the storage
 * type where a stored value is produced.  OpenMP splits independent output
 * rows across threads; every sum is still taken in index order by one thread,
 * so results do not depend on the thread count.
 *
 * Sources (web pages, cited by title and section):
 *  [RL]  "Recover-LoRA: 4-bit 压缩掉的精度, Edge0 怎么找回来", sections 一 (4-bit
 *        group-64 affine weights with per-group scale and zero-point; 8-bit
 *        mlp.gate and shared_expert_gate) and 二 (frozen base + unmerged LoRA).
 *  [G35] Edge0-35B-A3B preview guide (trdm.cn), sections 三大核心机制 (switch_mlp
 *        gate/up/down projections with scales and biases), 模型规格与仓库构成
 *        (40 layers, 256 experts, hidden 2048, expert and shared intermediate
 *        512, shared_expert_gate) and 量化实现.
 *  [D1A] "d1a-e2b-it-qat-4bit 的 MLX 4-bit 逐比特移植原理", sections 4-bit 分组量化
 *        (bf16 scale and bias per group, packed words) and 0.0 反量化误差.
 *  [REV] "Edge0 项目推荐" review, 亮点三 (unmerged parallel LoRA delta), the
 *        framework paragraph (MoESpec SOFTMAX_TOPK routing) and 优点 (the
 *        _swiglu(up, gate) argument order).
 *  [ER]  "EDGERAZOR 深度解读", section 2.1 SQMP (super-group allocation, ternary
 *        and 4-bit quantisers, the matmul decomposition).
 *  [PR]  "Edge0 项目推荐" review, 亮点一 (the prerouter head: features, fc1, exact
 *        erf GELU, fc2, the linear_init skip, fp16 weights, the double shift).
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_MAX_RANK 64

static int g_mutation = 0;

void orc_set_mutation(int mutation) { g_mutation = mutation; }

int orc_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------ bf16 */

double orc_bf16_value(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* The float next to v in direction dir (-1: largest float <= v, +1: smallest >= v). */
static float f32_directed(double v, int dir) {
    float f = (float)v;
    if (dir < 0 && (double)f > v) f = nextafterf(f, -INFINITY);
    if (dir > 0 && (double)f < v) f = nextafterf(f, INFINITY);
    return f;
}

/* bf16 is float with the low 16 bits dropped, so dropping them truncates toward
 * zero; a directed rounding adds one unit in the last place when truncation went
 * the wrong way.  Rounding double->float->bf16 in the same direction is exact
 * because the bf16 grid is a subset of the float grid. */
static uint16_t bf16_directed(double v, int dir) {
    float f = f32_directed(v, dir);
    uint32_t u;
    memcpy(&u, &f, 4);
    uint16_t t = (uint16_t)(u >> 16);
    if ((u & 0xFFFFu) == 0) return t;
    int neg = (int)(u >> 31);
    if (dir < 0) return neg ? (uint16_t)(t + 1) : t;
    return neg ? t : (uint16_t)(t + 1);
}

uint16_t orc_bf16_round_down(double v) { return bf16_directed(v, -1); }
uint16_t orc_bf16_round_up(double v) { return bf16_directed(v, +1); }

/* Nearest bf16, ties to the even bit pattern. */
uint16_t orc_bf16_round_nearest(double v) {
    uint16_t lo = bf16_directed(v, -1), hi = bf16_directed(v, +1);
    if (lo == hi) return lo;
    double dl = v - orc_bf16_value(lo), dh = orc_bf16_value(hi) - v;
    if (dl < dh) return lo;
    if (dh < dl) return hi;
    return (lo & 1u) ? hi : lo;
}

/* ------------------------------------------------ affine group quantiser */

/*
 * [RL §一], [G35 量化实现], [D1A 4-bit 分组量化]: every `group` consecutive
 * elements along the input dimension share one bf16 scale s and one bf16 bias
 * b, and w is stored as an unsigned integer q with w ~ s*q + b.  The pages give
 * no rule for choosing s and b; this reading takes the group minimum rounded
 * down as b and the range over 2^bits - 1 rounded up as s, so that every q
 * lands in range and |w - (s*q + b)| <= s/2.
 */
int orc_quant_affine(const float* W, int64_t rows, int in, int bits, int group, uint32_t* packed,
                     uint16_t* scales, uint16_t* biases) {
    if (bits != 4 && bits != 8) return -1;
    const int per_word = 32 / bits;
    if (group <= 0 || in <= 0 || in % group != 0 || group % per_word != 0) return -1;
    const int qmax = (1 << bits) - 1;
    const int words = in / per_word, ngroups = in / group;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const float* w = W + r * in;
        uint32_t* pw = packed + r * words;
        memset(pw, 0, (size_t)words * 4);
        for (int g = 0; g < ngroups; ++g) {
            const float* wg = w + (int64_t)g * group;
            double lo = wg[0], hi = wg[0];
            for (int j = 1; j < group; ++j) {
                if (wg[j] < lo) lo = wg[j];
                if (wg[j] > hi) hi = wg[j];
            }
            if (lo == 0.0) lo = 0.0; /* a minimum of -0 and +0 stores the bias +0 */
            uint16_t b16 = orc_bf16_round_down(lo);
            double b = orc_bf16_value(b16);
            double d = hi - b;
            uint16_t s16 = 0;
            double s = 0.0;
            if (d > 0.0) {
                s16 = orc_bf16_round_up(d / (double)qmax);
                s = orc_bf16_value(s16);
            }
            scales[r * ngroups + g] = s16;
            biases[r * ngroups + g] = b16;
            for (int j = 0; j < group; ++j) {
                int q = 0;
                if (s > 0.0) {
                    double t = rint(((double)wg[j] - b) / s);
                    if (t < 0.0) t = 0.0;
                    if (t > (double)qmax) t = (double)qmax;
                    q = (int)t;
                }
                int col = g * group + j;
                pw[col / per_word] |= (uint32_t)q << ((col % per_word) * bits);
            }
        }
    }
    return 0;
}

void orc_unpack_codes(const uint32_t* packed, int64_t rows, int in, int bits, int32_t* q) {
    const int per_word = 32 / bits;
    const uint32_t mask = (1u << bits) - 1u;
    const int words = in / per_word;
    for (int64_t r = 0; r < rows; ++r)
        for (int j = 0; j < in; ++j)
            q[r * in + j] = (int32_t)((packed[r * words + j / per_word] >> ((j % per_word) * bits)) & mask);
}

/* Dequantised weight as stored: s*q + b is exact in fp64, then rounded once to fp32. */
static inline double affine_weight(double s, double b, uint32_t q) {
    return (double)(float)(s * (double)q + b);
}

void orc_dequant_affine(const uint32_t* packed, const uint16_t* scales, const uint16_t* biases,
                        int64_t rows, int in, int bits, int group, float* w_hat) {
    const int per_word = 32 / bits;
    const uint32_t mask = (1u << bits) - 1u;
    const int words = in / per_word, ngroups = in / group;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int j = 0; j < in; ++j) {
            double s = orc_bf16_value(scales[r * ngroups + j / group]);
            double b = orc_bf16_value(biases[r * ngroups + j / group]);
            uint32_t q = (packed[r * words + j / per_word] >> ((j % per_word) * bits)) & mask;
            w_hat[r * in + j] = (float)affine_weight(s, b, q);
        }
}

/* sum_j w_hat[row][j] * x[j], index order, fp64. */
static double qmat_row_dot(const orc_qmat* m, int64_t mat, int row, const double* x) {
    const int per_word = 32 / m->bits;
    const uint32_t mask = (1u << m->bits) - 1u;
    const int words = m->in / per_word, ngroups = m->in / m->group;
    const int64_t r = mat * m->out + row;
    const uint32_t* pw = m->packed + r * words;
    const uint16_t* sc = m->scales + r * ngroups;
    const uint16_t* bi = m->biases + r * ngroups;
    double acc = 0.0;
    for (int j = 0; j < m->in; ++j) {
        int g = j / m->group;
        uint32_t q = (pw[j / per_word] >> ((j % per_word) * m->bits)) & mask;
        acc += affine_weight(orc_bf16_value(sc[g]), orc_bf16_value(bi[g]), q) * x[j];
    }
    return acc;
}

/* ------------------------------------------- EdgeRazor mixed super-groups */

/* [ER §2.1 超组分配]: every floor(1/rho) consecutive output channels form a
 * super-group holding exactly one 4-bit channel; rho = 0 means all ternary. */
int orc_mixed_group(double rho) {
    if (rho <= 0.0) return 0;
    return (int)floor(1.0 / rho + 1e-9);
}

int64_t orc_mixed_row_offset(int row, int in, int G) {
    const int64_t w4 = in / 8, w2 = in / 16;
    if (G == 0) return (int64_t)row * w2;
    const int64_t sg = row / G, pos = row % G;
    const int64_t base = sg * (w4 + (int64_t)(G - 1) * w2);
    return pos == 0 ? base : base + w4 + (pos - 1) * w2;
}

int64_t orc_mixed_words(int out, int in, double rho) {
    const int G = orc_mixed_group(rho);
    const int64_t w4 = in / 8, w2 = in / 16;
    if (G == 0) return (int64_t)out * w2;
    const int64_t full = out / G, rem = out % G;
    return full * (w4 + (int64_t)(G - 1) * w2) + (rem ? w4 + (rem - 1) * w2 : 0);
}

static inline int mixed_is4(int row, int G) { return G > 0 && row % G == 0; }

/*
 * [ER §2.1 量化公式]: the 4-bit channel uses s = max(max|w| / (2^{n-1} - 1), eps)
 * with n = 4 and q = round(w / s); the ternary channels use
 * s = max(beta * mean|w|, eps) with beta = 2 and q = clip(round(w / s), -1, 1).
 * Reading: one scale per output channel, stored as the nearest bf16; q of the
 * 4-bit channel clipped to [-7, 7]; eps = 1e-5.
 */
int orc_quant_mixed(const float* W, int out, int in, double rho, uint32_t* packed, uint16_t* scales) {
    if (rho < 0.0 || rho > 1.0 || in <= 0 || in % 16 != 0 || out <= 0) return -1;
    const int G = orc_mixed_group(rho);
    const double eps = 1e-5;
    memset(packed, 0, (size_t)orc_mixed_words(out, in, rho) * 4);
    #pragma omp parallel for schedule(static)
    for (int o = 0; o < out; ++o) {
        const float* w = W + (int64_t)o * in;
        uint32_t* pw = packed + orc_mixed_row_offset(o, in, G);
        double s;
        if (mixed_is4(o, G)) {
            double m = 0.0;
            for (int j = 0; j < in; ++j) m = fmax(m, fabs((double)w[j]));
            uint16_t s16 = orc_bf16_round_nearest(fmax(m / 7.0, eps));
            scales[o] = s16;
            s = orc_bf16_value(s16);
            for (int j = 0; j < in; ++j) {
                double t = rint((double)w[j] / s);
                if (t < -7.0) t = -7.0;
                if (t > 7.0) t = 7.0;
                pw[j / 8] |= (uint32_t)((int)t + 8) << ((j % 8) * 4);
            }
        } else {
            double sum = 0.0;
            for (int j = 0; j < in; ++j) sum += fabs((double)w[j]);
            uint16_t s16 = orc_bf16_round_nearest(fmax(2.0 * (sum / (double)in), eps));
            scales[o] = s16;
            s = orc_bf16_value(s16);
            for (int j = 0; j < in; ++j) {
                double t = rint((double)w[j] / s);
                if (t < -1.0) t = -1.0;
                if (t > 1.0) t = 1.0;
                pw[j / 16] |= (uint32_t)((int)t + 1) << ((j % 16) * 2);
            }
        }
    }
    return 0;
}

void orc_mixed_codes(const uint32_t* packed, int out, int in, double rho, int32_t* q) {
    const int G = orc_mixed_group(rho);
    for (int o = 0; o < out; ++o) {
        const uint32_t* pw = packed + orc_mixed_row_offset(o, in, G);
        for (int j = 0; j < in; ++j) {
            if (mixed_is4(o, G))
                q[(int64_t)o * in + j] = (int32_t)((pw[j / 8] >> ((j % 8) * 4)) & 15u) - 8;
            else
                q[(int64_t)o * in + j] = (int32_t)((pw[j / 16] >> ((j % 16) * 2)) & 3u) - 1;
        }
    }
}

void orc_dequant_mixed(const uint32_t* packed, const uint16_t* scales, int out, int in, double rho,
                       float* w_hat) {
    int32_t* q = (int32_t*)malloc((size_t)out * in * sizeof(int32_t));
    orc_mixed_codes(packed, out, in, rho, q);
    for (int o = 0; o < out; ++o) {
        double s = orc_bf16_value(scales[o]);
        for (int j = 0; j < in; ++j) w_hat[(int64_t)o * in + j] = (float)(s * (double)q[(int64_t)o * in + j]);
    }
    free(q);
}

/* [ER §2.1 矩阵乘法分解]: with weight-only quantisation (activation scale 1)
 * the product is the 16-bit channel scale times an integer-code dot product:
 * y_o = s_o * sum_j q_oj x_j. */
static void mixed_linear_f64(const uint32_t* packed, const uint16_t* scales, int out, int in, int G,
                             const double* x, double* y) {
    #pragma omp parallel for schedule(static)
    for (int o = 0; o < out; ++o) {
        const uint32_t* pw = packed + orc_mixed_row_offset(o, in, G);
        double acc = 0.0;
        for (int j = 0; j < in; ++j) {
            int q = mixed_is4(o, G) ? (int)((pw[j / 8] >> ((j % 8) * 4)) & 15u) - 8
                                    : (int)((pw[j / 16] >> ((j % 16) * 2)) & 3u) - 1;
            acc += (double)q * x[j];
        }
        y[o] = orc_bf16_value(scales[o]) * acc;
    }
}

void orc_mixed_linear(const uint32_t* packed, const uint16_t* scales, int out, int in, double rho,
                      const uint16_t* x, int T, double* y) {
    const int G = orc_mixed_group(rho);
    double* xd = (double*)malloc((size_t)in * sizeof(double));
    for (int t = 0; t < T; ++t) {
        for (int j = 0; j < in; ++j) xd[j] = orc_bf16_value(x[(int64_t)t * in + j]);
        mixed_linear_f64(packed, scales, out, in, G, xd, y + (int64_t)t * out);
    }
    free(xd);
}

static double silu(double v) { return v / (1.0 + exp(-v)); }

/* SwiGLU MLP on mixed-layout weights: y = down(SiLU(gate x) * up x). */
int orc_mixed_mlp(const uint32_t* gp, const uint16_t* gs, const uint32_t* up, const uint16_t* us,
                  const uint32_t* dp, const uint16_t* ds, int H, int I, double rho, const uint16_t* x,
                  int T, double* y) {
    if (H % 16 || I % 16) return -1;
    const int G = orc_mixed_group(rho);
    double* xd = (double*)malloc((size_t)H * sizeof(double));
    double* g = (double*)malloc((size_t)I * sizeof(double));
    double* u = (double*)malloc((size_t)I * sizeof(double));
    for (int t = 0; t < T; ++t) {
        for (int j = 0; j < H; ++j) xd[j] = orc_bf16_value(x[(int64_t)t * H + j]);
        mixed_linear_f64(gp, gs, I, H, G, xd, g);
        mixed_linear_f64(up, us, I, H, G, xd, u);
        for (int i = 0; i < I; ++i) g[i] = (g_mutation == 1) ? silu(u[i]) * g[i] : silu(g[i]) * u[i];
        mixed_linear_f64(dp, ds, H, I, G, g, y + (int64_t)t * H);
    }
    free(xd);
    free(g);
    free(u);
    return 0;
}

/* ------------------------------------------------------------ RMSNorm */

/* Pre-norm between stacked layers (reading: unit weight), materialised in bf16. */
void orc_rmsnorm_bf16(const uint16_t* x, int T, int H, double eps, uint16_t* xn) {
    for (int t = 0; t < T; ++t) {
        const uint16_t* xr = x + (int64_t)t * H;
        double ss = 0.0;
        for (int j = 0; j < H; ++j) {
            double v = orc_bf16_value(xr[j]);
            ss += v * v;
        }
        double inv = 1.0 / sqrt(ss / (double)H + eps);
        for (int j = 0; j < H; ++j) xn[(int64_t)t * H + j] = orc_bf16_round_nearest(orc_bf16_value(xr[j]) * inv);
    }
}

int orc_mixed_block(const uint32_t* gp, const uint16_t* gs, const uint32_t* up, const uint16_t* us,
                    const uint32_t* dp, const uint16_t* ds, int H, int I, double rho, double eps,
                    const uint16_t* x, int T, uint16_t* x_out) {
    uint16_t* xn = (uint16_t*)malloc((size_t)T * H * 2);
    double* y = (double*)malloc((size_t)T * H * sizeof(double));
    orc_rmsnorm_bf16(x, T, H, eps, xn);
    int rc = orc_mixed_mlp(gp, gs, up, us, dp, ds, H, I, rho, xn, T, y);
    if (rc == 0)
        for (int64_t i = 0; i < (int64_t)T * H; ++i) x_out[i] = orc_bf16_round_nearest(orc_bf16_value(x[i]) + y[i]);
    free(xn);
    free(y);
    return rc;
}

/* ------------------------------------------------------------- router */

/* [RL §一], [G35 量化实现]: the router (mlp.gate) and the shared-expert gate are
 * 8-bit group-affine linear maps of the MoE input. */
void orc_router(const orc_layer* L, const uint16_t* x, int T, double* logits, double* gs) {
    double* xd = (double*)malloc((size_t)L->H * sizeof(double));
    for (int t = 0; t < T; ++t) {
        for (int j = 0; j < L->H; ++j) xd[j] = orc_bf16_value(x[(int64_t)t * L->H + j]);
        #pragma omp parallel for schedule(static)
        for (int e = 0; e < L->E; ++e)
            logits[(int64_t)t * L->E + e] =
                qmat_row_dot(&L->router, 0, e, xd) + (L->logit_bias ? (double)L->logit_bias[e] : 0.0);
        if (gs) gs[t] = L->shared_gate.packed ? qmat_row_dot(&L->shared_gate, 0, 0, xd) : 0.0;
    }
    free(xd);
}

static void softmax_row(const double* z, int E, double* p) {
    double m = z[0];
    for (int e = 1; e < E; ++e) m = fmax(m, z[e]);
    double s = 0.0;
    for (int e = 0; e < E; ++e) {
        p[e] = exp(z[e] - m);
        s += p[e];
    }
    for (int e = 0; e < E; ++e) p[e] /= s;
}

/* SOFTMAX_TOPK routing ([REV] framework paragraph): p = softmax(z); the K
 * largest in descending order, equal logits going to the lower expert index;
 * weights renormalised over the chosen K. */
void orc_topk(const double* logits, int T, int E, int K, int32_t* idx, double* w) {
    double* p = (double*)malloc((size_t)E * sizeof(double));
    char* taken = (char*)malloc((size_t)E);
    for (int t = 0; t < T; ++t) {
        const double* z = logits + (int64_t)t * E;
        softmax_row(z, E, p);
        memset(taken, 0, (size_t)E);
        double psum = 0.0;
        for (int k = 0; k < K; ++k) {
            int best = -1;
            for (int e = 0; e < E; ++e)
                if (!taken[e] && (best < 0 || z[e] > z[best])) best = e;
            taken[best] = 1;
            idx[(int64_t)t * K + k] = best;
            psum += p[best];
        }
        for (int k = 0; k < K; ++k) w[(int64_t)t * K + k] = p[idx[(int64_t)t * K + k]] / psum;
    }
    free(p);
    free(taken);
}

/* ------------------------------------------------------- index build */

typedef struct { int32_t expert, arank, token, k, adapter; } orc_job;

static int job_cmp(const void* a, const void* b) {
    const orc_job* x = (const orc_job*)a;
    const orc_job* y = (const orc_job*)b;
    if (x->expert != y->expert) return x->expert < y->expert ? -1 : 1;
    if (x->arank != y->arank) return x->arank < y->arank ? -1 : 1;
    if (x->token != y->token) return x->token < y->token ? -1 : 1;
    return (x->k > y->k) - (x->k < y->k);
}

static int token_adapter(const int32_t* adapter_id, int t, int n_adapters) {
    if (adapter_id) return adapter_id[t];
    return n_adapters > 0 ? 0 : -1;
}

/*
 * Expert-grouped job list.  Every token contributes K routed jobs and one
 * shared-expert job (expert index E).  Jobs are ordered by (expert, adapter,
 * token, k), "no adapter" (-1) sorting after the real adapters.  counts[e] is
 * the number of jobs of expert e, offsets the exclusive prefix sum (E + 2
 * entries), and perm[p] = {token, k, adapter, expert} (k = K for the shared job).
 */
int orc_index_build(const int32_t* idx, const int32_t* adapter_id, int T, int K, int E, int n_adapters,
                    int32_t* counts, int32_t* offsets, int32_t* perm) {
    const int64_t n = (int64_t)T * (K + 1);
    orc_job* jobs = (orc_job*)malloc((size_t)(n ? n : 1) * sizeof(orc_job));
    for (int t = 0; t < T; ++t) {
        int a = token_adapter(adapter_id, t, n_adapters);
        if (a >= n_adapters || a < -1) {
            free(jobs);
            return -2;
        }
        int arank = a < 0 ? n_adapters : a;
        for (int k = 0; k <= K; ++k) {
            int e = (k < K) ? idx[(int64_t)t * K + k] : E;
            if (e < 0 || e > E || (k < K && e == E)) {
                free(jobs);
                return -2;
            }
            orc_job j = {e, arank, t, k, a};
            jobs[(int64_t)t * (K + 1) + k] = j;
        }
    }
    qsort(jobs, (size_t)n, sizeof(orc_job), job_cmp);
    for (int e = 0; e <= E; ++e) counts[e] = 0;
    for (int64_t p = 0; p < n; ++p) counts[jobs[p].expert]++;
    offsets[0] = 0;
    for (int e = 0; e <= E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    for (int64_t p = 0; p < n; ++p) {
        perm[4 * p + 0] = jobs[p].token;
        perm[4 * p + 1] = jobs[p].k;
        perm[4 * p + 2] = jobs[p].adapter;
        perm[4 * p + 3] = jobs[p].expert;
    }
    free(jobs);
    return 0;
}

/* ------------------------------------------------------------- experts */

static const orc_lora_proj* pick_lora(const orc_layer* L, int a, int shared, int proj) {
    if (a < 0 || a >= L->n_adapters || L->rank <= 0) return NULL;
    const orc_adapter* ad = &L->adapters[a];
    const orc_lora_proj* p;
    if (proj == 0) p = shared ? &ad->s_gate : &ad->gate;
    else if (proj == 1) p = shared ? &ad->s_up : &ad->up;
    else p = shared ? &ad->s_down : &ad->down;
    return (p->A && p->B) ? p : NULL;
}

/* t_k = sum_j A[mat][k][j] v[j] */
static void lora_down_proj(const orc_lora_proj* lp, int64_t mat, int rank, int in, const double* v, double* t) {
    for (int k = 0; k < rank; ++k) {
        const uint16_t* a = lp->A + (mat * rank + k) * (int64_t)in;
        double acc = 0.0;
        for (int j = 0; j < in; ++j) acc += orc_bf16_value(a[j]) * v[j];
        t[k] = acc;
    }
}

/* (alpha / r) * sum_k B[mat][row][k] t_k */
static double lora_up_row(const orc_lora_proj* lp, int64_t mat, int rank, int out, int row, const double* t,
                          double scale) {
    const uint16_t* b = lp->B + (mat * out + row) * (int64_t)rank;
    double acc = 0.0;
    for (int k = 0; k < rank; ++k) acc += orc_bf16_value(b[k]) * t[k];
    return scale * acc;
}

/*
 * One SwiGLU expert with the unmerged LoRA delta on every projection
 * ([RL §二], [REV 亮点三]): g = W_g x + (alpha/r) B_g A_g x,
 * u = W_u x + (alpha/r) B_u A_u x, h = SiLU(g) * u (SiLU on the gate branch,
 * [REV 优点]), y = W_d h + (alpha/r) B_d A_d h.
 */
static void expert_forward(const orc_layer* L, int shared, int e, int a, const double* x, double* y) {
    const orc_qmat* Wg = shared ? &L->s_gate : &L->gate;
    const orc_qmat* Wu = shared ? &L->s_up : &L->up;
    const orc_qmat* Wd = shared ? &L->s_down : &L->down;
    const int I = shared ? L->Is : L->I;
    const int H = L->H;
    const int64_t mat = shared ? 0 : e;
    const orc_lora_proj* lg = pick_lora(L, a, shared, 0);
    const orc_lora_proj* lu = pick_lora(L, a, shared, 1);
    const orc_lora_proj* ld = pick_lora(L, a, shared, 2);
    const double scale = L->rank > 0 ? L->alpha / (double)L->rank : 0.0;
    double tg[ORC_MAX_RANK], tu[ORC_MAX_RANK], td[ORC_MAX_RANK];
    double* h = (double*)malloc((size_t)I * sizeof(double));
    if (lg) lora_down_proj(lg, mat, L->rank, H, x, tg);
    if (lu) lora_down_proj(lu, mat, L->rank, H, x, tu);
    #pragma omp parallel for schedule(static)
    for (int i = 0; i < I; ++i) {
        double g = qmat_row_dot(Wg, mat, i, x) + (lg ? lora_up_row(lg, mat, L->rank, I, i, tg, scale) : 0.0);
        double u = qmat_row_dot(Wu, mat, i, x) + (lu ? lora_up_row(lu, mat, L->rank, I, i, tu, scale) : 0.0);
        h[i] = (g_mutation == 1) ? silu(u) * g : silu(g) * u;
    }
    if (ld) lora_down_proj(ld, mat, L->rank, I, h, td);
    #pragma omp parallel for schedule(static)
    for (int o = 0; o < H; ++o)
        y[o] = qmat_row_dot(Wd, mat, o, h) + (ld ? lora_up_row(ld, mat, L->rank, H, o, td, scale) : 0.0);
    free(h);
}

static int layer_valid(const orc_layer* L) {
    if (L->H <= 0 || L->E <= 0 || L->K <= 0 || L->K > L->E || L->I <= 0) return 0;
    if (L->n_adapters < 0 || L->n_adapters > ORC_MAX_ADAPTERS) return 0;
    if (L->n_adapters > 0 && (L->rank <= 0 || L->rank > ORC_MAX_RANK)) return 0;
    return 1;
}

/*
 * The MoE FFN of one layer for T tokens:
 *   y = sum_k w_k E_{idx_k}(x) + sigma(g_s) * S(x),
 * with (idx, w) from SOFTMAX_TOPK routing of the 8-bit router logits, g_s the
 * 8-bit shared_expert_gate logit and S the shared expert ([G35 模型规格与仓库构成]).
 * `select` (nullable, [T][K]) replaces the top-K choice by a caller-supplied
 * expert set, with w renormalised over that set; tests use it to evaluate the
 * alternatives of a near-tied routing decision.
 */
int orc_moe_ffn(const orc_layer* L, const uint16_t* x, const int32_t* adapter_id, int T, const int32_t* select,
                double* y, int32_t* idx_out, double* w_out, double* sg_out, double* logits_out) {
    if (!layer_valid(L)) return -1;
    const int H = L->H, E = L->E, K = L->K;
    double* z = (double*)malloc((size_t)E * sizeof(double));
    double* p = (double*)malloc((size_t)E * sizeof(double));
    double* ye = (double*)malloc((size_t)H * sizeof(double));
    double* xd = (double*)malloc((size_t)H * sizeof(double));
    int32_t idx[64];
    double w[64];
    int rc = 0;
    if (K > 64) rc = -1;
    for (int t = 0; t < T && rc == 0; ++t) {
        double gs;
        orc_router(L, x + (int64_t)t * H, 1, z, &gs);
        if (select) {
            softmax_row(z, E, p);
            double psum = 0.0;
            for (int k = 0; k < K; ++k) {
                idx[k] = select[(int64_t)t * K + k];
                if (idx[k] < 0 || idx[k] >= E) rc = -2;
                else psum += p[idx[k]];
            }
            for (int k = 0; k < K && rc == 0; ++k) w[k] = p[idx[k]] / psum;
        } else {
            orc_topk(z, 1, E, K, idx, w);
        }
        if (rc) break;
        int a = token_adapter(adapter_id, t, L->n_adapters);
        if (a >= L->n_adapters || a < -1) {
            rc = -2;
            break;
        }
        double sg = L->shared_gate.packed ? 1.0 / (1.0 + exp(-gs)) : 1.0;
        for (int j = 0; j < H; ++j) xd[j] = orc_bf16_value(x[(int64_t)t * H + j]);
        double* yt = y + (int64_t)t * H;
        for (int j = 0; j < H; ++j) yt[j] = 0.0;
        for (int k = 0; k < K; ++k) {
            expert_forward(L, 0, idx[k], a, xd, ye);
            for (int j = 0; j < H; ++j) yt[j] += w[k] * ye[j];
        }
        if (L->s_gate.packed) {
            expert_forward(L, 1, 0, a, xd, ye);
            for (int j = 0; j < H; ++j) yt[j] += sg * ye[j];
        }
        for (int k = 0; k < K; ++k) {
            if (idx_out) idx_out[(int64_t)t * K + k] = idx[k];
            if (w_out) w_out[(int64_t)t * K + k] = w[k];
        }
        if (sg_out) sg_out[t] = sg;
        if (logits_out)
            for (int e = 0; e < E; ++e) logits_out[(int64_t)t * E + e] = z[e];
    }
    free(z);
    free(p);
    free(ye);
    free(xd);
    return rc;
}

/* Pre-norm residual block used between stacked layers (reading):
 * x_out = bf16(x + FFN(bf16(RMSNorm(x)))). */
int orc_moe_block(const orc_layer* L, const uint16_t* x, const int32_t* adapter_id, int T, double eps,
                  uint16_t* x_out) {
    const int H = L->H;
    uint16_t* xn = (uint16_t*)malloc((size_t)T * H * 2 + 2);
    double* y = (double*)malloc((size_t)T * H * sizeof(double) + 8);
    orc_rmsnorm_bf16(x, T, H, eps, xn);
    int rc = orc_moe_ffn(L, xn, adapter_id, T, NULL, y, NULL, NULL, NULL, NULL);
    if (rc == 0)
        for (int64_t i = 0; i < (int64_t)T * H; ++i) x_out[i] = orc_bf16_round_nearest(orc_bf16_value(x[i]) + y[i]);
    free(xn);
    free(y);
    return rc;
}

/* ------------------------------------------------------- prerouter head */

/* IEEE 754 binary16 bit pattern -> value: sign, 5-bit exponent (bias 15), 10-bit
 * fraction; exponent 0 is subnormal (fraction * 2^-24), exponent 31 is inf/NaN. */
double orc_fp16_value(uint16_t h) {
    const int sign = (h >> 15) & 1, ex = (h >> 10) & 31, fr = h & 1023;
    double v;
    if (ex == 0) v = ldexp((double)fr, -24);
    else if (ex == 31) v = fr ? NAN : INFINITY;
    else v = ldexp(1024.0 + fr, ex - 25);
    return sign ? -v : v;
}

/* GELU in its exact form, x * Phi(x) with Phi the standard normal CDF written
 * through erf ([PR]: "精确 erf 形式的 GELU"). */
double orc_gelu_erf(double v) { return 0.5 * v * (1.0 + erf(v / sqrt(2.0))); }

/* [PR]: layer N's head takes f = [h, onehot(executed top-K of this token),
 * onehot(executed top-K of the previous token)] and predicts layer N+1's router
 * logits, logits = linear_init(f) + fc2(gelu_erf(fc1(f))).  Every weight is fp16
 * ([PR]: fp16 in training and in production); the sums here are fp64 in index
 * order.  prev_idx NULL is an all-zero previous-token one-hot.  An expert listed
 * twice in one top-K still sets a single one. */
int orc_prerouter(const orc_prerouter_head* P, const uint16_t* h, const int32_t* exec_idx, const int32_t* prev_idx,
                  int T, double* logits) {
    const int H = P->H, E = P->E, K = P->K, D = P->D, F = H + 2 * E;
    if (H <= 0 || E <= 0 || K <= 0 || K > E || D <= 0 || !P->w1 || !P->w2 || !P->wl) return -1;
    double* f = (double*)malloc((size_t)F * sizeof(double));
    double* g = (double*)malloc((size_t)D * sizeof(double));
    int rc = 0;
    for (int t = 0; t < T && rc == 0; ++t) {
        for (int j = 0; j < H; ++j) f[j] = orc_bf16_value(h[(int64_t)t * H + j]);
        for (int j = H; j < F; ++j) f[j] = 0.0;
        for (int k = 0; k < K; ++k) {
            const int e = exec_idx[(int64_t)t * K + k];
            const int q = prev_idx ? prev_idx[(int64_t)t * K + k] : 0;
            if (e < 0 || e >= E || (prev_idx && (q < 0 || q >= E))) rc = -2;
            else {
                f[H + e] = 1.0;
                if (prev_idx) f[H + E + q] = 1.0;
            }
        }
        if (rc) break;
        #pragma omp parallel for schedule(static)
        for (int d = 0; d < D; ++d) {
            double a = P->b1 ? orc_fp16_value(P->b1[d]) : 0.0;
            for (int j = 0; j < F; ++j) a += orc_fp16_value(P->w1[(int64_t)d * F + j]) * f[j];
            g[d] = orc_gelu_erf(a);
        }
        #pragma omp parallel for schedule(static)
        for (int e = 0; e < E; ++e) {
            double z = (P->bl ? orc_fp16_value(P->bl[e]) : 0.0) + (P->b2 ? orc_fp16_value(P->b2[e]) : 0.0);
            for (int j = 0; j < F; ++j) z += orc_fp16_value(P->wl[(int64_t)e * F + j]) * f[j];
            for (int d = 0; d < D; ++d) z += orc_fp16_value(P->w2[(int64_t)e * D + d]) * g[d];
            logits[(int64_t)t * E + e] = z;
        }
    }
    free(f);
    free(g);
    return rc;
}

/* ------------------------------------- weight-activation mixed layer (W + 8-bit A) */

/* [ER §2.1 量化公式] applied to activations at n = 8 (the "-8-8" rows of the page's
 * weight-activation table), reading: one symmetric scale per token row,
 * s_X = max(max|x| / (2^7 - 1), eps) and q = clip(round(x / s_X), -127, 127).  The
 * scale and the codes are decided in fp32 (IEEE division, round half to even), the
 * precision the kernel decides them in, so the codes agree bit for bit. */
void orc_quant_act8(const float* x, int T, int n, int8_t* q, float* s) {
    for (int t = 0; t < T; ++t) {
        const float* xr = x + (int64_t)t * n;
        float m = 0.0f;
        for (int j = 0; j < n; ++j) m = fmaxf(m, fabsf(xr[j]));
        volatile float st = m / 127.0f;  /* one IEEE fp32 division, no contraction */
        float sc = fmaxf(st, 1e-5f);
        s[t] = sc;
        for (int j = 0; j < n; ++j) {
            volatile float v = xr[j] / sc;
            float r = rintf(v);
            if (r > 127.0f) r = 127.0f;
            if (r < -127.0f) r = -127.0f;
            q[(int64_t)t * n + j] = (int8_t)r;
        }
    }
}

/* [ER §2.1 矩阵乘法分解]: Y = sum (s_W s_X) Q(W)^T Q(X): the integer dot product of
 * the weight codes and the 8-bit activation codes, scaled once by the channel scale
 * and the token scale. */
static void mixed_linear_a8(const uint32_t* packed, const uint16_t* scales, int out, int in, int G,
                            const int8_t* qx, double sx, double* y) {
    #pragma omp parallel for schedule(static)
    for (int o = 0; o < out; ++o) {
        const uint32_t* pw = packed + orc_mixed_row_offset(o, in, G);
        int64_t acc = 0;
        for (int j = 0; j < in; ++j) {
            int q = mixed_is4(o, G) ? (int)((pw[j / 8] >> ((j % 8) * 4)) & 15u) - 8
                                    : (int)((pw[j / 16] >> ((j % 16) * 2)) & 3u) - 1;
            acc += (int64_t)q * qx[j];
        }
        y[o] = orc_bf16_value(scales[o]) * sx * (double)acc;
    }
}

void orc_mixed_linear_a8(const uint32_t* packed, const uint16_t* scales, int out, int in, double rho,
                         const uint16_t* x, int T, double* y) {
    const int G = orc_mixed_group(rho);
    float* xf = (float*)malloc((size_t)in * sizeof(float));
    int8_t* q = (int8_t*)malloc((size_t)in);
    for (int t = 0; t < T; ++t) {
        float sx;
        for (int j = 0; j < in; ++j) xf[j] = (float)orc_bf16_value(x[(int64_t)t * in + j]);
        orc_quant_act8(xf, 1, in, q, &sx);
        mixed_linear_a8(packed, scales, out, in, G, q, (double)sx, y + (int64_t)t * out);
    }
    free(xf);
    free(q);
}

/* The SwiGLU MLP with every linear layer in weight-activation form: x and the
 * intermediate h = SiLU(gate x) * up x are each quantised to 8 bits per token (h
 * rounded to fp32 first, the width the kernel holds it in). */
int orc_mixed_mlp_a8(const uint32_t* gp, const uint16_t* gs, const uint32_t* up, const uint16_t* us,
                     const uint32_t* dp, const uint16_t* ds, int H, int I, double rho, const uint16_t* x, int T,
                     double* y) {
    if (H % 16 || I % 16) return -1;
    const int G = orc_mixed_group(rho);
    float* xf = (float*)malloc((size_t)(H > I ? H : I) * sizeof(float));
    int8_t* q = (int8_t*)malloc((size_t)(H > I ? H : I));
    double* g = (double*)malloc((size_t)I * sizeof(double));
    double* u = (double*)malloc((size_t)I * sizeof(double));
    for (int t = 0; t < T; ++t) {
        float sx;
        for (int j = 0; j < H; ++j) xf[j] = (float)orc_bf16_value(x[(int64_t)t * H + j]);
        orc_quant_act8(xf, 1, H, q, &sx);
        mixed_linear_a8(gp, gs, I, H, G, q, (double)sx, g);
        mixed_linear_a8(up, us, I, H, G, q, (double)sx, u);
        for (int i = 0; i < I; ++i) xf[i] = (float)(silu(g[i]) * u[i]);
        orc_quant_act8(xf, 1, I, q, &sx);
        mixed_linear_a8(dp, ds, H, I, G, q, (double)sx, y + (int64_t)t * H);
    }
    free(xf);
    free(q);
    free(g);
    free(u);
    return 0;
}

int orc_mixed_block_a8(const uint32_t* gp, const uint16_t* gs, const uint32_t* up, const uint16_t* us,
                       const uint32_t* dp, const uint16_t* ds, int H, int I, double rho, double eps,
                       const uint16_t* x, int T, uint16_t* x_out) {
    uint16_t* xn = (uint16_t*)malloc((size_t)T * H * 2);
    double* y = (double*)malloc((size_t)T * H * sizeof(double));
    orc_rmsnorm_bf16(x, T, H, eps, xn);
    int rc = orc_mixed_mlp_a8(gp, gs, up, us, dp, ds, H, I, rho, xn, T, y);
    if (rc == 0)
        for (int64_t i = 0; i < (int64_t)T * H; ++i) x_out[i] = orc_bf16_round_nearest(orc_bf16_value(x[i]) + y[i]);
    free(xn);
    free(y);
    return rc;
}
