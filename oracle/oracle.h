/*
 * oracle.h - fp64 CPU reference for the int4 group-affine MoE expert FFN and
 * the EdgeRazor mixed ternary / 4-bit linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this code; only the tests, the smoke check and the benchmark's CPU
 * baseline do.  It shares no source with the CUDA library: the storage
 * formats below are re-declared here on purpose (an interface both sides must
 * agree on), and every routine is written out directly from the definitions on
 * the pages it cites.
 *
 * Storage formats (the interface):
 *   affine  : packed uint32 [rows][in*bits/32], element j of a row in word j/(32/bits),
 *             bit field (j % (32/bits)) * bits, lowest field first;
 *             scales, biases: bf16 bit patterns [rows][in/group]; w = s*q + b.
 *   mixed   : per super-group of G = floor(1/rho) output rows, one 4-bit row
 *             (in/8 words, nibble = q+8, q in [-7,7]) followed by G-1 ternary
 *             rows (in/16 words, 2-bit code = q+1, q in {-1,0,1}), lowest
 *             field first; bf16 scale per row; w = s*q.
 *   LoRA    : A bf16 [n][rank][in], B bf16 [n][out][rank].
 */
#ifndef ORACLE_H
#define ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
    const uint32_t* packed;
    const uint16_t* scales;
    const uint16_t* biases;
    int32_t n, out, in, bits, group;
} orc_qmat;

typedef struct {
    const uint16_t* A; /* [n][rank][in]  (NULL: no delta on this projection) */
    const uint16_t* B; /* [n][out][rank] */
} orc_lora_proj;

typedef struct {
    orc_lora_proj gate, up, down;       /* routed experts, n = E */
    orc_lora_proj s_gate, s_up, s_down; /* shared expert,  n = 1 */
} orc_adapter;

#define ORC_MAX_ADAPTERS 16

typedef struct {
    int32_t H, E, K, I, Is;
    orc_qmat router;      /* 8-bit [E][H] */
    orc_qmat shared_gate; /* 8-bit [1][H]; packed NULL: shared output not gated */
    orc_qmat gate, up, down;       /* int4 [E][I][H], [E][I][H], [E][H][I] */
    orc_qmat s_gate, s_up, s_down; /* int4 [1][Is][H], ..., [1][H][Is]; packed NULL: no shared expert */
    const float* logit_bias;       /* [E] or NULL */
    int32_t n_adapters, rank;
    double alpha;
    orc_adapter adapters[ORC_MAX_ADAPTERS];
} orc_layer;

/* 0 = exact definition; 1 = planted mistake: SiLU applied to up instead of gate. */
void orc_set_mutation(int mutation);

int orc_quant_affine(const float* W, int64_t rows, int in, int bits, int group,
                     uint32_t* packed, uint16_t* scales, uint16_t* biases);
void orc_dequant_affine(const uint32_t* packed, const uint16_t* scales, const uint16_t* biases,
                        int64_t rows, int in, int bits, int group, float* w_hat);
void orc_unpack_codes(const uint32_t* packed, int64_t rows, int in, int bits, int32_t* q);

int orc_mixed_group(double rho);
int64_t orc_mixed_words(int out, int in, double rho);
int64_t orc_mixed_row_offset(int row, int in, int G);
int orc_quant_mixed(const float* W, int out, int in, double rho, uint32_t* packed, uint16_t* scales);
void orc_mixed_codes(const uint32_t* packed, int out, int in, double rho, int32_t* q);
void orc_dequant_mixed(const uint32_t* packed, const uint16_t* scales, int out, int in, double rho,
                       float* w_hat);
void orc_mixed_linear(const uint32_t* packed, const uint16_t* scales, int out, int in, double rho,
                      const uint16_t* x, int T, double* y);
int orc_mixed_mlp(const uint32_t* gp, const uint16_t* gs, const uint32_t* up, const uint16_t* us,
                  const uint32_t* dp, const uint16_t* ds, int H, int I, double rho,
                  const uint16_t* x, int T, double* y);
int orc_mixed_block(const uint32_t* gp, const uint16_t* gs, const uint32_t* up, const uint16_t* us,
                    const uint32_t* dp, const uint16_t* ds, int H, int I, double rho, double eps,
                    const uint16_t* x, int T, uint16_t* x_out);

/* Weight-activation form of the mixed layer ("EDGERAZOR 深度解读" section 2.1 and
 * the W/A table of section 3.1): 8-bit per-token activation codes. */
void orc_quant_act8(const float* x, int T, int n, int8_t* q, float* s);
void orc_mixed_linear_a8(const uint32_t* packed, const uint16_t* scales, int out, int in, double rho,
                         const uint16_t* x, int T, double* y);
int orc_mixed_mlp_a8(const uint32_t* gp, const uint16_t* gs, const uint32_t* up, const uint16_t* us,
                     const uint32_t* dp, const uint16_t* ds, int H, int I, double rho, const uint16_t* x, int T,
                     double* y);
int orc_mixed_block_a8(const uint32_t* gp, const uint16_t* gs, const uint32_t* up, const uint16_t* us,
                       const uint32_t* dp, const uint16_t* ds, int H, int I, double rho, double eps,
                       const uint16_t* x, int T, uint16_t* x_out);

void orc_router(const orc_layer* L, const uint16_t* x, int T, double* logits, double* gs);
void orc_topk(const double* logits, int T, int E, int K, int32_t* idx, double* w);
int orc_index_build(const int32_t* idx, const int32_t* adapter_id, int T, int K, int E,
                    int n_adapters, int32_t* counts, int32_t* offsets, int32_t* perm);
int orc_moe_ffn(const orc_layer* L, const uint16_t* x, const int32_t* adapter_id, int T,
                const int32_t* select, double* y, int32_t* idx_out, double* w_out,
                double* sg_out, double* logits_out);
void orc_rmsnorm_bf16(const uint16_t* x, int T, int H, double eps, uint16_t* xn);
int orc_moe_block(const orc_layer* L, const uint16_t* x, const int32_t* adapter_id, int T,
                  double eps, uint16_t* x_out);

/* Prerouter head of layer N ("Edge0 项目推荐" review, 亮点一): fp16 weights
 * fc1 w1 [D][F], b1 [D]; fc2 w2 [E][D], b2 [E]; linear_init wl [E][F], bl [E];
 * F = H + 2E (biases may be NULL). */
typedef struct {
    int32_t H, E, K, D;
    const uint16_t *w1, *b1, *w2, *b2, *wl, *bl;
} orc_prerouter_head;
double orc_fp16_value(uint16_t h);
double orc_gelu_erf(double v);
int orc_prerouter(const orc_prerouter_head* P, const uint16_t* h, const int32_t* exec_idx, const int32_t* prev_idx,
                  int T, double* logits);

uint16_t orc_bf16_round_down(double v);
uint16_t orc_bf16_round_up(double v);
uint16_t orc_bf16_round_nearest(double v);
double orc_bf16_value(uint16_t h);
int orc_threads(void);

#ifdef __cplusplus
}
#endif
#endif
