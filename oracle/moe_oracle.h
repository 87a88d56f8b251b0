/*
 * moe_oracle.h -- plain, slow CPU oracle for the streaming-experts MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes
 * or calls this code; only the tests, the smoke check and the benchmark's CPU
 * baseline use it.  It shares no code with the CUDA path.
 *
 * Sources (web pages about the Flash-MoE "streaming experts" engine):
 *   [toolarium] "Streaming experts: как запустить триллионную модель на MacBook"
 *               (toolarium.ru): sections "Mixture of Experts и почему SSD
 *               достаточно", "Flash-MoE: чистый C, Metal и никакого Python",
 *               "Бенчмарки на MacBook Pro" (table), "Оптимизации, которые
 *               сработали".
 *   [hakusoku]  "Flash-MoE: ラップトップでの397Bパラメータモデルの実行"
 *               (hakusoku.com): sections "モデルアーキテクチャ" (model
 *               architecture), "主要技術" (key techniques), "パイプライン概要"
 *               (pipeline overview), "試行錯誤と最適化" (experiments).
 *
 * Arithmetic: every floating-point result is computed in double precision
 * (the pages fix no precision).  Two decisions that produce integers are taken
 * in single precision, the precision of the product kernels: the quantiser's
 * code choice, and the router's top-K ordering (on logits rounded to float).
 *
 * Packed expert format (the oracle's own statement of it; see
 * orc_expert_bytes for the section table).  One blob per expert holds six
 * sections, each starting on a 256-byte boundary:
 *   0 gate codes  [I][H*b/8]     1 up codes   [I][H*b/8]
 *   2 down codes  [H][I*b/8]     3 gate scales [I][H/G] (uint32)
 *   4 up scales   [I][H/G]       5 down scales [H][I/G]
 * Codes come in blocks of 8 rows x 64 columns (row-block major, then column
 * group), 64*b bytes per block; inside a block the four codes that a
 * tensor-core B fragment takes for one 16-column step share one 32-bit word
 * (exact positions: code_pos in moe_oracle.c).  Scale words are stored
 * [row block][group][row % 8]; a scale word holds the bf16 scale s in bits
 * 0..15 and the bf16 bias beta in bits 16..31.  The dequantised weight is
 * q*s + beta ([toolarium] "Оптимизации, которые сработали": the "(nibble x
 * scale + bias)" form).  Group size 64, H and I multiples of 64.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  int hidden;     /* H */
  int inter;      /* I, expert intermediate size */
  int n_experts;  /* E */
  int top_k;      /* K */
  int bits;       /* b: 2 or 4 */
  int group;      /* G: weights per (scale, bias) group along the input dim */
  float eps;      /* RMSNorm epsilon */
  int has_shared; /* 1 if a bf16 shared expert is present */
} orc_cfg;

/* Byte size of one packed expert blob; 0 if the shape is not representable. */
size_t orc_expert_bytes(const orc_cfg* c);
/* Offsets of the six sections (see header comment). */
void orc_section_offsets(const orc_cfg* c, size_t off[6]);

/* bf16 helpers (round to nearest even; NaN stays NaN). */
uint16_t orc_f32_to_bf16(float f);
double orc_bf16_to_f64(uint16_t h);
/* Double to bf16 in one rounding (nearest, ties to even; finite inputs). */
uint16_t orc_f64_to_bf16(double v);
/* RMSNorm before the layer: x[t] = h[t] / sqrt(mean(h[t]^2) + eps) * gamma_pre,
 * h and gamma bf16, x double [T][H]. */
void orc_prenorm(const orc_cfg* c, const uint16_t* h_bf16, const uint16_t* gamma_bf16, int T,
                 double* x);

/* Quantise one expert from float weights w_gate [I][H], w_up [I][H],
 * w_down [H][I] into blob (orc_expert_bytes bytes, zero padding).  Returns 0. */
int orc_quantize_expert(const orc_cfg* c, const float* w_gate, const float* w_up,
                        const float* w_down, uint8_t* blob);

/* Dequantised weight of matrix m (0 gate, 1 up, 2 down) at (row, col). */
double orc_dequant(const orc_cfg* c, const uint8_t* blob, int m, int row, int col);
/* Code (integer) at (row, col) of matrix m. */
int orc_code(const orc_cfg* c, const uint8_t* blob, int m, int row, int col);
/* Whole dequantised matrix, rows x cols doubles. */
void orc_dequant_matrix(const orc_cfg* c, const uint8_t* blob, int m, double* out);

/* Router: logits[t][e] = float(sum_h x[t][h]*wr[e][h] + bias[e]) (bias may be
 * NULL), then top-K and renormalised weights.  Any of logits/idx/w may be NULL. */
void orc_router(const orc_cfg* c, const uint16_t* x_bf16, const uint16_t* wr_bf16,
                const float* bias, int T, float* logits, int32_t* idx, float* w);
/* Top-K on given float logits [T][E]; w_f64 (may be NULL) gets the weights in
 * double precision, w (may be NULL) the same rounded to float. */
void orc_topk(const orc_cfg* c, const float* logits, int T, int32_t* idx, float* w,
              double* w_f64);

/* One routed expert: y[H] = Wd * (silu(Wg x) * (Wu x)), x[H] in double. */
void orc_expert_ffn(const orc_cfg* c, const uint8_t* blob, const double* x, double* y);
/* Same through the fused-multiply-add form fma(q, s*x, beta*x): an independent
 * restatement used by the tests. */
void orc_expert_ffn_fma_form(const orc_cfg* c, const uint8_t* blob, const double* x,
                             double* y);
/* Intermediate activation only: a[I] = silu(Wg x) * (Wu x). */
void orc_expert_act(const orc_cfg* c, const uint8_t* blob, const double* x, double* a);
/* Shared expert with bf16 weights gate [I][H], up [I][H], down [H][I]. */
void orc_shared_ffn(const orc_cfg* c, const uint16_t* wg, const uint16_t* wu,
                    const uint16_t* wd, const double* x, double* y);

/* Full layer for T tokens.  experts[e] points at expert e's blob.  Outputs:
 * idx [T][K], w [T][K] (float), h_out [T][H] = residual + sum_k w_k y_k + y_s,
 * y_norm [T][H] = RMSNorm(h_out) * gamma.  Any output pointer may be NULL.
 * If idx_in is non-NULL it replaces the oracle's own routing (indices and
 * double weights w_in) so outputs can be compared under a given routing. */
void orc_layer_forward(const orc_cfg* c, const uint8_t* const* experts,
                       const uint16_t* wr_bf16, const float* bias,
                       const uint16_t* shared_gate, const uint16_t* shared_up,
                       const uint16_t* shared_down, const uint16_t* gamma_bf16,
                       const uint16_t* x_bf16, const uint16_t* residual_bf16, int T,
                       const int32_t* idx_in, const double* w_in, int32_t* idx,
                       float* w, double* h_out, double* y_norm);
/* The same layer with the shared expert's two optional forms: shared_blob
 * (a packed blob like the routed experts') replaces the bf16 weights, and
 * shared_gate_w (bf16 [H]) scales the shared output by sigmoid(x . g).
 * Either may be NULL; with both NULL this is orc_layer_forward. */
void orc_layer_forward_ex(const orc_cfg* c, const uint8_t* const* experts,
                          const uint16_t* wr_bf16, const float* bias,
                          const uint16_t* shared_gate, const uint16_t* shared_up,
                          const uint16_t* shared_down, const uint8_t* shared_blob,
                          const uint16_t* shared_gate_w, const uint16_t* gamma_bf16,
                          const uint16_t* x_bf16, const uint16_t* residual_bf16, int T,
                          const int32_t* idx_in, const double* w_in, int32_t* idx,
                          float* w, double* h_out, double* y_norm);

#ifdef __cplusplus
}
#endif
#endif
