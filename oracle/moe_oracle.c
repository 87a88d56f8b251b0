/*
 * moe_oracle.c -- plain, slow CPU oracle for the streaming-experts MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY (tests, smoke check, benchmark CPU baseline).  It
 * shares no code with the CUDA library and neither includes the other.
 * Citations name the page and its section; the page titles are listed in
 * moe_oracle.h.  Every function states the definition it writes out.
 *
 * Parity status: every function here is pinned by the CPU tests (hand-packed
 * examples, brute-force nearest codes, brute-force top-K, closed forms, dense
 * and one-hot special cases, the FMA identity).  No function is unpinned.
 */
#include "moe_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ORC_MUTANT selects one planted mistake; it is compiled only by the tests
 * that check the pins catch it (0 = the oracle as written). */
#ifndef ORC_MUTANT
#define ORC_MUTANT 0
#endif

static size_t round_up_256(size_t n) { return (n + 255u) & ~(size_t)255u; }

static int cfg_ok(const orc_cfg* c) {
  if (c->bits != 2 && c->bits != 4) return 0;
  if (c->group != 64 || c->hidden <= 0 || c->inter <= 0) return 0; /* layout blocks are 8 x 64 */
  if (c->hidden % c->group || c->inter % c->group) return 0;
  /* whole 32-bit code words per row */
  if ((c->hidden * c->bits) % 32 || (c->inter * c->bits) % 32) return 0;
  return 1;
}

/* Section sizes: codes take b bits per weight, one 4-byte (scale, bias) word
 * per group.  [toolarium] "Flash-MoE: чистый C, Metal и никакого Python"
 * prints ~6.75 MB per 4-bit expert, which this table reproduces exactly for
 * H=4096, I=1024, G=64 (3*4096*1024/2 + 3*4096*1024/64*4 = 7,077,888 B). */
static void section_sizes(const orc_cfg* c, size_t sz[6]) {
  size_t H = (size_t)c->hidden, I = (size_t)c->inter, b = (size_t)c->bits;
  size_t G = (size_t)c->group;
  sz[0] = I * H * b / 8;
  sz[1] = I * H * b / 8;
  sz[2] = H * I * b / 8;
  sz[3] = I * (H / G) * 4;
  sz[4] = I * (H / G) * 4;
  sz[5] = H * (I / G) * 4;
}

void orc_section_offsets(const orc_cfg* c, size_t off[6]) {
  size_t sz[6];
  size_t pos = 0;
  section_sizes(c, sz);
  for (int i = 0; i < 6; ++i) {
    off[i] = pos;
    pos = round_up_256(pos + sz[i]);
  }
}

size_t orc_expert_bytes(const orc_cfg* c) {
  size_t sz[6], off[6];
  if (!cfg_ok(c)) return 0;
  section_sizes(c, sz);
  orc_section_offsets(c, off);
  return round_up_256(off[5] + sz[5]);
}

/* ---- bf16 ------------------------------------------------------------- */

uint16_t orc_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) {
    return (uint16_t)((u >> 16) | 0x0040u); /* quiet NaN */
  }
  /* round to nearest, ties to even, on the 16 discarded bits */
  uint32_t lower = u & 0xffffu;
  uint32_t upper = u >> 16;
  if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;
  return (uint16_t)upper;
}

static float bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

double orc_bf16_to_f64(uint16_t h) { return (double)bf16_to_f32(h); }

/* ---- quantiser ---------------------------------------------------------- */

/* Group-affine quantiser for one group of n weights (the pages give the
 * dequant form q*scale + bias, [toolarium] "Оптимизации, которые сработали",
 * and the bit widths 4 and 2, [toolarium] "Бенчмарки на MacBook Pro"; they do
 * not print the quantiser, so this is the plain min/max affine one):
 *   scale = bf16((max - min) / (2^b - 1)),  bias = bf16(min),
 *   q = clamp(round_half_even((w - bias) / scale), 0, 2^b - 1), q = 0 if
 *   scale == 0.  All arithmetic of the code decision is single precision. */
static void quantize_group(const float* w, int n, int bits, uint16_t* s_out,
                           uint16_t* b_out, int* q) {
  float mn = w[0], mx = w[0];
  for (int i = 1; i < n; ++i) {
    if (w[i] < mn) mn = w[i];
    if (w[i] > mx) mx = w[i];
  }
  float qmax = (float)((1 << bits) - (ORC_MUTANT == 7 ? 0 : 1));
  volatile float range = mx - mn; /* volatile: keep each step a separate float rounding */
  volatile float sf_raw = range / qmax;
  uint16_t s = orc_f32_to_bf16(sf_raw);
  uint16_t beta = orc_f32_to_bf16(mn);
  float sf = bf16_to_f32(s), bf = bf16_to_f32(beta);
  for (int i = 0; i < n; ++i) {
    if (sf == 0.0f) {
      q[i] = 0;
      continue;
    }
    volatile float num = w[i] - bf;
    volatile float ratio = num / sf;
    float r = rintf(ratio); /* default rounding mode: to nearest even */
    if (r < 0.0f) r = 0.0f;
    if (r > qmax) r = qmax;
    q[i] = (int)r;
  }
  *s_out = s;
  *b_out = beta;
}

/* Where code (row, col) of a [rows][cols] matrix lives: byte offset of its
 * 32-bit little-endian word inside the code section, and its bit position.
 * Blocks of 8 rows x 64 columns, row-block major then column group; a block
 * holds 64*b bytes, 64*b/32 bytes per "lane" l = 4*(row % 8) + t.  Inside the
 * group, column c = 16*s + cc (k-step s = 0..3):
 *   cc in 0..7 : t = cc / 2, e = cc % 2, "first" slot;  cc in 8..15:
 *   t = (cc - 8) / 2, e = cc % 2, "second" slot.
 * 4-bit: word h = s / 2 of the lane, j = s % 2; first slot nibble 2j + 4e,
 *        second slot nibble 2j + 1 + 4e.
 * 2-bit: the lane's single word; first slot code 2s + 8e, second slot code
 *        2s + 1 + 8e.
 * (This places the four codes a lane needs for one 16-column step of a
 * tensor-core B fragment in one word; the dequantised value is unaffected.) */
static void code_pos(int bits, int cols, int row, int col, size_t* byte_off, int* shift) {
  int rb = row / 8, n = row % 8, g = col / 64, cg = col % 64;
  int s = cg / 16, cc = cg % 16;
  int second = cc >= 8;
  int t = (second ? cc - 8 : cc) / 2, e = cc % 2;
  int lane = 4 * n + t;
  size_t block = (size_t)rb * (cols / 64) + g;
  size_t lane_bytes = (size_t)(64 * bits) / 32;
  size_t off = block * (size_t)(64 * bits) + (size_t)lane * lane_bytes;
  int m;
  if (bits == 4) {
    int h = s / 2, j = s % 2;
    off += 4 * (size_t)h;
    m = second ? 2 * j + 1 + 4 * e : 2 * j + 4 * e;
  } else {
    m = second ? 2 * s + 1 + 8 * e : 2 * s + 8 * e;
  }
  *byte_off = off;
  *shift = m * bits;
}

/* Scale word of (row, group): [row block][group][row % 8], 4 bytes each. */
static size_t scale_pos(int cols, int row, int g) {
  return (((size_t)(row / 8) * (cols / 64) + g) * 8 + row % 8) * 4;
}

static void put_code(uint8_t* codes, int cols, int row, int col, int bits, int q) {
  size_t off;
  int shift;
  code_pos(bits, cols, row, col, &off, &shift);
  uint32_t v;
  memcpy(&v, codes + off, 4); /* little-endian host */
  v |= ((uint32_t)q & ((1u << bits) - 1u)) << shift;
  memcpy(codes + off, &v, 4);
}

static void quantize_matrix(const orc_cfg* c, const float* w, int rows, int cols,
                            uint8_t* codes, uint8_t* scales) {
  int G = c->group, b = c->bits;
  int* q = (int*)malloc(sizeof(int) * G);
  for (int r = 0; r < rows; ++r) {
    for (int g = 0; g < cols / G; ++g) {
      uint16_t s, beta;
      quantize_group(w + (size_t)r * cols + (size_t)g * G, G, b, &s, &beta, q);
      for (int i = 0; i < G; ++i) put_code(codes, cols, r, g * G + i, b, q[i]);
      uint32_t word = (uint32_t)s | ((uint32_t)beta << 16);
      memcpy(scales + scale_pos(cols, r, g), &word, 4);
    }
  }
  free(q);
}

int orc_quantize_expert(const orc_cfg* c, const float* w_gate, const float* w_up,
                        const float* w_down, uint8_t* blob) {
  size_t off[6];
  size_t total = orc_expert_bytes(c);
  if (total == 0) return -1;
  memset(blob, 0, total);
  orc_section_offsets(c, off);
  quantize_matrix(c, w_gate, c->inter, c->hidden, blob + off[0], blob + off[3]);
  quantize_matrix(c, w_up, c->inter, c->hidden, blob + off[1], blob + off[4]);
  quantize_matrix(c, w_down, c->hidden, c->inter, blob + off[2], blob + off[5]);
  return 0;
}

/* ---- dequantiser -------------------------------------------------------- */

static void mat_shape(const orc_cfg* c, int m, int* rows, int* cols) {
  if (m == 2) {
    *rows = c->hidden;
    *cols = c->inter;
  } else {
    *rows = c->inter;
    *cols = c->hidden;
  }
}

int orc_code(const orc_cfg* c, const uint8_t* blob, int m, int row, int col) {
  size_t off[6], pos;
  int rows, cols, shift;
  orc_section_offsets(c, off);
  mat_shape(c, m, &rows, &cols);
  int b = c->bits;
  code_pos(b, cols, row, ORC_MUTANT == 2 ? (col ^ 1) : col, &pos, &shift);
  uint32_t v;
  memcpy(&v, blob + off[m] + pos, 4);
  return (int)((v >> shift) & ((1u << b) - 1u));
}

/* w = q*s + beta, the "(nibble x scale + bias)" form of [toolarium]
 * "Оптимизации, которые сработали"; exact in double precision. */
double orc_dequant(const orc_cfg* c, const uint8_t* blob, int m, int row, int col) {
  size_t off[6];
  int rows, cols;
  orc_section_offsets(c, off);
  mat_shape(c, m, &rows, &cols);
  uint32_t word;
  memcpy(&word, blob + off[3 + m] + scale_pos(cols, row, col / c->group), 4);
  double s = orc_bf16_to_f64((uint16_t)(word & 0xffffu));
  double beta = orc_bf16_to_f64((uint16_t)(word >> 16));
  return (double)orc_code(c, blob, m, row, col) * s + (ORC_MUTANT == 1 ? 0.0 : beta);
}

void orc_dequant_matrix(const orc_cfg* c, const uint8_t* blob, int m, double* out) {
  int rows, cols;
  mat_shape(c, m, &rows, &cols);
  for (int r = 0; r < rows; ++r)
    for (int k = 0; k < cols; ++k) out[(size_t)r * cols + k] = orc_dequant(c, blob, m, r, k);
}

/* ---- router ------------------------------------------------------------- */

/* "a" ranks before "b": larger logit first, ties to the lower index; a NaN
 * logit ranks as -infinity.  The pages choose 4 of 512 experts per token by
 * softmax/top-K on the CPU ([hakusoku] "パイプライン概要"; [toolarium]
 * "Mixture of Experts и почему SSD достаточно"); order and ties are not
 * printed, so the plain total order above is used. */
static int ranks_before(float la, int ia, float lb, int ib) {
  double a = isnan(la) ? -INFINITY : (double)la;
  double b = isnan(lb) ? -INFINITY : (double)lb;
  if (a != b) return a > b;
  return ORC_MUTANT == 4 ? ia > ib : ia < ib;
}

/* Softmax over all E logits followed by renormalisation over the K chosen
 * ones equals a softmax over the K chosen logits (the full denominator
 * cancels); written here as the K-only softmax, in double precision. */
void orc_topk(const orc_cfg* c, const float* logits, int T, int32_t* idx, float* w,
              double* w_f64) {
  int E = c->n_experts, K = c->top_k;
  char* taken = (char*)malloc((size_t)E);
  int* sel = (int*)malloc(sizeof(int) * K);
  for (int t = 0; t < T; ++t) {
    const float* l = logits + (size_t)t * E;
    memset(taken, 0, (size_t)E);
    for (int k = 0; k < K; ++k) { /* selection: K passes of "best remaining" */
      int best = -1;
      for (int e = 0; e < E; ++e) {
        if (taken[e]) continue;
        if (best < 0 || ranks_before(l[e], e, l[best], best)) best = e;
      }
      taken[best] = 1;
      sel[k] = best;
    }
    double lmax = isnan(l[sel[0]]) ? -INFINITY : (double)l[sel[0]];
    double den = 0.0;
    for (int k = 0; k < K; ++k) {
      double lk = isnan(l[sel[k]]) ? -INFINITY : (double)l[sel[k]];
      den += exp(lk - lmax);
    }
    for (int k = 0; k < K; ++k) {
      double lk = isnan(l[sel[k]]) ? -INFINITY : (double)l[sel[k]];
      double wk = exp(lk - lmax) / den;
      if (idx) idx[(size_t)t * K + k] = sel[k];
      if (w) w[(size_t)t * K + k] = (float)wk;
      if (w_f64) w_f64[(size_t)t * K + k] = wk;
    }
  }
  free(sel);
  free(taken);
}

/* logits = x . Wr^T + bias, accumulated in double (each bf16 x bf16 product is
 * exact in double), then rounded to float: the router projection that the
 * pages compute on the GPU next to the shared expert ([hakusoku]
 * "パイプライン概要", CMD2 "routing"). */
static void router_logits(const orc_cfg* c, const uint16_t* x, const uint16_t* wr,
                          const float* bias, int T, float* logits) {
  int H = c->hidden, E = c->n_experts;
  for (int t = 0; t < T; ++t)
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int h = 0; h < H; ++h)
        acc += orc_bf16_to_f64(x[(size_t)t * H + h]) *
               orc_bf16_to_f64(wr[ORC_MUTANT == 10 ? (size_t)h * E + e : (size_t)e * H + h]);
      if (bias && ORC_MUTANT != 11) acc += (double)bias[e];
      logits[(size_t)t * E + e] = (float)acc;
    }
}

void orc_router(const orc_cfg* c, const uint16_t* x_bf16, const uint16_t* wr_bf16,
                const float* bias, int T, float* logits, int32_t* idx, float* w) {
  float* l = (float*)malloc(sizeof(float) * (size_t)T * c->n_experts + 1);
  router_logits(c, x_bf16, wr_bf16, bias, T, l);
  if (logits) memcpy(logits, l, sizeof(float) * (size_t)T * c->n_experts);
  if (idx || w) orc_topk(c, l, T, idx, w, NULL);
  free(l);
}

/* ---- expert FFN --------------------------------------------------------- */

/* silu(z) = z / (1 + exp(-z)), the SwiGLU gate ([hakusoku] "主要技術": SwiGLU
 * activation among the hand-written kernels). */
static double silu(double z) {
  if (ORC_MUTANT == 12) return 1.0 / (1.0 + exp(-z));
  return z / (1.0 + exp(ORC_MUTANT == 3 ? z : -z));
}

/* a[i] = silu(sum_h Wg[i][h] x[h]) * (sum_h Wu[i][h] x[h]) */
void orc_expert_act(const orc_cfg* c, const uint8_t* blob, const double* x, double* a) {
  int H = c->hidden, I = c->inter;
  for (int i = 0; i < I; ++i) {
    double g = 0.0, u = 0.0;
    for (int h = 0; h < H; ++h) {
      g += orc_dequant(c, blob, 0, i, h) * x[h];
      u += orc_dequant(c, blob, 1, i, h) * x[h];
    }
    a[i] = ORC_MUTANT == 9 ? silu(u) * g : silu(g) * u;
  }
}

/* y = Wd a: dequantise, then multiply ([toolarium] "Оптимизации, которые
 * сработали": the base form (nibble x scale + bias) x x). */
void orc_expert_ffn(const orc_cfg* c, const uint8_t* blob, const double* x, double* y) {
  int H = c->hidden, I = c->inter;
  double* a = (double*)malloc(sizeof(double) * I);
  orc_expert_act(c, blob, x, a);
  for (int r = 0; r < H; ++r) {
    double acc = 0.0;
    for (int i = 0; i < I; ++i) acc += orc_dequant(c, blob, 2, r, i) * a[i];
    y[r] = acc;
  }
  free(a);
}

/* The same product written as fma(q, s*x, beta*x) per weight, the rewritten
 * form of [toolarium] "Оптимизации, которые сработали" and [hakusoku]
 * "主要技術" (FMA dequant kernel).  Kept separate so the tests can check the
 * identity (q*s + beta)*x == q*(s*x) + beta*x. */
static double fma_form_dot(const orc_cfg* c, const uint8_t* blob, int m, int row,
                           const double* x, int n) {
  size_t off[6];
  orc_section_offsets(c, off);
  double acc = 0.0;
  for (int k = 0; k < n; ++k) {
    uint32_t word;
    memcpy(&word, blob + off[3 + m] + scale_pos(n, row, k / c->group), 4);
    double s = orc_bf16_to_f64((uint16_t)(word & 0xffffu));
    double beta = orc_bf16_to_f64((uint16_t)(word >> 16));
    double q = (double)orc_code(c, blob, m, row, k);
    acc += fma(q, s * x[k], beta * x[k]);
  }
  return acc;
}

void orc_expert_ffn_fma_form(const orc_cfg* c, const uint8_t* blob, const double* x,
                             double* y) {
  int H = c->hidden, I = c->inter;
  double* a = (double*)malloc(sizeof(double) * I);
  for (int i = 0; i < I; ++i) {
    double g = fma_form_dot(c, blob, 0, i, x, H);
    double u = fma_form_dot(c, blob, 1, i, x, H);
    a[i] = silu(g) * u;
  }
  for (int r = 0; r < H; ++r) y[r] = fma_form_dot(c, blob, 2, r, a, I);
  free(a);
}

/* Shared expert: same SwiGLU FFN with bf16 weights, weight 1, no gate
 * ([hakusoku] "モデルアーキテクチャ": K=4 routed experts plus a shared one). */
void orc_shared_ffn(const orc_cfg* c, const uint16_t* wg, const uint16_t* wu,
                    const uint16_t* wd, const double* x, double* y) {
  int H = c->hidden, I = c->inter;
  double* a = (double*)malloc(sizeof(double) * I);
  for (int i = 0; i < I; ++i) {
    double g = 0.0, u = 0.0;
    for (int h = 0; h < H; ++h) {
      g += orc_bf16_to_f64(wg[(size_t)i * H + h]) * x[h];
      u += orc_bf16_to_f64(wu[(size_t)i * H + h]) * x[h];
    }
    a[i] = silu(g) * u;
  }
  for (int r = 0; r < H; ++r) {
    double acc = 0.0;
    for (int i = 0; i < I; ++i)
      acc += orc_bf16_to_f64(ORC_MUTANT == 8 ? wd[(size_t)i * H + r] : wd[(size_t)r * I + i]) * a[i];
    y[r] = acc;
  }
  free(a);
}

/* ---- RMSNorm before the layer --------------------------------------------- */

/* x = h / sqrt(mean(h^2) + eps) * gamma_pre, per token: the normalisation that
 * the GPU command before the experts runs together with the router and the
 * shared expert ([hakusoku] "パイプライン概要").  The layer then takes x rounded
 * to bf16 as its input and h itself as the residual. */
void orc_prenorm(const orc_cfg* c, const uint16_t* h_bf16, const uint16_t* gamma_bf16, int T,
                 double* x) {
  int H = c->hidden;
  for (int t = 0; t < T; ++t) {
    double ss = 0.0;
    for (int r = 0; r < H; ++r) {
      double v = orc_bf16_to_f64(h_bf16[(size_t)t * H + r]);
      ss += v * v;
    }
    double inv = ORC_MUTANT == 13 ? 1.0 / sqrt(ss + (double)c->eps) : 1.0 / sqrt(ss / H + (double)c->eps);
    for (int r = 0; r < H; ++r) {
      double g = ORC_MUTANT == 14 ? 1.0 : orc_bf16_to_f64(gamma_bf16[r]);
      x[(size_t)t * H + r] = orc_bf16_to_f64(h_bf16[(size_t)t * H + r]) * inv * g;
    }
  }
}

/* Round a double to bf16, to nearest with ties to even, in one step (no
 * intermediate float).  Finite inputs only. */
uint16_t orc_f64_to_bf16(double v) {
  if (v == 0.0) return signbit(v) ? 0x8000u : 0u;
  int e;
  (void)frexp(fabs(v), &e); /* |v| = m * 2^e, m in [0.5, 1) */
  /* bf16 keeps 8 significant bits: units of 2^(e-8) for normal results */
  int ue = e - 8;
  if (ue < -133) ue = -133; /* subnormal bf16: units of 2^-133 */
  double q = ldexp(fabs(v), -ue);
  double fl = floor(q), fr = q - fl;
  if (fr > 0.5 || (fr == 0.5 && fmod(fl, 2.0) != 0.0)) fl += 1.0;
  float f = (float)ldexp(fl, ue); /* exact: at most 9 significant bits */
  uint32_t u;
  memcpy(&u, &f, 4);
  if (v < 0) u |= 0x80000000u;
  return (uint16_t)(u >> 16);
}

/* ---- whole layer ---------------------------------------------------------- */

/* h_out = residual + sum_k w_k * expert_{idx_k}(x) + shared(x);
 * y_norm = h_out / sqrt(mean(h_out^2) + eps) * gamma.
 * The pages fuse "combine + residual + normalization" into one GPU kernel
 * whose output feeds the next layer ([toolarium] "Оптимизации, которые
 * сработали"; [hakusoku] "主要技術", deferred expert computation).
 * The shared expert is the bf16 FFN, or, when shared_blob is given, the same
 * FFN with packed weights as the routed experts; when shared_gate_w (bf16
 * [H]) is given its output is scaled by sigmoid(x . shared_gate_w) (the
 * pages name the shared expert next to the K routed ones and compute it in
 * the command with the router, [hakusoku] "モデルアーキテクチャ",
 * "パイプライン概要"; neither form is printed there). */
void orc_layer_forward_ex(const orc_cfg* c, const uint8_t* const* experts,
                          const uint16_t* wr_bf16, const float* bias,
                          const uint16_t* shared_gate, const uint16_t* shared_up,
                          const uint16_t* shared_down, const uint8_t* shared_blob,
                          const uint16_t* shared_gate_w, const uint16_t* gamma_bf16,
                          const uint16_t* x_bf16, const uint16_t* residual_bf16, int T,
                          const int32_t* idx_in, const double* w_in, int32_t* idx,
                          float* w, double* h_out, double* y_norm) {
  int H = c->hidden, E = c->n_experts, K = c->top_k;
  int32_t* sel = (int32_t*)malloc(sizeof(int32_t) * (size_t)T * K + 4);
  double* wsel = (double*)malloc(sizeof(double) * (size_t)T * K + 8);
  if (idx_in) {
    memcpy(sel, idx_in, sizeof(int32_t) * (size_t)T * K);
    memcpy(wsel, w_in, sizeof(double) * (size_t)T * K);
  } else {
    float* l = (float*)malloc(sizeof(float) * (size_t)T * E + 4);
    router_logits(c, x_bf16, wr_bf16, bias, T, l);
    orc_topk(c, l, T, sel, NULL, wsel);
    free(l);
  }
  if (idx) memcpy(idx, sel, sizeof(int32_t) * (size_t)T * K);
  if (w)
    for (size_t i = 0; i < (size_t)T * K; ++i) w[i] = (float)wsel[i];

  double* x = (double*)malloc(sizeof(double) * H);
  double* y = (double*)malloc(sizeof(double) * H);
  double* h = (double*)malloc(sizeof(double) * H);
  for (int t = 0; t < T; ++t) {
    for (int r = 0; r < H; ++r) {
      x[r] = orc_bf16_to_f64(x_bf16[(size_t)t * H + r]);
      h[r] = ORC_MUTANT == 5 ? 0.0 : orc_bf16_to_f64(residual_bf16[(size_t)t * H + r]);
    }
    for (int k = 0; k < K; ++k) {
      orc_expert_ffn(c, experts[sel[(size_t)t * K + k]], x, y);
      for (int r = 0; r < H; ++r) h[r] += wsel[(size_t)t * K + k] * y[r];
    }
    if (c->has_shared) {
      if (shared_blob && ORC_MUTANT != 17)
        orc_expert_ffn(c, shared_blob, x, y);
      else
        orc_shared_ffn(c, shared_gate, shared_up, shared_down, x, y);
      double gs = 1.0;
      if (shared_gate_w) {
        double z = 0.0;
        for (int r = 0; r < H; ++r) z += x[r] * orc_bf16_to_f64(shared_gate_w[r]);
        gs = ORC_MUTANT == 15 ? z / (1.0 + exp(-z)) : 1.0 / (1.0 + exp(-z));
      }
      for (int r = 0; r < H; ++r) h[r] += (ORC_MUTANT == 16 ? 1.0 : gs) * y[r];
    }
    double ss = 0.0;
    for (int r = 0; r < H; ++r) ss += h[r] * h[r];
    double inv = ORC_MUTANT == 6 ? 1.0 / (sqrt(ss / H) + (double)c->eps)
                                 : 1.0 / sqrt(ss / H + (double)c->eps);
    for (int r = 0; r < H; ++r) {
      if (h_out) h_out[(size_t)t * H + r] = h[r];
      if (y_norm) y_norm[(size_t)t * H + r] = h[r] * inv * orc_bf16_to_f64(gamma_bf16[r]);
    }
  }
  free(h);
  free(y);
  free(x);
  free(wsel);
  free(sel);
}

void orc_layer_forward(const orc_cfg* c, const uint8_t* const* experts,
                       const uint16_t* wr_bf16, const float* bias,
                       const uint16_t* shared_gate, const uint16_t* shared_up,
                       const uint16_t* shared_down, const uint16_t* gamma_bf16,
                       const uint16_t* x_bf16, const uint16_t* residual_bf16, int T,
                       const int32_t* idx_in, const double* w_in, int32_t* idx,
                       float* w, double* h_out, double* y_norm) {
  orc_layer_forward_ex(c, experts, wr_bf16, bias, shared_gate, shared_up, shared_down, NULL, NULL,
                       gamma_bf16, x_bf16, residual_bf16, T, idx_in, w_in, idx, w, h_out, y_norm);
}
