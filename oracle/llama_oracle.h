/*
 * CPU oracle for one autoregressive decode step of a Llama-style decoder.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link or
 * call this code; it exists to check the GPU engine.  It shares no header,
 * helper or table with the engine.
 *
 * Every function exists twice: suffix _f64 (all arithmetic in double: the
 * definition the GPU is compared against) and _f32 (the same steps in float
 * with sequential accumulation, used to bound the effect of fp32 arithmetic).
 * Weights are bf16 bit patterns widened exactly; only the KV cache is stored
 * rounded (bf16, round-to-nearest-even).
 */
#ifndef LLAMA_ORACLE_H
#define LLAMA_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  int n_layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn, vocab;
  double rms_eps, rope_theta;
} orc_shape;

typedef struct {
  const uint16_t *attn_norm, *wq, *wk, *wv, *wo, *ffn_norm, *w_gate, *w_up, *w_down;
} orc_layer;

typedef struct {
  orc_shape shape;
  const uint16_t *embed, *lm_head, *final_norm;
  const orc_layer *layers; /* [n_layers] */
} orc_model;

/* One sequence's slice of a bf16 cache; position stride = head_dim. */
typedef struct {
  uint16_t *k, *v;
  int64_t layer_stride, head_stride; /* in elements */
} orc_kv;

/* Optional per-stage values of one decode step (any pointer may be NULL). */
typedef struct {
  double *q;       /* [L][q_dim]  after RoPE */
  double *k;       /* [L][kv_dim] after RoPE, before bf16 rounding */
  double *v;       /* [L][kv_dim] */
  double *attn;    /* [L][q_dim]  attention output (input of the O projection) */
  double *x_attn;  /* [L][H]      residual after O projection */
  double *act;     /* [L][F]      silu(gate) * up */
  double *x_out;   /* [L][H]      residual after down projection */
  double *final_a; /* [H]         final RMSNorm output (input of the LM head) */
} orc_dump;

#define ORC_DECL(S, R)                                                              \
  R orc_bf16_to_real##S(uint16_t b);                                               \
  uint16_t orc_real_to_bf16##S(R x);                                               \
  void orc_matvec##S(const uint16_t *W, const R *x, int rows, int cols, R *y);     \
  void orc_rmsnorm##S(const R *x, const uint16_t *gamma, int n, double eps, R *y); \
  void orc_rope##S(R *v, int d, int pos, double theta);                            \
  void orc_attention_head##S(const R *q, const uint16_t *K, const uint16_t *V,     \
                             int n_pos, int d, R *o);                              \
  R orc_silu##S(R z);                                                              \
  int orc_decode_step##S(const orc_model *m, const orc_kv *kv, int token, int pos, \
                         double *logits, const orc_dump *dump);                    \
  int orc_prefill##S(const orc_model *m, const orc_kv *kv, const int32_t *tokens,  \
                     int n, double *logits_all, double *logits_last);

ORC_DECL(_f64, double)
ORC_DECL(_f32, float)

/* Index of the first maximal element (ties go to the lowest index). */
int orc_argmax(const double *x, int n);

#ifdef __cplusplus
}
#endif
#endif
