/*
 * Body of the CPU oracle, included twice by llama_oracle.c with
 *   R = double, S = _f64   and   R = float, S = _f32.
 * TEST INFRASTRUCTURE ONLY (see llama_oracle.h).
 *
 * Sources.  The operations and their order come from the decode forward pass
 * the megakernel pages fuse: "Hazy megakernel summary" page (yaoshibet.com),
 * section 四(二) "融合大爆炸" lists the instructions (fused RMSNorm + QKV +
 * RoPE, attention, ...) and section 五(二) the RMSNorm + matrix-vector work.
 * The pages never write the formulas out, so each one below is the textbook
 * Llama reading of the named operation; every such reading is marked READING.
 */
#define CAT_(a, b) a##b
#define CAT(a, b) CAT_(a, b)
#define F(name) CAT(name, S)

R F(orc_bf16_to_real)(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (R)f; /* exact: every bf16 value is a float value */
}

/* Round-to-nearest-even of x to the bf16 grid, computed directly from R. */
uint16_t F(orc_real_to_bf16)(R x) {
  if (x == 0) return (uint16_t)(signbit(x) ? 0x8000u : 0u);
  int e;
  double m = frexp((double)x, &e); /* x = m * 2^e, 0.5 <= |m| < 1 */
  /* bf16 keeps 8 significant bits; scale them above the binary point and
     round half to even (nearbyint in the default rounding mode). */
  double r = ldexp(nearbyint(ldexp(m, 8)), e - 8);
  float f = (float)r; /* exact: r has at most 9 significant bits */
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}

/* y[r] = sum_c W[r][c] * x[c], W bf16 row-major [rows][cols], summed in
   order c = 0, 1, ... (a plain dot product per output row). */
void F(orc_matvec)(const uint16_t *W, const R *x, int rows, int cols, R *y) {
#pragma omp parallel for schedule(static)
  for (int r = 0; r < rows; ++r) {
    const uint16_t *w = W + (int64_t)r * cols;
    R acc = 0;
    for (int c = 0; c < cols; ++c) acc += F(orc_bf16_to_real)(w[c]) * x[c];
    y[r] = acc;
  }
}

/* READING (RMSNorm): y_i = x_i / sqrt(mean_j x_j^2 + eps) * gamma_i. */
void F(orc_rmsnorm)(const R *x, const uint16_t *gamma, int n, double eps, R *y) {
  R ss = 0;
  for (int i = 0; i < n; ++i) ss += x[i] * x[i];
  R inv = (R)1 / (R)sqrt((double)(ss / (R)n + (R)eps));
  for (int i = 0; i < n; ++i) y[i] = x[i] * inv * F(orc_bf16_to_real)(gamma[i]);
}

/* READING (RoPE, rotate-half): for i < d/2 the pair (v_i, v_{i+d/2}) turns by
   angle pos * theta^(-2i/d); the angle and its cos/sin are taken in double
   and then rounded to R. */
void F(orc_rope)(R *v, int d, int pos, double theta) {
  int h = d / 2;
  for (int i = 0; i < h; ++i) {
    double ang = (double)pos * pow(theta, -2.0 * (double)i / (double)d);
    R c = (R)cos(ang), s = (R)sin(ang);
    R u = v[i], w = v[i + h];
    v[i] = u * c - w * s;
    v[i + h] = u * s + w * c;
  }
}

/* READING (decode attention of one query head over n_pos cached positions):
   s_j = q.K_j / sqrt(d); w = softmax(s) (max subtracted); o = sum_j w_j V_j.
   K and V rows are bf16, row stride d. */
void F(orc_attention_head)(const R *q, const uint16_t *K, const uint16_t *V, int n_pos,
                           int d, R *o) {
  R *s = (R *)malloc(sizeof(R) * (size_t)(n_pos > 0 ? n_pos : 1));
  R scale = (R)1 / (R)sqrt((double)d);
  R mx = -(R)INFINITY;
  for (int j = 0; j < n_pos; ++j) {
    R dot = 0;
    for (int t = 0; t < d; ++t) dot += q[t] * F(orc_bf16_to_real)(K[(int64_t)j * d + t]);
    s[j] = dot * scale;
    if (s[j] > mx) mx = s[j];
  }
  R sum = 0;
  for (int j = 0; j < n_pos; ++j) {
    s[j] = (R)exp((double)(s[j] - mx));
    sum += s[j];
  }
  for (int t = 0; t < d; ++t) o[t] = 0;
  for (int j = 0; j < n_pos; ++j) {
    R w = s[j] / sum;
    for (int t = 0; t < d; ++t) o[t] += w * F(orc_bf16_to_real)(V[(int64_t)j * d + t]);
  }
  free(s);
}

/* READING (SwiGLU activation): silu(z) = z / (1 + e^-z). */
R F(orc_silu)(R z) { return z / ((R)1 + (R)exp(-(double)z)); }

/* ------------------------------------------------------------------------ */

static uint16_t *F(kv_row)(const orc_kv *kv, int which, int layer, int g, int pos, int d) {
  uint16_t *base = which ? kv->v : kv->k;
  return base + (int64_t)layer * kv->layer_stride + (int64_t)g * kv->head_stride +
         (int64_t)pos * d;
}

static void F(copy_out)(double *dst, const R *src, int n) {
  if (dst)
    for (int i = 0; i < n; ++i) dst[i] = (double)src[i];
}

/*
 * One decode step of one sequence: token `token` at position `pos`.
 * Writes this token's K/V (bf16) at `pos` in every layer, attends over
 * positions 0..pos, and returns the logits (double, [vocab]).
 * Step order per layer (the forward pass the pages fuse):
 *   a = rms(x) * g1;  q,k,v = Wq a, Wk a, Wv a;  RoPE(q), RoPE(k);
 *   cache[pos] = bf16(k), bf16(v);
 *   o_h = attention(q_h, K[g(h)], V[g(h)]) over 0..pos, g(h) = h / (nq/nkv);
 *   x += Wo o;  b = rms(x) * g2;  x += Wd (silu(Wg b) * (Wu b)).
 * Then logits = Wlm (rms(x) * gf).  Returns 0, or -1 on a bad argument.
 */
int F(orc_decode_step)(const orc_model *m, const orc_kv *kv, int token, int pos,
                       double *logits, const orc_dump *dump) {
  const orc_shape *sh = &m->shape;
  const int H = sh->hidden, d = sh->head_dim, nq = sh->n_q_heads, nkv = sh->n_kv_heads;
  const int qd = nq * d, kvd = nkv * d, Fd = sh->ffn;
  if (token < 0 || token >= sh->vocab || pos < 0 || nq % nkv) return -1;
  const int grp = nq / nkv;
  R *x = (R *)malloc(sizeof(R) * H), *a = (R *)malloc(sizeof(R) * H);
  R *q = (R *)malloc(sizeof(R) * qd), *k = (R *)malloc(sizeof(R) * kvd);
  R *v = (R *)malloc(sizeof(R) * kvd), *o = (R *)malloc(sizeof(R) * qd);
  R *t = (R *)malloc(sizeof(R) * H), *g = (R *)malloc(sizeof(R) * Fd);
  R *u = (R *)malloc(sizeof(R) * Fd);

  for (int i = 0; i < H; ++i) x[i] = F(orc_bf16_to_real)(m->embed[(int64_t)token * H + i]);

  for (int l = 0; l < sh->n_layers; ++l) {
    const orc_layer *L = &m->layers[l];
    F(orc_rmsnorm)(x, L->attn_norm, H, sh->rms_eps, a);
    F(orc_matvec)(L->wq, a, qd, H, q);
    F(orc_matvec)(L->wk, a, kvd, H, k);
    F(orc_matvec)(L->wv, a, kvd, H, v);
    for (int h = 0; h < nq; ++h) F(orc_rope)(q + h * d, d, pos, sh->rope_theta);
    for (int h = 0; h < nkv; ++h) F(orc_rope)(k + h * d, d, pos, sh->rope_theta);
    if (dump) {
      F(copy_out)(dump->q ? dump->q + (int64_t)l * qd : NULL, q, qd);
      F(copy_out)(dump->k ? dump->k + (int64_t)l * kvd : NULL, k, kvd);
      F(copy_out)(dump->v ? dump->v + (int64_t)l * kvd : NULL, v, kvd);
    }
    for (int h = 0; h < nkv; ++h) {
      uint16_t *kr = F(kv_row)(kv, 0, l, h, pos, d), *vr = F(kv_row)(kv, 1, l, h, pos, d);
      for (int i = 0; i < d; ++i) {
        kr[i] = F(orc_real_to_bf16)(k[h * d + i]);
        vr[i] = F(orc_real_to_bf16)(v[h * d + i]);
      }
    }
    for (int h = 0; h < nq; ++h) {
      int gh = h / grp; /* READING: contiguous query-head groups share a KV head */
      F(orc_attention_head)(q + h * d, F(kv_row)(kv, 0, l, gh, 0, d), F(kv_row)(kv, 1, l, gh, 0, d),
                            pos + 1, d, o + h * d);
    }
    if (dump) F(copy_out)(dump->attn ? dump->attn + (int64_t)l * qd : NULL, o, qd);
    F(orc_matvec)(L->wo, o, H, qd, t);
    for (int i = 0; i < H; ++i) x[i] += t[i];
    if (dump) F(copy_out)(dump->x_attn ? dump->x_attn + (int64_t)l * H : NULL, x, H);
    F(orc_rmsnorm)(x, L->ffn_norm, H, sh->rms_eps, a);
    F(orc_matvec)(L->w_gate, a, Fd, H, g);
    F(orc_matvec)(L->w_up, a, Fd, H, u);
    for (int i = 0; i < Fd; ++i) g[i] = F(orc_silu)(g[i]) * u[i];
    if (dump) F(copy_out)(dump->act ? dump->act + (int64_t)l * Fd : NULL, g, Fd);
    F(orc_matvec)(L->w_down, g, H, Fd, t);
    for (int i = 0; i < H; ++i) x[i] += t[i];
    if (dump) F(copy_out)(dump->x_out ? dump->x_out + (int64_t)l * H : NULL, x, H);
  }
  F(orc_rmsnorm)(x, m->final_norm, H, sh->rms_eps, a);
  if (dump) F(copy_out)(dump->final_a, a, H);
  {
    R *lg = (R *)malloc(sizeof(R) * (size_t)sh->vocab);
    F(orc_matvec)(m->lm_head, a, sh->vocab, H, lg);
    for (int i = 0; i < sh->vocab; ++i) logits[i] = (double)lg[i];
    free(lg);
  }
  free(x); free(a); free(q); free(k); free(v); free(o); free(t); free(g); free(u);
  return 0;
}

/*
 * Full causal forward over a prompt (positions 0..n-1), computed layer by
 * layer over all positions at once: every position's K/V of a layer is
 * produced and rounded into the cache before any position of that layer
 * attends, and position t attends over 0..t.  This is the "full recompute"
 * of the whole prefix; its last row must equal decode_step at the last
 * position.  logits_all ([n][vocab]) and logits_last ([vocab]) may be NULL.
 */
int F(orc_prefill)(const orc_model *m, const orc_kv *kv, const int32_t *tokens, int n,
                   double *logits_all, double *logits_last) {
  const orc_shape *sh = &m->shape;
  const int H = sh->hidden, d = sh->head_dim, nq = sh->n_q_heads, nkv = sh->n_kv_heads;
  const int qd = nq * d, kvd = nkv * d, Fd = sh->ffn;
  if (n <= 0 || nq % nkv) return -1;
  for (int i = 0; i < n; ++i)
    if (tokens[i] < 0 || tokens[i] >= sh->vocab) return -1;
  const int grp = nq / nkv;
  R *X = (R *)malloc(sizeof(R) * (size_t)n * H);
  R *Q = (R *)malloc(sizeof(R) * (size_t)n * qd);
  R *a = (R *)malloc(sizeof(R) * H), *k = (R *)malloc(sizeof(R) * kvd);
  R *v = (R *)malloc(sizeof(R) * kvd), *o = (R *)malloc(sizeof(R) * qd);
  R *t = (R *)malloc(sizeof(R) * H), *g = (R *)malloc(sizeof(R) * Fd);
  R *u = (R *)malloc(sizeof(R) * Fd), *lg = (R *)malloc(sizeof(R) * (size_t)sh->vocab);

  for (int p = 0; p < n; ++p)
    for (int i = 0; i < H; ++i)
      X[(int64_t)p * H + i] = F(orc_bf16_to_real)(m->embed[(int64_t)tokens[p] * H + i]);

  for (int l = 0; l < sh->n_layers; ++l) {
    const orc_layer *L = &m->layers[l];
    /* projections for every position first */
    for (int p = 0; p < n; ++p) {
      R *x = X + (int64_t)p * H, *q = Q + (int64_t)p * qd;
      F(orc_rmsnorm)(x, L->attn_norm, H, sh->rms_eps, a);
      F(orc_matvec)(L->wq, a, qd, H, q);
      F(orc_matvec)(L->wk, a, kvd, H, k);
      F(orc_matvec)(L->wv, a, kvd, H, v);
      for (int h = 0; h < nq; ++h) F(orc_rope)(q + h * d, d, p, sh->rope_theta);
      for (int h = 0; h < nkv; ++h) F(orc_rope)(k + h * d, d, p, sh->rope_theta);
      for (int h = 0; h < nkv; ++h) {
        uint16_t *kr = F(kv_row)(kv, 0, l, h, p, d), *vr = F(kv_row)(kv, 1, l, h, p, d);
        for (int i = 0; i < d; ++i) {
          kr[i] = F(orc_real_to_bf16)(k[h * d + i]);
          vr[i] = F(orc_real_to_bf16)(v[h * d + i]);
        }
      }
    }
    /* causal attention, then the rest of the layer, per position */
    for (int p = 0; p < n; ++p) {
      R *x = X + (int64_t)p * H, *q = Q + (int64_t)p * qd;
      for (int h = 0; h < nq; ++h) {
        int gh = h / grp;
        F(orc_attention_head)(q + h * d, F(kv_row)(kv, 0, l, gh, 0, d),
                              F(kv_row)(kv, 1, l, gh, 0, d), p + 1, d, o + h * d);
      }
      F(orc_matvec)(L->wo, o, H, qd, t);
      for (int i = 0; i < H; ++i) x[i] += t[i];
      F(orc_rmsnorm)(x, L->ffn_norm, H, sh->rms_eps, a);
      F(orc_matvec)(L->w_gate, a, Fd, H, g);
      F(orc_matvec)(L->w_up, a, Fd, H, u);
      for (int i = 0; i < Fd; ++i) g[i] = F(orc_silu)(g[i]) * u[i];
      F(orc_matvec)(L->w_down, g, H, Fd, t);
      for (int i = 0; i < H; ++i) x[i] += t[i];
    }
  }
  for (int p = 0; p < n; ++p) {
    if (!logits_all && p != n - 1) continue;
    F(orc_rmsnorm)(X + (int64_t)p * H, m->final_norm, H, sh->rms_eps, a);
    F(orc_matvec)(m->lm_head, a, sh->vocab, H, lg);
    if (logits_all)
      for (int i = 0; i < sh->vocab; ++i) logits_all[(int64_t)p * sh->vocab + i] = (double)lg[i];
    if (logits_last && p == n - 1)
      for (int i = 0; i < sh->vocab; ++i) logits_last[i] = (double)lg[i];
  }
  free(X); free(Q); free(a); free(k); free(v); free(o); free(t); free(g); free(u); free(lg);
  return 0;
}

#undef F
#undef CAT
#undef CAT_
