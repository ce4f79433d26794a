/*
 * nc_oracle.c — CPU oracle for the forward pass of the nanochat-style
 * KV-cache inference Engine (prefill and single-token decode).
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may link, load or
 * call this file; only the tests, the package's smoke() check and the bench's
 * CPU-baseline leg use it. It shares no code, header or table with the CUDA
 * engine.
 *
 * What it computes follows the architecture list Karpathy gives in the
 * launch Q&A of the nanochat news page ("nanochat" launch article, section
 * "技術細節與問答", the answer listing the model features):
 *   dense Transformer, "basically Llama-like"; rotary embeddings (RoPE) and no
 *   positional embedding; QK norm; untied embedding/unembedding; a norm right
 *   after the token embedding; relu^2 in the MLP; RMSNorm without learnable
 *   parameters; no bias in the linears; multi-query attention; logit softcap.
 * The Engine does KV-cache prefill/decode (same page, list of pipeline
 * stages, "高效推理"). The pages give no formulas, so every constant and
 * step below that they leave open is a stated reading:
 *   - RMSNorm: y = x / sqrt(mean(x^2) + eps), eps = 1e-6 (the config's).
 *   - pre-norm residual blocks ("Llama-like") plus a final norm before lm_head.
 *   - RoPE: split-half pairs (i, i + hd/2), theta_i = base^(-2i/hd), angle
 *     pos*theta_i, (a, b) -> (a cos - b sin, a sin + b cos).
 *   - QK norm: the same RMSNorm over each head of q and of k, after RoPE
 *     (the two commute: rotation is orthogonal and the norm has no gain).
 *   - attention scale 1/sqrt(hd), softmax with max subtraction, causal.
 *   - MLP: x += relu(h Wfc^T)^2 Wproj^T.
 *   - logits = cap * tanh(z / cap).
 *   - token pick: argmax(logits + g) (g optional noise), lowest index on ties.
 *
 * Precision: activations, accumulators and logits are double; weights are
 * read as stored (fp32, or bf16 widened exactly to double).
 *
 * Two independent evaluation orders are provided:
 *   orc_step          token-at-a-time through a per-sequence KV cache;
 *   orc_forward_full  whole sequence layer by layer with an explicit causal
 *                     score matrix and no cache.
 * Their agreement is one of the oracle's pins.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  int depth, d_model, n_head, n_kv_head, head_dim, mlp_hidden, vocab;
  double rope_base, softcap, norm_eps;
  int dtype; /* 0: fp32 weights, 1: bf16 weights */
} orc_config;

typedef struct {
  orc_config c;
  const void *blob; /* borrowed: caller keeps it alive */
  size_t off_wte, off_lm;
  size_t *off_layer; /* 6 per layer: wq, wk, wv, wo, wfc, wproj */
} orc_model;

typedef struct {
  int max_seq, len;
  double *k, *v; /* [depth][max_seq][n_kv_head*head_dim] */
} orc_seq;

/* ---------------------------------------------------------------- weights */
static inline double orc_w(const orc_model *m, size_t i) {
  if (m->c.dtype == 0) return (double)((const float *)m->blob)[i];
  uint32_t bits = ((uint32_t)((const uint16_t *)m->blob)[i]) << 16;
  float f;
  memcpy(&f, &bits, 4);
  return (double)f;
}

/* y[r] = sum_c W[r, c] x[c] for W = blob tensor at `off`, row-major [rows, cols]. */
static void orc_matvec(const orc_model *m, size_t off, int rows, int cols, const double *x, double *y) {
#pragma omp parallel for schedule(static) if ((long)rows * cols >= (1L << 18))
  for (int r = 0; r < rows; r++) {
    double acc = 0.0;
    size_t base = off + (size_t)r * cols;
    for (int c = 0; c < cols; c++) acc += orc_w(m, base + c) * x[c];
    y[r] = acc;
  }
}

/* ------------------------------------------------------------ primitives */
void orc_rmsnorm(const double *x, int n, double eps, double *y) {
  double ss = 0.0;
  for (int i = 0; i < n; i++) ss += x[i] * x[i];
  double inv = 1.0 / sqrt(ss / n + eps);
  for (int i = 0; i < n; i++) y[i] = x[i] * inv;
}

void orc_rope(double *v, int hd, double pos, double base) {
  int half = hd / 2;
  for (int i = 0; i < half; i++) {
    double theta = pow(base, -2.0 * i / hd);
    double ang = pos * theta;
    double c = cos(ang), s = sin(ang);
    double a = v[i], b = v[i + half];
    v[i] = a * c - b * s;
    v[i + half] = a * s + b * c;
  }
}

double orc_softcap(double z, double cap) { return cap * tanh(z / cap); }

/* One query head against n cached keys/values (rows `stride` apart):
 * y = sum_j softmax_j(q.k_j / sqrt(hd)) v_j. */
void orc_attend(const double *q, const double *K, const double *V, int n, int hd, int stride, double *y) {
  double *s = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  double mx = -INFINITY, scale = 1.0 / sqrt((double)hd);
  for (int j = 0; j < n; j++) {
    double d = 0.0;
    for (int i = 0; i < hd; i++) d += q[i] * K[(size_t)j * stride + i];
    s[j] = d * scale;
    if (s[j] > mx) mx = s[j];
  }
  double z = 0.0;
  for (int j = 0; j < n; j++) { s[j] = exp(s[j] - mx); z += s[j]; }
  for (int i = 0; i < hd; i++) y[i] = 0.0;
  for (int j = 0; j < n; j++)
    for (int i = 0; i < hd; i++) y[i] += s[j] / z * V[(size_t)j * stride + i];
  free(s);
}

/* Lowest index of max(v + g); g may be NULL. */
int orc_argmax(const double *v, const float *g, int n) {
  int best = 0;
  double bv = v[0] + (g ? (double)g[0] : 0.0);
  for (int i = 1; i < n; i++) {
    double x = v[i] + (g ? (double)g[i] : 0.0);
    if (x > bv) { bv = x; best = i; }
  }
  return best;
}

/* Sampled token pick with temperature and top-k. The launch article lists
 * sampling in the Engine ("高效推理") and gives no details; the reading is the
 * usual one: keep the top_k largest logits (top_k <= 0 or >= n keeps all;
 * at a tie on the cut the lower index is kept) and draw from the softmax of
 * z / temperature over them. With g_v i.i.d. standard Gumbel noise the draw
 * is argmax_v (z_v / temperature + g_v) (Gumbel-max), so the noise is an
 * input, as for orc_argmax. temperature == 0 is the greedy pick argmax_v z_v.
 * The decision is taken in fp32, the precision of the logits it is made on:
 * score_v = fl(fl(z_v / temperature) + g_v), lowest index on ties. */
static const float *g_sample_z;  /* key of the ordering below (qsort has no context argument) */

static int by_logit_desc(const void *a, const void *b) {
  const int i = *(const int *)a, j = *(const int *)b;
  const float zi = g_sample_z[i], zj = g_sample_z[j];
  if (zi > zj) return -1;
  if (zi < zj) return 1;
  return (i > j) - (i < j);
}

int orc_sample_topk(const float *z, const float *g, int n, float temperature, int top_k) {
  if (n <= 0) return -1;
  if (temperature == 0.0f) {
    int best = 0;
    for (int i = 1; i < n; i++)
      if (z[i] > z[best]) best = i;
    return best;
  }
  const int k = (top_k <= 0 || top_k >= n) ? n : top_k;
  int *order = (int *)malloc(sizeof(int) * (size_t)n);
  if (!order) return -1;
  for (int i = 0; i < n; i++) order[i] = i;
  g_sample_z = z;
  qsort(order, (size_t)n, sizeof(int), by_logit_desc);
  int best = -1;
  float best_s = 0.0f;
  for (int r = 0; r < k; r++) {
    const int v = order[r];
    const float scaled = z[v] / temperature;
    const float s = scaled + (g ? g[v] : 0.0f);
    if (best < 0 || s > best_s || (s == best_s && v < best)) {
      best = v;
      best_s = s;
    }
  }
  free(order);
  return best;
}

/* ----------------------------------------------------------------- model */
orc_model *orc_model_create(const orc_config *c, const void *blob) {
  if (!c || !blob || c->depth < 0 || c->d_model <= 0 || c->n_head <= 0 || c->n_kv_head <= 0 ||
      c->head_dim <= 0 || (c->head_dim & 1) || c->n_head % c->n_kv_head != 0 || c->mlp_hidden <= 0 ||
      c->vocab <= 0)
    return NULL;
  orc_model *m = (orc_model *)calloc(1, sizeof(orc_model));
  if (!m) return NULL;
  m->c = *c;
  m->blob = blob;
  m->off_layer = (size_t *)calloc((size_t)(c->depth > 0 ? c->depth : 1) * 6, sizeof(size_t));
  size_t d = c->d_model, qd = (size_t)c->n_head * c->head_dim, kd = (size_t)c->n_kv_head * c->head_dim;
  size_t F = c->mlp_hidden, off = 0;
  m->off_wte = off;
  off += (size_t)c->vocab * d;
  for (int l = 0; l < c->depth; l++) {
    size_t *o = m->off_layer + 6 * l;
    o[0] = off; off += qd * d;
    o[1] = off; off += kd * d;
    o[2] = off; off += kd * d;
    o[3] = off; off += d * qd;
    o[4] = off; off += F * d;
    o[5] = off; off += d * F;
  }
  m->off_lm = off;
  return m;
}

size_t orc_model_num_params(const orc_model *m) { return m->off_lm + (size_t)m->c.vocab * m->c.d_model; }

void orc_model_destroy(orc_model *m) {
  if (!m) return;
  free(m->off_layer);
  free(m);
}

orc_seq *orc_seq_create(const orc_model *m, int max_seq) {
  orc_seq *s = (orc_seq *)calloc(1, sizeof(orc_seq));
  if (!s) return NULL;
  size_t n = (size_t)(m->c.depth > 0 ? m->c.depth : 1) * max_seq * m->c.n_kv_head * m->c.head_dim;
  s->max_seq = max_seq;
  s->k = (double *)calloc(n, sizeof(double));
  s->v = (double *)calloc(n, sizeof(double));
  if (!s->k || !s->v) { free(s->k); free(s->v); free(s); return NULL; }
  return s;
}

void orc_seq_destroy(orc_seq *s) {
  if (!s) return;
  free(s->k);
  free(s->v);
  free(s);
}

int orc_seq_len(const orc_seq *s) { return s->len; }

/* Deep copy of src's cache into dst (same model, dst->max_seq >= src->len). */
int orc_seq_copy(const orc_model *m, const orc_seq *src, orc_seq *dst) {
  if (dst->max_seq < src->len) return -1;
  int kd = m->c.n_kv_head * m->c.head_dim;
  for (int l = 0; l < m->c.depth; l++) {
    size_t so = (size_t)l * src->max_seq * kd, doff = (size_t)l * dst->max_seq * kd;
    memcpy(dst->k + doff, src->k + so, sizeof(double) * (size_t)src->len * kd);
    memcpy(dst->v + doff, src->v + so, sizeof(double) * (size_t)src->len * kd);
  }
  dst->len = src->len;
  return 0;
}

/* Final norm, lm_head and softcap for one residual vector. */
static void orc_head(const orc_model *m, const double *x, double *logits) {
  const orc_config *c = &m->c;
  double *h = (double *)malloc(sizeof(double) * c->d_model);
  orc_rmsnorm(x, c->d_model, c->norm_eps, h);
  orc_matvec(m, m->off_lm, c->vocab, c->d_model, h, logits);
  for (int i = 0; i < c->vocab; i++) logits[i] = orc_softcap(logits[i], c->softcap);
  free(h);
}

/* Feed `token` at RoPE position `pos` into sequence s (stored at cache slot
 * s->len); writes the [vocab] logits for the next token. Returns 0, or -1 if
 * the cache is full or the token is out of range. */
int orc_step(const orc_model *m, orc_seq *s, int token, int pos, double *logits) {
  const orc_config *c = &m->c;
  if (s->len >= s->max_seq || token < 0 || token >= c->vocab) return -1;
  int d = c->d_model, hd = c->head_dim, H = c->n_head, Hkv = c->n_kv_head, F = c->mlp_hidden;
  int qd = H * hd, kd = Hkv * hd, group = H / Hkv, t = s->len;
  double *x = (double *)malloc(sizeof(double) * d), *h = (double *)malloc(sizeof(double) * d);
  double *q = (double *)malloc(sizeof(double) * qd), *k = (double *)malloc(sizeof(double) * kd);
  double *v = (double *)malloc(sizeof(double) * kd), *y = (double *)malloc(sizeof(double) * qd);
  double *f = (double *)malloc(sizeof(double) * F), *o = (double *)malloc(sizeof(double) * d);

  /* token embedding, then the norm that follows it */
  for (int i = 0; i < d; i++) x[i] = orc_w(m, m->off_wte + (size_t)token * d + i);
  orc_rmsnorm(x, d, c->norm_eps, x);

  for (int l = 0; l < c->depth; l++) {
    const size_t *W = m->off_layer + 6 * l;
    /* attention sub-block */
    orc_rmsnorm(x, d, c->norm_eps, h);
    orc_matvec(m, W[0], qd, d, h, q);
    orc_matvec(m, W[1], kd, d, h, k);
    orc_matvec(m, W[2], kd, d, h, v);
    for (int a = 0; a < H; a++) {
      orc_rope(q + a * hd, hd, pos, c->rope_base);
      orc_rmsnorm(q + a * hd, hd, c->norm_eps, q + a * hd);
    }
    for (int a = 0; a < Hkv; a++) {
      orc_rope(k + a * hd, hd, pos, c->rope_base);
      orc_rmsnorm(k + a * hd, hd, c->norm_eps, k + a * hd);
    }
    double *Kc = s->k + (size_t)l * s->max_seq * kd, *Vc = s->v + (size_t)l * s->max_seq * kd;
    memcpy(Kc + (size_t)t * kd, k, sizeof(double) * kd);
    memcpy(Vc + (size_t)t * kd, v, sizeof(double) * kd);
    for (int a = 0; a < H; a++) {
      int g = a / group;
      orc_attend(q + a * hd, Kc + g * hd, Vc + g * hd, t + 1, hd, kd, y + a * hd);
    }
    orc_matvec(m, W[3], d, qd, y, o);
    for (int i = 0; i < d; i++) x[i] += o[i];
    /* MLP sub-block */
    orc_rmsnorm(x, d, c->norm_eps, h);
    orc_matvec(m, W[4], F, d, h, f);
    for (int i = 0; i < F; i++) f[i] = f[i] > 0.0 ? f[i] * f[i] : 0.0;
    orc_matvec(m, W[5], d, F, f, o);
    for (int i = 0; i < d; i++) x[i] += o[i];
  }
  orc_head(m, x, logits);
  s->len = t + 1;
  free(x); free(h); free(q); free(k); free(v); free(y); free(f); free(o);
  return 0;
}

/* Whole-sequence forward without reading a cache: positions pos0 .. pos0+T-1.
 * Layer-major order with an explicit T x T causal score matrix per head.
 * Logits go to logits[T, vocab] if all_positions, else logits[vocab] for the
 * last position only. If `fill` is non-NULL (an empty sequence with room for
 * T tokens), the rotated/normed keys and the values are also written into its
 * cache slots 0..T-1, so that orc_step can continue from there.
 * Returns 0 or -1. */
int orc_forward_full(const orc_model *m, const int *tokens, int T, int pos0, int all_positions,
                     double *logits, orc_seq *fill) {
  const orc_config *c = &m->c;
  int d = c->d_model, hd = c->head_dim, H = c->n_head, Hkv = c->n_kv_head, F = c->mlp_hidden;
  int qd = H * hd, kd = Hkv * hd, group = H / Hkv;
  if (T <= 0) return -1;
  if (fill && (fill->len != 0 || fill->max_seq < T)) return -1;
  for (int t = 0; t < T; t++)
    if (tokens[t] < 0 || tokens[t] >= c->vocab) return -1;
  double *X = (double *)malloc(sizeof(double) * (size_t)T * d);
  double *Hn = (double *)malloc(sizeof(double) * (size_t)T * d);
  double *Q = (double *)malloc(sizeof(double) * (size_t)T * qd);
  double *K = (double *)malloc(sizeof(double) * (size_t)T * kd);
  double *V = (double *)malloc(sizeof(double) * (size_t)T * kd);
  double *Y = (double *)malloc(sizeof(double) * (size_t)T * qd);
  double *Fh = (double *)malloc(sizeof(double) * (size_t)T * F);
  double *S = (double *)malloc(sizeof(double) * (size_t)T * T);
  double scale = 1.0 / sqrt((double)hd);

  for (int t = 0; t < T; t++) {
    for (int i = 0; i < d; i++) X[(size_t)t * d + i] = orc_w(m, m->off_wte + (size_t)tokens[t] * d + i);
    orc_rmsnorm(X + (size_t)t * d, d, c->norm_eps, X + (size_t)t * d);
  }
  for (int l = 0; l < c->depth; l++) {
    const size_t *W = m->off_layer + 6 * l;
    for (int t = 0; t < T; t++) {
      double *hn = Hn + (size_t)t * d;
      orc_rmsnorm(X + (size_t)t * d, d, c->norm_eps, hn);
      orc_matvec(m, W[0], qd, d, hn, Q + (size_t)t * qd);
      orc_matvec(m, W[1], kd, d, hn, K + (size_t)t * kd);
      orc_matvec(m, W[2], kd, d, hn, V + (size_t)t * kd);
      for (int a = 0; a < H; a++) {
        double *qa = Q + (size_t)t * qd + a * hd;
        orc_rope(qa, hd, pos0 + t, c->rope_base);
        orc_rmsnorm(qa, hd, c->norm_eps, qa);
      }
      for (int a = 0; a < Hkv; a++) {
        double *ka = K + (size_t)t * kd + a * hd;
        orc_rope(ka, hd, pos0 + t, c->rope_base);
        orc_rmsnorm(ka, hd, c->norm_eps, ka);
      }
    }
    if (fill) {
      double *Kc = fill->k + (size_t)l * fill->max_seq * kd, *Vc = fill->v + (size_t)l * fill->max_seq * kd;
      memcpy(Kc, K, sizeof(double) * (size_t)T * kd);
      memcpy(Vc, V, sizeof(double) * (size_t)T * kd);
    }
    for (int a = 0; a < H; a++) {
      int g = a / group;
      /* scores with the causal mask: S[i][j] = -inf for j > i */
#pragma omp parallel for schedule(static) if ((long)T * T * hd >= (1L << 18))
      for (int i = 0; i < T; i++) {
        const double *qi = Q + (size_t)i * qd + a * hd;
        double mx = -INFINITY, z = 0.0;
        for (int j = 0; j < T; j++) {
          if (j > i) { S[(size_t)i * T + j] = -INFINITY; continue; }
          const double *kj = K + (size_t)j * kd + g * hd;
          double dot = 0.0;
          for (int e = 0; e < hd; e++) dot += qi[e] * kj[e];
          S[(size_t)i * T + j] = dot * scale;
          if (S[(size_t)i * T + j] > mx) mx = S[(size_t)i * T + j];
        }
        for (int j = 0; j < T; j++) {
          double p = (j > i) ? 0.0 : exp(S[(size_t)i * T + j] - mx);
          S[(size_t)i * T + j] = p;
          z += p;
        }
        double *yi = Y + (size_t)i * qd + a * hd;
        for (int e = 0; e < hd; e++) {
          double acc = 0.0;
          for (int j = 0; j < T; j++) acc += S[(size_t)i * T + j] * V[(size_t)j * kd + g * hd + e];
          yi[e] = acc / z;
        }
      }
    }
    for (int t = 0; t < T; t++) {
      double *xt = X + (size_t)t * d, *hn = Hn + (size_t)t * d, *ft = Fh + (size_t)t * F;
      orc_matvec(m, W[3], d, qd, Y + (size_t)t * qd, hn);
      for (int i = 0; i < d; i++) xt[i] += hn[i];
      orc_rmsnorm(xt, d, c->norm_eps, hn);
      orc_matvec(m, W[4], F, d, hn, ft);
      for (int i = 0; i < F; i++) ft[i] = ft[i] > 0.0 ? ft[i] * ft[i] : 0.0;
      orc_matvec(m, W[5], d, F, ft, hn);
      for (int i = 0; i < d; i++) xt[i] += hn[i];
    }
  }
  if (all_positions)
    for (int t = 0; t < T; t++) orc_head(m, X + (size_t)t * d, logits + (size_t)t * c->vocab);
  else
    orc_head(m, X + (size_t)(T - 1) * d, logits);
  if (fill) fill->len = T;
  free(X); free(Hn); free(Q); free(K); free(V); free(Y); free(Fh); free(S);
  return 0;
}

int orc_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Threads of the parallel loops from now on (n >= 1). Every output element
 * is computed by one thread in a fixed order, so results do not depend on it. */
void orc_set_threads(int n) {
#ifdef _OPENMP
  extern void omp_set_num_threads(int);
  if (n >= 1) omp_set_num_threads(n);
#else
  (void)n;
#endif
}
