// nc_api.cu — the C ABI (include/nc.h): objects, argument checks, and the
// prefill / decode / fork call sequences over the engine's kernels.
#include <math.h>
#include <stdlib.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <map>
#include <mutex>
#include <string>
#include <utility>

#include "nc_internal.h"
#include "nc_kernels.h"

namespace {

thread_local std::string g_err;

int fail(int code, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

#define NC_CUDA_TRY(expr)                                                                       \
  do {                                                                                          \
    cudaError_t e_ = (expr);                                                                    \
    if (e_ != cudaSuccess) return fail(NC_ECUDA, "%s: %s", #expr, cudaGetErrorString(e_));     \
  } while (0)

int check_config(const nc_config *c) {
  if (!c) return fail(NC_EINVAL, "config is NULL");
  if (c->depth < 0 || c->d_model <= 0 || c->n_head <= 0 || c->n_kv_head <= 0 || c->head_dim <= 0 ||
      c->mlp_hidden <= 0 || c->vocab <= 0)
    return fail(NC_EINVAL, "config has a non-positive size");
  if (c->head_dim % 2) return fail(NC_EINVAL, "head_dim must be even (RoPE pairs)");
  if (c->n_head * c->head_dim != c->d_model) return fail(NC_EINVAL, "n_head * head_dim != d_model");
  if (c->n_head % c->n_kv_head) return fail(NC_EINVAL, "n_kv_head must divide n_head");
  if (c->dtype != NC_F32 && c->dtype != NC_BF16) return fail(NC_EINVAL, "dtype must be NC_F32 or NC_BF16");
  if (!(c->softcap > 0.f) || !(c->rope_base > 0.f) || !(c->norm_eps >= 0.f))
    return fail(NC_EINVAL, "softcap and rope_base must be > 0, norm_eps >= 0");
  return NC_OK;
}

size_t blob_elems(const nc_config &c) {
  size_t d = c.d_model, qd = (size_t)c.n_head * c.head_dim, kd = (size_t)c.n_kv_head * c.head_dim;
  size_t F = c.mlp_hidden, V = c.vocab;
  size_t per_layer = qd * d + 2 * kd * d + d * qd + F * d + d * F;
  return 2 * V * d + per_layer * (size_t)c.depth;
}

inline cudaStream_t as_stream(void *s) { return (cudaStream_t)s; }

cudaEvent_t take_event(nc_model *m) {
  if (!m->event_pool.empty()) {
    cudaEvent_t e = m->event_pool.back();
    m->event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Brackets the launches issued in its lifetime with CUDA events when the
// model's profiling is on (nc_profile_enable); a no-op otherwise.
struct ProfScope {
  nc_model *m;
  int cls;
  cudaStream_t s;
  cudaEvent_t a = nullptr;
  unsigned long long n0 = 0;
  ProfScope(nc_model *m_, int cls_, cudaStream_t s_) : m(m_), cls(cls_), s(s_) {
    if (m->prof) {
      a = take_event(m);
      n0 = nc::g_launches.load();
      cudaEventRecord(a, s);
    }
  }
  ~ProfScope() {
    if (!a) return;
    cudaEvent_t b = take_event(m);
    cudaEventRecord(b, s);
    m->prof_recs.push_back({cls, (long long)(nc::g_launches.load() - n0), a, b});
  }
};

inline void *layer_ptr(const nc_kv *kv, void *base, int l) {
  return (char *)base + (size_t)l * kv->layer_elems * kv->model->elem;
}

// Where layer l's shared-prefix rows of kv's sequences live (len == nullptr
// when kv has no links).
nc::KvPrefix prefix_view(const nc_kv *kv, int l) {
  nc::KvPrefix p;
  const nc_kv *r = kv->prefix_src;
  if (!r) return p;
  p.k = layer_ptr(r, r->k, l);
  p.v = layer_ptr(r, r->v, l);
  p.seq = kv->pre_seq;
  p.len = kv->pre_len;
  p.max_seq = r->max_seq;
  return p;
}

void free_kv(nc_kv *kv);

void free_kv(nc_kv *kv) {
  cudaDeviceSynchronize();
  if (kv->graph) cudaGraphExecDestroy(kv->graph);
  if (kv->cap_stream) cudaStreamDestroy(kv->cap_stream);
  void *ps[] = {kv->k,      kv->v,      kv->len,  kv->valid,    kv->rope,   kv->x,     kv->h,
                kv->qkv,    kv->q,      kv->y,    kv->f,        kv->logits, kv->pos_ws, kv->ss,
                kv->part,   kv->counters, kv->cand_v, kv->cand_i, kv->xl,     kv->step_maps, kv->step_ws,
                kv->row_ss,   kv->pre_seq, kv->pre_len};
  for (void *p : ps) cudaFree(p);
  delete kv;
}

// Sequence b of kv stops reading rows of its prefix cache (host bookkeeping;
// the device table is reset by the kernel that replaces the sequence). A
// source cache destroyed while linked is freed with its last link.
void unlink_seq(nc_kv *kv, int b) {
  if (kv->link_seq.empty() || kv->link_seq[b] < 0) return;
  nc_kv *src = kv->prefix_src;
  src->dep_count[kv->link_seq[b]]--;
  src->n_dependents--;
  kv->link_seq[b] = -1;
  if (--kv->n_links == 0) kv->prefix_src = nullptr;
  if (src->destroy_pending && src->n_dependents == 0) free_kv(src);
}

// Sequences [first, first + n) of kv are about to be replaced: refuse if
// another sequence still reads shared rows from one of them (links from
// sequences inside the range itself end with the replacement).
bool replace_blocked(const nc_kv *kv, int first, int n, int *who) {
  for (int b = first; b < first + n; b++) {
    int inside = 0;
    if (kv->prefix_src == kv)
      for (int b2 = first; b2 < first + n; b2++) inside += kv->link_seq[b2] == b;
    if (kv->dep_count[b] - inside > 0) {
      *who = b;
      return true;
    }
  }
  return false;
}

// Each step below takes its sm_100a kernel when the shapes allow it and the
// generic kernel otherwise; a failed launch of either is returned (never
// retried on the other kernel, so a broken fast path cannot hide).

// Linear layer out (epi) A[M,K] * W[N,K]^T: tcgen05 kernel for bf16 models
// once there is at least one full 128-row tile, the generic kernel otherwise.
cudaError_t linear(nc_model *m, int epi, const void *A, int lda, const void *W, int M, int N, int K, void *out,
                   int ldo, float cap, const uint8_t *valid, cudaStream_t s) {
  if (m->fast && M >= 128 && !valid && nc::gemm_tc_supported(M, N, K, lda))
    return nc::k_gemm_tc(epi, A, lda, W, M, N, K, out, ldo, cap, m->status, m->num_sms, s);
  nc::k_gemm_generic(m->cfg.dtype, epi, A, lda, W, M, N, K, out, ldo, cap, valid, s);
  return cudaGetLastError();
}

// h = bf16/fp32 rmsnorm of the M rows of x.
cudaError_t norm_rows(nc_model *m, nc_kv *kv, int M, cudaStream_t s) {
  const nc_config &c = m->cfg;
  if (nc::rowops_supported(c)) return nc::k_rows_norm_bf16(kv->x, M, c.d_model, c.norm_eps, kv->h, s);
  nc::k_rmsnorm_rows(c.dtype, kv->x, M, c.d_model, 1, 0, c.norm_eps, kv->h, s);
  return cudaGetLastError();
}

// RoPE + QK norm of the M rows of kv->qkv, q out, K/V appended to the cache.
cudaError_t rope_append(nc_model *m, nc_kv *kv, void *kc, void *vc, int M, nc::RowMap rm, cudaStream_t s) {
  const nc_config &c = m->cfg;
  if (!rm.pos && !rm.off && c.n_kv_head == 1 && nc::rowops_supported(c))
    return nc::k_rope_qk_bf16(kv->qkv, M, rm.T, c.n_head, kv->rope, kv->q, kc, vc, kv->max_seq, c.norm_eps, s);
  nc::k_rope_qknorm_append(c.dtype, kv->qkv, rm, M, c.n_head, c.n_kv_head, c.head_dim, kv->rope, kv->q, kc, vc,
                           kv->max_seq, kv->valid, c.norm_eps, s);
  return cudaGetLastError();
}

// The layer whose K cache starts at kc.
int layer_of(const nc_kv *kv, const void *kc) {
  return (int)(((const char *)kc - (const char *)kv->k) / (ptrdiff_t)(kv->layer_elems * kv->model->elem));
}

// Causal attention of the M rows in kv->q (H query heads in groups of H/Hkv
// per KV head) against layer cache kc/vc.
cudaError_t attention(nc_model *m, nc_kv *kv, void *kc, void *vc, int M, nc::RowMap rm, cudaStream_t s) {
  const nc_config &c = m->cfg;
  // prefill rows, and appended chunks of a cache that reads no shared prefix
  if (m->fast && !rm.pos && (!rm.off || !kv->prefix_src) &&
      nc::attn_prefill_tc_supported(c.n_head, c.n_kv_head, c.head_dim))
    return nc::k_attn_prefill_tc(kv->q, kc, vc, M / rm.T, rm.T, c.n_head, c.n_kv_head, kv->max_batch, kv->max_seq,
                                 kv->y, m->status, s, rm.off);
  // decode rows and appended chunks may read shared-prefix rows; prefill rows
  // replace their sequences
  const nc::KvPrefix pre = (rm.pos || rm.off) ? prefix_view(kv, layer_of(kv, kc)) : nc::KvPrefix{};
  nc::k_attention_generic(c.dtype, kv->q, kc, vc, rm, M, c.n_head, c.n_kv_head, c.head_dim, kv->max_seq, kv->y, s,
                          &pre);
  return cudaGetLastError();
}

// The fused prefill layer sequence of bf16 head_dim-128 models, when every
// GEMM of the layer takes the tensor-core kernel:
//   QKV  = GEMM(h) with RoPE + QK norm + cache append in its epilogue, h the
//          normed x (layer 0) or bf16(x) scaled per row by its RMS factor
//   attention
//   x   += GEMM(y) (O projection), writing h = bf16(x) and row sums of squares
//   f    = relu(GEMM(h) * rms factor)^2
//   x   += GEMM(f) (MLP projection), again writing h and the sums of squares
//          except in the last layer
bool fused_layers_ok(const nc_model *m, const nc_kv *kv, int M, nc::RowMap rm) {
  const nc_config &c = m->cfg;
  const int d = c.d_model, q = c.n_head * 128, F = c.mlp_hidden, qkv = q + 256 * c.n_kv_head;
  // appended chunks too, unless the cache reads rows of a shared prefix
  return m->fast && !rm.pos && (!rm.off || !kv->prefix_src) && M >= 128 && kv->row_ss && nc::rowops_supported(c) &&
         nc::attn_prefill_tc_supported(c.n_head, c.n_kv_head, c.head_dim) && nc::gemm_tc_supported(M, qkv, d, d) &&
         nc::gemm_tc_supported(M, d, q, q) && nc::gemm_tc_supported(M, F, d, d) && nc::gemm_tc_supported(M, d, F, F);
}

int run_blocks_fused(nc_model *m, nc_kv *kv, int M, nc::RowMap rm, cudaStream_t s) {
  const nc_config &c = m->cfg;
  const int d = c.d_model, H = c.n_head, F = c.mlp_hidden, q = H * 128, qkv = q + 256 * c.n_kv_head;
  nc::GemmFuse fz;
  fz.eps = c.norm_eps;
  fz.xb = kv->h;
  fz.ss_out = kv->row_ss;
  fz.rope = kv->rope;
  fz.q = kv->q;
  fz.T = rm.T;
  fz.H = H;
  fz.Hkv = c.n_kv_head;
  fz.max_seq = kv->max_seq;
  fz.off = rm.off;
  fz.valid = rm.off ? kv->valid : nullptr;
  const int nss = (d + 127) / 128;
  cudaError_t e = cudaSuccess;
  auto gemm = [&](int epi, const void *A, int lda, const void *W, int N, int K, void *out) {
    if (e == cudaSuccess)
      e = nc::k_gemm_tc(epi, A, lda, W, M, N, K, out, N, 0.f, m->status, m->num_sms, s, &fz);
  };
  for (int l = 0; l < c.depth && e == cudaSuccess; l++) {
    const nc_layer_w &w = m->layers[l];
    fz.kc = layer_ptr(kv, kv->k, l);
    fz.vc = layer_ptr(kv, kv->v, l);
    if (l == 0) {
      ProfScope p(m, NC_K_MISC, s);
      e = norm_rows(m, kv, M, s);
    }
    {
      ProfScope p(m, NC_K_GEMM, s);
      fz.ss_in = kv->row_ss;
      fz.nss = l == 0 ? 0 : nss;
      gemm(nc::EPI_QKV, kv->h, d, w.wqkv, qkv, d, nullptr);
    }
    if (e == cudaSuccess) {
      ProfScope p(m, NC_K_ATTN, s);
      e = attention(m, kv, fz.kc, fz.vc, M, rm, s);
    }
    {
      ProfScope p(m, NC_K_GEMM, s);
      gemm(nc::EPI_RESID_X, kv->y, q, w.wo, d, q, kv->x);
      fz.nss = nss;
      gemm(nc::EPI_RELU2, kv->h, d, w.wfc, F, d, kv->f);
      gemm(l + 1 < c.depth ? nc::EPI_RESID_X : nc::EPI_RESID, kv->f, F, w.wproj, d, F, kv->x);
    }
  }
  if (e != cudaSuccess) return nc::set_error(NC_ECUDA, cudaGetErrorString(e));
  return NC_OK;
}

// The transformer blocks for M rows already embedded into kv->x.
int run_blocks(nc_model *m, nc_kv *kv, int M, nc::RowMap rm, cudaStream_t s) {
  if (fused_layers_ok(m, kv, M, rm)) return run_blocks_fused(m, kv, M, rm, s);
  const nc_config &c = m->cfg;
  int d = c.d_model, H = c.n_head, Hkv = c.n_kv_head, hd = c.head_dim, F = c.mlp_hidden;
  int qkv_w = (H + 2 * Hkv) * hd;
  cudaError_t e = cudaSuccess;
  auto step = [&](int cls, auto &&launch) {
    if (e != cudaSuccess) return;
    ProfScope p(m, cls, s);
    e = launch();
  };
  for (int l = 0; l < c.depth && e == cudaSuccess; l++) {
    const nc_layer_w &w = m->layers[l];
    void *kc = layer_ptr(kv, kv->k, l), *vc = layer_ptr(kv, kv->v, l);
    step(NC_K_MISC, [&] { return norm_rows(m, kv, M, s); });
    step(NC_K_GEMM, [&] { return linear(m, nc::EPI_STORE, kv->h, d, w.wqkv, M, qkv_w, d, kv->qkv, qkv_w, 0.f, nullptr, s); });
    step(NC_K_MISC, [&] { return rope_append(m, kv, kc, vc, M, rm, s); });
    step(NC_K_ATTN, [&] { return attention(m, kv, kc, vc, M, rm, s); });
    step(NC_K_GEMM, [&] { return linear(m, nc::EPI_RESID, kv->y, H * hd, w.wo, M, d, H * hd, kv->x, d, 0.f, nullptr, s); });
    step(NC_K_MISC, [&] { return norm_rows(m, kv, M, s); });
    step(NC_K_GEMM, [&] { return linear(m, nc::EPI_RELU2, kv->h, d, w.wfc, M, F, d, kv->f, F, 0.f, nullptr, s); });
    step(NC_K_GEMM, [&] { return linear(m, nc::EPI_RESID, kv->f, F, w.wproj, M, d, F, kv->x, d, 0.f, nullptr, s); });
  }
  if (e != cudaSuccess) return nc::set_error(NC_ECUDA, cudaGetErrorString(e));
  return NC_OK;
}

// Final norm of `rows` rows of x (row r taken from x row r*stride + offset),
// lm_head with softcap into logits (row-major, ldo = V), argmax into next.
cudaError_t run_head(nc_model *m, nc_kv *kv, int rows, int stride, int offset, float *logits, const uint8_t *valid,
                     cudaStream_t s) {
  const nc_config &c = m->cfg;
  ProfScope p(m, NC_K_HEAD, s);
  nc::k_rmsnorm_rows(c.dtype, kv->x, rows, c.d_model, stride, offset, c.norm_eps, kv->h, s);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return linear(m, nc::EPI_SOFTCAP, kv->h, c.d_model, m->wlm, rows, c.vocab, c.d_model, logits, c.vocab, c.softcap,
                valid, s);
}

// With sampling parameters set on the cache (nc_kv_set_sampling), replace the
// argmax pick in next[] by the sampled pick over the same logits and noise.
cudaError_t sampled_pick(nc_model *m, nc_kv *kv, const float *logits, int B, int V, long long stride,
                         const float *noise, const uint8_t *valid, int32_t *next, cudaStream_t s) {
  if (!next || !kv->sampling()) return cudaSuccess;
  ProfScope p(m, NC_K_HEAD, s);
  return nc::k_sample_topk(logits, B, V, stride, noise, kv->temperature, kv->top_k, valid, next, s);
}

// The decode step on the sm_100a decode kernels (bf16, head_dim 128, B <= 32).
cudaError_t decode_fast_launches(nc_model *m, nc_kv *kv, const int32_t *tokens, const int32_t *positions, int B,
                                 const float *noise, float *logits, int32_t *next, cudaStream_t s) {
  const nc_config &c = m->cfg;
  const int d = c.d_model, H = c.n_head, F = c.mlp_hidden, V = c.vocab, sms = m->num_sms;
  const float eps = c.norm_eps;
  cudaError_t e;
  if (kv->step_grid > 0 && nc::decode_step_supported(c, B)) {
    {
      ProfScope p(m, NC_K_STEP, s);
      const nc_kv *pre = kv->prefix_src ? kv->prefix_src : kv;
      e = nc::k_decode_step(m, kv->step_plan, B, kv->max_batch, kv->max_seq, kv->step_maps, kv->step_ws, tokens,
                            positions, kv->len, kv->k, kv->v, kv->rope, logits, noise, next, kv->step_trace,
                            kv->valid, kv->pre_seq, kv->pre_len, pre->max_batch, pre->max_seq, s);
    }
    return e == cudaSuccess ? sampled_pick(m, kv, logits, B, V, V, noise, kv->valid, next, s) : e;
  }
  {
    ProfScope p(m, NC_K_MISC, s);
    e = nc::k_dec_embed(tokens, positions, kv->len, kv->pos_ws, kv->valid, B, kv->max_seq, m->wte, d, V, eps, kv->x,
                        kv->ss, 32, m->status, s);
    if (e != cudaSuccess) return e;
  }
  for (int l = 0; l < c.depth; l++) {
    const nc_layer_w &w = m->layers[l];
    void *kc = layer_ptr(kv, kv->k, l), *vc = layer_ptr(kv, kv->v, l);
    {
      ProfScope p(m, NC_K_GEMM, s);
      e = nc::k_dec_linear(0 /*norm*/, 0 /*qkv*/, w.wqkv, (H + 2) * 128, d, B, kv->x, kv->ss, 32, eps, nullptr,
                           kv->part, kv->counters, nullptr, nullptr, kv->q, kc, vc, kv->max_seq, H, kv->pos_ws,
                           kv->valid, kv->rope, nullptr, nullptr, 0.f, nullptr, nullptr, nullptr, m->status, sms, s);
      if (e != cudaSuccess) return e;
    }
    {
      ProfScope p(m, NC_K_ATTN, s);
      const nc::KvPrefix pre = prefix_view(kv, l);
      e = nc::k_dec_attn(kv->q, kc, vc, kv->pos_ws, kv->valid, B, H, kv->max_seq, kv->attn_chunk, kv->attn_splits,
                         kv->part, kv->counters, kv->y, s, &pre);
      if (e != cudaSuccess) return e;
    }
    {
      ProfScope p(m, NC_K_GEMM, s);
      e = nc::k_dec_linear(1 /*bf16*/, 1 /*resid*/, w.wo, d, H * 128, B, nullptr, nullptr, 32, eps, kv->y, kv->part,
                           kv->counters, kv->x, kv->ss, nullptr, nullptr, nullptr, kv->max_seq, H, kv->pos_ws,
                           kv->valid, kv->rope, nullptr, nullptr, 0.f, nullptr, nullptr, nullptr, m->status, sms, s);
      if (e != cudaSuccess) return e;
      e = nc::k_dec_linear(0 /*norm*/, 2 /*relu2*/, w.wfc, F, d, B, kv->x, kv->ss, 32, eps, nullptr, kv->part,
                           kv->counters, nullptr, nullptr, kv->f, nullptr, nullptr, kv->max_seq, H, kv->pos_ws,
                           kv->valid, kv->rope, nullptr, nullptr, 0.f, nullptr, nullptr, nullptr, m->status, sms, s);
      if (e != cudaSuccess) return e;
      e = nc::k_dec_linear(1 /*bf16*/, 1 /*resid*/, w.wproj, d, F, B, nullptr, nullptr, 32, eps, kv->f, kv->part,
                           kv->counters, kv->x, kv->ss, nullptr, nullptr, nullptr, kv->max_seq, H, kv->pos_ws,
                           kv->valid, kv->rope, nullptr, nullptr, 0.f, nullptr, nullptr, nullptr, m->status, sms, s);
      if (e != cudaSuccess) return e;
    }
  }
  {
    ProfScope p(m, NC_K_HEAD, s);
    e = nc::k_dec_linear(0 /*norm*/, 3 /*lmhead*/, m->wlm, V, d, B, kv->x, kv->ss, 32, eps, nullptr, kv->part,
                         kv->counters, nullptr, nullptr, nullptr, nullptr, nullptr, kv->max_seq, H, kv->pos_ws,
                         kv->valid, kv->rope, logits, noise, c.softcap, kv->cand_v, kv->cand_i, next, m->status, sms,
                         s);
  }
  return e == cudaSuccess ? sampled_pick(m, kv, logits, B, V, V, noise, kv->valid, next, s) : e;
}

// Replay the cached graph of the decode step when the call matches the last
// captured one; otherwise capture a new graph (on the cache's own stream) and
// launch it. Profiling runs the launches directly so that events can bracket
// them.
int decode_fast(nc_model *m, nc_kv *kv, const int32_t *tokens, const int32_t *positions, int B, const float *noise,
                float *logits, int32_t *next, cudaStream_t s) {
  if (m->prof) {
    cudaError_t e = decode_fast_launches(m, kv, tokens, positions, B, noise, logits, next, s);
    if (e != cudaSuccess) return fail(NC_ECUDA, "decode launch failed: %s", cudaGetErrorString(e));
    return NC_OK;
  }
  nc_kv::GraphKey key;
  memset(&key, 0, sizeof key);  // compared bytewise, padding included
  key.tokens = tokens;
  key.positions = positions;
  key.noise = noise;
  key.logits = logits;
  key.next = next;
  key.B = B;
  key.temperature = kv->temperature;
  key.top_k = kv->top_k;
  const bool same = memcmp(&key, &kv->graph_key, sizeof key) == 0;
  if (!same || !kv->graph_ready) {
    // a new call shape runs directly; the graph is captured once it repeats
    if (kv->graph) {
      cudaGraphExecDestroy(kv->graph);
      kv->graph = nullptr;
    }
    kv->graph_key = key;
    kv->graph_ready = true;
    cudaError_t e = decode_fast_launches(m, kv, tokens, positions, B, noise, logits, next, s);
    if (e != cudaSuccess) return fail(NC_ECUDA, "decode launch failed: %s", cudaGetErrorString(e));
    return NC_OK;
  }
  if (!kv->graph) {
    if (kv->graph) {
      cudaGraphExecDestroy(kv->graph);
      kv->graph = nullptr;
    }
    unsigned long long n0 = nc::g_launches.load();
    NC_CUDA_TRY(cudaStreamBeginCapture(kv->cap_stream, cudaStreamCaptureModeThreadLocal));
    cudaError_t e = decode_fast_launches(m, kv, tokens, positions, B, noise, logits, next, kv->cap_stream);
    cudaGraph_t g = nullptr;
    cudaError_t e2 = cudaStreamEndCapture(kv->cap_stream, &g);
    if (e != cudaSuccess || e2 != cudaSuccess) {
      if (g) cudaGraphDestroy(g);
      cudaGetLastError();
      return fail(NC_ECUDA, "decode graph capture failed: %s",
                  cudaGetErrorString(e != cudaSuccess ? e : e2));
    }
    cudaError_t e3 = cudaGraphInstantiate(&kv->graph, g, 0);
    cudaGraphDestroy(g);
    if (e3 != cudaSuccess) {
      kv->graph = nullptr;
      cudaGetLastError();
      return fail(NC_ECUDA, "decode graph instantiate failed: %s", cudaGetErrorString(e3));
    }
    kv->graph_kernels = nc::g_launches.load() - n0;
    nc::g_launches.fetch_sub(kv->graph_kernels);  // counted when the graph runs
  }
  NC_CUDA_TRY(cudaGraphLaunch(kv->graph, s));
  nc::count_launch(kv->graph_kernels);
  return NC_OK;
}

// The outputs of a prefill (or an appended chunk) whose B * T rows are in
// kv->x: logits of the last or of every position, and the next token.
int prefill_tail(nc_model *m, nc_kv *kv, int B, int T, int logits_mode, float *d_logits, int32_t *d_next,
                 const float *d_noise, cudaStream_t s) {
  const nc_config &c = m->cfg;
  const int M = B * T;
  float *logits;
  long long last_off, row_stride;
  cudaError_t eh = cudaSuccess;
  if (logits_mode == 1) {
    if (d_logits) {
      eh = run_head(m, kv, M, 1, 0, d_logits, nullptr, s);
      logits = d_logits;
      last_off = (long long)(T - 1) * c.vocab;
      row_stride = (long long)T * c.vocab;
    } else {
      eh = run_head(m, kv, B, T, T - 1, kv->logits, nullptr, s);
      logits = kv->logits;
      last_off = 0;
      row_stride = c.vocab;
    }
  } else {
    logits = d_logits ? d_logits : kv->logits;
    if (kv->dec_fast && B <= 32) {
      // last rows -> fused norm + lm_head + softcap + argmax (the decode head kernel)
      ProfScope p(m, NC_K_HEAD, s);
      cudaError_t e = nc::k_gather_rows_ss(kv->x, B, c.d_model, T, T - 1, kv->xl, kv->ss, 32, s);
      if (e == cudaSuccess)
        e = nc::k_dec_linear(0 /*norm*/, 3 /*lmhead*/, m->wlm, c.vocab, c.d_model, B, kv->xl, kv->ss, 32, c.norm_eps,
                             nullptr, kv->part, kv->counters, nullptr, nullptr, nullptr, nullptr, nullptr, kv->max_seq,
                             c.n_head, kv->pos_ws, kv->valid, kv->rope, logits, d_noise, c.softcap, kv->cand_v,
                             kv->cand_i, d_next, m->status, m->num_sms, s);
      if (e == cudaSuccess) e = sampled_pick(m, kv, logits, B, c.vocab, c.vocab, d_noise, nullptr, d_next, s);
      if (e != cudaSuccess) return fail(NC_ECUDA, "prefill head launch failed: %s", cudaGetErrorString(e));
      return NC_OK;
    }
    eh = run_head(m, kv, B, T, T - 1, logits, nullptr, s);
    last_off = 0;
    row_stride = c.vocab;
  }
  if (eh != cudaSuccess) return fail(NC_ECUDA, "prefill head launch failed: %s", cudaGetErrorString(eh));
  if (d_next) {
    if (kv->sampling()) {
      NC_CUDA_TRY(sampled_pick(m, kv, logits + last_off, B, c.vocab, row_stride, d_noise, nullptr, d_next, s));
    } else {
      ProfScope p(m, NC_K_HEAD, s);
      nc::k_argmax_rows(logits + last_off, B, c.vocab, row_stride, d_noise, d_next, nullptr, s);
    }
  }
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

}  // namespace

namespace nc {
// Record a message for nc_last_error() from other translation units.
int set_error(int code, const char *msg) { return fail(code, "%s", msg); }

cudaError_t ensure_smem_attr(const void *func, size_t bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static std::mutex mu;
  static std::map<std::pair<const void *, int>, size_t> done;
  std::lock_guard<std::mutex> lock(mu);
  size_t &have = done[std::make_pair(func, dev)];
  if (bytes <= have) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) have = bytes;
  return e;
}
}  // namespace nc

extern "C" {

const char *nc_last_error(void) { return g_err.c_str(); }

int nc_model_create(const nc_config *cfg, const void *host_blob, size_t blob_bytes, nc_model **out) {
  if (!out) return fail(NC_EINVAL, "out is NULL");
  *out = nullptr;
  int rc = check_config(cfg);
  if (rc) return rc;
  if (!host_blob) return fail(NC_EINVAL, "blob is NULL");
  size_t elem = cfg->dtype == NC_F32 ? 4 : 2;
  size_t want = blob_elems(*cfg) * elem;
  if (blob_bytes != want)
    return fail(NC_EINVAL, "blob has %zu bytes, config needs %zu", blob_bytes, want);
  nc_model *m = new nc_model();
  m->cfg = *cfg;
  m->elem = elem;
  m->blob_bytes = blob_bytes;
  cudaError_t e = cudaGetDevice(&m->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&m->num_sms, cudaDevAttrMultiProcessorCount, m->device);
  if (e == cudaSuccess) e = cudaMalloc(&m->blob, blob_bytes);
  if (e == cudaSuccess) e = cudaMemcpy(m->blob, host_blob, blob_bytes, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMalloc(&m->status, sizeof(uint32_t));
  if (e == cudaSuccess) e = cudaMemset(m->status, 0, sizeof(uint32_t));
  if (e != cudaSuccess) {
    int code = (e == cudaErrorMemoryAllocation) ? NC_ENOMEM : NC_ECUDA;
    nc_model_destroy(m);
    cudaGetLastError();
    return fail(code, "model allocation/copy failed: %s", cudaGetErrorString(e));
  }
  const nc_config &c = *cfg;
  size_t d = c.d_model, qd = (size_t)c.n_head * c.head_dim, kd = (size_t)c.n_kv_head * c.head_dim;
  size_t F = c.mlp_hidden, V = c.vocab;
  char *p = (char *)m->blob;
  m->wte = p;
  p += V * d * elem;
  m->layers.resize(c.depth);
  for (int l = 0; l < c.depth; l++) {
    nc_layer_w &w = m->layers[l];
    w.wqkv = p;
    p += (qd + 2 * kd) * d * elem;
    w.wo = p;
    p += d * qd * elem;
    w.wfc = p;
    p += F * d * elem;
    w.wproj = p;
    p += d * F * elem;
  }
  m->wlm = p;
  m->fast = c.dtype == NC_BF16;
  *out = m;
  return NC_OK;
}

void nc_model_destroy(nc_model *m) {
  if (!m) return;
  cudaDeviceSynchronize();
  for (auto &r : m->prof_recs) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  for (cudaEvent_t e : m->event_pool) cudaEventDestroy(e);
  cudaFree(m->blob);
  cudaFree(m->status);
  delete m;
}

int nc_device_status(nc_model *m, uint32_t *out_bits) {
  if (!m || !out_bits) return fail(NC_EINVAL, "null argument");
  NC_CUDA_TRY(cudaDeviceSynchronize());
  NC_CUDA_TRY(cudaMemcpy(out_bits, m->status, sizeof(uint32_t), cudaMemcpyDeviceToHost));
  NC_CUDA_TRY(cudaMemset(m->status, 0, sizeof(uint32_t)));
  return NC_OK;
}

int nc_kv_create(const nc_model *model, int max_batch, int max_seq, nc_kv **out) {
  if (!out) return fail(NC_EINVAL, "out is NULL");
  *out = nullptr;
  if (!model) return fail(NC_EINVAL, "model is NULL");
  if (max_batch <= 0 || max_seq <= 0) return fail(NC_EINVAL, "max_batch and max_seq must be positive");
  const nc_config &c = model->cfg;
  nc_kv *kv = new nc_kv();
  kv->model = const_cast<nc_model *>(model);
  kv->max_batch = max_batch;
  kv->max_seq = max_seq;
  size_t kd = (size_t)c.n_kv_head * c.head_dim, elem = model->elem;
  kv->layer_elems = (size_t)max_batch * max_seq * kd;
  kv->max_rows = (size_t)max_batch * max_seq;
  size_t rows = kv->max_rows, d = c.d_model, qd = (size_t)c.n_head * c.head_dim;
  size_t qkv_w = qd + 2 * kd, F = c.mlp_hidden, half = c.head_dim / 2;
  size_t cache_bytes = kv->layer_elems * elem * (size_t)(c.depth > 0 ? c.depth : 1);
  cudaError_t e = cudaSuccess;
  auto alloc = [&](void **p, size_t bytes) {
    if (e == cudaSuccess) e = cudaMalloc(p, bytes ? bytes : 16);
  };
  alloc(&kv->k, cache_bytes);
  alloc(&kv->v, cache_bytes);
  alloc((void **)&kv->len, sizeof(int32_t) * max_batch);
  alloc((void **)&kv->valid, max_batch);
  alloc((void **)&kv->rope, sizeof(float2) * max_seq * half);
  alloc((void **)&kv->x, sizeof(float) * rows * d);
  alloc(&kv->h, elem * rows * (d > qd ? d : qd));
  alloc(&kv->qkv, elem * rows * qkv_w);
  alloc(&kv->q, elem * rows * qd);
  alloc(&kv->y, elem * rows * qd);
  alloc(&kv->f, elem * rows * F);
  alloc((void **)&kv->logits, sizeof(float) * (size_t)max_batch * c.vocab);
  alloc((void **)&kv->pos_ws, sizeof(int32_t) * max_batch);
  alloc((void **)&kv->pre_seq, sizeof(int32_t) * max_batch);
  alloc((void **)&kv->pre_len, sizeof(int32_t) * max_batch);
  kv->link_seq.assign(max_batch, -1);
  kv->dep_count.assign(max_batch, 0);
  if (model->fast && nc::rowops_supported(c)) alloc((void **)&kv->row_ss, sizeof(float) * ((d + 127) / 128) * rows);
  kv->dec_fast = nc::decode_head_supported(c);
  if (kv->dec_fast) {
    int nb = max_batch < 32 ? max_batch : 32;
    kv->part_floats = nc::decode_part_floats(c, nb, max_seq, model->num_sms, &kv->attn_splits, &kv->attn_chunk);
    alloc((void **)&kv->ss, sizeof(float) * (size_t)(c.d_model / 128) * 32);
    alloc((void **)&kv->part, sizeof(float) * kv->part_floats);
    alloc((void **)&kv->counters, sizeof(unsigned) * 1024);
    alloc((void **)&kv->cand_v, sizeof(float) * (size_t)(c.vocab / 128) * 32);
    alloc((void **)&kv->cand_i, sizeof(int) * (size_t)(c.vocab / 128) * 32);
    alloc((void **)&kv->xl, sizeof(float) * (size_t)32 * c.d_model);
    if (e == cudaSuccess) e = cudaMemset(kv->counters, 0, sizeof(unsigned) * 1024);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&kv->cap_stream, cudaStreamNonBlocking);
    // whole-step kernel: tensor maps of the weights and of this cache
    if (e == cudaSuccess && nc::decode_step_plan(c, model->num_sms, &kv->step_plan)) {
      const int nmaps = nc::decode_step_maps_count(c);
      std::vector<CUtensorMap> maps(nmaps);
      alloc((void **)&kv->step_maps, sizeof(CUtensorMap) * nmaps);
      alloc(&kv->step_ws, kv->step_plan.ws_bytes);
      if (e == cudaSuccess) e = cudaMemset(kv->step_ws, 0, kv->step_plan.ws_bytes);
      if (e == cudaSuccess && nc::decode_step_build_maps(model, kv->k, kv->v, max_batch, max_seq, kv->step_plan,
                                                          kv->step_ws, maps.data())) {
        e = cudaMemcpy(kv->step_maps, maps.data(), sizeof(CUtensorMap) * nmaps, cudaMemcpyHostToDevice);
        if (e == cudaSuccess) kv->step_grid = nc::decode_step_grid(kv->step_plan, model->num_sms);
        const char *sw = getenv("NC_DECODE_STEP_KERNEL");
        if (sw && sw[0] == '0') kv->step_grid = 0;  // per-kernel decode launches instead
      }
    }
  }
  // zeroed caches: attention may read (and mask) slots past a sequence's length
  if (e == cudaSuccess) e = cudaMemset(kv->k, 0, cache_bytes);
  if (e == cudaSuccess) e = cudaMemset(kv->v, 0, cache_bytes);
  if (e == cudaSuccess) e = cudaMemset(kv->len, 0, sizeof(int32_t) * max_batch);
  if (e == cudaSuccess) e = cudaMemset(kv->pre_seq, 0, sizeof(int32_t) * max_batch);
  if (e == cudaSuccess) e = cudaMemset(kv->pre_len, 0, sizeof(int32_t) * max_batch);
  if (e == cudaSuccess) e = cudaMemset(kv->valid, 0, max_batch);
  if (e == cudaSuccess) {
    // RoPE table: angle pos * base^(-2i/hd) in double, stored as (cos, sin).
    float2 *tab = (float2 *)malloc(sizeof(float2) * max_seq * half);
    if (!tab) {
      e = cudaErrorMemoryAllocation;
    } else {
      for (int p = 0; p < max_seq; p++)
        for (size_t i = 0; i < half; i++) {
          double theta = pow((double)c.rope_base, -2.0 * (double)i / (double)c.head_dim);
          double a = (double)p * theta;
          tab[p * half + i] = make_float2((float)cos(a), (float)sin(a));
        }
      e = cudaMemcpy(kv->rope, tab, sizeof(float2) * max_seq * half, cudaMemcpyHostToDevice);
      free(tab);
    }
  }
  if (e != cudaSuccess) {
    int code = (e == cudaErrorMemoryAllocation) ? NC_ENOMEM : NC_ECUDA;
    nc_kv_destroy(kv);
    cudaGetLastError();
    return fail(code, "kv allocation failed: %s", cudaGetErrorString(e));
  }
  *out = kv;
  return NC_OK;
}


void nc_kv_destroy(nc_kv *kv) {
  if (!kv) return;
  cudaDeviceSynchronize();
  // this cache's own links end; a cache others still read from is freed
  // with their last link
  for (int b = 0; b < (int)kv->link_seq.size(); b++) unlink_seq(kv, b);
  if (kv->n_dependents > 0) {
    kv->destroy_pending = true;
    return;
  }
  free_kv(kv);
}

int nc_kv_lengths(const nc_kv *kv, int n, int32_t *out) {
  if (!kv || !out || n < 0) return fail(NC_EINVAL, "bad argument");
  if (n > kv->max_batch) return fail(NC_ERANGE, "n=%d > max_batch=%d", n, kv->max_batch);
  NC_CUDA_TRY(cudaDeviceSynchronize());
  NC_CUDA_TRY(cudaMemcpy(out, kv->len, sizeof(int32_t) * n, cudaMemcpyDeviceToHost));
  return NC_OK;
}

int nc_prefill(nc_model *m, nc_kv *kv, const int32_t *d_tokens, int B, int T, int logits_mode, float *d_logits,
               int32_t *d_next, const float *d_noise, void *stream) {
  if (!m || !kv || !d_tokens) return fail(NC_EINVAL, "null model, kv or tokens");
  if (kv->model != m) return fail(NC_EINVAL, "kv belongs to another model");
  if (B < 1 || T < 1) return fail(NC_EINVAL, "B and T must be >= 1");
  if (logits_mode != 0 && logits_mode != 1) return fail(NC_EINVAL, "logits_mode must be 0 (last) or 1 (all)");
  if (B > kv->max_batch) return fail(NC_ERANGE, "B=%d > max_batch=%d", B, kv->max_batch);
  if (T > kv->max_seq) return fail(NC_ERANGE, "T=%d > max_seq=%d", T, kv->max_seq);
  int who = -1;
  if (replace_blocked(kv, 0, B, &who))
    return fail(NC_EINVAL, "sequence %d is the shared prefix of another sequence (nc_kv_fork_shared)", who);
  for (int b = 0; b < B; b++) unlink_seq(kv, b);
  const nc_config &c = m->cfg;
  cudaStream_t s = as_stream(stream);
  int M = B * T;
  {
    ProfScope p(m, NC_K_MISC, s);
    nc::k_prefill_begin(kv->len, kv->valid, kv->pre_len, B, T, s);
    nc::k_embed_norm(c.dtype, d_tokens, M, m->wte, c.d_model, c.vocab, c.norm_eps, kv->x, m->status, s);
  }
  nc::RowMap rm{T, nullptr};
  const int rc = run_blocks(m, kv, M, rm, s);
  if (rc != NC_OK) return rc;
  return prefill_tail(m, kv, B, T, logits_mode, d_logits, d_next, d_noise, s);
}

int nc_prefill_extend(nc_model *m, nc_kv *kv, const int32_t *d_tokens, int B, int T, int logits_mode,
                      float *d_logits, int32_t *d_next, const float *d_noise, void *stream) {
  if (!m || !kv || !d_tokens) return fail(NC_EINVAL, "null model, kv or tokens");
  if (kv->model != m) return fail(NC_EINVAL, "kv belongs to another model");
  if (B < 1 || T < 1) return fail(NC_EINVAL, "B and T must be >= 1");
  if (logits_mode != 0 && logits_mode != 1) return fail(NC_EINVAL, "logits_mode must be 0 (last) or 1 (all)");
  if (B > kv->max_batch) return fail(NC_ERANGE, "B=%d > max_batch=%d", B, kv->max_batch);
  if (T > kv->max_seq) return fail(NC_ERANGE, "T=%d > max_seq=%d", T, kv->max_seq);
  const nc_config &c = m->cfg;
  cudaStream_t s = as_stream(stream);
  const int M = B * T;
  {
    ProfScope p(m, NC_K_MISC, s);
    nc::k_extend_begin(kv->len, kv->valid, kv->pos_ws, B, T, kv->max_seq, m->status, s);
    nc::k_embed_norm(c.dtype, d_tokens, M, m->wte, c.d_model, c.vocab, c.norm_eps, kv->x, m->status, s);
  }
  nc::RowMap rm{T, nullptr, kv->pos_ws};  // rows at positions len[b] + t
  const int rc = run_blocks(m, kv, M, rm, s);
  if (rc != NC_OK) return rc;
  return prefill_tail(m, kv, B, T, logits_mode, d_logits, d_next, d_noise, s);
}

int nc_decode_step(nc_model *m, nc_kv *kv, const int32_t *d_tokens, const int32_t *d_positions, int B,
                   const float *d_noise, float *d_logits, int32_t *d_next, void *stream) {
  if (!m || !kv || !d_tokens) return fail(NC_EINVAL, "null model, kv or tokens");
  if (kv->model != m) return fail(NC_EINVAL, "kv belongs to another model");
  if (B < 1) return fail(NC_EINVAL, "B must be >= 1");
  if (B > kv->max_batch) return fail(NC_ERANGE, "B=%d > max_batch=%d", B, kv->max_batch);
  const nc_config &c = m->cfg;
  cudaStream_t s = as_stream(stream);
  float *logits = d_logits ? d_logits : kv->logits;
  if (kv->dec_fast && ((kv->step_grid > 0 && nc::decode_step_supported(c, B)) || nc::decode_fast_supported(c, B)))
    return decode_fast(m, kv, d_tokens, d_positions, B, d_noise, logits, d_next, s);
  if (!d_positions) {
    // positions default to the current lengths
    NC_CUDA_TRY(cudaMemcpyAsync(kv->pos_ws, kv->len, sizeof(int32_t) * B, cudaMemcpyDeviceToDevice, s));
    d_positions = kv->pos_ws;
  }
  {
    ProfScope p(m, NC_K_MISC, s);
    nc::k_decode_begin(d_positions, kv->len, kv->valid, B, kv->max_seq, m->status, s);
    nc::k_embed_norm(c.dtype, d_tokens, B, m->wte, c.d_model, c.vocab, c.norm_eps, kv->x, m->status, s);
  }
  nc::RowMap rm{1, d_positions};
  const int rc = run_blocks(m, kv, B, rm, s);
  if (rc != NC_OK) return rc;
  const cudaError_t eh = run_head(m, kv, B, 1, 0, logits, kv->valid, s);
  if (eh != cudaSuccess) return fail(NC_ECUDA, "decode head launch failed: %s", cudaGetErrorString(eh));
  if (d_next) {
    if (kv->sampling()) {
      NC_CUDA_TRY(sampled_pick(m, kv, logits, B, c.vocab, c.vocab, d_noise, kv->valid, d_next, s));
    } else {
      ProfScope p(m, NC_K_HEAD, s);
      nc::k_argmax_rows(logits, B, c.vocab, c.vocab, d_noise, d_next, kv->valid, s);
    }
  }
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

namespace {
int kv_fork_impl(nc_kv *src, int src_seq, nc_kv *dst, int dst_first, int n, bool shared, void *stream) {
  if (!src || !dst) return fail(NC_EINVAL, "null cache");
  if (src->model != dst->model) return fail(NC_EINVAL, "caches belong to different models");
  if (n < 1) return fail(NC_EINVAL, "n must be >= 1");
  if (src_seq < 0 || src_seq >= src->max_batch) return fail(NC_ERANGE, "src_seq out of range");
  if (dst_first < 0 || dst_first + n > dst->max_batch) return fail(NC_ERANGE, "destinations out of range");
  if (dst->max_seq < src->max_seq)
    return fail(NC_ERANGE, "destination max_seq %d < source max_seq %d", dst->max_seq, src->max_seq);
  if (src == dst && src_seq >= dst_first && src_seq < dst_first + n)
    return fail(NC_EINVAL, "source sequence is among the destinations");
  int who = -1;
  if (replace_blocked(dst, dst_first, n, &who))
    return fail(NC_EINVAL, "sequence %d is the shared prefix of another sequence (nc_kv_fork_shared)", who);
  // shared rows are read from the source's own prefix sequence if it has one
  nc_kv *root = shared && src->link_seq[src_seq] >= 0 ? src->prefix_src : src;
  const int root_seq = shared && src->link_seq[src_seq] >= 0 ? src->link_seq[src_seq] : src_seq;
  if (shared) {
    if (root == dst && root_seq >= dst_first && root_seq < dst_first + n)
      return fail(NC_EINVAL, "the shared prefix's sequence is among the destinations");
    int inside = 0;
    for (int b = dst_first; b < dst_first + n; b++) inside += dst->link_seq[b] >= 0;
    if (dst->prefix_src && dst->prefix_src != root && dst->n_links - inside > 0)
      return fail(NC_EINVAL, "the destination cache already shares prefixes with another cache");
  }
  const nc_config &c = src->model->cfg;
  cudaStream_t s = as_stream(stream);
  // the source's shared rows, as they are before any link changes below
  const nc::KvPrefix src_pre = prefix_view(src, 0);
  const size_t pre_layer = src->prefix_src ? src->prefix_src->layer_elems : 0;
  for (int b = dst_first; b < dst_first + n; b++) unlink_seq(dst, b);
  if (shared) {
    if (dst->prefix_src != root) {
      // the step kernel reads shared rows through the prefix cache's maps
      if (dst->step_maps && dst->step_grid > 0) {
        std::vector<CUtensorMap> pm(2);
        if (!nc::decode_step_prefix_maps(root->k, root->v, c, root->max_batch, root->max_seq, pm.data()))
          return fail(NC_ECUDA, "tensor maps of the shared prefix");
        NC_CUDA_TRY(cudaMemcpy(dst->step_maps + nc::decode_step_prefix_map_index(c), pm.data(),
                               sizeof(CUtensorMap) * 2, cudaMemcpyHostToDevice));
      }
      if (dst->graph) {  // the captured step carries the old prefix shape
        cudaGraphExecDestroy(dst->graph);
        dst->graph = nullptr;
      }
      dst->graph_ready = false;
    }
    dst->prefix_src = root;
    for (int b = dst_first; b < dst_first + n; b++) {
      dst->link_seq[b] = root_seq;
      dst->n_links++;
      root->dep_count[root_seq]++;
      root->n_dependents++;
    }
  }
  ProfScope p(src->model, NC_K_MISC, s);
  nc::k_kv_fork((int)src->model->elem, src->k, src->v, src->layer_elems, src->max_seq, src_seq, src->len, src_pre,
                pre_layer, dst->k, dst->v, dst->layer_elems, dst->max_seq, dst_first, n, dst->len, dst->pre_seq,
                dst->pre_len, shared, c.depth, c.n_kv_head * c.head_dim, src->model->status, s);
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}
}  // namespace

int nc_kv_fork(nc_kv *src, int src_seq, nc_kv *dst, int dst_first, int n, void *stream) {
  return kv_fork_impl(src, src_seq, dst, dst_first, n, false, stream);
}

int nc_kv_fork_shared(nc_kv *src, int src_seq, nc_kv *dst, int dst_first, int n, void *stream) {
  return kv_fork_impl(src, src_seq, dst, dst_first, n, true, stream);
}

int nc_kv_set_sampling(nc_kv *kv, float temperature, int top_k) {
  if (!kv) return fail(NC_EINVAL, "kv is NULL");
  if (!(temperature >= 0.f) || !isfinite(temperature)) return fail(NC_EINVAL, "temperature must be finite and >= 0");
  if (top_k < 0) return fail(NC_EINVAL, "top_k must be >= 0");
  kv->temperature = temperature;
  kv->top_k = top_k;
  return NC_OK;
}

int nc_decode_trace(nc_kv *kv, unsigned long long *d_buf, size_t n_words, int *grid, int *phases) {
  if (!kv) return fail(NC_EINVAL, "kv is NULL");
  const nc_config &c = kv->model->cfg;
  const int g = kv->step_grid, P = 3 + 5 * c.depth;
  if (grid) *grid = g;
  if (phases) *phases = P;
  if (d_buf && g == 0) return fail(NC_EUNSUP, "this cache has no whole-step decode kernel to trace");
  if (d_buf && n_words < (size_t)g * P * 8)
    return fail(NC_ERANGE, "trace buffer holds %zu words, the step kernel writes %zu", n_words, (size_t)g * P * 8);
  kv->step_trace = d_buf;
  if (kv->graph) {  // the captured launch carries the old trace pointer
    cudaGraphExecDestroy(kv->graph);
    kv->graph = nullptr;
  }
  kv->graph_ready = false;
  return NC_OK;
}

int nc_profile_enable(nc_model *m, int on) {
  if (!m) return fail(NC_EINVAL, "model is NULL");
  m->prof = on != 0;
  return NC_OK;
}

int nc_profile_read(nc_model *m, double *ms, long long *launches) {
  if (!m) return fail(NC_EINVAL, "model is NULL");
  NC_CUDA_TRY(cudaDeviceSynchronize());
  double t[NC_K_COUNT] = {0};
  long long n[NC_K_COUNT] = {0};
  for (auto &r : m->prof_recs) {
    float e = 0.f;
    if (cudaEventElapsedTime(&e, r.a, r.b) == cudaSuccess) t[r.cls] += e;
    n[r.cls] += r.launches;
    m->event_pool.push_back(r.a);
    m->event_pool.push_back(r.b);
  }
  m->prof_recs.clear();
  cudaGetLastError();
  for (int i = 0; i < NC_K_COUNT; i++) {
    if (ms) ms[i] = t[i];
    if (launches) launches[i] = n[i];
  }
  return NC_OK;
}

unsigned long long nc_launch_count(void) { return nc::g_launches.load(); }

static int kernel_status_init(uint32_t **status, int *sms) {
  static uint32_t *st = nullptr;
  static int n = 0;
  if (!st) {
    int dev = 0;
    NC_CUDA_TRY(cudaGetDevice(&dev));
    NC_CUDA_TRY(cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev));
    NC_CUDA_TRY(cudaMalloc(&st, sizeof(uint32_t)));
    NC_CUDA_TRY(cudaMemset(st, 0, sizeof(uint32_t)));
  }
  *status = st;
  *sms = n;
  return NC_OK;
}

int nc_attention_prefill_bf16(const void *d_q, const void *d_k, const void *d_v, int B, int T, int H, int hd,
                              int max_seq, void *d_y, void *stream) {
  if (!d_q || !d_k || !d_v || !d_y) return fail(NC_EINVAL, "null pointer");
  if (B <= 0 || T <= 0 || H <= 0 || hd <= 0 || (hd & 1) || max_seq < T) return fail(NC_EINVAL, "bad attention shape");
  uint32_t *status;
  int sms;
  int rc = kernel_status_init(&status, &sms);
  if (rc) return rc;
  cudaStream_t s = as_stream(stream);
  if (nc::attn_prefill_tc_supported(H, 1, hd)) {
    const cudaError_t e = nc::k_attn_prefill_tc(d_q, d_k, d_v, B, T, H, 1, B, max_seq, d_y, status, s);
    if (e != cudaSuccess) return fail(NC_ECUDA, "attention launch failed: %s", cudaGetErrorString(e));
    return NC_OK;
  }
  nc::RowMap rm{T, nullptr};
  nc::k_attention_generic(NC_BF16, d_q, d_k, d_v, rm, B * T, H, 1, hd, max_seq, d_y, s);
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

static int device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return n;
}

size_t nc_attention_decode_workspace_bytes(int B, int max_seq) {
  if (B <= 0 || max_seq <= 0) return 0;
  int sms = device_sms(), chunk, splits;
  if (sms <= 0) sms = 148;
  nc::attn_decode_plan(B, max_seq, sms, &chunk, &splits);
  return nc::attn_decode_partial_floats(B, splits) * sizeof(float) + sizeof(unsigned) * (size_t)B;
}

int nc_attention_decode_bf16(const void *d_q, const void *d_k, const void *d_v, const int32_t *d_pos, int B, int H,
                             int max_seq, void *d_y, void *d_workspace, size_t workspace_bytes, void *stream) {
  if (!d_q || !d_k || !d_v || !d_pos || !d_y || !d_workspace) return fail(NC_EINVAL, "null pointer");
  if (B <= 0 || H <= 0 || H > 16 || max_seq <= 0) return fail(NC_EINVAL, "bad decode attention shape");
  int sms = device_sms(), chunk, splits;
  if (sms <= 0) return fail(NC_ECUDA, "no CUDA device");
  nc::attn_decode_plan(B, max_seq, sms, &chunk, &splits);
  const size_t part = nc::attn_decode_partial_floats(B, splits);
  if (workspace_bytes < part * sizeof(float) + sizeof(unsigned) * (size_t)B)
    return fail(NC_EINVAL, "workspace of %zu bytes is too small", workspace_bytes);
  float *pf = (float *)d_workspace;
  unsigned *counters = (unsigned *)(pf + part);
  cudaError_t e = nc::k_dec_attn(d_q, d_k, d_v, d_pos, nullptr, B, H, max_seq, chunk, splits, pf, counters, d_y,
                                 as_stream(stream));
  if (e != cudaSuccess) return fail(NC_ECUDA, "decode attention launch: %s", cudaGetErrorString(e));
  return NC_OK;
}

int nc_sample_topk(const float *d_logits, int B, int V, long long row_stride, const float *d_noise, float temperature,
                   int top_k, int32_t *d_next, void *stream) {
  if (!d_logits || !d_next) return fail(NC_EINVAL, "null pointer");
  if (B < 1 || V < 1 || row_stride < V) return fail(NC_EINVAL, "bad shape (B, V >= 1, row_stride >= V)");
  if (!(temperature >= 0.f) || !isfinite(temperature)) return fail(NC_EINVAL, "temperature must be finite and >= 0");
  if (top_k < 0) return fail(NC_EINVAL, "top_k must be >= 0");
  const cudaError_t e =
      nc::k_sample_topk(d_logits, B, V, row_stride, d_noise, temperature, top_k, nullptr, d_next, as_stream(stream));
  if (e != cudaSuccess) return fail(NC_ECUDA, "sampling launch failed: %s", cudaGetErrorString(e));
  return NC_OK;
}

int nc_gemm_bf16(const void *d_A, int lda, const void *d_W, int M, int N, int K, int epi, void *d_out, int ldo,
                 float cap, void *stream) {
  if (!d_A || !d_W || !d_out) return fail(NC_EINVAL, "null pointer");
  if (M <= 0 || N <= 0 || K <= 0 || lda < K || ldo < N) return fail(NC_EINVAL, "bad GEMM shape");
  if (epi < NC_EPI_STORE || epi > NC_EPI_SOFTCAP) return fail(NC_EINVAL, "unknown epilogue %d", epi);
  uint32_t *status;
  int sms;
  int rc = kernel_status_init(&status, &sms);
  if (rc) return rc;
  cudaStream_t s = as_stream(stream);
  if (M >= 128 && nc::gemm_tc_supported(M, N, K, lda)) {
    const cudaError_t e = nc::k_gemm_tc(epi, d_A, lda, d_W, M, N, K, d_out, ldo, cap, status, sms, s);
    if (e != cudaSuccess) return fail(NC_ECUDA, "GEMM launch failed: %s", cudaGetErrorString(e));
    return NC_OK;
  }
  nc::k_gemm_generic(NC_BF16, epi, d_A, lda, d_W, M, N, K, d_out, ldo, cap, nullptr, s);
  NC_CUDA_TRY(cudaGetLastError());
  return NC_OK;
}

}  // extern "C"
