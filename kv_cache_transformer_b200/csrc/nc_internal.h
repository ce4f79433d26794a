// nc_internal.h — engine objects and kernel launchers (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <vector>

#include "nc.h"
#include "nc_common.cuh"
#include <cuda.h>

struct nc_layer_w {
  const void *wqkv;   // [(H + 2*Hkv)*hd, d]: Wq, Wk, Wv are adjacent in the blob
  const void *wo;     // [d, H*hd]
  const void *wfc;    // [F, d]
  const void *wproj;  // [d, F]
};

struct nc_model {
  nc_config cfg;
  int device = 0;
  int num_sms = 0;
  size_t elem = 4;             // bytes per stored element
  void *blob = nullptr;        // device copy of the whole weight blob
  size_t blob_bytes = 0;
  const void *wte = nullptr;   // [V, d]
  const void *wlm = nullptr;   // [V, d]
  std::vector<nc_layer_w> layers;
  uint32_t *status = nullptr;  // device status word (NC_DEV_* bits)
  bool fast = false;           // bf16 + shapes the sm_100a kernels cover
  // tracing (nc_profile_*)
  bool prof = false;
  struct ProfRec {
    int cls;
    long long launches;
    cudaEvent_t a, b;
  };
  std::vector<ProfRec> prof_recs;
  std::vector<cudaEvent_t> event_pool;
};

namespace nc {
// Shared-prefix view for attention (nc_kv_fork_shared): key/value row j < len[b]
// of sequence b is row j of sequence seq[b] of the prefix cache (k, v: that
// cache's K and V at the layer being read, max_seq rows per sequence). len ==
// nullptr: every row is the sequence's own.
struct KvPrefix {
  const void *k = nullptr, *v = nullptr;
  const int32_t *seq = nullptr, *len = nullptr;
  int max_seq = 0;
};

// Launch plan of the whole-step decode kernel (nc_step.cu): CTAs, the rows
// each CTA owns in every linear phase, its shared-memory ring and the layout
// of its device workspace.
struct StepPlan {
  int grid = 0;                      // CTAs, one per SM (0 = no plan)
  int n_qkv = 0, r_q = 0;            // QKV units of r_q rows (r_q / 2 RoPE pairs of one head)
  int r_o = 0, r_f = 0, r_p = 0;     // rows per CTA: O projection, MLP fc, MLP projection
  int s_p = 0;                       // K splits of the MLP projection
  int r_h = 0;                       // lm_head rows per CTA
  int n_o = 0, n_f = 0, n_p = 0, n_h = 0;  // units of each phase
  int slots = 0;                     // 32 KB ring slots
  size_t smem = 0;                   // dynamic shared memory per CTA
  size_t ws_bytes = 0;               // device workspace
  size_t off_ctr = 0, off_x0 = 0, off_x1 = 0, off_xb0 = 0, off_xb1 = 0, off_y = 0, off_f = 0, off_qk = 0,
         off_cv = 0, off_ci = 0, off_ap = 0, off_pp = 0;
};
}  // namespace nc

struct nc_kv {
  nc_model *model = nullptr;
  int max_batch = 0, max_seq = 0;
  size_t layer_elems = 0;      // max_batch * max_seq * Hkv * hd
  void *k = nullptr, *v = nullptr;  // [depth][max_batch][max_seq][Hkv*hd]
  int32_t *len = nullptr;      // device [max_batch]
  uint8_t *valid = nullptr;    // device [max_batch]: row takes part in this decode step
  float2 *rope = nullptr;      // device [max_seq][hd/2] (cos, sin), angles in double on the host
  // workspace sized for max_rows = max_batch * max_seq activation rows
  size_t max_rows = 0;
  float *x = nullptr;          // [rows, d] fp32 residual stream
  void *h = nullptr;           // [rows, max(d, H*hd)] normed activations (storage type)
  void *qkv = nullptr;         // [rows, (H + 2*Hkv)*hd]
  void *q = nullptr;           // [rows, H*hd] rotated + normed queries
  void *y = nullptr;           // [rows, H*hd] attention output
  void *f = nullptr;           // [rows, F] relu^2 hidden
  float *logits = nullptr;     // [max_batch, V] when the caller passes no logits buffer
  // decode fast path (bf16, head_dim 128, one KV head, B <= 32)
  bool dec_fast = false;
  int32_t *pos_ws = nullptr;   // [max_batch] positions of the current step
  float *ss = nullptr;         // [d/128][32] partial sums of squares of x rows
  float *part = nullptr;       // split-K / split-KV partials
  size_t part_floats = 0;
  unsigned *counters = nullptr;  // [1024], zero between launches
  float *cand_v = nullptr;     // [V/128][32] per-tile argmax winners
  int *cand_i = nullptr;
  float *xl = nullptr;         // [32][d] last-position rows of a prefill, for the fused lm_head
  float *row_ss = nullptr;     // [ceil(d/128)][max_rows] per-128-column sums of squares of x rows (prefill)
  // whole-step decode kernel (nc_step.cu)
  int step_grid = 0;           // CTAs of the step kernel, 0 = not available
  nc::StepPlan step_plan;
  CUtensorMap *step_maps = nullptr;  // device copy of the step kernel's tensor maps
  void *step_ws = nullptr;     // its workspace (activations, partials, counters)
  unsigned long long *step_trace = nullptr;  // caller's phase-timestamp buffer (nc_decode_trace), or null
  // shared prefixes (nc_kv_fork_shared): sequence b reads its first
  // pre_len[b] key/value rows of every layer from sequence pre_seq[b] of
  // prefix_src (a multiple of 64; 0 = none)
  int32_t *pre_seq = nullptr, *pre_len = nullptr;  // device [max_batch]
  nc_kv *prefix_src = nullptr;   // the cache those rows live in (host bookkeeping below mirrors the device)
  std::vector<int> link_seq;     // per sequence: the prefix_src sequence it reads from, -1 none
  int n_links = 0;               // live links of this cache into prefix_src
  std::vector<int> dep_count;    // per sequence: live links of any cache into it
  int n_dependents = 0;          // live links of any cache into this one
  bool destroy_pending = false;  // destroyed while links into it were live: freed with the last link
  // sampled token pick (nc_kv_set_sampling): temperature 1 and top_k 0 are
  // the plain argmax(logits + noise)
  float temperature = 1.f;
  int top_k = 0;
  bool sampling() const { return temperature != 1.f || top_k > 0; }
  int attn_chunk = 0, attn_splits = 0;
  // CUDA graph of the last decode step's launches, replayed while the call's
  // pointers and batch stay the same
  cudaStream_t cap_stream = nullptr;
  cudaGraphExec_t graph = nullptr;
  struct GraphKey {
    const void *tokens, *positions, *noise, *logits, *next;
    int B;
    float temperature;
    int top_k;
  } graph_key = {};
  bool graph_ready = false;    // graph_key has run once directly
  unsigned long long graph_kernels = 0;
};

namespace nc {

// Set the message returned by nc_last_error(); returns code.
int set_error(int code, const char *msg);

// Raise a kernel's dynamic shared-memory limit to at least `bytes` on the
// current device. The attribute is per device, so it is tracked per (kernel,
// device); thread-safe.
cudaError_t ensure_smem_attr(const void *func, size_t bytes);

// Kernels launched by this library (nc_launch_count).
extern std::atomic<unsigned long long> g_launches;
inline void count_launch(unsigned long long n = 1) { g_launches.fetch_add(n, std::memory_order_relaxed); }

enum Epi { EPI_STORE = 0, EPI_RELU2 = 1, EPI_RESID = 2, EPI_SOFTCAP = 3, EPI_QKV = 4, EPI_RESID_X = 5 };

// Extra operands of the fused prefill epilogues of the tensor-core GEMM.
//  ss_in/nss   the A rows are bf16(x) of an un-normed residual row: every
//              accumulator row is scaled by 1/sqrt(sum_j ss_in[j*M + row]/K + eps)
//              (nss = 0: A is already normed, no scaling); EPI_STORE, EPI_RELU2
//              and EPI_QKV
//  EPI_QKV     columns are the q heads, the k head and the v head (128 each):
//              RoPE + RMS norm of q and k, q to q[row][H][128], k and v to the
//              caches at (row / T, row % T) with row pitch 128, max_seq rows
//              per sequence
//  EPI_RESID_X x += acc as EPI_RESID, plus xb = bf16(x) (row pitch N) and
//              ss_out[j*M + row] = sum of squares of the new x over columns
//              128j .. 128j+127
struct GemmFuse {
  const float *ss_in = nullptr;
  int nss = 0;
  float eps = 0.f;
  void *xb = nullptr;
  float *ss_out = nullptr;
  const float2 *rope = nullptr;
  void *q = nullptr, *kc = nullptr, *vc = nullptr;
  int T = 1, H = 0, Hkv = 1, max_seq = 0;  // query heads, KV heads (the cache row holds Hkv heads)
  // appended chunks: row t of sequence b sits at position off[b] + t, and its
  // keys and values are written only where valid[b] (null: from position 0, all)
  const int32_t *off = nullptr;
  const uint8_t *valid = nullptr;
};

// ---- generic kernels (any even head_dim; fp32 or bf16 storage) ----
void k_prefill_begin(int32_t *len, uint8_t *valid, int32_t *pre_len, int B, int T, cudaStream_t s);
void k_extend_begin(int32_t *len, uint8_t *valid, int32_t *off, int B, int T, int max_seq, uint32_t *status,
                    cudaStream_t s);
void k_decode_begin(const int32_t *positions, int32_t *len, uint8_t *valid, int B, int max_seq,
                    uint32_t *status, cudaStream_t s);
void k_embed_norm(int dtype, const int32_t *tokens, int M, const void *wte, int d, int vocab, float eps,
                  float *x, uint32_t *status, cudaStream_t s);
void k_rmsnorm_rows(int dtype, const float *x, int rows, int d, int src_stride, int src_offset, float eps,
                    void *out, cudaStream_t s);
void k_gemm_generic(int dtype, int epi, const void *A, int lda, const void *W, int M, int N, int K, void *out,
                    int ldo, float cap, const uint8_t *valid_rows, cudaStream_t s);
void k_rope_qknorm_append(int dtype, const void *qkv, RowMap rm, int M, int H, int Hkv, int hd,
                          const float2 *rope, void *q_out, void *kc, void *vc, int max_seq,
                          const uint8_t *valid, float eps, cudaStream_t s);
void k_attention_generic(int dtype, const void *q, const void *kc, const void *vc, RowMap rm, int M, int H,
                         int Hkv, int hd, int max_seq, void *y, cudaStream_t s, const KvPrefix *pre = nullptr);
void k_argmax_rows(const float *logits, int rows, int V, long long row_stride, const float *noise,
                   int32_t *next, const uint8_t *valid, cudaStream_t s);
// Copy (shared == false) or share (true) the rows of sequence src_seq into
// sequences dst_first .. dst_first + n - 1. Copy: every row, the source's
// shared rows read from its prefix cache (src_pre, layer 0 pointers, with
// its per-layer stride pre_layer_elems); the destinations own all their rows.
// Share: the destinations read rows below the shared length (the source's
// own shared length if it has one, else its length rounded down to 64) from
// the source's prefix sequence or the source itself (dst_pre_seq/len set on
// the device) and get a copy of the rest.
void k_kv_fork(int elem_bytes, const void *src_k, const void *src_v, size_t src_layer_elems, int src_max_seq,
               int src_seq, const int32_t *src_len, const KvPrefix &src_pre, size_t pre_layer_elems, void *dst_k,
               void *dst_v, size_t dst_layer_elems, int dst_max_seq, int dst_first, int n, int32_t *dst_len,
               int32_t *dst_pre_seq, int32_t *dst_pre_len, bool shared, int depth, int kd, uint32_t *status,
               cudaStream_t s);


// ---- sm_100a tensor-core GEMM (nc_gemm_tc.cu) ----
bool gemm_tc_supported(int M, int N, int K, int lda);
cudaError_t k_gemm_tc(int epi, const void *A, int lda, const void *W, int M, int N, int K, void *out, int ldo,
                      float cap, uint32_t *status, int num_sms, cudaStream_t s, const GemmFuse *fz = nullptr);


// ---- sm_100a causal MQA / GQA prefill attention (nc_attn_tc.cu) ----
bool attn_prefill_tc_supported(int H, int Hkv, int hd);
cudaError_t k_attn_prefill_tc(const void *q, const void *kc, const void *vc, int B, int T, int H, int Hkv,
                              int max_batch, int max_seq, void *y, uint32_t *status, cudaStream_t s,
                              const int32_t *off = nullptr);


// ---- row-wise prefill kernels for bf16 head_dim-128 models (nc_rowops.cu) ----
bool rowops_supported(const nc_config &c);
cudaError_t k_rows_norm_bf16(const float *x, int rows, int d, float eps, void *h, cudaStream_t s);
cudaError_t k_rope_qk_bf16(const void *qkv, int M, int T, int H, const float2 *rope, void *q_out, void *kc, void *vc,
                           int max_seq, float eps, cudaStream_t s);
cudaError_t k_gather_rows_ss(const float *x, int rows, int d, int stride, int offset, float *xl, float *ss, int ssb,
                             cudaStream_t s);

// ---- decode step kernels (nc_decode.cu) ----
// the per-kernel decode launches (one KV head)
bool decode_fast_supported(const nc_config &c, int B);
// the decode scratch and the fused last-row lm_head + argmax kernel (any KV heads)
bool decode_head_supported(const nc_config &c);
size_t decode_part_floats(const nc_config &c, int max_batch, int max_seq, int num_sms, int *attn_splits,
                          int *attn_chunk);
cudaError_t k_dec_embed(const int32_t *tokens, const int32_t *positions, int32_t *len, int32_t *pos_ws,
                        uint8_t *valid, int B, int max_seq, const void *wte, int d, int vocab, float eps, float *x,
                        float *ss, int ssb, uint32_t *status, cudaStream_t s);
cudaError_t k_dec_linear(int src, int epi, const void *W, int N, int K, int B, const float *x, const float *ss, int ssb,
                         float eps, const void *act, float *part, unsigned *counters, float *xres, float *ss_out,
                         void *out, void *kc, void *vc, int max_seq, int H, const int32_t *pos, const uint8_t *valid,
                         const float2 *rope, float *logits, const float *noise, float cap, float *cand_v, int *cand_i,
                         int32_t *next, uint32_t *status, int num_sms, cudaStream_t s);
void attn_decode_plan(int B, int max_seq, int num_sms, int *chunk, int *splits);
size_t attn_decode_partial_floats(int B, int splits);
cudaError_t k_dec_attn(const void *q, const void *kc, const void *vc, const int32_t *pos, const uint8_t *valid, int B,
                       int H, int max_seq, int chunk, int splits, float *part, unsigned *counters, void *y,
                       cudaStream_t s, const KvPrefix *pre = nullptr);


// ---- sampled token pick (nc_sample.cu) ----
// next[b] = argmax over the top_k largest logits of row b (all when top_k <= 0
// or >= V; the lower index on a tie at the cut) of fl(fl(z / temperature) +
// noise), lowest index on ties; temperature 0 is argmax z. Logit rows are
// `stride` floats apart, noise rows V; rows with valid[b] == 0 are skipped.
cudaError_t k_sample_topk(const float *logits, int B, int V, long long stride, const float *noise, float temperature,
                          int top_k, const uint8_t *valid, int32_t *next, cudaStream_t s);

// ---- whole decode step in one persistent kernel (nc_step.cu) ----
bool decode_step_supported(const nc_config &c, int B);
bool decode_step_plan(const nc_config &c, int num_sms, StepPlan *plan);
int decode_step_maps_count(const nc_config &c);
int decode_step_prefix_map_index(const nc_config &c);
bool decode_step_prefix_maps(const void *kcache, const void *vcache, const nc_config &c, int max_batch, int max_seq,
                             CUtensorMap *out);
bool decode_step_build_maps(const nc_model *m, const void *kcache, const void *vcache, int max_batch, int max_seq,
                            const StepPlan &p, void *ws, CUtensorMap *out);
int decode_step_grid(const StepPlan &p, int num_sms);
cudaError_t k_decode_step(const nc_model *m, const StepPlan &pl, int B, int max_batch, int max_seq,
                          const CUtensorMap *maps_dev, void *ws, const int32_t *tokens, const int32_t *positions,
                          int32_t *len, void *kc, void *vc, const float2 *rope, float *logits, const float *noise,
                          int32_t *next, unsigned long long *trace, uint8_t *valid_out, const int32_t *pre_seq,
                          const int32_t *pre_len, int pmax_batch, int pmax_seq, cudaStream_t s);

}  // namespace nc
