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
  CUtensorMap *step_maps = nullptr;  // device copy of the step kernel's tensor maps
  unsigned long long *step_bar = nullptr;  // its grid-barrier counter and split counters
  float *step_part = nullptr;  // split-K partials of its MLP proj phase
  float *step_ss = nullptr;    // [2*depth+1][16][32] per-128-column sums of squares
  unsigned long long *step_trace = nullptr;  // caller's phase-timestamp buffer (nc_decode_trace), or null
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
  int T = 1, H = 0, max_seq = 0;
};

// ---- generic kernels (any even head_dim; fp32 or bf16 storage) ----
void k_prefill_begin(int32_t *len, uint8_t *valid, int B, int T, cudaStream_t s);
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
                         int Hkv, int hd, int max_seq, void *y, cudaStream_t s);
void k_argmax_rows(const float *logits, int rows, int V, long long row_stride, const float *noise,
                   int32_t *next, const uint8_t *valid, cudaStream_t s);
void k_kv_fork(int elem_bytes, const void *src_k, const void *src_v, size_t src_layer_elems, int src_max_seq,
               int src_seq, const int32_t *src_len, void *dst_k, void *dst_v, size_t dst_layer_elems,
               int dst_max_seq, int dst_first, int n, int32_t *dst_len, int depth, int kd, uint32_t *status,
               cudaStream_t s);


// ---- sm_100a tensor-core GEMM (nc_gemm_tc.cu) ----
bool gemm_tc_supported(int M, int N, int K, int lda);
cudaError_t k_gemm_tc(int epi, const void *A, int lda, const void *W, int M, int N, int K, void *out, int ldo,
                      float cap, uint32_t *status, int num_sms, cudaStream_t s, const GemmFuse *fz = nullptr);


// ---- sm_100a causal MQA prefill attention (nc_attn_tc.cu) ----
bool attn_prefill_tc_supported(int H, int Hkv, int hd);
cudaError_t k_attn_prefill_tc(const void *q, const void *kc, const void *vc, int B, int T, int H, int max_batch,
                              int max_seq, void *y, uint32_t *status, cudaStream_t s);


// ---- row-wise prefill kernels for bf16 head_dim-128 models (nc_rowops.cu) ----
bool rowops_supported(const nc_config &c);
cudaError_t k_rows_norm_bf16(const float *x, int rows, int d, float eps, void *h, cudaStream_t s);
cudaError_t k_rope_qk_bf16(const void *qkv, int M, int T, int H, const float2 *rope, void *q_out, void *kc, void *vc,
                           int max_seq, float eps, cudaStream_t s);
cudaError_t k_gather_rows_ss(const float *x, int rows, int d, int stride, int offset, float *xl, float *ss, int ssb,
                             cudaStream_t s);

// ---- decode step kernels (nc_decode.cu) ----
bool decode_fast_supported(const nc_config &c, int B);
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
                       cudaStream_t s);


// ---- sampled token pick (nc_sample.cu) ----
// next[b] = argmax over the top_k largest logits of row b (all when top_k <= 0
// or >= V; the lower index on a tie at the cut) of fl(fl(z / temperature) +
// noise), lowest index on ties; temperature 0 is argmax z. Logit rows are
// `stride` floats apart, noise rows V; rows with valid[b] == 0 are skipped.
cudaError_t k_sample_topk(const float *logits, int B, int V, long long stride, const float *noise, float temperature,
                          int top_k, const uint8_t *valid, int32_t *next, cudaStream_t s);

// ---- whole decode step in one persistent kernel (nc_step.cu) ----
bool decode_step_supported(const nc_config &c, int B);
int decode_step_maps_count(const nc_config &c);
bool decode_step_build_maps(const nc_model *m, const void *kcache, const void *vcache, int max_batch, int max_seq,
                            CUtensorMap *out);
int decode_step_grid(int num_sms);
cudaError_t k_decode_step(const nc_model *m, int B, int max_batch, int max_seq, const CUtensorMap *maps_dev,
                          const int32_t *tokens, const int32_t *positions, int32_t *len, float *x0, float *x1,
                          float *ss, void *q, void *y, void *f, void *kc, void *vc, const float2 *rope, float *logits,
                          const float *noise, int32_t *next, float *cand_v, int *cand_i, unsigned long long *bar,
                          float *split_part, int grid, unsigned long long *trace, uint8_t *valid_out,
                          cudaStream_t s);
size_t decode_step_bar_bytes();              // grid-barrier word + split counters, zeroed per launch
size_t decode_step_part_floats(int num_sms);  // split-K partials of the MLP proj phase

}  // namespace nc
