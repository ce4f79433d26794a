/*
 * nc_kernels.h — kernel-level entry points of the B200 engine library.
 *
 * These expose single building blocks of the forward pass for callers that
 * assemble their own pipeline (and for unit tests of the kernels). Same
 * conventions as nc.h: d_* are device pointers owned by the caller, work is
 * enqueued on `stream` (a cudaStream_t, NULL = legacy default stream),
 * return NC_OK or an NC_E* code with nc_last_error() set.
 */
#ifndef NC_KERNELS_H
#define NC_KERNELS_H

#include "nc.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Epilogues of nc_gemm_bf16. */
#define NC_EPI_STORE 0    /* d_out bf16 [M, ldo]: acc */
#define NC_EPI_RELU2 1    /* d_out bf16 [M, ldo]: relu(acc)^2 (the MLP activation) */
#define NC_EPI_RESID 2    /* d_out fp32 [M, ldo]: d_out += acc (residual add) */
#define NC_EPI_SOFTCAP 3  /* d_out fp32 [M, ldo]: cap * tanh(acc / cap) (logit softcap) */

/* Linear layer without bias (feature list: "no bias in the linear layers"):
 * acc[m, n] = sum_k A[m, k] * W[n, k], A bf16 [M, K] with row pitch lda
 * elements, W bf16 [N, K] row-major (a weight stored [out, in]), fp32
 * accumulation; the epilogue writes d_out. Runs on the tcgen05 tensor-core
 * kernel when M >= 128, K % 64 == 0, N % 32 == 0 and lda % 8 == 0 (16-byte
 * rows for TMA), otherwise on the generic kernel. Above 128 rows the tcgen05
 * kernel runs on CTA pairs (clusters of two CTAs, tcgen05.mma.cta_group::2);
 * the environment variable NC_GEMM_PAIR=0 keeps it on single CTAs. Device
 * pointers must be 16-byte aligned. Errors: NC_EINVAL (null pointer,
 * non-positive size, lda < K, ldo < N, unknown epilogue), NC_ECUDA. */
int nc_gemm_bf16(const void *d_A, int lda, const void *d_W, int M, int N, int K, int epi, void *d_out, int ldo,
                 float cap, void *stream);

/* Causal multi-query attention (one KV head shared by all H query heads;
 * feature list: "multi-query attention") for B sequences of T positions:
 *   y[b,t,h,:] = sum_{j<=t} softmax_j(q[b,t,h,:] . k[b,j,:] / sqrt(hd)) v[b,j,:]
 * d_q, d_y bf16 [B, T, H, hd] (queries after RoPE and QK norm); d_k, d_v bf16
 * [B, max_seq, hd] (keys after RoPE and QK norm; rows 0..T-1 of each sequence
 * are used, rows T..max_seq-1 must hold finite values). Runs on the tcgen05
 * kernel when hd == 128, else on the generic kernel. Errors: NC_EINVAL,
 * NC_ECUDA. */
int nc_attention_prefill_bf16(const void *d_q, const void *d_k, const void *d_v, int B, int T, int H, int hd,
                              int max_seq, void *d_y, void *stream);

/* Single-token (decode) multi-query attention for B sequences, head_dim 128,
 * H <= 16 query heads sharing one KV head:
 *   y[b,h,:] = sum_{j<=pos[b]} softmax_j(q[b,h,:] . k[b,j,:] / sqrt(128)) v[b,j,:]
 * split over the keys (flash decoding) with a merge of the partial softmax
 * states. d_q, d_y bf16 [B, H, 128]; d_k, d_v bf16 [B, max_seq, 128];
 * d_pos int32 [B], each in [0, max_seq) (clamped on the device otherwise).
 * d_workspace: device scratch of nc_attention_decode_workspace_bytes(B,
 * max_seq) bytes, zero-filled before its first use; the call leaves it ready
 * for the next one. Calls sharing a workspace must not overlap on the GPU.
 * Errors: NC_EINVAL (null pointer, bad shape, H > 16, workspace too small),
 * NC_ECUDA. */
size_t nc_attention_decode_workspace_bytes(int B, int max_seq);
int nc_attention_decode_bf16(const void *d_q, const void *d_k, const void *d_v, const int32_t *d_pos, int B, int H,
                             int max_seq, void *d_y, void *d_workspace, size_t workspace_bytes, void *stream);

/* Sampled token pick over fp32 logits (the pick nc_kv_set_sampling turns on
 * inside the engine): d_next[b] = argmax, over the top_k largest logits of
 * row b (all when top_k == 0 or >= V; at a tie on the cut the lower index is
 * kept), of fl(fl(d_logits[b, v] / temperature) + d_noise[b, v]), lowest
 * index on ties; temperature 0 gives argmax of the logits. d_logits rows are
 * row_stride floats apart (row_stride >= V); d_noise fp32 [B, V] contiguous
 * or NULL (no noise); d_next int32 [B]. One CTA per row re-reads the row from
 * memory four times (radix select of the cut, then the pick). Errors:
 * NC_EINVAL (null logits or next, B or V < 1, row_stride < V, temperature < 0
 * or not finite, top_k < 0), NC_ECUDA. */
int nc_sample_topk(const float *d_logits, int B, int V, long long row_stride, const float *d_noise, float temperature,
                   int top_k, int32_t *d_next, void *stream);

/* nc_attention_decode_bf16 without a workspace argument, for callers that
 * cannot allocate device memory (a serving runtime whose allocator owns all
 * of it, a plugin host without a workspace hook, a fixed-footprint
 * deployment). The pages have no counterpart: this is a packaging variant of
 * the decode attention above, with the same inputs, outputs and results.
 * Its scratch is a static array inside the library (about 4.3 MB, held on
 * every GPU that loads the library until the process exits); no call
 * allocates or frees device memory. Limits: B <= 32, H <= 16, and max_seq
 * small enough for 16 key splits (the split rule grows the chunk to fit).
 * Every call looks up the array's device address on the current device
 * (a host-side query), so a device reset in between is harmless; the first
 * call on a device also loads the library's code there, so make that first
 * call before any stream capture. All calls share the one
 * array: calls that overlap on the GPU (other streams, other threads) race
 * and must be serialised by the caller. Errors: NC_EINVAL (null pointer, bad
 * shape, B or max_seq beyond the limits), NC_ECUDA. */
int nc_attention_decode_bf16_static(const void *d_q, const void *d_k, const void *d_v, const int32_t *d_pos, int B,
                                    int H, int max_seq, void *d_y, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* NC_KERNELS_H */
