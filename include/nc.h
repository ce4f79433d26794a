/*
 * nc.h — C ABI of the B200 KV-cache Transformer inference engine.
 *
 * The engine runs the forward pass of the nanochat-style dense Transformer
 * (launch Q&A of "Karpathy再放大招：8000行代碼復現ChatGPT全棧..." : Llama-like,
 * RoPE and no positional embedding, QK norm, untied embedding/unembedding, a
 * norm after the token embedding, relu^2 MLP, RMSNorm without parameters, no
 * biases, multi-query attention, logit softcap) as the two operations the
 * same page names for its inference Engine: prefill and single-token decode
 * against a per-sequence KV cache ("高效推理": KV-cache engine with simple
 * prefill/decode). Forking a prefilled cache to N samples serves the RL
 * rollouts the page lists ("RL ... GRPO on GSM8K").
 *
 * Conventions for every call:
 *  - Pointers named d_* are DEVICE pointers (CUDA global memory on the
 *    model's device) owned by the caller; other pointers are host pointers.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream). Work is
 *    enqueued on it and the call returns without waiting; outputs are valid
 *    once the stream has been synchronised.
 *  - Return value: NC_OK (0) or an NC_E* code; nc_last_error() gives a
 *    message for the last failing call on this thread. Argument errors are
 *    detected on the host before anything is enqueued, so a failing call has
 *    changed nothing. Conditions only visible on the device (a token id out
 *    of range, a decode position that is not the sequence's current length)
 *    never fault: the kernels clamp/skip and set a bit in the model's device
 *    status word, read with nc_device_status().
 *  - The library owns the weights, KV caches and workspaces it allocates;
 *    calls on one model/cache must not overlap on different streams.
 *  - Only one GPU is used: the device current when the model is created.
 *  - A call whose shapes take one of the sm_100a kernels returns NC_ECUDA if
 *    that kernel fails to launch; the work is never retried on another
 *    kernel.
 *
 * Numerics. fp32 models compute in fp32 throughout. bf16 models keep the
 * weights, the activations fed to each matrix product and the KV cache in
 * bf16, and accumulate, keep the residual stream and produce logits in fp32.
 * On the sm_100a prefill path, an RMS norm followed by a linear layer is
 * evaluated as (bf16(x) . W) * (1 / rms(x)) rather than bf16(x / rms(x)) . W.
 * Both round each input once, so the error is of the same size; the
 * results differ in the last bf16 bits. The QK-norm factor is taken before
 * RoPE, which keeps each pair's sum of squares.
 */
#ifndef NC_H
#define NC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. */
#define NC_OK 0
#define NC_EINVAL 1   /* null pointer, bad shape, config/blob mismatch */
#define NC_ERANGE 2   /* batch or length beyond what the cache was created for */
#define NC_ENOMEM 3   /* device allocation failed */
#define NC_ECUDA 4    /* a CUDA runtime call failed (message has the CUDA error) */
#define NC_EUNSUP 5   /* valid config that this build has no kernel for */

/* Device status bits (nc_device_status). */
#define NC_DEV_BAD_TOKEN 1u     /* a token id was outside [0, vocab): clamped */
#define NC_DEV_BAD_POSITION 2u  /* decode position != current length or >= max_seq: sequence skipped */
#define NC_DEV_TIMEOUT 4u       /* a bounded in-kernel wait ran out (pipeline error) */

/* Storage type of weights, activations and KV cache. Accumulation is fp32. */
#define NC_F32 0
#define NC_BF16 1

/* Model shape. Fields follow the feature list above; n_kv_head = 1 is the
 * page's multi-query attention. n_kv_head > 1 groups the query heads: head h
 * reads KV head h / (n_head / n_kv_head) (grouped-query attention; n_kv_head
 * = n_head is multi-head attention, the reading under which the lineage
 * article "Karpathy 的 nano 諧系" pretraining bullet's d20 of about 560M
 * parameters comes out). Constants the pages leave open are inputs:
 * rope_base (10000), softcap (15), norm_eps (1e-6, inside the sqrt of every
 * RMSNorm). */
typedef struct {
  int depth;       /* number of Transformer blocks (>= 0) */
  int d_model;     /* residual width d */
  int n_head;      /* query heads H; n_head * head_dim == d_model */
  int n_kv_head;   /* KV heads; must divide n_head. The sm_100a decode step takes
                      up to 16 query heads per KV head, the tensor-core prefill
                      attention a group size dividing 128 (or one KV head);
                      other shapes run the generic kernels */
  int head_dim;    /* hd, even */
  int mlp_hidden;  /* F (4*d in the presets) */
  int vocab;       /* V */
  float rope_base;
  float softcap;
  float norm_eps;
  int dtype;       /* NC_F32 or NC_BF16 */
} nc_config;

typedef struct nc_model nc_model;
typedef struct nc_kv nc_kv;

/* Create a model on the current CUDA device from a host weight blob.
 * Blob: tensors back to back, row-major [out, in], element type cfg->dtype
 * (fp32, or bf16 bit patterns), in this order: wte[V,d]; for each layer
 * Wq[H*hd,d], Wk[Hkv*hd,d], Wv[Hkv*hd,d], Wo[d,H*hd], Wfc[F,d], Wproj[d,F];
 * then the untied lm_head Wlm[V,d]. blob_bytes must match exactly. The blob
 * is copied to the device before the call returns; the caller keeps
 * ownership of it. Errors: NC_EINVAL (null, inconsistent config, size
 * mismatch), NC_EUNSUP, NC_ENOMEM, NC_ECUDA. */
int nc_model_create(const nc_config *cfg, const void *host_blob, size_t blob_bytes, nc_model **out);

/* Free the model (waits for the device to finish). NULL is ignored. */
void nc_model_destroy(nc_model *model);

/* Read and clear the model's device status word (NC_DEV_* bits) raised by
 * kernels since the last call. Synchronises the device. */
int nc_device_status(nc_model *model, uint32_t *out_bits);

/* Create a KV cache for up to max_batch sequences of up to max_seq tokens,
 * plus the workspace prefill/decode need (sized for max_batch*max_seq
 * prefill rows). Layout per layer: K and V [max_batch][max_seq][Hkv*hd] of
 * the model's dtype, K stored after RoPE and QK norm. All lengths start at
 * 0. A bf16 decode step of up to 32 sequences runs as one persistent kernel
 * (NC_K_STEP); with the environment variable NC_DECODE_STEP_KERNEL=0 set
 * when the cache is created, it runs as one launch per layer step instead
 * (one KV head) or on the generic kernels (several KV heads): a diagnostic
 * switch, same results within the stated tolerances.
 * Errors: NC_EINVAL, NC_ENOMEM, NC_ECUDA. */
int nc_kv_create(const nc_model *model, int max_batch, int max_seq, nc_kv **out);

/* Free a cache (waits for the device). NULL is ignored. */
void nc_kv_destroy(nc_kv *kv);

/* Copy the current lengths of sequences 0..n-1 to host memory out[n].
 * Synchronises the device. Errors: NC_EINVAL, NC_ERANGE (n > max_batch). */
int nc_kv_lengths(const nc_kv *kv, int n, int32_t *out);

/* Prefill: run the prompts d_tokens[B,T] (int32, row-major) from position 0
 * into sequences 0..B-1 of `kv`, replacing whatever they held; afterwards
 * each has length T. Outputs (each may be NULL):
 *   d_logits  fp32 softcapped logits: [B,V] for the last position when
 *             logits_mode == 0, or [B,T,V] for every position when 1;
 *   d_next    int32 [B]: argmax over the vocabulary of the last position's
 *             logits (+ d_noise[b,:] if given), lowest index on ties;
 *   d_noise   fp32 [B,V] additive noise for d_next (e.g. Gumbel), or NULL.
 * Errors: NC_EINVAL (null kv/model/tokens, B or T < 1, bad logits_mode, a
 * sequence among 0..B-1 is the shared prefix of another, nc_kv_fork_shared),
 * NC_ERANGE (B > max_batch, T > max_seq), NC_ECUDA. */
int nc_prefill(nc_model *model, nc_kv *kv, const int32_t *d_tokens, int B, int T, int logits_mode,
               float *d_logits, int32_t *d_next, const float *d_noise, void *stream);

/* Append a chunk: run d_tokens[B,T] at positions len[b] .. len[b] + T - 1
 * of sequences 0..B-1, after whatever each already holds (its prompt,
 * earlier chunks, decode steps). This is how the Engine feeds tokens into a
 * running sequence (the launch article's "高效推理" item: tool use, whose
 * outputs go back into the conversation). Each sequence's K/V rows for the
 * chunk are appended and its length grows by T. Outputs as in nc_prefill:
 * d_logits [B,V] for the chunk's last position (logits_mode 0) or [B,T,V]
 * for all of its positions (1), d_next from the last position (+ d_noise,
 * or the sampled pick of nc_kv_set_sampling). A sequence whose chunk does
 * not fit (len + T > max_seq) is skipped: its cache and length stay
 * unchanged, NC_DEV_BAD_POSITION is raised, and its outputs are not
 * meaningful. A sequence reading a shared prefix (nc_kv_fork_shared) may be
 * extended. On bf16 head_dim-128 models with at least 128 chunk rows, the
 * chunk runs the same fused tensor-core layers as nc_prefill (RoPE, QK norm
 * and the cache append in the QKV GEMM's epilogue, tcgen05 attention over the
 * cached prefix and the chunk), unless the cache reads a shared prefix; then,
 * and for smaller chunks, RoPE/QK norm and attention run on the shape-generic
 * kernels.
 * Errors: as nc_prefill. */
int nc_prefill_extend(nc_model *model, nc_kv *kv, const int32_t *d_tokens, int B, int T, int logits_mode,
                      float *d_logits, int32_t *d_next, const float *d_noise, void *stream);

/* Decode one token for each of sequences 0..B-1: d_tokens[B] are fed at
 * d_positions[B] (int32, device). positions[b] must equal sequence b's
 * current length (< max_seq); the token's K/V are appended there and the
 * length becomes positions[b]+1. Positions may differ between sequences.
 * Outputs as in nc_prefill: d_logits fp32 [B,V], d_next int32 [B] (argmax of
 * logits + d_noise[b,:] when d_noise is non-NULL). A sequence whose position
 * is wrong is skipped (outputs untouched, cache unchanged) and
 * NC_DEV_BAD_POSITION is raised. Errors: NC_EINVAL, NC_ERANGE (B >
 * max_batch), NC_ECUDA. */
int nc_decode_step(nc_model *model, nc_kv *kv, const int32_t *d_tokens, const int32_t *d_positions, int B,
                   const float *d_noise, float *d_logits, int32_t *d_next, void *stream);

/* Fork: copy sequence src_seq of `src` (its first len tokens, every layer,
 * K and V) into sequences dst_first .. dst_first+n-1 of `dst` and set their
 * lengths to len. src and dst may be the same cache (the source must not be
 * among the destinations). Both caches must belong to the same model.
 * Errors: NC_EINVAL, NC_ERANGE (indices out of range, len > dst max_seq),
 * NC_ECUDA. */
int nc_kv_fork(nc_kv *src, int src_seq, nc_kv *dst, int dst_first, int n, void *stream);

/* Fork by sharing the prefix (the RL rollouts of the launch article's
 * pipeline list sample many continuations of one prompt, and the lineage
 * page's GRPO stage does the same): like nc_kv_fork, with the same results
 * in every later call, but the destinations get no copy of the source's
 * first P key/value rows of every layer, P = its length rounded down to a
 * multiple of 64. Their attention reads those rows from the source sequence
 * in `src` (one read of the shared rows serves every sample through the L2
 * cache), and only the remaining len - P < 64 rows are copied. If the source
 * sequence itself reads a shared prefix, the destinations read the same one
 * (P is the source's). src and dst may be the same cache.
 * The link lasts until the destination is replaced (nc_prefill over it, a
 * fork into it) or its cache is destroyed. While any sequence reads shared
 * rows from a sequence, that sequence may take decode steps (they append
 * past the shared rows) but may not be replaced: nc_prefill and the forks
 * return NC_EINVAL. A cache reads shared rows from one cache at a time. A
 * source cache destroyed while others still read from it keeps its memory
 * until the last such link ends.
 * Errors: as nc_kv_fork, plus NC_EINVAL (the prefix's sequence among the
 * destinations, dst already shares prefixes with another cache). */
int nc_kv_fork_shared(nc_kv *src, int src_seq, nc_kv *dst, int dst_first, int n, void *stream);

/* Sampled token pick for nc_prefill and nc_decode_step on this cache. The
 * launch article's Engine samples its tokens ("高效推理"; the pages give no
 * details); the usual temperature / top-k reading is taken. From now on
 * d_next[b] is the argmax, over the top_k largest logits of row b (all of
 * them when top_k == 0 or >= V; at a tie on the cut the lower index is
 * kept), of fl(fl(logit / temperature) + d_noise[b, v]) in fp32, lowest
 * index on ties. With d_noise i.i.d. standard Gumbel this draws from
 * softmax(logits / temperature) restricted to the top_k (Gumbel-max); with
 * d_noise NULL the noise is 0. temperature 0 is the greedy pick argmax of
 * the logits. temperature 1 with top_k 0 (the default) is the plain
 * argmax(logits + noise) pick. The logits returned are unchanged (softcapped,
 * untempered). Errors: NC_EINVAL (temperature < 0 or not finite, top_k < 0). */
int nc_kv_set_sampling(nc_kv *kv, float temperature, int top_k);

/* ---- tracing ----
 * Kernel classes for nc_profile_read. */
#define NC_K_GEMM 0   /* linear layers: QKV, O-proj, MLP fc, MLP proj */
#define NC_K_ATTN 1   /* attention, prefill or decode (with any split combine) */
#define NC_K_HEAD 2   /* final norm, lm_head with softcap, token pick */
#define NC_K_MISC 3   /* embedding, norms, RoPE/QK norm/KV append, bookkeeping, fork */
#define NC_K_STEP 4   /* a whole decode step run as one persistent kernel */
#define NC_K_COUNT 5

/* Turn per-class device timing on (1) or off (0) for calls on this model.
 * When on, every launch (or fused group of launches) is bracketed by CUDA
 * events on the call's stream; the events add no work on the device. */
int nc_profile_enable(nc_model *model, int on);

/* Sum of event-timed durations in ms (ms[NC_K_COUNT]) and kernel launch
 * counts (launches[NC_K_COUNT]) per class since profiling was enabled or
 * last read; then resets them. Synchronises the device. Either output may be
 * NULL. */
int nc_profile_read(nc_model *model, double *ms, long long *launches);

/* Phase timestamps of the whole-step decode kernel (NC_K_STEP). With d_buf
 * non-NULL, every later nc_decode_step on `kv` that runs that kernel writes,
 * for each CTA c and phase p, eight %globaltimer readings (ns) to
 * d_buf[(c * phases + p) * 8 + slot]: slot 0 phase start (after the previous
 * grid barrier), 1 inputs staged (linear phases) or first cache tile in
 * (attention), 2 products done (linear) or keys done (attention), 3 the
 * reduction over the compute warps or the merge of the key splits done, 4
 * phase work done (barrier entry), 5 and 6 the TMA producer's first and last
 * load of the phase, 7 unused. Slots a CTA does not reach in a
 * phase keep their old contents (clear the buffer first). Phases are EMBED,
 * then per layer QKV, ATTN, O-proj, MLP fc, MLP proj, then HEAD and MERGE.
 * d_buf = NULL turns tracing off. *grid and *phases (host, may be NULL)
 * receive the kernel's CTA count and phase count; d_buf needs grid * phases
 * * 8 words. Errors: NC_EINVAL, NC_EUNSUP (no step kernel on this cache),
 * NC_ERANGE (buffer too small). */
int nc_decode_trace(nc_kv *kv, unsigned long long *d_buf, size_t n_words, int *grid, int *phases);

/* Number of kernels this library has launched in this process so far
 * (a CUDA graph replay counts each of its kernel nodes). */
unsigned long long nc_launch_count(void);

/* Message for the last failing nc_* call on this thread ("" if none). */
const char *nc_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* NC_H */
