// nc_generic.cu — shape-generic CUDA kernels of the engine.
//
// These cover every config the C ABI accepts (fp32 or bf16 storage, any even
// head_dim). The bf16 head_dim-128 models run the specialised sm_100a kernels
// for their hot ops and use these only for the cheap row-wise steps.
//
// Model (nanochat launch Q&A feature list): pre-norm blocks; RMSNorm without
// gain, y = x / sqrt(mean(x^2) + eps); a norm right after the token
// embedding; RoPE on split-half pairs (i, i + hd/2) followed by QK norm;
// multi-query causal attention with scale 1/sqrt(hd); relu^2 MLP; final
// norm, untied lm_head and softcap cap*tanh(z/cap).
#include <math.h>

#include <type_traits>

#include "nc_internal.h"

namespace nc {

std::atomic<unsigned long long> g_launches{0};

// --------------------------------------------------------------- sequences
__global__ void prefill_begin_kernel(int32_t *len, uint8_t *valid, int32_t *pre_len, int B, int T) {
  int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) {
    len[b] = T;
    valid[b] = 1;
    pre_len[b] = 0;  // a replaced sequence owns all its rows
  }
}

void k_prefill_begin(int32_t *len, uint8_t *valid, int32_t *pre_len, int B, int T, cudaStream_t s) {
  count_launch();
  prefill_begin_kernel<<<(B + 127) / 128, 128, 0, s>>>(len, valid, pre_len, B, T);
}

// A chunk of T tokens is appended to sequence b at its current length:
// off[b] = len[b]; the sequence takes part iff the chunk fits (len + T <=
// max_seq), and then its length advances by T.
__global__ void extend_begin_kernel(int32_t *len, uint8_t *valid, int32_t *off, int B, int T, int max_seq,
                                    uint32_t *status) {
  int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const int l = len[b];
  const bool ok = l >= 0 && l + T <= max_seq;
  off[b] = ok ? l : 0;
  valid[b] = ok ? 1 : 0;
  if (ok) len[b] = l + T;
  else atomicOr(status, (unsigned)NC_DEV_BAD_POSITION);
}

void k_extend_begin(int32_t *len, uint8_t *valid, int32_t *off, int B, int T, int max_seq, uint32_t *status,
                    cudaStream_t s) {
  count_launch();
  extend_begin_kernel<<<(B + 127) / 128, 128, 0, s>>>(len, valid, off, B, T, max_seq, status);
}

// A decode row is valid iff its position is the sequence's current length and
// inside the cache; valid rows advance their length by one.
__global__ void decode_begin_kernel(const int32_t *positions, int32_t *len, uint8_t *valid, int B, int max_seq,
                                    uint32_t *status) {
  int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  int p = positions[b];
  bool ok = p >= 0 && p < max_seq && p == len[b];
  valid[b] = ok ? 1 : 0;
  if (ok) len[b] = p + 1;
  else atomicOr(status, (unsigned)NC_DEV_BAD_POSITION);
}

void k_decode_begin(const int32_t *positions, int32_t *len, uint8_t *valid, int B, int max_seq,
                    uint32_t *status, cudaStream_t s) {
  count_launch();
  decode_begin_kernel<<<(B + 127) / 128, 128, 0, s>>>(positions, len, valid, B, max_seq, status);
}

// ------------------------------------------------------------ embed + norm
template <typename T>
__global__ void embed_norm_kernel(const int32_t *tokens, const T *wte, int d, int vocab, float eps, float *x,
                                  uint32_t *status) {
  __shared__ float red[32];
  int m = blockIdx.x;
  int tok = tokens[m];
  if (tok < 0 || tok >= vocab) {
    if (threadIdx.x == 0) atomicOr(status, (unsigned)NC_DEV_BAD_TOKEN);
    tok = tok < 0 ? 0 : vocab - 1;
  }
  const T *row = wte + (size_t)tok * d;
  float ss = 0.f;
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    float v = to_f32(row[i]);
    ss += v * v;
  }
  ss = block_sum(ss, red);
  float inv = rsqrtf(ss / d + eps);
  for (int i = threadIdx.x; i < d; i += blockDim.x) x[(size_t)m * d + i] = to_f32(row[i]) * inv;
}

// bf16 tables with d a multiple of 8: one warp per row, 16-byte loads of 8
// elements, the row kept in registers between the sum of squares and the
// scaled fp32 stores (d <= 8 * 32 * EC).
template <int EC>
__global__ void embed_norm_bf16_kernel(const int32_t *tokens, const bf16 *wte, int M, int d, int vocab, float eps,
                                       float *x, uint32_t *status) {
  const int lane = threadIdx.x & 31, m = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (m >= M) return;
  int tok = tokens[m];
  if (tok < 0 || tok >= vocab) {
    if (lane == 0) atomicOr(status, (unsigned)NC_DEV_BAD_TOKEN);
    tok = tok < 0 ? 0 : vocab - 1;
  }
  const uint4 *row = reinterpret_cast<const uint4 *>(wte + (size_t)tok * d);
  const int nc = d / 8;
  float v[EC][8];
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < EC; j++) {
    const int c = lane + 32 * j;
    uint4 u = c < nc ? __ldg(row + c) : make_uint4(0, 0, 0, 0);
    const bf16 *h = reinterpret_cast<const bf16 *>(&u);
#pragma unroll
    for (int q = 0; q < 8; q++) {
      v[j][q] = __bfloat162float(h[q]);
      ss = fmaf(v[j][q], v[j][q], ss);
    }
  }
  const float inv = rsqrtf(warp_sum(ss) / d + eps);
  float4 *dst = reinterpret_cast<float4 *>(x + (size_t)m * d);
#pragma unroll
  for (int j = 0; j < EC; j++) {
    const int c = lane + 32 * j;
    if (c < nc) {
      dst[2 * c] = make_float4(v[j][0] * inv, v[j][1] * inv, v[j][2] * inv, v[j][3] * inv);
      dst[2 * c + 1] = make_float4(v[j][4] * inv, v[j][5] * inv, v[j][6] * inv, v[j][7] * inv);
    }
  }
}

void k_embed_norm(int dtype, const int32_t *tokens, int M, const void *wte, int d, int vocab, float eps,
                  float *x, uint32_t *status, cudaStream_t s) {
  if (M <= 0) return;
  count_launch();
  if (dtype == NC_BF16 && d % 8 == 0 && d <= 8 * 32 * 8) {
    const int grid = (M + 7) / 8;
    if (d <= 8 * 32 * 4)
      embed_norm_bf16_kernel<4><<<grid, 256, 0, s>>>(tokens, (const bf16 *)wte, M, d, vocab, eps, x, status);
    else
      embed_norm_bf16_kernel<8><<<grid, 256, 0, s>>>(tokens, (const bf16 *)wte, M, d, vocab, eps, x, status);
    return;
  }
  if (dtype == NC_F32)
    embed_norm_kernel<float><<<M, 256, 0, s>>>(tokens, (const float *)wte, d, vocab, eps, x, status);
  else
    embed_norm_kernel<bf16><<<M, 256, 0, s>>>(tokens, (const bf16 *)wte, d, vocab, eps, x, status);
}

// ------------------------------------------------------------------ norm
// out[r, :] = x[r*src_stride + src_offset, :] / rms (no gain), storage type.
template <typename T>
__global__ void rmsnorm_rows_kernel(const float *x, int d, int src_stride, int src_offset, float eps, T *out) {
  __shared__ float red[32];
  int r = blockIdx.x;
  const float *src = x + ((size_t)r * src_stride + src_offset) * d;
  float ss = 0.f;
  for (int i = threadIdx.x; i < d; i += blockDim.x) ss += src[i] * src[i];
  ss = block_sum(ss, red);
  float inv = rsqrtf(ss / d + eps);
  for (int i = threadIdx.x; i < d; i += blockDim.x) out[(size_t)r * d + i] = from_f32<T>(src[i] * inv);
}

void k_rmsnorm_rows(int dtype, const float *x, int rows, int d, int src_stride, int src_offset, float eps,
                    void *out, cudaStream_t s) {
  if (rows <= 0) return;
  count_launch();
  if (dtype == NC_F32)
    rmsnorm_rows_kernel<float><<<rows, 256, 0, s>>>(x, d, src_stride, src_offset, eps, (float *)out);
  else
    rmsnorm_rows_kernel<bf16><<<rows, 256, 0, s>>>(x, d, src_stride, src_offset, eps, (bf16 *)out);
}

// ------------------------------------------------------------------ GEMM
// out[m, n] (epilogue) acc[m, n] = sum_k A[m, k] * W[n, k]; W row-major [N, K].
// 64x64 output tile per block, 16-deep K slices, 4x4 outputs per thread.
template <typename T, int EPI>
__global__ void __launch_bounds__(256) gemm_generic_kernel(const T *A, int lda, const T *W, int M, int N, int K,
                                                           void *out, int ldo, float cap, const uint8_t *valid) {
  __shared__ float As[16][68];
  __shared__ float Ws[16][68];
  int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; i++)
#pragma unroll
    for (int j = 0; j < 4; j++) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 1024; i += 256) {
      int r = i >> 4, c = i & 15, gk = k0 + c;
      int gm = m0 + r, gn = n0 + r;
      As[c][r] = (gm < M && gk < K) ? to_f32(A[(size_t)gm * lda + gk]) : 0.f;
      Ws[c][r] = (gn < N && gk < K) ? to_f32(W[(size_t)gn * K + gk]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; kk++) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; i++) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; j++) b[j] = Ws[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; i++)
#pragma unroll
        for (int j = 0; j < 4; j++) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; i++) {
    int m = m0 + ty * 4 + i;
    if (m >= M) continue;
    if (EPI == EPI_SOFTCAP && valid && !valid[m]) continue;
#pragma unroll
    for (int j = 0; j < 4; j++) {
      int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float v = acc[i][j];
      size_t o = (size_t)m * ldo + n;
      if (EPI == EPI_STORE) {
        ((T *)out)[o] = from_f32<T>(v);
      } else if (EPI == EPI_RELU2) {
        float r = fmaxf(v, 0.f);
        ((T *)out)[o] = from_f32<T>(r * r);
      } else if (EPI == EPI_RESID) {
        ((float *)out)[o] += v;
      } else {
        ((float *)out)[o] = cap * tanhf(v / cap);
      }
    }
  }
}

template <typename T>
static void gemm_generic_t(int epi, const void *A, int lda, const void *W, int M, int N, int K, void *out, int ldo,
                           float cap, const uint8_t *valid, cudaStream_t s) {
  dim3 grid((N + 63) / 64, (M + 63) / 64);
  const T *a = (const T *)A, *w = (const T *)W;
  switch (epi) {
    case EPI_STORE: count_launch(); gemm_generic_kernel<T, EPI_STORE><<<grid, 256, 0, s>>>(a, lda, w, M, N, K, out, ldo, cap, valid); break;
    case EPI_RELU2: count_launch(); gemm_generic_kernel<T, EPI_RELU2><<<grid, 256, 0, s>>>(a, lda, w, M, N, K, out, ldo, cap, valid); break;
    case EPI_RESID: count_launch(); gemm_generic_kernel<T, EPI_RESID><<<grid, 256, 0, s>>>(a, lda, w, M, N, K, out, ldo, cap, valid); break;
    default: count_launch(); gemm_generic_kernel<T, EPI_SOFTCAP><<<grid, 256, 0, s>>>(a, lda, w, M, N, K, out, ldo, cap, valid); break;
  }
}

void k_gemm_generic(int dtype, int epi, const void *A, int lda, const void *W, int M, int N, int K, void *out,
                    int ldo, float cap, const uint8_t *valid_rows, cudaStream_t s) {
  if (M <= 0 || N <= 0) return;
  if (dtype == NC_F32) gemm_generic_t<float>(epi, A, lda, W, M, N, K, out, ldo, cap, valid_rows, s);
  else gemm_generic_t<bf16>(epi, A, lda, W, M, N, K, out, ldo, cap, valid_rows, s);
}

// --------------------------------------------- RoPE + QK norm + KV append
// One block per row: rotate every q and k head at the row's position, RMS-
// normalise each head, write q and append k, v to the row's sequence.
template <typename T>
__global__ void rope_qknorm_kernel(const T *qkv, RowMap rm, int H, int Hkv, int hd, const float2 *rope, T *q_out,
                                   T *kc, T *vc, int max_seq, const uint8_t *valid, float eps) {
  extern __shared__ float sm[];
  int m = blockIdx.x, W = (H + 2 * Hkv) * hd, nh = H + Hkv, half = hd / 2;
  int b = rm.seq(m), pos = rm.position(m);
  int pc = pos < 0 ? 0 : (pos >= max_seq ? max_seq - 1 : pos);
  float *inv = sm + W;
  const T *row = qkv + (size_t)m * W;
  for (int i = threadIdx.x; i < W; i += blockDim.x) sm[i] = to_f32(row[i]);
  __syncthreads();
  for (int p = threadIdx.x; p < nh * half; p += blockDim.x) {
    int hh = p / half, i = p % half;
    float2 cs = rope[(size_t)pc * half + i];
    float a = sm[hh * hd + i], c = sm[hh * hd + i + half];
    sm[hh * hd + i] = a * cs.x - c * cs.y;
    sm[hh * hd + i + half] = a * cs.y + c * cs.x;
  }
  __syncthreads();
  int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int hh = wid; hh < nh; hh += nw) {
    float ss = 0.f;
    for (int e = lane; e < hd; e += 32) ss += sm[hh * hd + e] * sm[hh * hd + e];
    ss = warp_sum(ss);
    if (lane == 0) inv[hh] = rsqrtf(ss / hd + eps);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < H * hd; i += blockDim.x)
    q_out[(size_t)m * H * hd + i] = from_f32<T>(sm[i] * inv[i / hd]);
  bool ok = (valid ? valid[b] != 0 : true) && pos >= 0 && pos < max_seq;
  if (ok) {
    int kd = Hkv * hd;
    size_t base = ((size_t)b * max_seq + pos) * kd;
    for (int i = threadIdx.x; i < kd; i += blockDim.x) {
      kc[base + i] = from_f32<T>(sm[H * hd + i] * inv[H + i / hd]);
      vc[base + i] = from_f32<T>(sm[(H + Hkv) * hd + i]);
    }
  }
}

void k_rope_qknorm_append(int dtype, const void *qkv, RowMap rm, int M, int H, int Hkv, int hd,
                          const float2 *rope, void *q_out, void *kc, void *vc, int max_seq,
                          const uint8_t *valid, float eps, cudaStream_t s) {
  if (M <= 0) return;
  size_t smem = sizeof(float) * ((size_t)(H + 2 * Hkv) * hd + H + Hkv);
  count_launch();
  if (dtype == NC_F32)
    rope_qknorm_kernel<float><<<M, 128, smem, s>>>((const float *)qkv, rm, H, Hkv, hd, rope, (float *)q_out,
                                                   (float *)kc, (float *)vc, max_seq, valid, eps);
  else
    rope_qknorm_kernel<bf16><<<M, 128, smem, s>>>((const bf16 *)qkv, rm, H, Hkv, hd, rope, (bf16 *)q_out,
                                                  (bf16 *)kc, (bf16 *)vc, max_seq, valid, eps);
}

// ------------------------------------------------------------- attention
// One block per (row, query head): softmax over the row's causal keys
// 0..pos of its sequence (exact scores kept in shared memory).
template <typename T>
__global__ void attn_generic_kernel(const T *q, const T *kc, const T *vc, RowMap rm, int H, int Hkv, int hd,
                                    int max_seq, T *y, KvPrefix pre) {
  extern __shared__ float sm[];
  __shared__ float red[32];
  int m = blockIdx.x, h = blockIdx.y;
  int b = rm.seq(m), pos = rm.position(m);
  pos = pos < 0 ? 0 : (pos >= max_seq ? max_seq - 1 : pos);
  int n = pos + 1, g = h / (H / Hkv), kd = Hkv * hd;
  float *qs = sm, *s = sm + hd;
  for (int e = threadIdx.x; e < hd; e += blockDim.x) qs[e] = to_f32(q[((size_t)m * H + h) * hd + e]);
  __syncthreads();
  const T *K = kc + (size_t)b * max_seq * kd + g * hd;
  const T *V = vc + (size_t)b * max_seq * kd + g * hd;
  // rows below the shared length live in the prefix cache's sequence
  const int plen = pre.len ? pre.len[b] : 0;
  const T *PK = plen ? (const T *)pre.k + (size_t)pre.seq[b] * pre.max_seq * kd + g * hd : K;
  const T *PV = plen ? (const T *)pre.v + (size_t)pre.seq[b] * pre.max_seq * kd + g * hd : V;
  float scale = 1.0f / sqrtf((float)hd), mx = -INFINITY;
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    float dot = 0.f;
    const T *Kj = (j < plen ? PK : K) + (size_t)j * kd;
    for (int e = 0; e < hd; e++) dot = fmaf(qs[e], to_f32(Kj[e]), dot);
    s[j] = dot * scale;
    mx = fmaxf(mx, s[j]);
  }
  mx = block_max(mx, red);
  float z = 0.f;
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    float p = expf(s[j] - mx);
    s[j] = p;
    z += p;
  }
  z = block_sum(z, red);
  __syncthreads();
  for (int e = threadIdx.x; e < hd; e += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j < n; j++) acc = fmaf(s[j], to_f32((j < plen ? PV : V)[(size_t)j * kd + e]), acc);
    y[((size_t)m * H + h) * hd + e] = from_f32<T>(acc / z);
  }
}

void k_attention_generic(int dtype, const void *q, const void *kc, const void *vc, RowMap rm, int M, int H,
                         int Hkv, int hd, int max_seq, void *y, cudaStream_t s, const KvPrefix *pre) {
  if (M <= 0) return;
  const KvPrefix pv = pre ? *pre : KvPrefix{};
  size_t smem = sizeof(float) * ((size_t)hd + max_seq);
  dim3 grid(M, H);
  if (dtype == NC_F32) {
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(attn_generic_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    count_launch();
    attn_generic_kernel<float><<<grid, 128, smem, s>>>((const float *)q, (const float *)kc, (const float *)vc, rm,
                                                       H, Hkv, hd, max_seq, (float *)y, pv);
  } else {
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(attn_generic_kernel<bf16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    count_launch();
    attn_generic_kernel<bf16><<<grid, 128, smem, s>>>((const bf16 *)q, (const bf16 *)kc, (const bf16 *)vc, rm, H,
                                                      Hkv, hd, max_seq, (bf16 *)y, pv);
  }
}

// ---------------------------------------------------------------- argmax
// next[r] = argmax_v logits[r*row_stride + v] (+ noise[r*V + v]), lowest index
// on ties; rows with valid[r] == 0 are left untouched.
__global__ void argmax_rows_kernel(const float *logits, int V, long long row_stride, const float *noise,
                                   int32_t *next, const uint8_t *valid) {
  __shared__ float sv[32];
  __shared__ int si[32];
  int r = blockIdx.x;
  if (valid && !valid[r]) return;
  const float *row = logits + (size_t)r * row_stride;
  const float *nz = noise ? noise + (size_t)r * V : nullptr;
  ArgMax best{-INFINITY, 0x7fffffff};
  for (int v = threadIdx.x; v < V; v += blockDim.x) {
    float x = row[v] + (nz ? nz[v] : 0.f);
    best = argmax_merge(best, ArgMax{x, v});
  }
  best = warp_argmax(best);
  int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if (lane == 0) { sv[wid] = best.v; si[wid] = best.i; }
  __syncthreads();
  if (wid == 0) {
    ArgMax a = lane < nw ? ArgMax{sv[lane], si[lane]} : ArgMax{-INFINITY, 0x7fffffff};
    a = warp_argmax(a);
    if (lane == 0) next[r] = a.i;
  }
}

void k_argmax_rows(const float *logits, int rows, int V, long long row_stride, const float *noise,
                   int32_t *next, const uint8_t *valid, cudaStream_t s) {
  if (rows <= 0) return;
  count_launch();
  argmax_rows_kernel<<<rows, 512, 0, s>>>(logits, V, row_stride, noise, next, valid);
}

// ------------------------------------------------------------------ fork
struct ForkArgs {
  const uint32_t *src_k, *src_v;          // source cache at layer 0, sequence src_seq
  size_t src_layer_words;
  const int32_t *src_len;                  // &len[src_seq]
  const int32_t *src_pre_len, *src_pre_seq;  // &pre_len[src_seq], &pre_seq[src_seq] (null: none)
  const uint32_t *pre_k, *pre_v;           // the source's prefix cache at layer 0
  size_t pre_layer_words, pre_seq_words;
  uint32_t *dst_k, *dst_v;                 // destination cache at layer 0
  size_t dst_layer_words, dst_seq_words;
  int dst_first, dst_max_seq, row_words, src_seq;
  int32_t *dst_len, *dst_pre_seq, *dst_pre_len;
  int shared;                              // 1: share the rows below the shared length
  uint32_t *status;
};

// One (layer, K or V, destination) per blockIdx.(y, z): copy the rows the
// destination owns; the source's rows below its own shared length come from
// its prefix cache. Lengths and prefix tables are read on the device. Words
// are W x 32 bits (W = 4: 16-byte copies when every row offset allows it).
template <int W>
__global__ void kv_fork_kernel(ForkArgs f) {
  using Vec = typename std::conditional<W == 4, uint4, uint32_t>::type;
  const int layer = blockIdx.y >> 1, which = blockIdx.y & 1, i = blockIdx.z;
  int len = *f.src_len;
  if (len > f.dst_max_seq) {
    if (blockIdx.x == 0 && threadIdx.x == 0 && layer == 0 && which == 0) atomicOr(f.status, (unsigned)NC_DEV_BAD_POSITION);
    len = f.dst_max_seq;
  }
  if (len < 0) len = 0;
  const int spl = f.src_pre_len ? *f.src_pre_len : 0;  // rows of the source living in its prefix cache
  const int first = f.shared ? (spl > 0 ? spl : len / 64 * 64) : 0;
  const uint32_t *own = (which ? f.src_v : f.src_k) + layer * f.src_layer_words;
  const uint32_t *pre = spl > 0 ? (which ? f.pre_v : f.pre_k) + layer * f.pre_layer_words +
                                      (size_t)*f.src_pre_seq * f.pre_seq_words
                                : own;
  uint32_t *dst = (which ? f.dst_v : f.dst_k) + layer * f.dst_layer_words + (size_t)(f.dst_first + i) * f.dst_seq_words;
  const size_t w0 = (size_t)first * f.row_words / W, total = (size_t)len * f.row_words / W,
               wsh = (size_t)spl * f.row_words / W;
  const Vec *ownv = reinterpret_cast<const Vec *>(own), *prev = reinterpret_cast<const Vec *>(pre);
  Vec *dstv = reinterpret_cast<Vec *>(dst);
  for (size_t w = w0 + (size_t)blockIdx.x * blockDim.x + threadIdx.x; w < total; w += (size_t)gridDim.x * blockDim.x)
    dstv[w] = w < wsh ? prev[w] : ownv[w];
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
    f.dst_len[f.dst_first + i] = len;
    f.dst_pre_len[f.dst_first + i] = first;
    f.dst_pre_seq[f.dst_first + i] = spl > 0 ? *f.src_pre_seq : f.src_seq;
  }
}

void k_kv_fork(int elem_bytes, const void *src_k, const void *src_v, size_t src_layer_elems, int src_max_seq,
               int src_seq, const int32_t *src_len, const KvPrefix &src_pre, size_t pre_layer_elems, void *dst_k,
               void *dst_v, size_t dst_layer_elems, int dst_max_seq, int dst_first, int n, int32_t *dst_len,
               int32_t *dst_pre_seq, int32_t *dst_pre_len, bool shared, int depth, int kd, uint32_t *status,
               cudaStream_t s) {
  if (n <= 0) return;
  const size_t per = (size_t)elem_bytes / 2;  // 16-bit units per element
  // all row sizes are whole 32-bit words: kd is even
  const int row_words = (int)((size_t)kd * elem_bytes / 4);
  ForkArgs f;
  f.src_layer_words = src_layer_elems * per / 2;
  const size_t src_seq_words = (size_t)src_max_seq * row_words;
  f.src_k = (const uint32_t *)src_k + (size_t)src_seq * src_seq_words;
  f.src_v = (const uint32_t *)src_v + (size_t)src_seq * src_seq_words;
  f.src_len = src_len + src_seq;
  f.src_pre_len = src_pre.len ? src_pre.len + src_seq : nullptr;
  f.src_pre_seq = src_pre.seq ? src_pre.seq + src_seq : nullptr;
  f.pre_k = (const uint32_t *)src_pre.k;
  f.pre_v = (const uint32_t *)src_pre.v;
  f.pre_layer_words = pre_layer_elems * per / 2;
  f.pre_seq_words = (size_t)src_pre.max_seq * row_words;
  f.dst_k = (uint32_t *)dst_k;
  f.dst_v = (uint32_t *)dst_v;
  f.dst_layer_words = dst_layer_elems * per / 2;
  f.dst_seq_words = (size_t)dst_max_seq * row_words;
  f.dst_first = dst_first;
  f.dst_max_seq = dst_max_seq;
  f.row_words = depth > 0 ? row_words : 0;
  f.src_seq = src_seq;
  f.dst_len = dst_len;
  f.dst_pre_seq = dst_pre_seq;
  f.dst_pre_len = dst_pre_len;
  f.shared = shared ? 1 : 0;
  f.status = status;
  // 16-byte copies when rows, sequences, layers and the bases are 16-byte aligned
  const bool vec = row_words % 4 == 0 && ((uintptr_t)src_k | (uintptr_t)src_v | (uintptr_t)dst_k |
                                          (uintptr_t)dst_v | (uintptr_t)(src_pre.k ? src_pre.k : src_k) |
                                          (uintptr_t)(src_pre.v ? src_pre.v : src_v)) % 16 == 0;
  // blocks along the rows: about four vectors per thread at the longest length
  const size_t words = (size_t)dst_max_seq * row_words / (vec ? 4 : 1);
  unsigned bx = (unsigned)((words + 4 * 256 - 1) / (4 * 256));
  bx = bx < 1 ? 1 : (bx > 64 ? 64 : bx);
  dim3 grid(bx, (unsigned)(depth > 0 ? depth * 2 : 1), (unsigned)n);
  count_launch();
  if (vec) kv_fork_kernel<4><<<grid, 256, 0, s>>>(f);
  else kv_fork_kernel<1><<<grid, 256, 0, s>>>(f);
}

}  // namespace nc
