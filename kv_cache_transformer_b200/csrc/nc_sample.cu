// nc_sample.cu — sampled token pick over fp32 logits: temperature and top-k.
//
// The launch article lists sampling in its inference Engine ("高效推理") and
// gives no details; the pick made here is the usual one. Keep the top_k
// largest logits (ties on the cut keep the lower index), draw from
// softmax(z / temperature) over them. The draw is taken as the Gumbel-max
// argmax_v (z_v / temperature + g_v) with the noise g supplied by the caller,
// the same convention as the engine's argmax(logits + noise) pick;
// temperature 0 is the greedy pick.
//
// One CTA of 1024 threads per row. Each warp owns a contiguous slice of the
// row and reads it 32 consecutive logits at a time (coalesced), so the
// lowest-index rule on the cut is a prefix sum over the warps plus a ballot
// within each read; the row is re-read from L2 on every pass (it was just
// written by the lm_head):
//   select   the top_k-th largest logit by radix select on an order-preserving
//            32-bit key, 11 + 11 + 10 bits, histograms in shared memory with
//            warp-aggregated increments;
//   pick     among keys above the cut (and the first `need` keys equal to it),
//            the largest fl(fl(z / T) + g), lowest index on ties.
#include "nc_internal.h"
#include "nc_kernels.h"

namespace nc {
namespace {

constexpr int ST = 1024;   // threads per row
constexpr int NBIN = 2048;  // histogram bins (11-bit digits)

// Order-preserving key of a logit: larger z, larger key; -0 is keyed as +0 so
// that equal logits have equal keys.
__device__ __forceinline__ uint32_t order_key(float z) {
  const uint32_t u = __float_as_uint(z == 0.f ? 0.f : z);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix sum of v over the block's threads in thread order; every
// thread also gets the total. `wsum` holds 32 ints of shared memory.
__device__ __forceinline__ int block_excl_scan(int v, int *wsum, int *total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) wsum[w] = x;
  __syncthreads();
  if (w == 0) {
    int s = wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    wsum[lane] = s;  // inclusive over warps
  }
  __syncthreads();
  *total = wsum[31];
  return x - v + (w > 0 ? wsum[w - 1] : 0);
}

__global__ void __launch_bounds__(ST, 1)
    sample_topk_kernel(const float *__restrict__ logits, long long stride, int V, const float *__restrict__ noise,
                       float temperature, int top_k, const uint8_t *__restrict__ valid, int32_t *__restrict__ next) {
  const int row = blockIdx.x;
  if (valid && !valid[row]) return;
  __shared__ int hist[NBIN];
  __shared__ int wsum[32];
  __shared__ uint32_t s_digit;
  __shared__ int s_above, s_count;
  __shared__ ArgMax s_best[ST / 32];
  const float *z = logits + (size_t)row * (size_t)stride;
  const float *g = noise ? noise + (size_t)row * (size_t)V : nullptr;
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  // warp w reads [w0, w1) in rounds of 32 consecutive logits
  const int per_w = ((V + ST / 32 - 1) / (ST / 32) + 31) / 32 * 32;
  const int w0 = min(V, w * per_w), w1 = min(V, w0 + per_w);
  const bool greedy = temperature == 0.f;
  const int K = (top_k <= 0 || top_k >= V) ? V : top_k;

  // ---- select: the K-th largest key (tau), how many keys lie above it, and
  // how many keys equal to it are kept (need)
  uint32_t tau = 0;
  int need = 0, n_eq = 0;
  const bool cut = !greedy && K < V;
  if (cut) {
    uint32_t prefix = 0;
    int rem = K;
    const int shifts[3] = {21, 10, 0}, widths[3] = {11, 11, 10};
    for (int pass = 0; pass < 3; pass++) {
      const int sh = shifts[pass], nb = 1 << widths[pass];
      const int hi_sh = sh + widths[pass];  // bits above this digit, fixed by earlier passes
      for (int i = t; i < NBIN; i += ST) hist[i] = 0;
      __syncthreads();
      for (int i = w0 + lane; i < w0 + per_w; i += 32) {
        const bool in = i < w1;
        const uint32_t key = in ? order_key(__ldg(z + i)) : 0u;
        const bool take = in && (pass == 0 || (key >> hi_sh) == prefix);
        const uint32_t digit = (key >> sh) & (uint32_t)(nb - 1);
        const unsigned m = __ballot_sync(0xffffffffu, take);
        if (take) {
          const unsigned peers = __match_any_sync(m, digit);
          if (lane == __ffs(peers) - 1) atomicAdd(&hist[digit], __popc(peers));
        }
      }
      __syncthreads();
      // bins from the top: thread t owns bins nb-1-2t and nb-2-2t
      int c0 = 0, c1 = 0;
      const int b0 = nb - 1 - 2 * t, b1 = nb - 2 - 2 * t;
      if (b0 >= 0) c0 = hist[b0];
      if (b1 >= 0) c1 = hist[b1];
      int tot;
      const int above = block_excl_scan(c0 + c1, wsum, &tot);
      if (b0 >= 0 && above < rem && rem <= above + c0) {
        s_digit = (uint32_t)b0;
        s_above = above;
        s_count = c0;
      } else if (b1 >= 0 && above + c0 < rem && rem <= above + c0 + c1) {
        s_digit = (uint32_t)b1;
        s_above = above + c0;
        s_count = c1;
      }
      __syncthreads();
      prefix = (prefix << widths[pass]) | s_digit;
      rem -= s_above;
      n_eq = s_count;
      __syncthreads();
    }
    tau = prefix;
    need = rem;  // keys equal to tau that are kept (the lowest indices)
  }

  // ---- pick
  const bool tie = cut && need < n_eq;
  int eq_base = 0;  // keys equal to tau in the warps before this one
  if (tie) {        // a tie on the cut: rank the equal keys by index
    int mine = 0;
    for (int i = w0 + lane; i < w0 + per_w; i += 32)
      mine += __popc(__ballot_sync(0xffffffffu, i < w1 && order_key(__ldg(z + i)) == tau));
    int tot;
    eq_base = block_excl_scan(lane == 0 ? mine : 0, wsum, &tot);
    eq_base = __shfl_sync(0xffffffffu, eq_base, 0);
  }
  ArgMax best{-INFINITY, 0x7fffffff};
  int eq_seen = 0;  // equal keys in this warp's earlier rounds
  for (int i = w0 + lane; i < w0 + per_w; i += 32) {
    const bool in = i < w1;
    const float zi = in ? __ldg(z + i) : 0.f;
    bool member = in;
    if (cut) {
      const uint32_t key = order_key(zi);
      const bool eq = in && key == tau;
      if (tie) {
        const unsigned eqm = __ballot_sync(0xffffffffu, eq);
        const int rank = eq_base + eq_seen + __popc(eqm & ((1u << lane) - 1u));
        eq_seen += __popc(eqm);
        member = in && (eq ? rank < need : key > tau);
      } else {
        member = in && (eq || key > tau);
      }
    }
    if (!member) continue;
    const float s = greedy ? zi : __fadd_rn(__fdiv_rn(zi, temperature), g ? __ldg(g + i) : 0.f);
    best = argmax_merge(best, ArgMax{s, i});
  }
  best = warp_argmax(best);
  if (lane == 0) s_best[t >> 5] = best;
  __syncthreads();
  if (t < 32) {
    ArgMax b = t < ST / 32 ? s_best[t] : ArgMax{-INFINITY, 0x7fffffff};
    b = warp_argmax(b);
    if (t == 0) next[row] = b.i;
  }
}

}  // namespace

cudaError_t k_sample_topk(const float *logits, int B, int V, long long stride, const float *noise, float temperature,
                          int top_k, const uint8_t *valid, int32_t *next, cudaStream_t s) {
  count_launch();
  sample_topk_kernel<<<B, ST, 0, s>>>(logits, stride, V, noise, temperature, top_k, valid, next);
  return cudaGetLastError();
}

}  // namespace nc
