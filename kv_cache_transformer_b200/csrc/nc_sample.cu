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
// row and reads it 32 consecutive logits at a time (coalesced), eight such
// rounds in flight before any is used, so the lowest-index rule on the cut is
// a prefix sum over the warps plus a ballot within each round; the row is
// re-read from L2 (it was just written by the lm_head):
//   select   the top_k-th largest logit by radix select on an order-preserving
//            32-bit key, four 8-bit digits; each warp counts into its own
//            histogram in shared memory (plain shared atomics), and the 32
//            histograms are added before the digit is chosen, so no two
//            warps contend for a bin. After the first digit, the keys whose
//            top digit is at or above the chosen one (every candidate of the
//            top_k) are compacted, in index order, into a list in shared
//            memory when they fit, and the remaining digits and the pick run
//            on that list; otherwise every pass re-reads the row;
//   pick     among keys above the cut (and the first `need` keys equal to it),
//            the largest fl(fl(z / T) + g), lowest index on ties.
#include "nc_internal.h"
#include "nc_kernels.h"

namespace nc {
namespace {

constexpr int ST = 1024;   // threads per row
constexpr int NBIN = 256;   // histogram bins (8-bit digits)
constexpr int NBAT = 8;     // rounds of 32 logits a warp loads before using them
constexpr int LCAP = 6144;  // candidate list entries (key, index)
constexpr size_t SMEM_BYTES = (size_t)LCAP * 8;  // the list, in dynamic shared memory

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

// VEC: rows start on 16-byte boundaries and V % 4 == 0, so the two full
// reads (top-digit histogram, compaction) load four logits per lane per round.
template <bool VEC>
__global__ void __launch_bounds__(ST, 1)
    sample_topk_kernel(const float *__restrict__ logits, long long stride, int V, const float *__restrict__ noise,
                       float temperature, int top_k, const uint8_t *__restrict__ valid, int32_t *__restrict__ next) {
  const int row = blockIdx.x;
  if (valid && !valid[row]) return;
  __shared__ int whist[ST / 32][NBIN];  // one histogram per warp
  __shared__ int part[4][NBIN];         // sums over warps 8q .. 8q+7
  __shared__ int wsum[32];
  __shared__ uint32_t s_digit;
  __shared__ int s_above, s_count;
  __shared__ ArgMax s_best[ST / 32];
  extern __shared__ uint32_t lmem[];
  uint32_t *lkey = lmem;                                 // [LCAP] candidate keys, in index order
  int *lidx = reinterpret_cast<int *>(lmem + LCAP);      // [LCAP] their indices
  const float *z = logits + (size_t)row * (size_t)stride;
  const float *g = noise ? noise + (size_t)row * (size_t)V : nullptr;
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  // warp w reads [w0, w1) in rounds of 32 consecutive logits, NBAT rounds a
  // batch (vector reads: rounds of 32 x 4, NBAT / 2 rounds a batch)
  const int per_w = ((V + ST / 32 - 1) / (ST / 32) + 64 * NBAT - 1) / (64 * NBAT) * (64 * NBAT);
  const int w0 = min(V, w * per_w), w1 = min(V, w0 + per_w);
  const bool greedy = temperature == 0.f;
  const int K = (top_k <= 0 || top_k >= V) ? V : top_k;

  // ---- select: the K-th largest key (tau), how many keys lie above it, and
  // how many keys equal to it are kept (need)
  uint32_t tau = 0;
  int need = 0, n_eq = 0;
  const bool cut = !greedy && K < V;
  bool compact = false;  // the candidates are in the list
  int n_list = 0;
  if (cut) {
    uint32_t prefix = 0;
    int rem = K;
    for (int pass = 0; pass < 4; pass++) {
      const int sh = 24 - 8 * pass;
      const int hi_sh = sh + 8;  // bits above this digit, fixed by earlier passes (pass >= 1)
#pragma unroll
      for (int i = lane; i < NBIN; i += 32) whist[w][i] = 0;
      __syncwarp();
      if (compact) {
        for (int e = t; e < n_list; e += ST) {
          const uint32_t key = lkey[e];
          if ((key >> hi_sh) == prefix) atomicAdd(&whist[w][(key >> sh) & (uint32_t)(NBIN - 1)], 1);
        }
      } else if (VEC && pass == 0) {
        constexpr int NB4 = NBAT / 2;
        for (int base = w0; base < w0 + per_w; base += 128 * NB4) {
          float4 zq[NB4];
#pragma unroll
          for (int r = 0; r < NB4; r++) {
            const int i = base + 128 * r + 4 * lane;
            zq[r] = i < w1 ? __ldg(reinterpret_cast<const float4 *>(z + i)) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int r = 0; r < NB4; r++) {
            if (base + 128 * r + 4 * lane >= w1) continue;
            atomicAdd(&whist[w][order_key(zq[r].x) >> 24], 1);
            atomicAdd(&whist[w][order_key(zq[r].y) >> 24], 1);
            atomicAdd(&whist[w][order_key(zq[r].z) >> 24], 1);
            atomicAdd(&whist[w][order_key(zq[r].w) >> 24], 1);
          }
        }
      } else
      for (int base = w0; base < w0 + per_w; base += 32 * NBAT) {
        uint32_t key[NBAT];
#pragma unroll
        for (int r = 0; r < NBAT; r++) {
          const int i = base + 32 * r + lane;
          key[r] = i < w1 ? order_key(__ldg(z + i)) : 0u;
        }
#pragma unroll
        for (int r = 0; r < NBAT; r++) {
          const bool take = base + 32 * r + lane < w1 && (pass == 0 ? true : (key[r] >> hi_sh) == prefix);
          const uint32_t digit = (key[r] >> sh) & (uint32_t)(NBIN - 1);
          if (take) atomicAdd(&whist[w][digit], 1);
        }
      }
      __syncthreads();
      {  // the warps' histograms added: thread t sums bin t % 256 over 8 warps
        const int bin = t & (NBIN - 1), q = t / NBIN;
        int c = 0;
#pragma unroll
        for (int v = 0; v < 8; v++) c += whist[8 * q + v][bin];
        part[q][bin] = c;
      }
      __syncthreads();
      // bins from the top: thread t < 256 owns bin 255 - t
      const int b0 = NBIN - 1 - t;
      const int c0 = t < NBIN ? part[0][b0] + part[1][b0] + part[2][b0] + part[3][b0] : 0;
      int tot;
      const int above = block_excl_scan(c0, wsum, &tot);
      if (t < NBIN && above < rem && rem <= above + c0) {
        s_digit = (uint32_t)b0;
        s_above = above;
        s_count = c0;
      }
      __syncthreads();
      prefix = (prefix << 8) | s_digit;
      rem -= s_above;
      n_eq = s_count;
      if (pass == 0 && s_above + s_count <= LCAP) {
        // compact the keys with top digit >= d0, in index order: each warp's
        // count from its own histogram, warp offsets by a block scan, then
        // positions within a warp by ballot
        const uint32_t d0 = s_digit;
        int cw = 0;
        for (int bin = (int)d0 + lane; bin < NBIN; bin += 32) cw += whist[w][bin];
        cw = __reduce_add_sync(0xffffffffu, cw);
        int tot;
        int wbase = block_excl_scan(lane == 0 ? cw : 0, wsum, &tot);
        wbase = __shfl_sync(0xffffffffu, wbase, 0);
        int seen = 0;
        if (VEC) {
          // a round is 128 consecutive logits, 4 per lane: a key's place is
          // the candidates of the lanes below plus those before it in its lane
          constexpr int NB4 = NBAT / 2;
          for (int base = w0; base < w0 + per_w; base += 128 * NB4) {
            float4 zq[NB4];
#pragma unroll
            for (int r = 0; r < NB4; r++) {
              const int i = base + 128 * r + 4 * lane;
              zq[r] = i < w1 ? __ldg(reinterpret_cast<const float4 *>(z + i)) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int r = 0; r < NB4; r++) {
              const int i = base + 128 * r + 4 * lane;
              const bool in = i < w1;
              const uint32_t k4[4] = {order_key(zq[r].x), order_key(zq[r].y), order_key(zq[r].z), order_key(zq[r].w)};
              int c = 0;
#pragma unroll
              for (int q = 0; q < 4; q++) c += in && (k4[q] >> 24) >= d0;
              int incl = c;  // inclusive prefix over the lanes
#pragma unroll
              for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
              }
              int at = wbase + seen + incl - c;
#pragma unroll
              for (int q = 0; q < 4; q++)
                if (in && (k4[q] >> 24) >= d0) {
                  lkey[at] = k4[q];
                  lidx[at] = i + q;
                  at++;
                }
              seen += __shfl_sync(0xffffffffu, incl, 31);
            }
          }
        } else
        for (int base = w0; base < w0 + per_w; base += 32 * NBAT) {
          uint32_t key[NBAT];
#pragma unroll
          for (int r = 0; r < NBAT; r++) {
            const int i = base + 32 * r + lane;
            key[r] = i < w1 ? order_key(__ldg(z + i)) : 0u;
          }
#pragma unroll
          for (int r = 0; r < NBAT; r++) {
            const int i = base + 32 * r + lane;
            const bool c = i < w1 && (key[r] >> 24) >= d0;
            const unsigned m = __ballot_sync(0xffffffffu, c);
            if (c) {
              const int at = wbase + seen + __popc(m & ((1u << lane) - 1u));
              lkey[at] = key[r];
              lidx[at] = i;
            }
            seen += __popc(m);
          }
        }
        n_list = tot;
        compact = true;
      }
      __syncthreads();
    }
    tau = prefix;
    need = rem;  // keys equal to tau that are kept (the lowest indices)
  }

  // ---- pick
  const bool tie = cut && need < n_eq;
  ArgMax best{-INFINITY, 0x7fffffff};
  if (compact) {
    // thread t takes a contiguous run of the list (index order), so the rank of
    // an equal key is a block prefix sum plus its place in the run
    const int per = (n_list + ST - 1) / ST;
    const int e0 = min(n_list, t * per), e1 = min(n_list, e0 + per);
    int eq_rank = 0;
    if (tie) {
      int mine = 0;
      for (int e = e0; e < e1; e++) mine += lkey[e] == tau;
      int tot;
      eq_rank = block_excl_scan(mine, wsum, &tot);
    }
    for (int e = e0; e < e1; e++) {
      const uint32_t key = lkey[e];
      const bool member = key == tau ? (!tie || eq_rank++ < need) : key > tau;
      if (!member) continue;
      const int i = lidx[e];
      const float sc = __fadd_rn(__fdiv_rn(__ldg(z + i), temperature), g ? __ldg(g + i) : 0.f);
      best = argmax_merge(best, ArgMax{sc, i});
    }
  } else {
  int eq_base = 0;  // keys equal to tau in the warps before this one
  if (tie) {        // a tie on the cut: rank the equal keys by index
    int mine = 0;
    for (int base = w0; base < w0 + per_w; base += 32 * NBAT) {
      uint32_t key[NBAT];
#pragma unroll
      for (int r = 0; r < NBAT; r++) {
        const int i = base + 32 * r + lane;
        key[r] = i < w1 ? order_key(__ldg(z + i)) : ~tau;
      }
#pragma unroll
      for (int r = 0; r < NBAT; r++) mine += __popc(__ballot_sync(0xffffffffu, key[r] == tau));
    }
    int tot;
    eq_base = block_excl_scan(lane == 0 ? mine : 0, wsum, &tot);
    eq_base = __shfl_sync(0xffffffffu, eq_base, 0);
  }
  int eq_seen = 0;  // equal keys in this warp's earlier rounds
  for (int base = w0; base < w0 + per_w; base += 32 * NBAT) {
    float zv[NBAT], gv[NBAT];
#pragma unroll
    for (int r = 0; r < NBAT; r++) {
      const int i = base + 32 * r + lane;
      zv[r] = i < w1 ? __ldg(z + i) : 0.f;
      gv[r] = (g && i < w1) ? __ldg(g + i) : 0.f;
    }
#pragma unroll
    for (int r = 0; r < NBAT; r++) {
      const int i = base + 32 * r + lane;
      const bool in = i < w1;
      bool member = in;
      if (cut) {
        const uint32_t key = order_key(zv[r]);
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
      if (member) {
        const float sc = greedy ? zv[r] : __fadd_rn(__fdiv_rn(zv[r], temperature), gv[r]);
        best = argmax_merge(best, ArgMax{sc, i});
      }
    }
  }
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
  const bool vec = V % 4 == 0 && stride % 4 == 0 && (uintptr_t)logits % 16 == 0;
  const void *fn = vec ? (const void *)sample_topk_kernel<true> : (const void *)sample_topk_kernel<false>;
  const cudaError_t e = ensure_smem_attr(fn, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  count_launch();
  if (vec) sample_topk_kernel<true><<<B, ST, SMEM_BYTES, s>>>(logits, stride, V, noise, temperature, top_k, valid, next);
  else sample_topk_kernel<false><<<B, ST, SMEM_BYTES, s>>>(logits, stride, V, noise, temperature, top_k, valid, next);
  return cudaGetLastError();
}

}  // namespace nc
