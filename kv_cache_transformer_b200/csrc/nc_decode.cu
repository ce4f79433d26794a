// nc_decode.cu — single-token decode step for bf16 models with head_dim 128,
// one KV head and up to 32 sequences.
//
// A decode step reads every weight once and each sequence's KV cache once, so
// it is bound by HBM bandwidth; the kernels are built to stream those bytes
// with all SMs busy and few launches per layer:
//
//   dec_embed      validate positions, token embedding + norm into the fp32
//                  residual x, per-128-column sums of squares of x
//   dec_linear     y[b, n] = sum_k X[b, k] W[n, k] with X = rmsnorm(x) or a
//                  bf16 activation: "swap-AB" tcgen05 MMA (M = 128 weight
//                  rows, N = 16/32 batch columns) over TMA-streamed weight
//                  tiles, split over K across CTAs; the last CTA of each
//                  128-row tile sums the fp32 partials and applies the fused
//                  epilogue:
//                    QKV     RoPE + QK norm, q out, K/V appended to the cache
//                    RESID   x += y and the sums of squares for the next norm
//                    RELU2   relu(y)^2 in bf16 (MLP hidden)
//                    LMHEAD  softcap, logits, (noise +) argmax: per-tile
//                            winners, merged by the last tile
//   dec_attn       split-KV flash decoding: Q (all H heads, one KV head) x
//                  K^T and P x V with mma.sync m16n8k16 on 64-key tiles in
//                  shared memory, online softmax; the last split of each
//                  sequence merges the partial (m, l, O) into y
//
// Every kernel is launched with programmatic stream serialization: it starts
// its weight prefetch while the previous kernel drains and waits
// (griddepcontrol.wait) before touching activations. Split-K and split-KV
// partials go to scratch owned by the cache object; the per-tile counters are
// reset by the CTA that consumes them, so the step can be replayed from a
// CUDA graph.
#include "nc_internal.h"
#include "nc_sm100.cuh"

namespace nc {
using namespace sm100;

namespace {

constexpr int DT = 128;           // weight rows per tile (MMA M)
constexpr int DSTAGES = 4;        // weight ring depth (16 KB tiles)
constexpr int WTILE = DT * 64 * 2;
constexpr int DTHREADS = 192;     // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t *r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ uint32_t pack_bf2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

}  // namespace

// ------------------------------------------------------------- arguments
struct DecLinArgs {
  int B, N, K, kblocks;
  int n_tiles, splits, kbs;  // k-blocks per split (the last split may have fewer)
  int units;                 // n_tiles * splits
  // X source
  const float *x;            // SRC_NORM: fp32 [B][K]
  const float *ss;           //           [K/128][ssb] partial sums of squares of x
  int ssb;
  float eps;
  const bf16 *act;           // SRC_BF16: [B][K]
  // scratch
  float *part;               // [units][NB][128]
  unsigned *counters;        // [n_tiles + 1], zero between launches
  // epilogue
  float *xres;               // RESID: x [B][N] (+=)
  float *ss_out;             // RESID: [N/128][ssb]
  bf16 *out;                 // RELU2: [B][N]; QKV: q [B][H][128]
  bf16 *kc, *vc;             // QKV: layer cache [max_batch][max_seq][128]
  int max_seq, H;
  const int32_t *pos;        // QKV: positions [B]
  const uint8_t *valid;      // [B]
  const float2 *rope;        // [max_seq][64]
  float *logits;             // LMHEAD: [B][V]
  const float *noise;        // LMHEAD: [B][V] or null
  float cap;
  float *cand_v;             // LMHEAD: [n_tiles][32]
  int *cand_i;
  int32_t *next;             // LMHEAD: [B] or null
  uint32_t *status;
};

enum { SRC_NORM = 0, SRC_BF16 = 1 };
enum { DEC_QKV = 0, DEC_RESID = 1, DEC_RELU2 = 2, DEC_LMHEAD = 3 };

template <int NB>
struct DecSmem {
  static constexpr int X_BYTES_PER_KB = NB * 128;  // one 64-column block of X, NB rows
};

// Finalize one 128-row output tile whose fp32 sums sit in tl[n * (NB+1) + b].
// Called by the 128 epilogue threads (e = 0..127 owns output row n = e).
template <int NB, int EPI>
__device__ void dec_finalize(const DecLinArgs &a, int nt, float *tl, float *red, int e) {
  const int lane = e & 31, w = e >> 5;
  const int col = nt * DT + e;
  if (EPI == DEC_RELU2) {
    for (int b = 0; b < a.B; b++) {
      float v = fmaxf(tl[e * (NB + 1) + b], 0.f);
      a.out[(size_t)b * a.N + col] = __float2bfloat16_rn(v * v);
    }
  } else if (EPI == DEC_RESID) {
    for (int b = 0; b < a.B; b++) {
      float v = a.xres[(size_t)b * a.N + col] + tl[e * (NB + 1) + b];
      a.xres[(size_t)b * a.N + col] = v;
      tl[e * (NB + 1) + b] = v * v;
    }
    epi_sync();
    for (int b = w; b < a.B; b += 4) {
      float s = tl[lane * (NB + 1) + b] + tl[(lane + 32) * (NB + 1) + b] + tl[(lane + 64) * (NB + 1) + b] +
                tl[(lane + 96) * (NB + 1) + b];
      s = warp_sum(s);
      if (lane == 0) a.ss_out[(size_t)nt * a.ssb + b] = s;
    }
  } else if (EPI == DEC_QKV) {
    const int head = nt;  // one 128-wide head per tile: q heads, then k, then v
    if (head <= a.H) {
      // RoPE on split-half pairs (e, e^64), then RMS norm over the head
      float rot[NB];
      const int i = e & 63;
#pragma unroll
      for (int b = 0; b < NB; b++) {
        rot[b] = 0.f;
        if (b < a.B) {
          int p = a.pos[b];
          p = p < 0 ? 0 : (p >= a.max_seq ? a.max_seq - 1 : p);
          float2 cs = a.rope[(size_t)p * 64 + i];
          float v = tl[e * (NB + 1) + b], u = tl[(e ^ 64) * (NB + 1) + b];
          rot[b] = e < 64 ? v * cs.x - u * cs.y : u * cs.y + v * cs.x;
        }
      }
      epi_sync();
#pragma unroll
      for (int b = 0; b < NB; b++) tl[e * (NB + 1) + b] = rot[b] * rot[b];
      epi_sync();
      for (int b = w; b < a.B; b += 4) {
        float s = tl[lane * (NB + 1) + b] + tl[(lane + 32) * (NB + 1) + b] + tl[(lane + 64) * (NB + 1) + b] +
                  tl[(lane + 96) * (NB + 1) + b];
        s = warp_sum(s);
        if (lane == 0) red[b] = rsqrtf(s * (1.0f / DT) + a.eps);
      }
      epi_sync();
#pragma unroll
      for (int b = 0; b < NB; b++) {
        if (b >= a.B) break;
        float v = rot[b] * red[b];
        if (head < a.H) {
          a.out[((size_t)b * a.H + head) * DT + e] = __float2bfloat16_rn(v);
        } else if (a.valid[b]) {
          int p = a.pos[b];
          if (p >= 0 && p < a.max_seq) a.kc[((size_t)b * a.max_seq + p) * DT + e] = __float2bfloat16_rn(v);
        }
      }
    } else {
      for (int b = 0; b < a.B; b++) {
        int p = a.pos[b];
        if (a.valid[b] && p >= 0 && p < a.max_seq)
          a.vc[((size_t)b * a.max_seq + p) * DT + e] = __float2bfloat16_rn(tl[e * (NB + 1) + b]);
      }
    }
  } else {  // DEC_LMHEAD
    const float inv = 1.0f / a.cap;
    for (int b = 0; b < a.B; b++) {
      float z = a.cap * tanhf(tl[e * (NB + 1) + b] * inv);
      if (a.valid[b]) a.logits[(size_t)b * a.N + col] = z;
      tl[e * (NB + 1) + b] = z + (a.noise ? a.noise[(size_t)b * a.N + col] : 0.f);
    }
    epi_sync();
    for (int b = w; b < a.B; b += 4) {
      ArgMax best{-INFINITY, 0x7fffffff};
#pragma unroll
      for (int q = 0; q < 4; q++) best = argmax_merge(best, ArgMax{tl[(lane + 32 * q) * (NB + 1) + b], nt * DT + lane + 32 * q});
      best = warp_argmax(best);
      if (lane == 0) {
        a.cand_v[(size_t)nt * 32 + b] = best.v;
        a.cand_i[(size_t)nt * 32 + b] = best.i;
      }
    }
    // the last finished tile merges every tile's winners
    __threadfence();
    epi_sync();
    __shared__ int last_tile;
    if (e == 0) last_tile = atomicAdd(&a.counters[a.n_tiles], 1u) == (unsigned)(a.n_tiles - 1);
    epi_sync();
    if (last_tile) {
      __threadfence();
      for (int b = w; b < a.B; b += 4) {
        ArgMax best{-INFINITY, 0x7fffffff};
        for (int t = lane; t < a.n_tiles; t += 32)
          best = argmax_merge(best, ArgMax{__ldcg(&a.cand_v[(size_t)t * 32 + b]), __ldcg(&a.cand_i[(size_t)t * 32 + b])});
        best = warp_argmax(best);
        if (lane == 0 && a.next && a.valid[b]) a.next[b] = best.i;
      }
      if (e == 0) a.counters[a.n_tiles] = 0;
    }
  }
}

template <int NB, int SRC, int EPI>
__global__ void __launch_bounds__(DTHREADS, 1) dec_linear_kernel(const __grid_constant__ CUtensorMap mapW, DecLinArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint32_t raw = smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw + 1023) & ~1023u) - raw);
  uint8_t *sW = smem;                                   // DSTAGES x 16 KB
  uint8_t *sX = smem + DSTAGES * WTILE;                 // kbs x NB x 128 B
  float *tl = reinterpret_cast<float *>(sX + a.kbs * NB * 128);  // [128][NB+1]
  uint64_t *full = reinterpret_cast<uint64_t *>(tl + DT * (NB + 1));
  uint64_t *empty = full + DSTAGES;
  uint64_t *afull = empty + DSTAGES;
  uint64_t *aempty = afull + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(aempty + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  float *red = reinterpret_cast<float *>(tmem_slot + 4);  // [32]
  int *flag = reinterpret_cast<int *>(red + 32);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sp = blockIdx.x % a.splits;                 // fixed split (grid % splits == 0)
  const int kb0 = sp * a.kbs;
  const int nkb = min(a.kbs, a.kblocks - kb0);
  int my_units = 0;
  for (int u = blockIdx.x; u < a.units; u += gridDim.x) my_units++;
  const int total_loads = my_units * nkb;

  if (threadIdx.x == 0) {
    for (int s = 0; s < DSTAGES; s++) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&afull[0], 1);
    mbar_init(&afull[1], 1);
    mbar_init(&aempty[0], 128);
    mbar_init(&aempty[1], 128);
    *abort_flag = 0;
    fence_barrier_init();
    // weights do not depend on the previous kernel: start streaming now
    for (int i = 0; i < total_loads && i < DSTAGES; i++) {
      const int u = blockIdx.x + (i / nkb) * gridDim.x;
      const int nt = u / a.splits;
      mbar_arrive_expect_tx(&full[i], WTILE);
      tma_load_2d(sW + i * WTILE, &mapW, (kb0 + i % nkb) * 64, nt * DT, &full[i]);
    }
  }
  if (warp == 1) tmem_alloc(tmem_slot, 2 * NB);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // ---- activations from the previous kernel: stage X (bf16, 128B swizzle)
  pdl_wait();
  if (SRC == SRC_NORM) {
    if (threadIdx.x < a.B) {
      float s = 0.f;
      for (int j = 0; j < a.K / DT; j++) s += a.ss[(size_t)j * a.ssb + threadIdx.x];
      red[threadIdx.x] = rsqrtf(s / a.K + a.eps);
    }
    __syncthreads();
  }
  for (int idx = threadIdx.x; idx < nkb * NB * 8; idx += DTHREADS) {
    const int c = idx & 7, b = (idx >> 3) % NB, kbl = idx / (8 * NB);
    const int k = (kb0 + kbl) * 64 + c * 8;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (b < a.B) {
      if (SRC == SRC_NORM) {
        const float4 *src = reinterpret_cast<const float4 *>(a.x + (size_t)b * a.K + k);
        float4 v0 = src[0], v1 = src[1];
        float r = red[b];
        val = make_uint4(pack_bf2(v0.x * r, v0.y * r), pack_bf2(v0.z * r, v0.w * r), pack_bf2(v1.x * r, v1.y * r),
                         pack_bf2(v1.z * r, v1.w * r));
      } else {
        val = *reinterpret_cast<const uint4 *>(a.act + (size_t)b * a.K + k);
      }
    }
    *reinterpret_cast<uint4 *>(sX + kbl * NB * 128 + b * 128 + ((c ^ (b & 7)) << 4)) = val;
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncthreads();
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      for (int i = DSTAGES; i < total_loads; i++) {
        const int s = i % DSTAGES;
        if (!mbar_wait(&empty[s], ((i / DSTAGES) - 1) & 1, abort_flag, a.status)) break;
        const int u = blockIdx.x + (i / nkb) * gridDim.x;
        const int nt = u / a.splits;
        mbar_arrive_expect_tx(&full[s], WTILE);
        tma_load_2d(sW + s * WTILE, &mapW, (kb0 + i % nkb) * 64, nt * DT, &full[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(DT, NB);
      const uint32_t x0 = smem_u32(sX);
      int i = 0;
      bool ok = true;
      for (int lu = 0; lu < my_units && ok; lu++) {
        const int acc = lu & 1;
        if (!mbar_wait(&aempty[acc], ((lu >> 1) & 1) ^ 1, abort_flag, a.status)) break;
        tc_fence_after();
        for (int kbl = 0; kbl < nkb; kbl++, i++) {
          const int s = i % DSTAGES;
          if (!mbar_wait(&full[s], (i / DSTAGES) & 1, abort_flag, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t w0 = smem_u32(sW + s * WTILE), xk = x0 + kbl * NB * 128;
#pragma unroll
          for (int k = 0; k < 4; k++)
            mma_bf16(tmem + acc * NB, desc_k_sw128(w0 + 32 * k), desc_k_sw128(xk + 32 * k), idesc, (kbl | k) != 0);
          mma_commit(&empty[s]);
        }
        mma_commit(&afull[acc]);
      }
    }
  } else {
    const int e = threadIdx.x - 64;          // 0..127: output row within the tile
    const int quarter = warp & 3;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int n = quarter * 32 + lane;       // TMEM lane = weight row
    int lu = 0;
    for (int u = blockIdx.x; u < a.units; u += gridDim.x, lu++) {
      const int acc = lu & 1;
      const int nt = u / a.splits;
      if (!mbar_wait(&afull[acc], (lu >> 1) & 1, abort_flag, a.status)) break;
      tc_fence_after();
      uint32_t r[NB];
      if constexpr (NB == 32) tmem_ld32(tmem + lane_off + acc * NB, r);
      else tmem_ld16(tmem + lane_off + acc * NB, r);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&aempty[acc]);
      if (a.splits == 1) {
#pragma unroll
        for (int b = 0; b < NB; b++) tl[n * (NB + 1) + b] = __uint_as_float(r[b]);
        epi_sync();
      } else {
        float *pp = a.part + (size_t)u * NB * DT;
#pragma unroll
        for (int b = 0; b < NB; b++) __stcg(&pp[b * DT + n], __uint_as_float(r[b]));
        __threadfence();
        epi_sync();
        if (e == 0) *flag = atomicAdd(&a.counters[nt], 1u) == (unsigned)(a.splits - 1);
        epi_sync();
        if (!*flag) continue;
        __threadfence();
        // sum the partials of every split of this tile, in split order
        float s[NB];
#pragma unroll
        for (int b = 0; b < NB; b++) s[b] = 0.f;
        for (int q = 0; q < a.splits; q++) {
          const float *pq = a.part + (size_t)(nt * a.splits + q) * NB * DT;
#pragma unroll
          for (int b = 0; b < NB; b++) s[b] += __ldcg(&pq[b * DT + e]);
        }
#pragma unroll
        for (int b = 0; b < NB; b++) tl[e * (NB + 1) + b] = s[b];
        if (e == 0) a.counters[nt] = 0;
        epi_sync();
      }
      dec_finalize<NB, EPI>(a, nt, tl, red, e);
      epi_sync();
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * NB);
  }
}

// -------------------------------------------------------------- embedding
// One block per sequence: validate the position, x = rmsnorm(wte[token]),
// per-128-column sums of squares of x for the first layer's norm.
__global__ void dec_embed_kernel(const int32_t *tokens, const int32_t *positions, int32_t *len, int32_t *pos_ws,
                                 uint8_t *valid, int max_seq, const bf16 *wte, int d, int vocab, float eps, float *x,
                                 float *ss, int ssb, uint32_t *status) {
  __shared__ float red[32];
  __shared__ float part[64];
  pdl_wait();
  const int b = blockIdx.x;
  if (threadIdx.x == 0) {
    int p = positions ? positions[b] : len[b];
    pos_ws[b] = p;
    bool ok = p >= 0 && p < max_seq && p == len[b];
    valid[b] = ok ? 1 : 0;
    if (ok) len[b] = p + 1;
    else atomicOr(status, (unsigned)NC_DEV_BAD_POSITION);
  }
  int tok = tokens[b];
  if (tok < 0 || tok >= vocab) {
    if (threadIdx.x == 0) atomicOr(status, (unsigned)NC_DEV_BAD_TOKEN);
    tok = tok < 0 ? 0 : vocab - 1;
  }
  const bf16 *row = wte + (size_t)tok * d;
  float s = 0.f;
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    float v = __bfloat162float(row[i]);
    s += v * v;
  }
  s = block_sum(s, red);
  const float inv = rsqrtf(s / d + eps);
  // blockDim.x == 128: thread i handles columns i, i+128, ... -> chunk j = column / 128
  const int nchunk = d / 128;
  for (int j = 0; j < nchunk; j++) {
    float v = __bfloat162float(row[j * 128 + threadIdx.x]) * inv;
    x[(size_t)b * d + j * 128 + threadIdx.x] = v;
    float q = warp_sum(v * v);
    if ((threadIdx.x & 31) == 0) part[(threadIdx.x >> 5)] = q;
    __syncthreads();
    if (threadIdx.x == 0) ss[(size_t)j * ssb + b] = part[0] + part[1] + part[2] + part[3];
    __syncthreads();
  }
  pdl_trigger();
}

// -------------------------------------------------------------- attention
struct DecAttnArgs {
  const bf16 *q;        // [B][H][128]
  const bf16 *kc, *vc;  // [max_batch][max_seq][128]
  const int32_t *pos;
  const uint8_t *valid;  // null: every sequence takes part
  int H, max_seq, chunk, splits;
  float scale_log2;
  float *part;          // [B][splits][16][130]: m, l, O[128] per head row
  unsigned *counters;   // [B]
  bf16 *y;              // [B][H][128]
  KvPrefix pre;         // shared prefixes (pre.len null: none)
};

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool pred) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(pred ? 16 : 0) : "memory");
}

constexpr int AKT = 64;                  // keys per shared-memory tile
constexpr int ATILE = AKT * 256;         // 64 keys x 128 dims bf16 = 16 KB
constexpr int ATHREADS = 128;

// Row `key` of a 256-byte-row tile, 16-byte chunk c, XOR-swizzled by key % 8.
__device__ __forceinline__ uint32_t atile_off(int key, int c) { return key * 256 + ((c ^ (key & 7)) << 4); }

__global__ void __launch_bounds__(ATHREADS) dec_attn_kernel(DecAttnArgs a) {
  extern __shared__ uint8_t smem_a[];
  uint8_t *sK = smem_a;                  // 2 stages
  uint8_t *sV = smem_a + 2 * ATILE;      // 2 stages
  __shared__ int is_last;
  const int split = blockIdx.x, b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3;
  pdl_wait();
  int pos = a.pos[b];
  const bool ok = a.valid ? a.valid[b] != 0 : true;
  pos = pos < 0 ? 0 : (pos >= a.max_seq ? a.max_seq - 1 : pos);
  const int n_keys = pos + 1;
  const int k_begin = split * a.chunk;
  const int k_end = min(k_begin + a.chunk, n_keys);
  const int n_tiles = k_end > k_begin ? (k_end - k_begin + AKT - 1) / AKT : 0;
  const bf16 *Kb = a.kc + (size_t)b * a.max_seq * 128;
  const bf16 *Vb = a.vc + (size_t)b * a.max_seq * 128;
  // keys below the shared length live in the prefix cache's sequence
  const int plen = a.pre.len ? a.pre.len[b] : 0;
  const bf16 *PK = plen ? (const bf16 *)a.pre.k + (size_t)a.pre.seq[b] * a.pre.max_seq * 128 : Kb;
  const bf16 *PV = plen ? (const bf16 *)a.pre.v + (size_t)a.pre.seq[b] * a.pre.max_seq * 128 : Vb;

  auto load_tile = [&](int it, int stage) {
    const int key0 = k_begin + it * AKT;
    const uint32_t kd = smem_u32(sK + stage * ATILE), vd = smem_u32(sV + stage * ATILE);
    for (int idx = threadIdx.x; idx < AKT * 16; idx += ATHREADS) {
      const int r = idx >> 4, c = idx & 15;
      const int key = key0 + r;
      const bool in = key < k_end;
      const size_t off = (size_t)(in ? key : 0) * 128 + c * 8;
      const bool sh = in && key < plen;
      cp_async16(kd + atile_off(r, c), (sh ? PK : Kb) + off, in);
      cp_async16(vd + atile_off(r, c), (sh ? PV : Vb) + off, in);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  // Q fragments (A operand, rows = heads, zero beyond H), 8 k-steps of 16 dims
  uint32_t qa[8][4];
  {
    const bf16 *qb = a.q + (size_t)b * a.H * 128;
#pragma unroll
    for (int ks = 0; ks < 8; ks++) {
      const int c0 = ks * 16 + t4 * 2;
      auto ld2 = [&](int row, int col) -> uint32_t {
        if (row >= a.H) return 0u;
        return *reinterpret_cast<const uint32_t *>(qb + (size_t)row * 128 + col);
      };
      qa[ks][0] = ld2(g, c0);
      qa[ks][1] = ld2(g + 8, c0);
      qa[ks][2] = ld2(g, c0 + 8);
      qa[ks][3] = ld2(g + 8, c0 + 8);
    }
  }
  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; i++) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  if (ok && n_tiles > 0) load_tile(0, 0);
  for (int it = 0; ok && it < n_tiles; it++) {
    const int stage = it & 1;
    if (it + 1 < n_tiles) {
      load_tile(it + 1, stage ^ 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    const uint32_t kbase = smem_u32(sK + stage * ATILE), vbase = smem_u32(sV + stage * ATILE);
    const int kw = warp * 16;                 // this warp's 16 keys of the tile
    const int key_glob0 = k_begin + it * AKT + kw;
    // S = Q K^T for 16 keys (two n8 tiles)
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < 8; ks++) {
      const int key = kw + (lane & 7) + ((lane >> 4) << 3);
      const int c = 2 * ks + ((lane >> 3) & 1);
      uint32_t b0, b1, b2, b3;
      ldsm_x4(kbase + atile_off(key, c), b0, b1, b2, b3);
      mma16816(s0, qa[ks], b0, b1);
      mma16816(s1, qa[ks], b2, b3);
    }
    // mask + online softmax; rows g (s*[0..1]) and g+8 (s*[2..3])
    float v[8] = {s0[0], s0[1], s1[0], s1[1], s0[2], s0[3], s1[2], s1[3]};
    const int kidx[4] = {key_glob0 + 2 * t4, key_glob0 + 2 * t4 + 1, key_glob0 + 8 + 2 * t4, key_glob0 + 9 + 2 * t4};
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const bool in = kidx[i] < k_end;
      v[i] = in ? v[i] * a.scale_log2 : -INFINITY;
      v[i + 4] = in ? v[i + 4] * a.scale_log2 : -INFINITY;
      mx0 = fmaxf(mx0, v[i]);
      mx1 = fmaxf(mx1, v[i + 4]);
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float al0 = mn0 == -INFINITY ? 1.f : exp2f(m0 - mn0), al1 = mn1 == -INFINITY ? 1.f : exp2f(m1 - mn1);
    float p[8];
#pragma unroll
    for (int i = 0; i < 4; i++) {
      p[i] = v[i] == -INFINITY ? 0.f : exp2f(v[i] - mn0);
      p[i + 4] = v[i + 4] == -INFINITY ? 0.f : exp2f(v[i + 4] - mn1);
    }
    l0 = l0 * al0 + p[0] + p[1] + p[2] + p[3];
    l1 = l1 * al1 + p[4] + p[5] + p[6] + p[7];
    m0 = mn0;
    m1 = mn1;
#pragma unroll
    for (int i = 0; i < 16; i++) {
      o[i][0] *= al0;
      o[i][1] *= al0;
      o[i][2] *= al1;
      o[i][3] *= al1;
    }
    uint32_t pa[4] = {pack_bf2(p[0], p[1]), pack_bf2(p[4], p[5]), pack_bf2(p[2], p[3]), pack_bf2(p[6], p[7])};
    // O += P V over this warp's 16 keys, 16 n8 tiles of dims
#pragma unroll
    for (int dt = 0; dt < 16; dt += 2) {
      const int key = kw + (lane & 7) + (((lane >> 3) & 1) << 3);
      const int c = dt + (lane >> 4);
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(vbase + atile_off(key, c), b0, b1, b2, b3);
      mma16816(o[dt], pa, b0, b1);
      mma16816(o[dt + 1], pa, b2, b3);
    }
    __syncthreads();
  }
  // row sums across the quad
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

  // combine the 4 warps in shared memory (reuse the K/V tiles): per warp
  // [16 rows][130] = m, l, O[128]
  float *cw = reinterpret_cast<float *>(smem_a);
  {
    float *mine = cw + warp * 16 * 130;
    if (t4 == 0) {
      mine[g * 130 + 0] = m0;
      mine[g * 130 + 1] = l0;
      mine[(g + 8) * 130 + 0] = m1;
      mine[(g + 8) * 130 + 1] = l1;
    }
#pragma unroll
    for (int dt = 0; dt < 16; dt++) {
      const int col = dt * 8 + 2 * t4;
      mine[g * 130 + 2 + col] = o[dt][0];
      mine[g * 130 + 2 + col + 1] = o[dt][1];
      mine[(g + 8) * 130 + 2 + col] = o[dt][2];
      mine[(g + 8) * 130 + 2 + col + 1] = o[dt][3];
    }
  }
  __syncthreads();
  float *dst = a.part + ((size_t)b * a.splits + split) * 16 * 130;
  for (int idx = threadIdx.x; idx < 16 * 128; idx += ATHREADS) {
    const int row = idx >> 7, col = idx & 127;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; w++) M = fmaxf(M, cw[w * 16 * 130 + row * 130]);
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < 4; w++) {
      const float mw = cw[w * 16 * 130 + row * 130];
      const float f = mw == -INFINITY ? 0.f : exp2f(mw - M);
      L += f * cw[w * 16 * 130 + row * 130 + 1];
      O += f * cw[w * 16 * 130 + row * 130 + 2 + col];
    }
    __stcg(&dst[row * 130 + 2 + col], O);
    if (col == 0) {
      __stcg(&dst[row * 130 + 0], M);
      __stcg(&dst[row * 130 + 1], L);
    }
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = atomicAdd(&a.counters[b], 1u) == (unsigned)(a.splits - 1);
  __syncthreads();
  pdl_trigger();
  if (!is_last) return;
  __threadfence();
  // merge the splits of sequence b into y
  const float *src = a.part + (size_t)b * a.splits * 16 * 130;
  for (int idx = threadIdx.x; idx < a.H * 128; idx += ATHREADS) {
    const int row = idx >> 7, col = idx & 127;
    float M = -INFINITY;
    for (int s = 0; s < a.splits; s++) M = fmaxf(M, __ldcg(&src[(s * 16 + row) * 130]));
    float L = 0.f, O = 0.f;
    for (int s = 0; s < a.splits; s++) {
      const float ms = __ldcg(&src[(s * 16 + row) * 130]);
      const float f = ms == -INFINITY ? 0.f : exp2f(ms - M);
      L += f * __ldcg(&src[(s * 16 + row) * 130 + 1]);
      O += f * __ldcg(&src[(s * 16 + row) * 130 + 2 + col]);
    }
    a.y[((size_t)b * a.H + row) * 128 + col] = __float2bfloat16_rn(L > 0.f ? O / L : 0.f);
  }
  if (threadIdx.x == 0) a.counters[b] = 0;
}

// ------------------------------------------------------------------ host
bool make_map_bf16_k64(CUtensorMap *map, const void *ptr, int rows, int cols, int ld, int box_rows);

namespace {

template <typename Kern, typename... Args>
cudaError_t launch_pdl(Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  count_launch();
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <int NB>
size_t dec_linear_smem(int kbs) {
  return 1024 + DSTAGES * WTILE + (size_t)kbs * NB * 128 + DT * (NB + 1) * 4 + 256 + 64 * 4;
}

// Pick the K split so that about two CTAs per SM stream equal weight slices.
void plan_split(int n_tiles, int kblocks, int num_sms, int &splits, int &kbs) {
  splits = 1;
  if (n_tiles < 2 * num_sms) {
    splits = (2 * num_sms) / n_tiles;
    if (splits > kblocks) splits = kblocks;
    if (splits < 1) splits = 1;
  }
  kbs = (kblocks + splits - 1) / splits;
  splits = (kblocks + kbs - 1) / kbs;  // no empty split
}

template <int NB, int SRC, int EPI>
cudaError_t launch_dec_linear_t(const CUtensorMap &map, DecLinArgs &a, int num_sms, cudaStream_t s) {
  size_t smem = dec_linear_smem<NB>(a.kbs);
  {
    const cudaError_t e = ensure_smem_attr((const void *)dec_linear_kernel<NB, SRC, EPI>, smem);
    if (e != cudaSuccess) return e;
  }
  int per_sm = smem * 2 + 2048 <= 227 * 1024 ? 2 : 1;
  int grid = a.units < per_sm * num_sms ? a.units : per_sm * num_sms;
  grid -= grid % a.splits;
  if (grid < a.splits) grid = a.splits;
  return launch_pdl(dec_linear_kernel<NB, SRC, EPI>, dim3(grid), dim3(DTHREADS), smem, s, map, a);
}

template <int NB>
cudaError_t launch_dec_linear_nb(int src, int epi, const CUtensorMap &map, DecLinArgs &a, int num_sms, cudaStream_t s) {
  if (src == SRC_NORM) {
    if (epi == DEC_QKV) return launch_dec_linear_t<NB, SRC_NORM, DEC_QKV>(map, a, num_sms, s);
    if (epi == DEC_RELU2) return launch_dec_linear_t<NB, SRC_NORM, DEC_RELU2>(map, a, num_sms, s);
    if (epi == DEC_LMHEAD) return launch_dec_linear_t<NB, SRC_NORM, DEC_LMHEAD>(map, a, num_sms, s);
  } else {
    if (epi == DEC_RESID) return launch_dec_linear_t<NB, SRC_BF16, DEC_RESID>(map, a, num_sms, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool decode_head_supported(const nc_config &c) {
  return c.dtype == NC_BF16 && c.head_dim == 128 && c.d_model % 128 == 0 && c.mlp_hidden % 128 == 0 &&
         c.vocab % 128 == 0 && c.d_model / 128 <= 64;
}

bool decode_fast_supported(const nc_config &c, int B) {
  return decode_head_supported(c) && c.n_kv_head == 1 && c.n_head <= 16 && B >= 1 && B <= 32;
}

// Scratch sizes for a cache of max_batch sequences (see DecodeScratch).
size_t decode_part_floats(const nc_config &c, int max_batch, int max_seq, int num_sms, int *attn_splits,
                          int *attn_chunk) {
  (void)max_batch;
  size_t need = 0;
  const int N[5] = {(c.n_head + 2 * c.n_kv_head) * 128, c.d_model, c.mlp_hidden, c.d_model, c.vocab};
  const int K[5] = {c.d_model, c.n_head * 128, c.d_model, c.mlp_hidden, c.d_model};
  for (int i = 0; i < 5; i++) {
    int splits, kbs;
    plan_split(N[i] / 128, K[i] / 64, num_sms, splits, kbs);
    size_t f = (size_t)(N[i] / 128) * splits * 32 * 128;
    if (splits > 1 && f > need) need = f;
  }
  // attention split-KV: about two CTAs per SM over the batch
  int chunk = AKT;
  while ((size_t)((max_seq + chunk - 1) / chunk) * max_batch > (size_t)2 * num_sms && chunk < max_seq) chunk += AKT;
  *attn_chunk = chunk;
  *attn_splits = (max_seq + chunk - 1) / chunk;
  size_t fa = (size_t)max_batch * (*attn_splits) * 16 * 130;
  return need > fa ? need : fa;
}

// Split-KV plan for the kernel-level decode attention entry points: keys in
// chunks of a multiple of 64, about two CTAs per SM over the batch, at most
// 16 splits per sequence.
void attn_decode_plan(int B, int max_seq, int num_sms, int *chunk, int *splits) {
  int c = AKT;
  while (((max_seq + c - 1) / c) * B > 2 * num_sms && c < max_seq) c += AKT;
  while ((max_seq + c - 1) / c > 16) c += AKT;
  *chunk = c;
  *splits = (max_seq + c - 1) / c;
}

size_t attn_decode_partial_floats(int B, int splits) { return (size_t)B * splits * 16 * 130; }

cudaError_t k_dec_embed(const int32_t *tokens, const int32_t *positions, int32_t *len, int32_t *pos_ws,
                        uint8_t *valid, int B, int max_seq, const void *wte, int d, int vocab, float eps, float *x,
                        float *ss, int ssb, uint32_t *status, cudaStream_t s) {
  return launch_pdl(dec_embed_kernel, dim3(B), dim3(128), 0, s, tokens, positions, len, pos_ws, valid, max_seq,
                    (const bf16 *)wte, d, vocab, eps, x, ss, ssb, status);
}

cudaError_t k_dec_linear(int src, int epi, const void *W, int N, int K, int B, const float *x, const float *ss, int ssb,
                         float eps, const void *act, float *part, unsigned *counters, float *xres, float *ss_out,
                         void *out, void *kc, void *vc, int max_seq, int H, const int32_t *pos, const uint8_t *valid,
                         const float2 *rope, float *logits, const float *noise, float cap, float *cand_v, int *cand_i,
                         int32_t *next, uint32_t *status, int num_sms, cudaStream_t s) {
  CUtensorMap map;
  if (!make_map_bf16_k64(&map, W, N, K, K, DT)) return cudaErrorInvalidValue;
  DecLinArgs a = {};
  a.B = B;
  a.N = N;
  a.K = K;
  a.kblocks = K / 64;
  a.n_tiles = N / DT;
  plan_split(a.n_tiles, a.kblocks, num_sms, a.splits, a.kbs);
  a.units = a.n_tiles * a.splits;
  a.x = x;
  a.ss = ss;
  a.ssb = ssb;
  a.eps = eps;
  a.act = (const bf16 *)act;
  a.part = part;
  a.counters = counters;
  a.xres = xres;
  a.ss_out = ss_out;
  a.out = (bf16 *)out;
  a.kc = (bf16 *)kc;
  a.vc = (bf16 *)vc;
  a.max_seq = max_seq;
  a.H = H;
  a.pos = pos;
  a.valid = valid;
  a.rope = rope;
  a.logits = logits;
  a.noise = noise;
  a.cap = cap;
  a.cand_v = cand_v;
  a.cand_i = cand_i;
  a.next = next;
  a.status = status;
  if (B <= 16) return launch_dec_linear_nb<16>(src, epi, map, a, num_sms, s);
  return launch_dec_linear_nb<32>(src, epi, map, a, num_sms, s);
}

cudaError_t k_dec_attn(const void *q, const void *kc, const void *vc, const int32_t *pos, const uint8_t *valid, int B,
                       int H, int max_seq, int chunk, int splits, float *part, unsigned *counters, void *y,
                       cudaStream_t s, const KvPrefix *pre) {
  DecAttnArgs a;
  a.pre = pre ? *pre : KvPrefix{};
  a.q = (const bf16 *)q;
  a.kc = (const bf16 *)kc;
  a.vc = (const bf16 *)vc;
  a.pos = pos;
  a.valid = valid;
  a.H = H;
  a.max_seq = max_seq;
  a.chunk = chunk;
  a.splits = splits;
  a.scale_log2 = 1.4426950408889634f / sqrtf(128.f);
  a.part = part;
  a.counters = counters;
  a.y = (bf16 *)y;
  const size_t smem = 4 * ATILE;
  {
    const cudaError_t e = ensure_smem_attr((const void *)dec_attn_kernel, smem);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(dec_attn_kernel, dim3(splits, B), dim3(ATHREADS), smem, s, a);
}

}  // namespace nc
