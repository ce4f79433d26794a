// nc_step.cu — the whole single-token decode step as one persistent kernel.
//
// A decode step of the nanochat Transformer is a chain of about 5 x depth
// all-to-all dependencies (QKV -> attention -> O-proj -> MLP fc -> MLP proj
// per layer); the bytes it must move (every weight once, each sequence's KV
// cache once) take ~0.24 ms on a B200. Launching each link as its own kernel
// costs more than the bytes. Here one kernel runs the whole step:
//
//  * as many 4-CTA clusters as the occupancy query places (33 on a B200:
//    132 CTAs, one per SM), one phase per link, separated by a grid barrier
//    (a counter zeroed before each launch, release increments, acquire
//    polling, bounded);
//  * warp 0 is a TMA producer that walks the same phase program as everyone
//    and streams every weight tile and KV-cache tile this CTA will need into
//    a 6-slot shared-memory ring, running ahead across phase barriers —
//    neither weights nor the cached keys depend on the step's activations
//    (the one new key per sequence is patched in from global memory);
//  * warp 1 issues the tensor-core work of linear layers: swap-AB tcgen05
//    MMA, M = 128 weight rows, N = 32 batch columns, fp32 in TMEM, two
//    accumulator sets so a CTA's next weight tile overlaps the current one's
//    reduction and epilogue;
//  * warps 2-5 stage the activations (once per phase: every weight tile of a
//    phase multiplies the same slice), read the accumulators and run the
//    epilogues and the attention. The four CTAs of a cluster split K
//    (linears) or the keys (attention); each CTA pushes the batch columns
//    (linears) or heads (attention) another CTA finishes straight into that
//    CTA's shared-memory inbox, so the finishing CTA reduces locally. The MLP
//    projection, with few weight tiles and a long K, also splits K over
//    several clusters per tile; the last cluster to arrive adds the partials
//    in split order.
//
// Phases: EMBED | depth x [QKV | ATTN | OPROJ | FC | PROJ] | HEAD | MERGE.
//   EMBED  validate positions, x0 = rmsnorm(wte[token]), sum of squares
//   QKV    rmsnorm(x0) . [Wq;Wk;Wv]^T; RoPE + QK norm; q out; K/V appended
//   ATTN   flash decoding over the cache with mma.sync (one KV head, all H
//          query heads), cluster merge of the key splits -> y
//   OPROJ  x1 = x0 + y . Wo^T, sums of squares of x1
//   FC     f = relu(rmsnorm(x1) . Wfc^T)^2
//   PROJ   x0 = x1 + f . Wproj^T, sums of squares of x0
//   HEAD   logits = cap * tanh(rmsnorm(x0) . Wlm^T / cap) (+ noise), per-tile
//          argmax winners
//   MERGE  next token per sequence, lengths advanced
// Every wait is bounded (~2 s): a timeout raises NC_DEV_TIMEOUT and all
// roles drain to the exit, where TMEM is freed.
#include <cooperative_groups.h>

#include "nc_internal.h"
#include "nc_sm100.cuh"

namespace cg = cooperative_groups;

namespace nc {
using namespace sm100;

namespace {

constexpr int CL = 4;                  // CTAs per cluster
constexpr int NB = 32;                 // batch columns of the MMA (B <= 32)
constexpr int RING = 6;                // 16 KB ring slots
constexpr int SLOT = 16384;
constexpr int XKB = 20;                // X staging capacity, 64-column blocks
constexpr int THREADS = 192;
constexpr int KT = 64;                 // keys per attention tile
constexpr int NACC = 4;                // TMEM accumulators the K loop rotates over
constexpr int SSN = 16;                // 128-column chunks of d_model (d <= 2048)
constexpr int SPLIT_TILES = 16;        // MLP proj n-tiles (d / 128) the cross-cluster K split supports
constexpr int SPLIT_MAX = 4;           // clusters per MLP proj n-tile at most

constexpr int OFF_RING = 0;
constexpr int OFF_X = OFF_RING + RING * SLOT;          // XKB * NB * 128 bytes
constexpr int OFF_RED = OFF_X + XKB * NB * 128;         // 16 KB, read by cluster peers
constexpr int OFF_TL = OFF_RED + 16384;                 // [128][NB+1] fp32
constexpr int OFF_BAR = OFF_TL + 128 * (NB + 1) * 4;
constexpr int SMEM_BYTES = OFF_BAR + 1024 + 1024;  // barriers and per-row tables, then alignment slack

enum Phase { P_EMBED = 0, P_QKV, P_ATTN, P_OPROJ, P_FC, P_PROJ, P_HEAD, P_MERGE };

struct StepArgs {
  int L, d, H, F, V, B, max_batch, max_seq, grid;
  float eps, cap, scale_log2;
  const bf16 *wte;
  const CUtensorMap *wmaps;   // [4L + 1]: per layer qkv, o, fc, proj; then lm_head
  const CUtensorMap *kvmaps;  // [2]: K and V cache as [L * max_batch * max_seq, 128]
  const int32_t *tokens, *positions;
  int32_t *len;
  float *x0, *x1;             // residual [32][d]: layer input, after attention
  float *ss;                  // [2L + 1][SSN][32]: per-128-column sums of squares for each norm
  bf16 *q, *y, *f;            // [32][H][128], [32][d], [32][F]
  bf16 *kc, *vc;              // [L][max_batch][max_seq][128]
  const float2 *rope;         // [max_seq][64]
  float *logits;              // [B][V]
  const float *noise;         // [B][V] or null
  int32_t *next;              // [B] or null
  float *cand_v;              // [V/128][32]
  int *cand_i;
  unsigned long long *bar;    // grid barrier counter, followed by split_cnt
  unsigned *split_cnt;        // [SPLIT_TILES][CL]: arrivals of the K-split MLP proj partials
  float *split_part;          // [n_tiles * S][CL][128][NB/CL]: their partial sums
  uint32_t *status;
  unsigned long long *trace;  // [grid][phases][8] phase timestamps (ns), or null
  uint8_t *valid_out;         // [B]: 1 where the sequence's position was valid (written by CTA 0)
};

// Phase timestamps for nc_decode_trace: slot 0 phase start (after the last
// barrier), 1 activations staged / first cache tile in, 2 first accumulator
// complete, 3 last cluster reduction done, 4 epilogue done (barrier entry),
// 5 producer's first load of the phase, 6 its last load, 7 the MMA issuer's
// last commit of the phase. Only written when a trace buffer is set.
__device__ __forceinline__ void trace_mark(const StepArgs &a, int p, int slot) {
  if (a.trace) a.trace[((size_t)blockIdx.x * (3 + 5 * a.L) + p) * 8 + slot] = global_ns();
}

struct Smem {
  uint64_t *full, *empty, *x_ready, *x_free, *red_full, *red_free;
  uint64_t *acc_full, *acc_empty;  // [2] each: one per TMEM accumulator set
  uint32_t *tmem_slot;
  int *abort_flag;
  int *pos, *valid;  // [32]
  float *inv;        // [32] per-row scale for X staging
  float *qn;         // [32] QK-norm factors of the QKV epilogue
  int *flag;
};

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_bf(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

// arrive (release, cluster scope) on the same-offset mbarrier of CTA `rank`
__device__ __forceinline__ void mbar_arrive_remote(uint64_t *bar, uint32_t rank) {
  asm volatile(
      "{\n .reg .b32 ra;\n mapa.shared::cluster.u32 ra, %0, %1;\n"
      " mbarrier.arrive.release.cluster.shared::cluster.b64 _, [ra];\n}" ::"r"(smem_u32(bar)),
      "r"(rank)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ bool mbar_wait_cluster(uint64_t *bar, uint32_t parity, volatile int *abort_flag, uint32_t *status) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait_cluster(a, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait_cluster(a, parity)) return true;
    if ((it & 63) == 63) {
      if (*abort_flag) return false;
      if (global_ns() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        atomicOr(status, (unsigned)NC_DEV_TIMEOUT);
        return false;
      }
    }
  }
}

// Grid barrier among the compute threads of every CTA (bounded), the one
// after phase p. The counter is zeroed before every launch, so the barrier is
// complete once it reaches (p + 1) * grid: each CTA adds 1 with a release
// reduction (no returned value, no round trip; the CTA barrier before it
// orders the other compute threads' writes ahead of it) and polls with
// acquire loads.
__device__ bool grid_sync(const StepArgs &a, volatile int *abort_flag, int e, int p) {
  epi_sync();
  if (e == 0) {
    const unsigned long long target = (unsigned long long)(p + 1) * (unsigned long long)a.grid;
    asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(a.bar) : "memory");
    const uint64_t t0 = global_ns();
    for (uint32_t it = 0;; ++it) {
      unsigned long long v;
      asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(a.bar) : "memory");
      if (v >= target) break;
      if ((it & 15) == 15) {
        if (*abort_flag) break;
        if (global_ns() - t0 > kWaitLimitNs) {
          *abort_flag = 1;
          atomicOr(a.status, (unsigned)NC_DEV_TIMEOUT);
          break;
        }
      }
    }
  }
  epi_sync();
  return *abort_flag == 0;
}

// ---------------------------------------------------------- phase program
__device__ __forceinline__ int n_phases(const StepArgs &a) { return 3 + 5 * a.L; }

__device__ __forceinline__ void phase_of(const StepArgs &a, int p, int &type, int &layer) {
  if (p == 0) { type = P_EMBED; layer = 0; return; }
  if (p == 1 + 5 * a.L) { type = P_HEAD; layer = a.L; return; }
  if (p == 2 + 5 * a.L) { type = P_MERGE; layer = a.L; return; }
  layer = (p - 1) / 5;
  type = P_QKV + (p - 1) % 5;
}

struct Gemm {
  int N, K, kb_total, n_tiles;
  int kb0, nkb;           // this CTA's k-blocks (split over the cluster; full K for HEAD)
  int nt0, nt_step;       // this CTA's n-tiles: nt0, nt0 + nt_step, ...
  int S, split;           // K also split over S clusters per n-tile; this cluster's part
  const CUtensorMap *map;
};

__device__ __forceinline__ Gemm gemm_of(const StepArgs &a, int type, int layer, int cid, int ncl, int rank) {
  Gemm g;
  if (type == P_QKV) { g.N = (a.H + 2) * 128; g.K = a.d; g.map = a.wmaps + 4 * layer; }
  else if (type == P_OPROJ) { g.N = a.d; g.K = a.H * 128; g.map = a.wmaps + 4 * layer + 1; }
  else if (type == P_FC) { g.N = a.F; g.K = a.d; g.map = a.wmaps + 4 * layer + 2; }
  else if (type == P_PROJ) { g.N = a.d; g.K = a.F; g.map = a.wmaps + 4 * layer + 3; }
  else { g.N = a.V; g.K = a.d; g.map = a.wmaps + 4 * a.L; }
  g.kb_total = g.K / 64;
  g.n_tiles = g.N / 128;
  g.S = 1;
  g.split = 0;
  if (type == P_HEAD) {
    g.kb0 = 0;
    g.nkb = g.kb_total;
    g.nt0 = cid * CL + rank;
    g.nt_step = ncl * CL;
  } else if (type == P_PROJ && ncl >= 2 * g.n_tiles && g.n_tiles <= SPLIT_TILES) {
    // few n-tiles, long K: S clusters per n-tile, each a contiguous K range
    // split again over its CTAs; the partials are summed after the phase's
    // cluster reduction by the last of the S clusters to arrive
    g.S = min(ncl / g.n_tiles, SPLIT_MAX);
    if (cid < g.n_tiles * g.S) {
      g.split = cid / g.n_tiles;
      g.nt0 = cid % g.n_tiles;
    } else {
      g.nt0 = g.n_tiles;  // no work in this phase
    }
    g.nt_step = g.n_tiles;
    const int s0 = g.split * g.kb_total / g.S, s1 = (g.split + 1) * g.kb_total / g.S;
    const int kbs = (s1 - s0 + CL - 1) / CL;
    g.kb0 = s0 + rank * kbs;
    g.nkb = max(0, min(kbs, s1 - g.kb0));
  } else {
    const int kbs = (g.kb_total + CL - 1) / CL;
    g.kb0 = rank * kbs;
    g.nkb = max(0, min(kbs, g.kb_total - g.kb0));
    g.nt0 = cid;
    g.nt_step = ncl;
  }
  return g;
}

// key range of cluster rank `rank` for sequence b (n keys)
__device__ __forceinline__ void key_range(int n, int rank, int &k0, int &k1) {
  int chunk = (n + CL - 1) / CL;
  chunk = (chunk + KT - 1) / KT * KT;
  k0 = min(n, rank * chunk);
  k1 = min(n, k0 + chunk);
}

__device__ __forceinline__ uint32_t kv_tile_off(int key, int c) {
  // 64-key tile loaded as two TMA boxes of 64 dims x 64 keys, 128-byte swizzle
  return (uint32_t)((c >> 3) * 8192 + key * 128 + (((c & 7) ^ (key & 7)) << 4));
}

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

// ------------------------------------------------------------- producer
__device__ void producer(const StepArgs &a, const Smem &s, uint8_t *ring, int cid, int ncl, int rank) {
  uint32_t t = 0;
  auto take = [&](uint32_t &slot) -> bool {
    slot = t % RING;
    const uint32_t ph = (t / RING) & 1;
    t++;
    return mbar_wait(&s.empty[slot], ph ^ 1, s.abort_flag, a.status);
  };
  const int P = n_phases(a);
  for (int p = 0; p < P; p++) {
    int type, layer;
    phase_of(a, p, type, layer);
    if (type == P_QKV || type == P_OPROJ || type == P_FC || type == P_PROJ || type == P_HEAD) {
      const Gemm g = gemm_of(a, type, layer, cid, ncl, rank);
      bool first = true;
      for (int nt = g.nt0; nt < g.n_tiles; nt += g.nt_step)
        for (int kb = g.kb0; kb < g.kb0 + g.nkb; kb++) {
          uint32_t slot;
          if (!take(slot)) return;
          if (first) trace_mark(a, p, 5);
          first = false;
          mbar_arrive_expect_tx(&s.full[slot], SLOT);
          tma_load_2d(ring + slot * SLOT, g.map, kb * 64, nt * 128, &s.full[slot]);
        }
      trace_mark(a, p, 6);
    } else if (type == P_ATTN) {
      for (int b = cid; b < a.B; b += ncl) {
        if (!s.valid[b]) continue;
        int k0, k1;
        key_range(s.pos[b] + 1, rank, k0, k1);
        const int row0 = (layer * a.max_batch + b) * a.max_seq;
        for (int key = k0; key < k1; key += KT)
          for (int which = 0; which < 2; which++) {
            uint32_t slot;
            if (!take(slot)) return;
            if (key == k0 && which == 0 && b == cid) trace_mark(a, p, 5);
            mbar_arrive_expect_tx(&s.full[slot], SLOT);
            uint8_t *dst = ring + slot * SLOT;
            tma_load_2d(dst, a.kvmaps + which, 0, row0 + key, &s.full[slot]);
            tma_load_2d(dst + 8192, a.kvmaps + which, 64, row0 + key, &s.full[slot]);
          }
      }
      trace_mark(a, p, 6);
    }
  }
}

// ------------------------------------------------------------ MMA issuer
__device__ void mma_issuer(const StepArgs &a, const Smem &s, uint8_t *ring, uint8_t *xs, uint32_t tmem, int cid,
                           int ncl, int rank) {
  uint32_t t = 0, xr = 0, units = 0;
  const uint32_t idesc = idesc_bf16_f32(128, NB);
  const int P = n_phases(a);
  for (int p = 0; p < P; p++) {
    int type, layer;
    phase_of(a, p, type, layer);
    if (type == P_QKV || type == P_OPROJ || type == P_FC || type == P_PROJ || type == P_HEAD) {
      const Gemm g = gemm_of(a, type, layer, cid, ncl, rank);
      // When this CTA's K range fits the staging buffer, X is staged once for
      // every n-tile of the phase (they all multiply the same X slice)
      const bool single = g.nkb <= XKB && g.nt0 < g.n_tiles;
      if (single) {
        if (!mbar_wait(s.x_ready, xr & 1, s.abort_flag, a.status)) return;
        xr++;
        tc_fence_after();
      }
      // k-blocks kb_lo .. kb_lo + cn - 1 of this unit, X staged from kb_lo
      auto issue = [&](uint32_t acc0, int kb_lo, int cn, bool fresh0) -> bool {
        // a wait's result takes ~160 cycles even when the slot is full: the
        // next slot is probed before this slot's MMAs, its answer read after
        bool ready = cn > 0 && mbar_try_wait(smem_u32(&s.full[t % RING]), (t / RING) & 1);
        for (int kb = 0; kb < cn; kb++) {
          const uint32_t slot = t % RING;
          if (!ready && !mbar_wait(&s.full[slot], (t / RING) & 1, s.abort_flag, a.status)) return false;
          t++;
          tc_fence_after();
          ready = kb + 1 < cn && mbar_try_wait(smem_u32(&s.full[t % RING]), (t / RING) & 1);
          const uint32_t w0 = smem_u32(ring + slot * SLOT), x0 = smem_u32(xs + (kb_lo + kb) * NB * 128);
          // the four 16-column steps of a block accumulate into four different
          // TMEM accumulators, so consecutive MMAs do not wait on one another;
          // the epilogue adds the accumulators up
          const bool fresh = fresh0 && kb == 0;
#pragma unroll
          for (int k = 0; k < 4; k++)
            mma_bf16(acc0 + (uint32_t)k * NB, desc_k_sw128(w0 + 32 * k), desc_k_sw128(x0 + 32 * k), idesc,
                     fresh ? 0 : 1);
          mma_commit(&s.empty[slot]);
        }
        return true;
      };
      for (int nt = g.nt0; nt < g.n_tiles; nt += g.nt_step, units++) {
        // two accumulator sets: this unit's MMAs may run while the compute
        // warps still reduce and store the previous unit
        const uint32_t set = units & 1;
        if (!mbar_wait(&s.acc_empty[set], ((units >> 1) & 1) ^ 1, s.abort_flag, a.status)) return;
        tc_fence_after();
        const uint32_t acc0 = tmem + set * (uint32_t)(NACC * NB);
        if (single) {
          if (!issue(acc0, 0, g.nkb, true)) return;
        } else {
          for (int c0 = 0; c0 < g.nkb || (c0 == 0 && g.nkb == 0); c0 += XKB) {
            if (!mbar_wait(s.x_ready, xr & 1, s.abort_flag, a.status)) return;
            xr++;
            tc_fence_after();
            if (!issue(acc0, 0, min(XKB, g.nkb - c0), c0 == 0)) return;
            mma_commit(s.x_free);
            if (g.nkb == 0) break;
          }
        }
        mma_commit(&s.acc_full[set]);
      }
      if (single) mma_commit(s.x_free);  // X is free once every unit's MMAs are done
      trace_mark(a, p, 7);
    } else if (type == P_ATTN) {
      // the compute warps consume this phase's ring slots; keep the count
      for (int b = cid; b < a.B; b += ncl) {
        if (!s.valid[b]) continue;
        int k0, k1;
        key_range(s.pos[b] + 1, rank, k0, k1);
        t += 2 * ((k1 - k0 + KT - 1) / KT);
      }
    }
  }
}

// ------------------------------------------------- compute-side helpers
// X staging: X[b][kb*64 + c] for this pass, NB rows, 128-byte swizzled. The
// normed inputs (QKV, FC, HEAD) are staged as bf16(x); their RMS factor is
// applied to the accumulator column in the epilogue, so staging does not
// wait for the row sums.
// Loads are issued in batches of U per thread before any is consumed, so a
// pass costs a few L2 round trips instead of one per item.
__device__ void stage_x(const StepArgs &a, const Smem &s, uint8_t *xs, int type, int kb_begin, int nkb, int e) {
  constexpr int U = 16;
  const bool norm = (type == P_QKV || type == P_FC || type == P_HEAD);
  const float *xsrc = (type == P_FC) ? a.x1 : a.x0;
  const bf16 *act = (type == P_OPROJ) ? a.y : a.f;
  const int K = (type == P_PROJ) ? a.F : a.d;
  const int total = nkb * NB * 8;
  for (int base = e; base < total; base += 128 * U) {
    if (norm) {
      float4 p[U], q[U];
#pragma unroll
      for (int u = 0; u < U; u++) {
        const int idx = base + u * 128;
        const int c = idx & 7, b = (idx >> 3) % NB, kbl = idx / (8 * NB);
        p[u] = q[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (idx < total && b < a.B) {
          const float4 *src = reinterpret_cast<const float4 *>(xsrc + (size_t)b * a.d + (kb_begin + kbl) * 64 + c * 8);
          p[u] = src[0];
          q[u] = src[1];
        }
      }
#pragma unroll
      for (int u = 0; u < U; u++) {
        const int idx = base + u * 128;
        if (idx >= total) break;
        const int c = idx & 7, b = (idx >> 3) % NB, kbl = idx / (8 * NB);
        const uint4 v = make_uint4(pack_bf(p[u].x, p[u].y), pack_bf(p[u].z, p[u].w), pack_bf(q[u].x, q[u].y),
                                   pack_bf(q[u].z, q[u].w));
        *reinterpret_cast<uint4 *>(xs + kbl * NB * 128 + b * 128 + ((c ^ (b & 7)) << 4)) = v;
      }
    } else {
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; u++) {
        const int idx = base + u * 128;
        const int c = idx & 7, b = (idx >> 3) % NB, kbl = idx / (8 * NB);
        v[u] = make_uint4(0, 0, 0, 0);
        if (idx < total && b < a.B)
          v[u] = *reinterpret_cast<const uint4 *>(act + (size_t)b * K + (kb_begin + kbl) * 64 + c * 8);
      }
#pragma unroll
      for (int u = 0; u < U; u++) {
        const int idx = base + u * 128;
        if (idx >= total) break;
        const int c = idx & 7, b = (idx >> 3) % NB, kbl = idx / (8 * NB);
        *reinterpret_cast<uint4 *>(xs + kbl * NB * 128 + b * 128 + ((c ^ (b & 7)) << 4)) = v[u];
      }
    }
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// per-row scale 1/rms from a complete sum of squares
__device__ void load_inv(const StepArgs &a, const Smem &s, const float *ss, int e) {
  if (e < NB) {
    float v[SSN];
#pragma unroll
    for (int j = 0; j < SSN; j++) v[j] = (j < a.d / 128 && e < a.B) ? ss[j * 32 + e] : 0.f;
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < SSN; j++) sum += v[j];
    s.inv[e] = e < a.B ? rsqrtf(sum / a.d + a.eps) : 0.f;
  }
  epi_sync();
}

// Epilogue of one reduced 128-row tile for the batch columns b in [b0, b1):
// tl[n * (NB+1) + j] holds row n (thread e = n), column b0 + j.
// Global operands of the epilogue, loaded before the cluster exchange so that
// their latency overlaps it.
struct EpiPre {
  float xv[NB / CL];   // residual inputs (OPROJ / PROJ)
  float2 cs[NB / CL];  // RoPE (cos, sin) of the row's pair at each column's position (QKV)
};

__device__ __forceinline__ void epi_preload(const StepArgs &a, const Smem &s, int type, int nt, int b0, int b1, int e,
                                            EpiPre &pre) {
  const int nb = b1 - b0, col = nt * 128 + e;
  if (type == P_OPROJ || type == P_PROJ) {
    const float *xin = type == P_OPROJ ? a.x0 : a.x1;
#pragma unroll
    for (int j = 0; j < NB / CL; j++) pre.xv[j] = j < nb ? xin[(size_t)(b0 + j) * a.d + col] : 0.f;
  } else if (type == P_QKV && nt <= a.H) {
#pragma unroll
    for (int j = 0; j < NB / CL; j++) {
      pre.cs[j] = make_float2(1.f, 0.f);
      if (j < nb) {
        const int p = min(max(s.pos[b0 + j], 0), a.max_seq - 1);
        pre.cs[j] = a.rope[(size_t)p * 64 + (e & 63)];
      }
    }
  }
}

__device__ void gemm_epilogue(const StepArgs &a, const Smem &s, int type, int layer, int nt, float *tl, int b0,
                              int b1, int e, const EpiPre &pre) {
  const int lane = e & 31, w = e >> 5, nb = b1 - b0;
  const int col = nt * 128 + e;
  if (type == P_FC) {
#pragma unroll
    for (int j = 0; j < NB / CL; j++) {
      if (j < nb) {
        const float v = fmaxf(tl[e * (NB + 1) + j] * s.inv[b0 + j], 0.f);
        a.f[(size_t)(b0 + j) * a.F + col] = __float2bfloat16_rn(v * v);
      }
    }
  } else if (type == P_OPROJ || type == P_PROJ) {
    float *xout = type == P_OPROJ ? a.x1 : a.x0;
    // this tile's sum of squares: one slot per (tile, column), added up in a
    // fixed order by the consumer, so results do not depend on timing
    float *ss = a.ss + ((size_t)(type == P_OPROJ ? 2 * layer + 1 : 2 * layer + 2) * SSN + nt) * 32;
#pragma unroll
    for (int j = 0; j < NB / CL; j++) {
      if (j < nb) {
        const float v = pre.xv[j] + tl[e * (NB + 1) + j];
        xout[(size_t)(b0 + j) * a.d + col] = v;
        tl[e * (NB + 1) + j] = v * v;
      }
    }
    epi_sync();
    for (int j = w; j < nb; j += 4) {
      float sum = tl[lane * (NB + 1) + j] + tl[(lane + 32) * (NB + 1) + j] + tl[(lane + 64) * (NB + 1) + j] +
                  tl[(lane + 96) * (NB + 1) + j];
      sum = warp_sum(sum);
      if (lane == 0) ss[b0 + j] = sum;
    }
  } else {  // P_QKV: one 128-wide head per tile: q heads, then k, then v
    const int head = nt;
    const size_t lay = (size_t)layer * a.max_batch * a.max_seq * 128;
    if (head <= a.H) {
      // RoPE on split-half pairs (e, e^64), then RMS norm over the head
      constexpr int MJ = NB / CL;
      float rot[MJ];
#pragma unroll
      for (int j = 0; j < MJ; j++) {
        rot[j] = 0.f;
        if (j < nb) {
          const float2 cs = pre.cs[j];
          const float r = s.inv[b0 + j];
          const float v = tl[e * (NB + 1) + j] * r, u = tl[(e ^ 64) * (NB + 1) + j] * r;
          rot[j] = e < 64 ? v * cs.x - u * cs.y : u * cs.y + v * cs.x;
        }
      }
      epi_sync();
#pragma unroll
      for (int j = 0; j < MJ; j++) tl[e * (NB + 1) + j] = rot[j] * rot[j];
      epi_sync();
      for (int j = w; j < nb; j += 4) {
        float sum = tl[lane * (NB + 1) + j] + tl[(lane + 32) * (NB + 1) + j] + tl[(lane + 64) * (NB + 1) + j] +
                    tl[(lane + 96) * (NB + 1) + j];
        sum = warp_sum(sum);
        if (lane == 0) s.qn[b0 + j] = rsqrtf(sum * (1.0f / 128) + a.eps);
      }
      epi_sync();
#pragma unroll
      for (int j = 0; j < MJ; j++) {
        if (j >= nb) break;
        const int b = b0 + j;
        const float v = rot[j] * s.qn[b];
        if (head < a.H) {
          a.q[((size_t)b * a.H + head) * 128 + e] = __float2bfloat16_rn(v);
        } else if (s.valid[b]) {
          a.kc[lay + ((size_t)b * a.max_seq + s.pos[b]) * 128 + e] = __float2bfloat16_rn(v);
        }
      }
      epi_sync();  // s.qn is rewritten by the next tile
    } else {
      for (int j = 0; j < nb; j++) {
        const int b = b0 + j;
        if (s.valid[b])
          a.vc[lay + ((size_t)b * a.max_seq + s.pos[b]) * 128 + e] =
              __float2bfloat16_rn(tl[e * (NB + 1) + j] * s.inv[b]);
      }
    }
  }
}

// LM head tile (full K, no reduction): softcap, logits, per-tile argmax.
// r holds tile row n (this thread's TMEM lane) for every batch column.
__device__ void head_epilogue(const StepArgs &a, const Smem &s, int nt, const uint32_t (&r)[NB], float *tl, int n,
                              int e) {
  const int lane = e & 31, w = e >> 5;
  const int col = nt * 128 + n;
  const float inv = 1.0f / a.cap;
  float nz[NB];
#pragma unroll
  for (int b = 0; b < NB; b++) nz[b] = (a.noise && b < a.B) ? a.noise[(size_t)b * a.V + col] : 0.f;
#pragma unroll
  for (int b = 0; b < NB; b++) {
    if (b < a.B) {
      const float z = a.cap * tanhf(__uint_as_float(r[b]) * s.inv[b] * inv);
      if (s.valid[b]) a.logits[(size_t)b * a.V + col] = z;
      tl[n * (NB + 1) + b] = z + nz[b];
    }
  }
  epi_sync();
  for (int b = w; b < a.B; b += 4) {
    ArgMax best{-INFINITY, 0x7fffffff};
#pragma unroll
    for (int q = 0; q < 4; q++)
      best = argmax_merge(best, ArgMax{tl[(lane + 32 * q) * (NB + 1) + b], nt * 128 + lane + 32 * q});
    best = warp_argmax(best);
    if (lane == 0) {
      a.cand_v[(size_t)nt * 32 + b] = best.v;
      a.cand_i[(size_t)nt * 32 + b] = best.i;
    }
  }
  epi_sync();
}

// ATTN phase: flash decoding over this CTA's key range of each sequence of
// the cluster (mma.sync m16n8k16: rows = query heads, padded to 16), then a
// cluster merge of the (m, l, O) states; rank r writes heads r, r+CL, ...
__device__ bool attention_phase(const StepArgs &a, const Smem &s, uint8_t *ring, uint8_t *xs, float *red, int layer,
                                int cid, int ncl, int rank, int e, uint32_t &t, uint32_t &rounds,
                                cg::cluster_group &cluster) {
  const int warp = e >> 5, lane = e & 31, g = lane >> 2, t4 = lane & 3;
  const size_t lay = (size_t)layer * a.max_batch * a.max_seq * 128;
  float *cw = reinterpret_cast<float *>(xs);  // [4 warps][16 rows][130]
  for (int b = cid; b < a.B; b += ncl) {
    if (!s.valid[b]) continue;  // the same in every CTA of the cluster
    const int n_keys = s.pos[b] + 1;
    int k0, k1;
    key_range(n_keys, rank, k0, k1);
    uint32_t qa[8][4];
    {
      const bf16 *qb = a.q + (size_t)b * a.H * 128;
#pragma unroll
      for (int ks = 0; ks < 8; ks++) {
        const int c0 = ks * 16 + t4 * 2;
        qa[ks][0] = g < a.H ? *reinterpret_cast<const uint32_t *>(qb + (size_t)g * 128 + c0) : 0u;
        qa[ks][1] = g + 8 < a.H ? *reinterpret_cast<const uint32_t *>(qb + (size_t)(g + 8) * 128 + c0) : 0u;
        qa[ks][2] = g < a.H ? *reinterpret_cast<const uint32_t *>(qb + (size_t)g * 128 + c0 + 8) : 0u;
        qa[ks][3] = g + 8 < a.H ? *reinterpret_cast<const uint32_t *>(qb + (size_t)(g + 8) * 128 + c0 + 8) : 0u;
      }
    }
    float o[16][4];
#pragma unroll
    for (int i = 0; i < 16; i++) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    for (int key0 = k0; key0 < k1; key0 += KT) {
      const uint32_t ks_ = t % RING, kph = (t / RING) & 1;
      t++;
      const uint32_t vs_ = t % RING, vph = (t / RING) & 1;
      t++;
      if (!mbar_wait(&s.full[ks_], kph, s.abort_flag, a.status)) return false;
      if (!mbar_wait(&s.full[vs_], vph, s.abort_flag, a.status)) return false;
      if (e == 0 && b == cid && key0 == k0) trace_mark(a, 2 + 5 * layer, 1);
      uint8_t *K = ring + ks_ * SLOT, *V = ring + vs_ * SLOT;
      // the key/value written by this step's QKV phase may postdate the
      // prefetch: copy that row from the cache
      const int pr = s.pos[b] - key0;
      if (pr >= 0 && pr < KT) {
        if (e < 32) {
          const int c = e & 15;
          const bf16 *src = (e < 16 ? a.kc : a.vc) + lay + ((size_t)b * a.max_seq + s.pos[b]) * 128 + c * 8;
          *reinterpret_cast<uint4 *>((e < 16 ? K : V) + kv_tile_off(pr, c)) = *reinterpret_cast<const uint4 *>(src);
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        epi_sync();
      }
      const uint32_t kb = smem_u32(K), vb = smem_u32(V);
      const int kw = warp * 16;
      const int kg = key0 + kw;
      float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < 8; ks++) {
        const int key = kw + (lane & 7) + ((lane >> 4) << 3);
        const int c = 2 * ks + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kb + kv_tile_off(key, c), b0, b1, b2, b3);
        mma16816(s0, qa[ks], b0, b1);
        mma16816(s1, qa[ks], b2, b3);
      }
      float v[8] = {s0[0], s0[1], s1[0], s1[1], s0[2], s0[3], s1[2], s1[3]};
      const int kidx[4] = {kg + 2 * t4, kg + 2 * t4 + 1, kg + 8 + 2 * t4, kg + 9 + 2 * t4};
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int i = 0; i < 4; i++) {
        const bool in = kidx[i] < k1;
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
      const float al0 = mn0 == -INFINITY ? 1.f : exp2f(m0 - mn0);
      const float al1 = mn1 == -INFINITY ? 1.f : exp2f(m1 - mn1);
      float pp[8];
#pragma unroll
      for (int i = 0; i < 4; i++) {
        pp[i] = v[i] == -INFINITY ? 0.f : exp2f(v[i] - mn0);
        pp[i + 4] = v[i + 4] == -INFINITY ? 0.f : exp2f(v[i + 4] - mn1);
      }
      l0 = l0 * al0 + pp[0] + pp[1] + pp[2] + pp[3];
      l1 = l1 * al1 + pp[4] + pp[5] + pp[6] + pp[7];
      m0 = mn0;
      m1 = mn1;
#pragma unroll
      for (int i = 0; i < 16; i++) {
        o[i][0] *= al0;
        o[i][1] *= al0;
        o[i][2] *= al1;
        o[i][3] *= al1;
      }
      uint32_t pa[4] = {pack_bf(pp[0], pp[1]), pack_bf(pp[4], pp[5]), pack_bf(pp[2], pp[3]), pack_bf(pp[6], pp[7])};
#pragma unroll
      for (int dt = 0; dt < 16; dt += 2) {
        const int key = kw + (lane & 7) + (((lane >> 3) & 1) << 3);
        const int c = dt + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vb + kv_tile_off(key, c), b0, b1, b2, b3);
        mma16816(o[dt], pa, b0, b1);
        mma16816(o[dt + 1], pa, b2, b3);
      }
      epi_sync();
      if (e == 0) {
        mbar_arrive(&s.empty[ks_]);
        mbar_arrive(&s.empty[vs_]);
      }
    }
    if (e == 0 && b == cid) trace_mark(a, 2 + 5 * layer, 2);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
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
    epi_sync();
    // this CTA's state (m, l, O per head row) is pushed into the inbox of the
    // rank that finishes that head (head h -> rank h % CL, inbox laid out
    // [source rank][h / CL][130]); the owner merges its inbox locally
    if (!mbar_wait_cluster(s.red_free, (rounds & 1) ^ 1, s.abort_flag, a.status)) return false;
    for (int idx = e; idx < a.H * 128; idx += 128) {
      const int row = idx >> 7, col = idx & 127;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < 4; w++) M = fmaxf(M, cw[w * 16 * 130 + row * 130]);
      float Ls = 0.f, O = 0.f;
#pragma unroll
      for (int w = 0; w < 4; w++) {
        const float mw = cw[w * 16 * 130 + row * 130];
        const float f = mw == -INFINITY ? 0.f : exp2f(mw - M);
        Ls += f * cw[w * 16 * 130 + row * 130 + 1];
        O += f * cw[w * 16 * 130 + row * 130 + 2 + col];
      }
      float *dst = cluster.map_shared_rank(red, row % CL) + (rank * (16 / CL) + row / CL) * 130;
      dst[2 + col] = O;
      if (col == 0) {
        dst[0] = M;
        dst[1] = Ls;
      }
    }
    epi_sync();
    if (e < CL) mbar_arrive_remote(s.red_full, e);
    if (!mbar_wait_cluster(s.red_full, rounds & 1, s.abort_flag, a.status)) return false;
    if (e == 0) trace_mark(a, 2 + 5 * layer, 3);
    for (int h = rank; h < a.H; h += CL) {
      const int slot = h / CL;
      float M = -INFINITY;
#pragma unroll
      for (int q = 0; q < CL; q++) M = fmaxf(M, red[(q * (16 / CL) + slot) * 130]);
      float Ls = 0.f, O = 0.f;
#pragma unroll
      for (int q = 0; q < CL; q++) {
        const float *pr = red + (q * (16 / CL) + slot) * 130;
        const float f = pr[0] == -INFINITY ? 0.f : exp2f(pr[0] - M);
        Ls += f * pr[1];
        O += f * pr[2 + e];
      }
      a.y[((size_t)b * a.H + h) * 128 + e] = __float2bfloat16_rn(Ls > 0.f ? O / Ls : 0.f);
    }
    epi_sync();
    if (e < CL) mbar_arrive_remote(s.red_free, e);
    rounds++;
  }
  return true;
}

// ------------------------------------------------------------ the kernel
__global__ void __cluster_dims__(CL, 1, 1) __launch_bounds__(THREADS, 1) decode_step_kernel(StepArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint32_t raw = smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw + 1023) & ~1023u) - raw);
  uint8_t *ring = smem + OFF_RING;
  uint8_t *xs = smem + OFF_X;
  float *red = reinterpret_cast<float *>(smem + OFF_RED);
  float *tl = reinterpret_cast<float *>(smem + OFF_TL);
  Smem s;
  {
    uint64_t *b = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    s.full = b;
    s.empty = b + RING;
    s.x_ready = b + 2 * RING;
    s.x_free = s.x_ready + 1;
    s.acc_full = s.x_ready + 2;   // [2]
    s.acc_empty = s.x_ready + 4;  // [2]
    s.red_full = s.x_ready + 6;
    s.red_free = s.x_ready + 7;
    s.tmem_slot = reinterpret_cast<uint32_t *>(s.x_ready + 8);
    s.abort_flag = reinterpret_cast<int *>(s.tmem_slot + 1);
    s.pos = s.abort_flag + 1;
    s.valid = s.pos + 32;
    s.inv = reinterpret_cast<float *>(s.valid + 32);
    s.qn = s.inv + 32;
    s.flag = reinterpret_cast<int *>(s.qn + 32);
  }
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int cid = blockIdx.x / CL, ncl = gridDim.x / CL;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < RING; i++) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    mbar_init(s.x_ready, 1);
    mbar_init(s.x_free, 1);
    for (int i = 0; i < 2; i++) {
      mbar_init(&s.acc_full[i], 1);
      mbar_init(&s.acc_empty[i], 128);
    }
    mbar_init(s.red_full, CL);
    mbar_init(s.red_free, CL);
    *s.abort_flag = 0;
    fence_barrier_init();
  }
  if (threadIdx.x < 32) {
    // positions and validity, identical in every CTA (the lengths only change
    // in the last phase)
    const int b = threadIdx.x;
    int p = 0, ok = 0;
    if (b < a.B) {
      p = a.positions ? a.positions[b] : a.len[b];
      ok = (p >= 0 && p < a.max_seq && p == a.len[b]) ? 1 : 0;
    }
    s.pos[b] = ok ? p : 0;
    s.valid[b] = ok;
    if (blockIdx.x == 0 && b < a.B) a.valid_out[b] = (uint8_t)ok;
  }
  if (warp == 1) tmem_alloc(s.tmem_slot, 2 * NB * NACC);
  tc_fence_before();
  __syncthreads();
  cluster.sync();  // peers' barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *s.tmem_slot;

  if (warp == 0) {
    if (lane == 0) producer(a, s, ring, cid, ncl, rank);
  } else if (warp == 1) {
    if (lane == 0) mma_issuer(a, s, ring, xs, tmem, cid, ncl, rank);
  } else {
    const int e = threadIdx.x - 64;
    const int quarter = warp & 3;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int n = quarter * 32 + lane;  // TMEM lane of this thread
    uint32_t t = 0;                     // ring slot counter, in the producer's order
    uint32_t xf = 0, units = 0, rounds = 0;
    bool x_pending = false;             // a staged X is waiting for x_free
    const int P = n_phases(a);
    bool ok = true;
    for (int p = 0; p < P && ok; p++) {
      int type, layer;
      phase_of(a, p, type, layer);
      if (e == 0) trace_mark(a, p, 0);
      if (type == P_EMBED) {
        for (int b = blockIdx.x; b < a.B; b += gridDim.x) {
          int tok = a.tokens[b];
          if (tok < 0 || tok >= a.V) {
            if (e == 0) atomicOr(a.status, (unsigned)NC_DEV_BAD_TOKEN);
            tok = tok < 0 ? 0 : a.V - 1;
          }
          const bf16 *row = a.wte + (size_t)tok * a.d;
          float sq = 0.f;
          for (int i = e; i < a.d; i += 128) {
            const float v = __bfloat162float(row[i]);
            sq += v * v;
          }
          sq = warp_sum(sq);
          if (lane == 0) tl[e >> 5] = sq;
          epi_sync();
          const float tot = tl[0] + tl[1] + tl[2] + tl[3];
          const float inv = rsqrtf(tot / a.d + a.eps);
          // x0 and its per-128-column sums of squares (norm 0 of layer 0)
          epi_sync();
          for (int j = 0; j < a.d / 128; j++) {
            const float v = __bfloat162float(row[j * 128 + e]) * inv;
            a.x0[(size_t)b * a.d + j * 128 + e] = v;
            const float q = warp_sum(v * v);
            if (lane == 0) tl[8 + 4 * j + (e >> 5)] = q;
          }
          epi_sync();
          if (e < a.d / 128) a.ss[(size_t)e * 32 + b] = tl[8 + 4 * e] + tl[9 + 4 * e] + tl[10 + 4 * e] + tl[11 + 4 * e];
          epi_sync();
        }
      } else if (type == P_ATTN) {
        ok = attention_phase(a, s, ring, xs, red, layer, cid, ncl, rank, e, t, rounds, cluster);
      } else if (type == P_MERGE) {
        for (int b = blockIdx.x; b < a.B; b += gridDim.x) {
          if (!s.valid[b]) continue;
          const int nt_count = a.V / 128;
          ArgMax best{-INFINITY, 0x7fffffff};
          for (int i = e; i < nt_count; i += 128)
            best = argmax_merge(best, ArgMax{__ldcg(&a.cand_v[(size_t)i * 32 + b]), __ldcg(&a.cand_i[(size_t)i * 32 + b])});
          best = warp_argmax(best);
          if (lane == 0) {
            tl[2 * (e >> 5)] = best.v;
            reinterpret_cast<int *>(tl)[2 * (e >> 5) + 1] = best.i;
          }
          epi_sync();
          if (e == 0) {
            ArgMax r{tl[0], reinterpret_cast<int *>(tl)[1]};
            for (int q = 1; q < 4; q++) r = argmax_merge(r, ArgMax{tl[2 * q], reinterpret_cast<int *>(tl)[2 * q + 1]});
            if (a.next) a.next[b] = r.i;
            a.len[b] = s.pos[b] + 1;
          }
          epi_sync();
        }
        for (int b = blockIdx.x; b < a.B; b += gridDim.x)
          if (!s.valid[b] && e == 0) atomicOr(a.status, (unsigned)NC_DEV_BAD_POSITION);
      } else {
        // linear layer: QKV, OPROJ, FC, PROJ (cluster split-K) or HEAD (full K)
        const Gemm g = gemm_of(a, type, layer, cid, ncl, rank);
        const bool norm = (type == P_QKV || type == P_FC || type == P_HEAD);
        bool inv_ready = !norm;
        const bool single = g.nkb <= XKB && g.nt0 < g.n_tiles;  // X staged once for the phase
        if (single) {
          if (x_pending) {
            if (!mbar_wait(s.x_free, xf & 1, s.abort_flag, a.status)) { ok = false; }
            xf++;
            x_pending = false;
          }
          if (ok && g.nkb > 0) stage_x(a, s, xs, type, g.kb0, g.nkb, e);
          epi_sync();
          if (e == 0) {
            mbar_arrive(s.x_ready);
            trace_mark(a, p, 1);
          }
          x_pending = true;
        }
        for (int nt = g.nt0; nt < g.n_tiles && ok; nt += g.nt_step, units++) {
          if (!single) {
            for (int c0 = 0; c0 < g.nkb || (c0 == 0 && g.nkb == 0); c0 += XKB) {
              if (x_pending) {
                if (!mbar_wait(s.x_free, xf & 1, s.abort_flag, a.status)) { ok = false; break; }
                xf++;
                x_pending = false;
              }
              const int cn = min(XKB, g.nkb - c0);
              if (cn > 0) stage_x(a, s, xs, type, g.kb0 + c0, cn, e);
              epi_sync();
              if (e == 0) mbar_arrive(s.x_ready);
              x_pending = true;
              if (g.nkb == 0) break;
            }
            if (!ok) break;
          }
          if (!inv_ready) {  // the row factors, computed while the MMAs run
            load_inv(a, s, a.ss + (size_t)(type == P_QKV ? 2 * layer : type == P_FC ? 2 * layer + 1 : 2 * a.L) * SSN * 32,
                     e);
            inv_ready = true;
          }
          t += g.nkb;  // the unit's weight tiles went through the ring (consumed by the MMA warp)
          const uint32_t set = units & 1;
          if (!mbar_wait(&s.acc_full[set], (units >> 1) & 1, s.abort_flag, a.status)) { ok = false; break; }
          tc_fence_after();
          if (e == 0 && nt == g.nt0) trace_mark(a, p, 2);
          const uint32_t tacc = tmem + set * (uint32_t)(NACC * NB) + lane_off;
          uint32_t r[NB];
          {
            const int nacc = g.nkb > 0 ? NACC : 1;
            tmem_ld32(tacc, r);
            for (int q = 1; q < nacc; q++) {
              uint32_t r2[NB];
              tmem_ld32(tacc + (uint32_t)q * NB, r2);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < NB; j++) r[j] = __float_as_uint(__uint_as_float(r[j]) + __uint_as_float(r2[j]));
            }
            tmem_ld_wait();
          }
          tc_fence_before();
          mbar_arrive(&s.acc_empty[set]);
          if (g.nkb == 0)
            for (int j = 0; j < NB; j++) r[j] = 0u;  // this rank holds no k-blocks
          if (type == P_HEAD) {
            head_epilogue(a, s, nt, r, tl, n, e);
            continue;
          }
          // cluster reduction over the K split: each CTA finishes NB/CL batch
          // columns. Every CTA pushes the columns rank q finishes straight into
          // q's inbox (red, laid out [source rank][row][NB/CL]) and arrives on
          // q's red_full; q then adds its inbox up from local shared memory.
          // (red_free: every destination has read its inbox of the last round.)
          constexpr int NC = NB / CL;
          if (!mbar_wait_cluster(s.red_free, (rounds & 1) ^ 1, s.abort_flag, a.status)) { ok = false; break; }
#pragma unroll
          for (int q = 0; q < CL; q++) {
            float4 *dst = reinterpret_cast<float4 *>(cluster.map_shared_rank(red, q) + (rank * 128 + n) * NC);
#pragma unroll
            for (int j4 = 0; j4 < NC / 4; j4++)
              dst[j4] = make_float4(__uint_as_float(r[q * NC + 4 * j4]), __uint_as_float(r[q * NC + 4 * j4 + 1]),
                                    __uint_as_float(r[q * NC + 4 * j4 + 2]), __uint_as_float(r[q * NC + 4 * j4 + 3]));
          }
          epi_sync();
          if (e < CL) mbar_arrive_remote(s.red_full, e);
          const int b0 = rank * NC, b1 = min(a.B, b0 + NC);
          EpiPre pre;
          epi_preload(a, s, type, nt, b0, b1, e, pre);
          if (!mbar_wait_cluster(s.red_full, rounds & 1, s.abort_flag, a.status)) { ok = false; break; }
          if (e == 0) trace_mark(a, p, 3);
          {
            float sum[NC];
#pragma unroll
            for (int j = 0; j < NC; j++) sum[j] = 0.f;
#pragma unroll
            for (int q = 0; q < CL; q++) {
              const float4 *src = reinterpret_cast<const float4 *>(red + (q * 128 + e) * NC);
#pragma unroll
              for (int j4 = 0; j4 < NC / 4; j4++) {
                const float4 v4 = src[j4];
                sum[4 * j4 + 0] += v4.x;
                sum[4 * j4 + 1] += v4.y;
                sum[4 * j4 + 2] += v4.z;
                sum[4 * j4 + 3] += v4.w;
              }
            }
#pragma unroll
            for (int j = 0; j < NC; j++) tl[e * (NB + 1) + j] = sum[j];
          }
          epi_sync();
          if (e < CL) mbar_arrive_remote(s.red_free, e);
          rounds++;
          if (g.S > 1) {
            // K split over S clusters: publish this cluster's partial of
            // (n-tile, rank); the last of the S to arrive adds them up in
            // split order (independent of the arrival order) and runs the
            // epilogue, the others are done
            float *part = a.split_part + ((size_t)(nt * g.S + g.split) * CL + rank) * 128 * NC;
#pragma unroll
            for (int j = 0; j < NC; j++) part[e * NC + j] = tl[e * (NB + 1) + j];
            epi_sync();
            if (e == 0) {
              unsigned old;
              asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                           : "=r"(old)
                           : "l"(a.split_cnt + nt * CL + rank)
                           : "memory");
              *s.flag = old == (unsigned)((layer + 1) * g.S - 1) ? 1 : 0;
            }
            epi_sync();
            if (!*s.flag) {
              epi_sync();  // s.flag is rewritten by the next unit
              continue;
            }
            float sum[NC];
#pragma unroll
            for (int j = 0; j < NC; j++) sum[j] = 0.f;
            for (int q = 0; q < g.S; q++) {
              if (q == g.split) {
#pragma unroll
                for (int j = 0; j < NC; j++) sum[j] += tl[e * (NB + 1) + j];
              } else {
                const float *src = a.split_part + ((size_t)(nt * g.S + q) * CL + rank) * 128 * NC + e * NC;
#pragma unroll
                for (int j = 0; j < NC; j++) sum[j] += __ldcg(src + j);
              }
            }
#pragma unroll
            for (int j = 0; j < NC; j++) tl[e * (NB + 1) + j] = sum[j];
            epi_sync();
          }
          if (b1 > b0) gemm_epilogue(a, s, type, layer, nt, tl, b0, b1, e, pre);
          epi_sync();
        }
      }
      if (e == 0) trace_mark(a, p, 4);
      if (ok && p + 1 < P) ok = grid_sync(a, s.abort_flag, e, p);
    }
    if (x_pending && ok) {
      mbar_wait(s.x_free, xf & 1, s.abort_flag, a.status);
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster.sync();  // no CTA leaves while a peer may still read its shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * NB * NACC);
  }
}

}  // namespace

bool make_map_bf16_k64(CUtensorMap *map, const void *ptr, int rows, int cols, int ld, int box_rows);

size_t decode_step_bar_bytes() { return sizeof(unsigned long long) + sizeof(unsigned) * SPLIT_TILES * CL; }

size_t decode_step_part_floats(int num_sms) {
  // n_tiles * S <= clusters; each (tile, split, rank) holds 128 rows x NB/CL columns
  return (size_t)(num_sms / CL + 1) * CL * 128 * (NB / CL);
}

bool decode_step_supported(const nc_config &c, int B) {
  return decode_fast_supported(c, B) && c.n_head <= 16 && c.d_model / 128 <= SSN;
}

int decode_step_maps_count(const nc_config &c) { return 4 * c.depth + 1 + 2; }

// Tensor maps of the step kernel, written to host memory `out` (to be copied
// to the device): per layer QKV, O, fc, proj weights, the lm_head, then the
// K and V caches viewed as [depth * max_batch * max_seq, 128].
bool decode_step_build_maps(const nc_model *m, const void *kcache, const void *vcache, int max_batch, int max_seq,
                            CUtensorMap *out) {
  const nc_config &c = m->cfg;
  const int d = c.d_model, F = c.mlp_hidden, H = c.n_head;
  for (int l = 0; l < c.depth; l++) {
    const nc_layer_w &w = m->layers[l];
    if (!make_map_bf16_k64(&out[4 * l + 0], w.wqkv, (H + 2) * 128, d, d, 128)) return false;
    if (!make_map_bf16_k64(&out[4 * l + 1], w.wo, d, H * 128, H * 128, 128)) return false;
    if (!make_map_bf16_k64(&out[4 * l + 2], w.wfc, F, d, d, 128)) return false;
    if (!make_map_bf16_k64(&out[4 * l + 3], w.wproj, d, F, F, 128)) return false;
  }
  if (!make_map_bf16_k64(&out[4 * c.depth], m->wlm, c.vocab, d, d, 128)) return false;
  const int rows = c.depth * max_batch * max_seq;
  if (!make_map_bf16_k64(&out[4 * c.depth + 1], kcache, rows, 128, 128, KT)) return false;
  if (!make_map_bf16_k64(&out[4 * c.depth + 2], vcache, rows, 128, 128, KT)) return false;
  return true;
}

// Number of CTAs: whole clusters, at most one CTA per SM, all co-resident.
int decode_step_grid(int num_sms) {
  cudaError_t e = ensure_smem_attr((const void *)decode_step_kernel, SMEM_BYTES);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((num_sms / CL) * CL);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  e = cudaOccupancyMaxActiveClusters(&clusters, decode_step_kernel, &cfg);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (clusters > num_sms / CL) clusters = num_sms / CL;
  return clusters * CL;
}

cudaError_t k_decode_step(const nc_model *m, int B, int max_batch, int max_seq, const CUtensorMap *maps_dev,
                          const int32_t *tokens, const int32_t *positions, int32_t *len, float *x0, float *x1,
                          float *ss, void *q, void *y, void *f, void *kc, void *vc, const float2 *rope, float *logits,
                          const float *noise, int32_t *next, float *cand_v, int *cand_i, unsigned long long *bar,
                          float *split_part, int grid, unsigned long long *trace, uint8_t *valid_out,
                          cudaStream_t s) {
  const nc_config &c = m->cfg;
  StepArgs a;
  a.L = c.depth;
  a.d = c.d_model;
  a.H = c.n_head;
  a.F = c.mlp_hidden;
  a.V = c.vocab;
  a.B = B;
  a.max_batch = max_batch;
  a.max_seq = max_seq;
  a.grid = grid;
  a.eps = c.norm_eps;
  a.cap = c.softcap;
  a.scale_log2 = 1.4426950408889634f / sqrtf(128.f);
  a.wte = (const bf16 *)m->wte;
  a.wmaps = maps_dev;
  a.kvmaps = maps_dev + 4 * c.depth + 1;
  a.tokens = tokens;
  a.positions = positions;
  a.len = len;
  a.x0 = x0;
  a.x1 = x1;
  a.ss = ss;
  a.q = (bf16 *)q;
  a.y = (bf16 *)y;
  a.f = (bf16 *)f;
  a.kc = (bf16 *)kc;
  a.vc = (bf16 *)vc;
  a.rope = rope;
  a.logits = logits;
  a.noise = noise;
  a.next = next;
  a.cand_v = cand_v;
  a.cand_i = cand_i;
  a.bar = bar;
  a.split_cnt = reinterpret_cast<unsigned *>(bar + 1);
  a.split_part = split_part;
  a.status = m->status;
  a.trace = trace;
  a.valid_out = valid_out;
  // grid-barrier counter and split counters from zero for every step
  cudaError_t e = cudaMemsetAsync(bar, 0, decode_step_bar_bytes(), s);
  if (e != cudaSuccess) return e;
  count_launch();
  decode_step_kernel<<<grid, THREADS, SMEM_BYTES, s>>>(a);
  return cudaGetLastError();
}

}  // namespace nc
