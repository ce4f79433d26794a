// nc_step.cu — the whole single-token decode step as one persistent kernel.
//
// A decode step of the nanochat Transformer is a chain of 5 x depth
// all-to-all dependencies (QKV -> attention -> O-proj -> MLP fc -> MLP proj
// per layer). Its bytes (every weight once, each sequence's KV cache once)
// take ~0.24 ms on a B200 at d20, B = 32; what bounds it is the latency of
// that chain. One kernel runs the whole step on one CTA per SM (a
// cooperative launch, so all CTAs are resident), one phase per link,
// separated by a grid barrier (a counter zeroed before each launch, release
// increments, acquire polling, bounded), and each phase is built to put as
// little as possible between its barrier and the next:
//
//  * warp 0 is a TMA producer that walks the same phase program as everyone
//    and streams every weight tile and KV-cache tile this CTA will need into
//    a ring of 32 KB slots (as deep as shared memory allows), running ahead
//    across phase barriers: neither the weights nor the cached keys depend
//    on the step's activations, so they are mostly resident when a phase
//    starts;
//  * linear layers split their output rows over all CTAs and keep the whole
//    K in each CTA, so no CTA waits for another's partial sums. A phase's
//    activation rows (bf16, [32][K]) arrive with one bulk tensor copy right
//    after the barrier; eight compute warps split K, multiply with mma.sync
//    m16n8k16 (M = the sequences, N = 8 weight rows) out of shared memory and
//    add their partials in a fixed order. A normed input's 1/rms per row is
//    computed from the staged bf16 rows themselves. The MLP projection
//    (K = 4d) splits K four ways instead; the last of the four CTAs of a row
//    block to arrive adds the partials in split order;
//  * attention runs per (sequence, KV head): the G = H/Hkv query heads of a
//    KV head are the rows of its MMAs (flash decoding with mma.sync); each
//    pair's keys are split over up to 8 CTAs. When there are more pairs than
//    CTAs, the pairs' 64-key tiles are dealt evenly instead (tile_deal): each
//    CTA takes a contiguous run of them, which may span several pairs. The
//    last split or segment of a pair to arrive merges the softmax states in
//    order.
// Every reduction has a fixed order, so results do not depend on timing.
//
// Measured costs behind the choice of mma.sync for the linear layers (the
// probes in kv_cache_transformer_b200/microbench, on a B200): a tcgen05.mma
// with N <= 128 takes ~72 cycles
// whatever its M and N, so at 32 sequences it consumes weights at ~57
// B/cycle; mma.sync m16n8k16 runs at 8 cycles per warp instruction per SM
// sub-partition (1024 MACs/cycle/SM), the same ~64 B/cycle of weights at 32
// sequences, without a per-instruction floor, so narrow row blocks with
// full K cost nothing extra.
//
// Phases: EMBED | depth x [QKV | ATTN | OPROJ | FC | PROJ] | HEAD | MERGE.
//   EMBED  validate positions, x0 = rmsnorm(wte[token]), bf16(x0)
//   QKV    (bf16(x0) . [Wq;Wk;Wv]^T) / rms(x0); RoPE on q and k (fp32 out);
//          v appended to the cache
//   ATTN   QK norm of q and of the new keys (appended to the cache), flash
//          decoding over the cache, merge of the key splits -> y
//   OPROJ  x1 = x0 + y . Wo^T, bf16(x1)
//   FC     f = relu((bf16(x1) . Wfc^T) / rms(x1))^2
//   PROJ   x0 = x1 + f . Wproj^T (four K splits), bf16(x0)
//   HEAD   logits = cap * tanh((bf16(x0) . Wlm^T) / rms(x0) / cap) (+ noise),
//          per-CTA argmax winners
//   MERGE  next token per sequence, lengths advanced
// Every wait is bounded (~2 s): a timeout raises NC_DEV_TIMEOUT and all
// roles drain to the exit.
#include <stdlib.h>

#include "nc_internal.h"
#include "nc_sm100.cuh"

namespace nc {
using namespace sm100;

namespace {

constexpr int NCW = 8;                  // compute warps (two per SM sub-partition)
constexpr int THREADS = 32 * (1 + NCW);  // warp 0: TMA producer
constexpr int SLOT = 32768;             // ring slot bytes: a 64-key K and V tile pair, or k-blocks of weights
constexpr int HKB = SLOT / (64 * 128);  // lm_head k-blocks per slot (64 rows each)
constexpr int KT = 64;                  // keys per attention tile
constexpr int MAXB = 32;                // sequences per step: rows of every staged activation
constexpr int MAX_SPLIT = 8;            // attention key splits per sequence
constexpr int SEGMAX = 8;               // attention segments of one CTA under the tile deal
constexpr int MAX_R = 64;               // weight rows per CTA in the K-split linears
constexpr int HG = 64;                  // lm_head rows per pass (16 per warp of each warp group)
constexpr int SMEM_CAP = 227 * 1024;
constexpr int MISC = 2048;              // barriers and per-sequence tables
constexpr int CTR_BYTES = 4096;         // counters zeroed before each launch
constexpr int MAX_HKV = 16;             // KV heads (attention arrival counters per sequence)
static_assert(64 + 4 * 32 * MAX_HKV + 4 * 256 <= CTR_BYTES, "counter region: barrier, attention, projection");
constexpr int AROW = 132;               // floats per attention state row: m, l, O[128], padding
// attention scratch: the warps' softmax states, q and the new key in bf16,
// per-row merge factors
constexpr int ATT_SCRATCH = NCW * 16 * AROW * 4 + 17 * 128 * 2 + (NCW + 2) * 16 * 4;

enum Phase { P_EMBED = 0, P_QKV, P_ATTN, P_OPROJ, P_FC, P_PROJ, P_HEAD, P_MERGE };

struct StepArgs {
  int L, d, H, F, V, B, max_batch, max_seq, grid;
  int Hkv, G;                 // KV heads, query heads per KV head (G = H / Hkv <= 16)
  int r_q, r_o, r_f, r_p, s_p, r_h, n_o, n_f, n_p, n_h, n_qkv;
  int slots, splits;
  int stream;                 // attention units outnumber the CTAs: deal their key tiles evenly
  float eps, cap, scale_log2;
  const bf16 *wte;
  const CUtensorMap *wmaps;   // [4L + 1]: per layer qkv (r_q/2-row box), o, fc, proj; then lm_head
  const CUtensorMap *kvmaps;  // [4]: K and V caches as [L * max_batch * max_seq][Hkv][128], then the
                              // same views of the prefix cache (shared rows, nc_kv_fork_shared)
  const CUtensorMap *amaps;   // [4]: xb0, y, xb1, f as [32][K], boxes of rb rows
  int rb;                     // activation rows staged: 16 for B <= 16, else 32
  const int32_t *pre_seq, *pre_len;  // [max_batch]: shared rows of each sequence (0: none)
  int pmax_batch, pmax_seq;   // shape of the prefix cache
  const int32_t *tokens, *positions;
  int32_t *len;
  float *x0, *x1;             // [32][d] fp32 residual: layer input, after attention
  bf16 *xb0, *xb1, *y, *f;    // [32][d], [32][d], [32][d], [32][F]
  float *qk;                  // [32][H + Hkv][128]: q heads and k heads after RoPE, before QK norm
  bf16 *kc, *vc;              // [L][max_batch][max_seq][Hkv][128]
  const float2 *rope;         // [max_seq][64]
  float *logits;              // [B][V]
  const float *noise;         // [B][V] or null
  int32_t *next;              // [B] or null
  float *cand_v;              // [grid][32]
  int *cand_i;
  float *apart;               // [32 * Hkv][MAX_SPLIT][G][AROW]: attention softmax states (m, l, O)
  float *ppart;               // [n_p][s_p][32][r_p]: MLP projection partial sums
  unsigned long long *bar;    // grid barrier counter
  unsigned *acnt;             // [32 * Hkv] attention arrivals, cumulative over layers
  unsigned *pcnt;             // [n_p] projection arrivals, cumulative over layers
  uint32_t *status;
  unsigned long long *trace;  // [grid][phases][8] phase timestamps (ns), or null
  uint8_t *valid_out;         // [B]: 1 where the sequence's position was valid (written by CTA 0)
};

// Phase timestamps for nc_decode_trace: slot 0 phase start (after the last
// barrier), 1 activations staged / first cache tile in, 2 multiply done /
// keys done, 3 reduction or merge done, 4 phase work done (barrier entry),
// 5 producer's first load of the phase, 6 its last load, 7 unused. Only
// written when a trace buffer is set.
__device__ __forceinline__ void trace_mark(const StepArgs &a, int p, int slot) {
  if (a.trace) a.trace[((size_t)blockIdx.x * (3 + 5 * a.L) + p) * 8 + slot] = global_ns();
}

struct Smem {
  uint64_t *full, *empty;  // [slots]
  uint64_t *x_bar;         // activation staging (tx count)
  int *abort_flag;
  int *pos, *valid;        // [32]
  float *inv;              // [32] per-sequence 1/rms of the phase's normed input
  float *red_ss;           // [NCW][32] per-warp sums of squares of the staged rows
  int *flag;
  int *nseg;               // this CTA's attention segments under the tile deal; -1: units dealt in rounds
  int *seg;                // [SEGMAX][6]: sequence, KV head, first key, end key, segment, segments of the unit
};

__device__ __forceinline__ void csync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_bf(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

// Grid barrier among the compute threads of every CTA (bounded), the one
// after phase p. The counter is zeroed before every launch, so the barrier is
// complete once it reaches (p + 1) * grid: each CTA adds 1 with a release
// reduction (the CTA barrier before it orders the other compute threads'
// writes ahead of it) and polls with acquire loads.
__device__ bool grid_sync(const StepArgs &a, volatile int *abort_flag, int e, int p) {
  csync();
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
  csync();
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

// This CTA's share of a linear phase: weight rows [r0, r0 + R) (QKV: rows
// r0 .. r0+R/2-1 and their RoPE partners 64 rows on, of one head), k-blocks
// [kb0, kb0 + nkb) of 64 columns, the weight map and the activation map it
// stages.
struct Unit {
  bool active;
  int u, split;   // unit index, K split (MLP projection)
  int r0, R, N;   // first row, rows per unit, rows of the layer
  int kb0, nkb;
  int sbox;       // k-blocks of the activation map's box (what one staging copy brings)
  const CUtensorMap *map, *amap;
};

__device__ __forceinline__ Unit unit_of(const StepArgs &a, int type, int layer, int c) {
  Unit u;
  u.active = false;
  u.split = 0;
  u.kb0 = 0;
  u.sbox = a.d / 64;
  if (type == P_QKV) {
    u.N = (a.H + 2 * a.Hkv) * 128;
    u.R = a.r_q;
    u.u = c;
    u.active = c < a.n_qkv;
    const int uph = 128 / a.r_q;  // units per head
    u.r0 = (c / uph) * 128 + (c % uph) * (a.r_q / 2);
    u.nkb = a.d / 64;
    u.map = a.wmaps + 4 * layer;
    u.amap = a.amaps + 0;
  } else if (type == P_OPROJ) {
    u.N = a.d;
    u.R = a.r_o;
    u.u = c;
    u.active = c < a.n_o;
    u.r0 = c * a.r_o;
    u.nkb = a.H * 2;  // K = H * 128
    u.map = a.wmaps + 4 * layer + 1;
    u.amap = a.amaps + 1;
  } else if (type == P_FC) {
    u.N = a.F;
    u.R = a.r_f;
    u.u = c;
    u.active = c < a.n_f;
    u.r0 = c * a.r_f;
    u.nkb = a.d / 64;
    u.map = a.wmaps + 4 * layer + 2;
    u.amap = a.amaps + 2;
  } else if (type == P_PROJ) {
    u.N = a.d;
    u.R = a.r_p;
    u.u = c % a.n_p;
    u.split = c / a.n_p;
    u.active = c < a.n_p * a.s_p;
    u.r0 = u.u * a.r_p;
    const int kbt = a.F / 64, kbs = (kbt + a.s_p - 1) / a.s_p;
    u.kb0 = u.split * kbs;
    u.nkb = max(0, min(kbs, kbt - u.kb0));
    u.sbox = kbs;
    u.map = a.wmaps + 4 * layer + 3;
    u.amap = a.amaps + 3;
  } else {  // P_HEAD
    u.N = a.V;
    u.R = a.r_h;
    u.u = c;
    u.r0 = c * a.r_h;
    u.active = c < a.n_h && u.r0 < a.V;
    u.nkb = a.d / 64;
    u.map = a.wmaps + 4 * a.L;
    u.amap = a.amaps + 0;
  }
  return u;
}

// key range of split `sp` of `ns` for a sequence with n keys (64-key tiles)
__device__ __forceinline__ void key_range(int n, int sp, int ns, int &k0, int &k1) {
  int chunk = (n + ns - 1) / ns;
  chunk = (chunk + KT - 1) / KT * KT;
  k0 = min(n, sp * chunk);
  k1 = min(n, k0 + chunk);
}

__device__ __forceinline__ uint32_t kv_tile_off(int key, int c) {
  // 64-key tile loaded as two TMA boxes of 64 dims x 64 keys, 128-byte swizzle
  return (uint32_t)((c >> 3) * 8192 + key * 128 + (((c & 7) ^ (key & 7)) << 4));
}

// (row r, 16-byte chunk c) of a 128-byte-swizzled tile of 128-byte rows
__device__ __forceinline__ uint32_t swz(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

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

__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t &r0, uint32_t &r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Tensor copies of rank 3 and 4 (one copy per ring slot, per cache tile, per
// staging), with an L2 cache hint for the streamed weights.
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int x, int y, int z, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_load_3d_hint(void *dst, const CUtensorMap *map, int x, int y, int z, uint64_t *bar,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tma_load_4d_hint(void *dst, const CUtensorMap *map, int x, int y, int z, int w,
                                                 uint64_t *bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// 1D bulk copy global -> shared (16-byte aligned, size a multiple of 16),
// completing on `bar`'s transaction count.
__device__ __forceinline__ void bulk_copy(void *smem_dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(smem_dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// ------------------------------------------------------------- producer
// Slot contents: a linear unit of R rows puts kps = SLOT / (R * 128) k-blocks
// in a slot, [kb][R rows][128 B], as one tensor copy whose box spans the
// k-blocks (the last slot of a unit may run past the unit's k-blocks: zero
// fill past K, or a few bytes of the next split that nobody reads); the
// lm_head puts HKB k-blocks of 64 rows; attention puts the K tile and then
// the V tile of 64 keys, each [half][key][128 B]. Few, large slots halve the
// per-slot waits and releases of every phase.
__host__ __device__ __forceinline__ int kps_of(int R) { return SLOT / (R * 128); }

// Ring position of the producer and of each consumer: the slot in the low 16
// bits, the parity of the slot's current fill in bit 16 (advanced without a
// division by the runtime slot count).
__device__ __forceinline__ uint32_t ring_slot(uint32_t t) { return t & 0xffffu; }
__device__ __forceinline__ uint32_t ring_ph(uint32_t t) { return t >> 16; }
__device__ __forceinline__ uint32_t ring_next(uint32_t t, int slots) {
  return (int)(t & 0xffffu) + 1 == slots ? ((t & 0x10000u) ^ 0x10000u) : t + 1;
}

__device__ void producer(const StepArgs &a, const Smem &s, uint8_t *ring) {
  uint64_t evict_first;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(evict_first));
  uint32_t t = 0;
  // the next slot, armed for `bytes`; false once the pipeline has aborted
  auto take = [&](uint32_t &slot, uint32_t bytes) -> bool {
    slot = ring_slot(t);
    const uint32_t ph = ring_ph(t);
    t = ring_next(t, a.slots);
    if (!mbar_wait(&s.empty[slot], ph ^ 1, s.abort_flag, a.status)) return false;
    mbar_arrive_expect_tx(&s.full[slot], bytes);
    return true;
  };
  const int c = blockIdx.x, P = n_phases(a);
  for (int p = 0; p < P; p++) {
    int type, layer;
    phase_of(a, p, type, layer);
    bool first = true;
    if (type == P_ATTN) {
      // this CTA's units (sequence, KV head, split) or segments of the tile
      // deal, in the consumers' order
      const int nseg = *s.nseg;
      const int nun = nseg >= 0 ? nseg : (a.B * a.Hkv * a.splits + a.grid - 1 - c) / a.grid;
      for (int iu = 0; iu < nun; iu++) {
        int b, j, k0, k1;
        if (nseg >= 0) {
          const int *sg = s.seg + 6 * iu;
          b = sg[0];
          j = sg[1];
          k0 = sg[2];
          k1 = sg[3];
        } else {
          const int un = c + iu * a.grid;
          b = un / (a.Hkv * a.splits);
          j = (un / a.splits) % a.Hkv;
          if (!s.valid[b]) continue;
          key_range(s.pos[b] + 1, un % a.splits, a.splits, k0, k1);
        }
        const int row0 = (layer * a.max_batch + b) * a.max_seq;
        // tiles below the shared length (a multiple of 64) come from the prefix cache
        const int plen = a.pre_len[b];
        const int prow0 = (layer * a.pmax_batch + a.pre_seq[b]) * a.pmax_seq;
        for (int key = k0; key < k1; key += KT) {  // K at the slot's start, V 16 KB on
          uint32_t slot;
          if (!take(slot, SLOT)) return;
          if (first) trace_mark(a, p, 5);
          first = false;
          const bool sh = key < plen;
          for (int which = 0; which < 2; which++)
            tma_load_4d(ring + slot * SLOT + which * (SLOT / 2), a.kvmaps + (sh ? 2 : 0) + which, 0,
                        (sh ? prow0 : row0) + key, 0, j, &s.full[slot]);
        }
      }
      if (!first) trace_mark(a, p, 6);
    } else if (type == P_QKV || type == P_OPROJ || type == P_FC || type == P_PROJ || type == P_HEAD) {
      const Unit u = unit_of(a, type, layer, c);
      if (!u.active) continue;
      if (type == P_HEAD) {
        const int rows = min(u.R, a.V - u.r0);
        for (int g0 = 0; g0 < rows; g0 += HG)
          for (int kb = 0; kb < u.nkb; kb += HKB) {
            uint32_t slot;
            if (!take(slot, HKB * HG * 128)) return;
            if (first) trace_mark(a, p, 5);
            first = false;
            tma_load_3d_hint(ring + slot * SLOT, u.map, 0, u.r0 + g0, kb, &s.full[slot], evict_first);
          }
      } else {
        const int kps = kps_of(u.R);
        for (int ch = 0; ch < u.nkb; ch += kps) {
          uint32_t slot;
          if (!take(slot, kps * u.R * 128)) return;
          if (first) trace_mark(a, p, 5);
          first = false;
          if (type == P_QKV)  // rows r0..r0+7 and their RoPE partners r0+64..r0+71
            tma_load_4d_hint(ring + slot * SLOT, u.map, 0, u.r0, 0, u.kb0 + ch, &s.full[slot], evict_first);
          else
            tma_load_3d_hint(ring + slot * SLOT, u.map, 0, u.r0, u.kb0 + ch, &s.full[slot], evict_first);
        }
      }
      trace_mark(a, p, 6);
    }
  }
}

// ------------------------------------------------- compute-side helpers
// Stage the phase's activation rows: sbox k-blocks of 64 columns x rb rows
// from k-block kb0 of the activation map into xs ([kb][rb rows][128 B],
// swizzled), one tensor copy issued right after the barrier. The writers' data
// was released through the grid barrier; the proxy fences order it (and this
// CTA's earlier generic accesses to xs) ahead of the copy.
__device__ __forceinline__ void stage_issue(const Smem &s, uint8_t *xs, const CUtensorMap *amap, int kb0, int sbox,
                                            int rb) {
  asm volatile("fence.proxy.async.global;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  mbar_arrive_expect_tx(s.x_bar, sbox * rb * 128);
  tma_load_3d(xs, amap, 0, 0, kb0, s.x_bar);
}

// 1/rms of each sequence's row from the staged bf16 row itself (the normed
// phases stage the whole row, K = d): warp w sums the squares of k-blocks w,
// w + 8, ... (lane = sequence), the warps' partials are added in warp order.
__device__ void smem_inv(const StepArgs &a, const Smem &s, const uint8_t *xs, int nkb, int warp, int lane, int e) {
  float acc = 0.f;
  for (int kb = warp; kb < nkb; kb += NCW) {
    // rows past rb belong to the next k-block (or lie past the staging):
    // their sums are not used
    const uint4 *row = reinterpret_cast<const uint4 *>(xs + kb * a.rb * 128 + lane * 128);
    // the row's 16-byte chunks in column order (the swizzle permutes them by
    // row), so every row sums in the same order and the lanes hit different banks
#pragma unroll
    for (int c = 0; c < 8; c++) {
      const uint4 v = row[c ^ (lane & 7)];
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; i++) {
        const float lo = __uint_as_float(w4[i] << 16), hi = __uint_as_float(w4[i] & 0xffff0000u);
        acc = fmaf(lo, lo, acc);
        acc = fmaf(hi, hi, acc);
      }
    }
  }
  s.red_ss[warp * 32 + lane] = acc;
  csync();
  if (e < MAXB) {
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < NCW; w++) sum += s.red_ss[w * 32 + e];
    s.inv[e] = e < a.B ? rsqrtf(sum / a.d + a.eps) : 0.f;
  }
  csync();
}

// The unit's product for every sequence, this warp's K part (k-blocks kb
// with kb % NCW == warp): NT n8 tiles of weight rows, MT m16 tiles of
// sequences, compile-time so that every fragment of a k-block is loaded before
// its MMAs. Consumes the unit's ring slots in the producer's order; the
// warp's partial goes to red[warp] as [32][R] (sequence b, row r at b*R + r).
template <int NT, int MT>
__device__ bool gemv_t(const StepArgs &a, const Smem &s, uint8_t *ring, const uint8_t *xs, const Unit &u, uint32_t &t,
                       float *red, int warp, int lane) {
  constexpr int R = NT * 8;
  float acc[MT][NT][4];
#pragma unroll
  for (int m = 0; m < MT; m++)
#pragma unroll
    for (int n = 0; n < NT; n++) acc[m][n][0] = acc[m][n][1] = acc[m][n][2] = acc[m][n][3] = 0.f;
  constexpr int kps = SLOT / (R * 128);
  for (int ch = 0; ch < u.nkb; ch += kps) {
    const uint32_t slot = ring_slot(t), ph = ring_ph(t);
    t = ring_next(t, a.slots);
    mbar_wait(&s.full[slot], ph, s.abort_flag, a.status);  // a timeout is raised at the next grid barrier
    const int n = min(kps, u.nkb - ch);
    const uint8_t *wslot = ring + slot * SLOT;
    for (int j = 0; j < n; j++) {
      const int kb = ch + j;
      if (kb % NCW != warp) continue;
      const uint32_t wb = smem_u32(wslot + j * R * 128), xb = smem_u32(xs + kb * a.rb * 128);
      uint32_t af[4][MT][4], bf[4][NT][2];
#pragma unroll
      for (int ks = 0; ks < 4; ks++) {
#pragma unroll
        for (int m = 0; m < MT; m++)
          ldsm_x4(xb + swz(m * 16 + (lane & 15), 2 * ks + (lane >> 4)), af[ks][m][0], af[ks][m][1], af[ks][m][2],
                  af[ks][m][3]);
#pragma unroll
        for (int nt = 0; nt < NT; nt++)
          ldsm_x2(wb + swz(nt * 8 + (lane & 7), 2 * ks + ((lane >> 3) & 1)), bf[ks][nt][0], bf[ks][nt][1]);
      }
#pragma unroll
      for (int ks = 0; ks < 4; ks++)
#pragma unroll
        for (int nt = 0; nt < NT; nt++)
#pragma unroll
          for (int m = 0; m < MT; m++) mma16816(acc[m][nt], af[ks][m], bf[ks][nt][0], bf[ks][nt][1]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.empty[slot]);
  }
  // every warp is done with the staged rows before any partial overlays them
  csync();
  const int g = lane >> 2, t4 = lane & 3;
  float *mine = red + (size_t)warp * MAXB * R;
#pragma unroll
  for (int m = 0; m < MT; m++)
#pragma unroll
    for (int nt = 0; nt < NT; nt++) {
      const int r = nt * 8 + 2 * t4, b = m * 16 + g;
      *reinterpret_cast<float2 *>(mine + b * R + r) = make_float2(acc[m][nt][0], acc[m][nt][1]);
      *reinterpret_cast<float2 *>(mine + (b + 8) * R + r) = make_float2(acc[m][nt][2], acc[m][nt][3]);
    }
  return true;
}

template <int MT>
__device__ bool gemv_mt(const StepArgs &a, const Smem &s, uint8_t *ring, const uint8_t *xs, const Unit &u,
                        uint32_t &t, float *red, int warp, int lane) {
  switch (u.R / 8) {
    case 1: return gemv_t<1, MT>(a, s, ring, xs, u, t, red, warp, lane);
    case 2: return gemv_t<2, MT>(a, s, ring, xs, u, t, red, warp, lane);
    case 3: return gemv_t<3, MT>(a, s, ring, xs, u, t, red, warp, lane);
    case 4: return gemv_t<4, MT>(a, s, ring, xs, u, t, red, warp, lane);
    case 5: return gemv_t<5, MT>(a, s, ring, xs, u, t, red, warp, lane);
    case 6: return gemv_t<6, MT>(a, s, ring, xs, u, t, red, warp, lane);
    case 7: return gemv_t<7, MT>(a, s, ring, xs, u, t, red, warp, lane);
    default: return gemv_t<8, MT>(a, s, ring, xs, u, t, red, warp, lane);
  }
}

// Add the four warps' partials (written by gemv_t) in warp order: the
// returned [32][R] block holds the full product of sequence b and weight row
// r0 + r at b * R + r.
__device__ float *reduce_warps(float *red, int R, int MT, int e) {
  csync();
  float *out = red + (size_t)NCW * MAXB * R;
  for (int i = e; i < MT * 16 * R; i += 32 * NCW) {
    float v = red[i];
#pragma unroll
    for (int w = 1; w < NCW; w++) v += red[(size_t)w * MAXB * R + i];
    out[i] = v;
  }
  csync();
  return out;
}

// ------------------------------------------------------------ attention
// Split `sp` of sequence b's keys: q and the new key get their QK norm here,
// the new key is appended to the cache by the split that holds it, then
// flash decoding over the split's 64-key tiles (mma.sync m16n8k16, rows =
// query heads padded to 16): warp group g (warps 4g .. 4g+3) takes the tiles
// of parity g, each warp 16 keys of a tile. The eight warps' softmax states
// are merged (per-row factors first), the split's state goes to apart, and
// the last split to arrive merges all splits in split order into y.
__device__ void attention_unit(const StepArgs &a, const Smem &s, uint8_t *ring, uint8_t *xs, int layer, int e,
                               uint32_t &t, uint32_t &xph, int p, int b, int j, int sp, int ns, int k0, int k1,
                               bool first) {
  const int warp = e >> 5, lane = e & 31, g = lane >> 2, t4 = lane & 3;
  const int grp = warp >> 2, wq = warp & 3;
  const int G = a.G, vs = b * a.Hkv + j;  // query heads j*G .. j*G+G-1 read KV head j
  const size_t lay = (size_t)layer * a.max_batch * a.max_seq * a.Hkv * 128;
  const size_t crow = ((size_t)b * a.max_seq + s.pos[b]) * a.Hkv + j;  // cache row of the new key / value
  const int pos = s.pos[b];
  float *cw = reinterpret_cast<float *>(xs);                                 // [8 warps][16 rows][AROW]
  bf16 *qs = reinterpret_cast<bf16 *>(xs + NCW * 16 * AROW * 4);             // [17][128]: q heads, the new key
  float *fac = reinterpret_cast<float *>(xs + NCW * 16 * AROW * 4 + 17 * 128 * 2);  // [NCW + 2][16]
  // QK norm of the G query heads and of the new key, in fp32, to bf16 (the
  // warp's heads w, w+8, w+16 are loaded before any is used)
  {
    float4 qv[3];
#pragma unroll
    for (int i = 0; i < 3; i++) {
      const int h = warp + NCW * i, src = h < G ? j * G + h : a.H + j;
      qv[i] = h <= G ? __ldcg(reinterpret_cast<const float4 *>(a.qk + ((size_t)b * (a.H + a.Hkv) + src) * 128) + lane)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int i = 0; i < 3; i++) {
      const int h = warp + NCW * i;
      if (h > G) break;
      const float4 v = qv[i];
      const float r = rsqrtf(warp_sum(v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w) * (1.0f / 128) + a.eps);
      *reinterpret_cast<uint2 *>(qs + h * 128 + 4 * lane) =
          make_uint2(pack_bf(v.x * r, v.y * r), pack_bf(v.z * r, v.w * r));
    }
  }
  csync();
  const bf16 *knew = qs + G * 128;
  if (pos >= k0 && pos < k1 && e < 16)  // this split holds the new key: append it to the cache
    *reinterpret_cast<uint4 *>(a.kc + lay + crow * 128 + e * 8) = *reinterpret_cast<const uint4 *>(knew + e * 8);
  uint32_t qa[8][4];
#pragma unroll
  for (int ks = 0; ks < 8; ks++) {
    const int c0 = ks * 16 + t4 * 2;
    qa[ks][0] = g < G ? *reinterpret_cast<const uint32_t *>(qs + g * 128 + c0) : 0u;
    qa[ks][1] = g + 8 < G ? *reinterpret_cast<const uint32_t *>(qs + (g + 8) * 128 + c0) : 0u;
    qa[ks][2] = g < G ? *reinterpret_cast<const uint32_t *>(qs + g * 128 + c0 + 8) : 0u;
    qa[ks][3] = g + 8 < G ? *reinterpret_cast<const uint32_t *>(qs + (g + 8) * 128 + c0 + 8) : 0u;
  }
  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; i++) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  int tile = 0;
  for (int key0 = k0; key0 < k1; key0 += KT, tile++) {
    const uint32_t ks_ = ring_slot(t), kph = ring_ph(t);
    t = ring_next(t, a.slots);
    // every warp waits for every tile (its arrival on the slot must follow the fill)
    mbar_wait(&s.full[ks_], kph, s.abort_flag, a.status);  // a timeout is raised at the next grid barrier
    if (first && e == 0 && key0 == k0) trace_mark(a, p, 1);
    uint8_t *K = ring + ks_ * SLOT, *V = K + SLOT / 2;
    // the new key (normed here) and value (written in the QKV phase) may
    // postdate the prefetch of their tile: patch that row
    const int pr = pos - key0;
    if (pr >= 0 && pr < KT) {
      if (e < 32) {
        const int cc = e & 15;
        const uint4 v = e < 16 ? *reinterpret_cast<const uint4 *>(knew + cc * 8)
                               : __ldcg(reinterpret_cast<const uint4 *>(a.vc + lay + crow * 128 + cc * 8));
        *reinterpret_cast<uint4 *>((e < 16 ? K : V) + kv_tile_off(pr, cc)) = v;
      }
      csync();
    }
    if ((tile & 1) == grp) {
      const uint32_t kb = smem_u32(K), vb = smem_u32(V);
      const int kw = wq * 16;
      const int kg = key0 + kw;
      float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < 8; ks++) {
        const int key = kw + (lane & 7) + ((lane >> 4) << 3);
        const int cc = 2 * ks + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kb + kv_tile_off(key, cc), b0, b1, b2, b3);
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
        const int cc = dt + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vb + kv_tile_off(key, cc), b0, b1, b2, b3);
        mma16816(o[dt], pa, b0, b1);
        mma16816(o[dt + 1], pa, b2, b3);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.empty[ks_]);
  }
  if (e == 0) trace_mark(a, p, 2);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  {
    float *mine = cw + warp * 16 * AROW;
    if (t4 == 0) {
      mine[g * AROW + 0] = m0;
      mine[g * AROW + 1] = l0;
      mine[(g + 8) * AROW + 0] = m1;
      mine[(g + 8) * AROW + 1] = l1;
    }
#pragma unroll
    for (int dt = 0; dt < 16; dt++) {
      const int col = dt * 8 + 2 * t4;
      *reinterpret_cast<float2 *>(mine + g * AROW + 2 + col) = make_float2(o[dt][0], o[dt][1]);
      *reinterpret_cast<float2 *>(mine + (g + 8) * AROW + 2 + col) = make_float2(o[dt][2], o[dt][3]);
    }
  }
  csync();
  // the eight warps' states merged: per-row factors, then the rows, to apart[b][sp]
  float *dst = a.apart + ((size_t)vs * MAX_SPLIT + sp) * G * AROW;
  if (e < G) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NCW; w++) M = fmaxf(M, cw[(w * 16 + e) * AROW]);
    float Ls = 0.f;
#pragma unroll
    for (int w = 0; w < NCW; w++) {
      const float mw = cw[(w * 16 + e) * AROW];
      const float f = mw == -INFINITY ? 0.f : exp2f(mw - M);
      fac[w * 16 + e] = f;
      Ls += f * cw[(w * 16 + e) * AROW + 1];
    }
    dst[e * AROW] = M;
    dst[e * AROW + 1] = Ls;
  }
  csync();
  for (int idx = e; idx < G * 128; idx += 32 * NCW) {
    const int row = idx >> 7, col = idx & 127;
    float O = 0.f;
#pragma unroll
    for (int w = 0; w < NCW; w++) O += fac[w * 16 + row] * cw[(w * 16 + row) * AROW + 2 + col];
    dst[row * AROW + 2 + col] = O;
  }
  csync();
  if (e == 0) {
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(a.acnt + vs) : "memory");
    *s.flag = old == (unsigned)((layer + 1) * ns - 1) ? 1 : 0;
  }
  csync();
  if (*s.flag) {  // the last split: merge all splits in split order
    // every split's G state rows in one bulk copy each, over the warp states
    // (free now: this split's state is in apart)
    float *st = cw;  // [splits][G][AROW]
    const uint32_t rows_bytes = (uint32_t)(G * AROW * 4);
    if (e == 0) {
      asm volatile("fence.proxy.async.global;" ::: "memory");
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive_expect_tx(s.x_bar, rows_bytes * ns);
      for (int q = 0; q < ns; q++)
        bulk_copy(st + q * G * AROW, a.apart + ((size_t)vs * MAX_SPLIT + q) * G * AROW, rows_bytes, s.x_bar);
    }
    mbar_wait(s.x_bar, xph & 1, s.abort_flag, a.status);
    xph++;
    if (e < G) {
      float M = -INFINITY;
      for (int q = 0; q < ns; q++) M = fmaxf(M, st[(q * G + e) * AROW]);
      float Ls = 0.f;
      for (int q = 0; q < ns; q++) {
        const float mq = st[(q * G + e) * AROW];
        const float f = mq == -INFINITY ? 0.f : exp2f(mq - M);
        fac[q * 16 + e] = f;
        Ls += f * st[(q * G + e) * AROW + 1];
      }
      fac[NCW * 16 + e] = Ls > 0.f ? 1.f / Ls : 0.f;
    }
    csync();
    for (int idx = e; idx < G * 128; idx += 32 * NCW) {
      const int row = idx >> 7, col = idx & 127;
      float O = 0.f;
      for (int q = 0; q < ns; q++) O += fac[q * 16 + row] * st[(q * G + row) * AROW + 2 + col];
      a.y[(size_t)b * a.d + (j * G + row) * 128 + col] = __float2bfloat16_rn(O * fac[NCW * 16 + row]);
    }
  }
  csync();  // s.flag and the scratch are rewritten by the next use
}

// The tile deal of the attention phases (one warp; positions are fixed for
// the whole step, so it holds for every layer). The units (sequence b, KV
// head j), in that order, hold n(u) = ceil((pos[b] + 1) / 64) key tiles, T in
// all; CTA c takes the tiles [c*T/grid, (c+1)*T/grid) of the concatenation,
// which cut the units into segments. A unit's segments are numbered by CTA
// (tile t belongs to CTA (t*grid + grid - 1) / T, so with T >= grid every CTA
// has tiles and a unit's CTAs are consecutive); the last one to finish merges
// them in that order. The deal is kept only when T >= grid, every unit has at
// most MAX_SPLIT segments and no CTA can have more than SEGMAX (conditions
// every CTA evaluates alike); otherwise nseg = -1 and the units are dealt in
// rounds of key splits.
__device__ void tile_deal(const StepArgs &a, const Smem &s, int lane) {
  const int units = a.B * a.Hkv;
  const long long G = a.grid, c = blockIdx.x;
  auto tiles_of = [&](int u) -> long long {
    const int b = u / a.Hkv;
    return s.valid[b] ? (s.pos[b] + 1 + KT - 1) / KT : 0;
  };
  long long T = 0, n_min = 1LL << 40;  // all tiles; fewest tiles of a unit that has any
  for (int u = lane; u < units; u += 32) {
    const long long n = tiles_of(u);
    T += n;
    if (n > 0 && n < n_min) n_min = n;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    T += __shfl_xor_sync(0xffffffffu, T, o);
    n_min = min(n_min, __shfl_xor_sync(0xffffffffu, n_min, o));
  }
  // every CTA takes the same decision: a range of at most ceil(T / grid)
  // tiles meets at most ceil(T / grid) / n_min + 2 units
  bool ok = a.stream && T >= G && ((T + G - 1) / G) / n_min + 2 <= SEGMAX;
  const long long lo = c * T / G, hi = (c + 1) * T / G;
  int count = 0, max_ns = 0;
  long long base = 0;  // tiles of the units before this chunk of 32
  for (int u0 = 0; ok && u0 < units; u0 += 32) {
    const int u = u0 + lane;
    const long long n = u < units ? tiles_of(u) : 0;
    long long incl = n;  // inclusive scan over the lanes
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const long long U = base + incl - n;  // first tile of unit u
    const long long o0 = n > 0 ? (U * G + G - 1) / T : 0;
    const int ns = n > 0 ? (int)(((U + n - 1) * G + G - 1) / T - o0 + 1) : 0;
    const bool mine = n > 0 && U < hi && U + n > lo;
    const unsigned mask = __ballot_sync(0xffffffffu, mine);
    if (mine) {
      const int slot = count + __popc(mask & ((1u << lane) - 1));
      if (slot < SEGMAX) {
        const int b = u / a.Hkv, n_keys = s.pos[b] + 1;
        const long long t0 = (U > lo ? U : lo) - U, t1 = (U + n < hi ? U + n : hi) - U;
        int *sg = s.seg + 6 * slot;
        sg[0] = b;
        sg[1] = u % a.Hkv;
        sg[2] = (int)(t0 * KT);
        sg[3] = (int)(t1 * KT < n_keys ? t1 * KT : n_keys);
        sg[4] = (int)(c - o0);
        sg[5] = ns;
      }
    }
    count += __popc(mask);
    int m = ns;
#pragma unroll
    for (int o = 16; o; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    max_ns = max(max_ns, m);
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  ok = ok && max_ns <= MAX_SPLIT;
  if (lane == 0) *s.nseg = ok ? count : -1;
}

// This CTA's attention units (sequence, KV head, split) or segments of the
// tile deal, in the producer's order.
__device__ bool attention_phase(const StepArgs &a, const Smem &s, uint8_t *ring, uint8_t *xs, int layer, int e,
                                uint32_t &t, uint32_t &xph, int p) {
  bool first = true;
  const int nseg = *s.nseg;
  if (nseg >= 0) {
    for (int i = 0; i < nseg; i++) {
      const int *sg = s.seg + 6 * i;
      attention_unit(a, s, ring, xs, layer, e, t, xph, p, sg[0], sg[1], sg[4], sg[5], sg[2], sg[3], first);
      first = false;
    }
  } else {
    for (int un = blockIdx.x; un < a.B * a.Hkv * a.splits; un += a.grid) {
      const int b = un / (a.Hkv * a.splits), j = (un / a.splits) % a.Hkv, sp = un % a.splits;
      if (!s.valid[b]) continue;
      int k0, k1;
      key_range(s.pos[b] + 1, sp, a.splits, k0, k1);
      attention_unit(a, s, ring, xs, layer, e, t, xph, p, b, j, sp, a.splits, k0, k1, first);
      first = false;
    }
  }
  if (e == 0) trace_mark(a, p, 3);
  return true;
}

// ------------------------------------------------------------- epilogues
// QKV: rows i and hq + i of the unit (hq = R / 2) are head rows j0 + i and
// j0 + 64 + i (a RoPE pair). q and k heads: scale by 1/rms(x0), rotate, to
// qk (fp32); a v head: scale, bf16, appended to its KV head's slot of the
// value cache.
__device__ void qkv_epilogue(const StepArgs &a, const Smem &s, const float *sum, const Unit &u, int layer, int e) {
  const int head = u.r0 >> 7, j0 = u.r0 & 127, hq = u.R / 2;
  const size_t lay = (size_t)layer * a.max_batch * a.max_seq * a.Hkv * 128;
  for (int idx = e; idx < a.B * hq; idx += 32 * NCW) {
    const int b = idx / hq, i = idx % hq;
    const float lo = sum[b * u.R + i] * s.inv[b], hi = sum[b * u.R + hq + i] * s.inv[b];
    if (head < a.H + a.Hkv) {
      const float2 cs = a.rope[(size_t)s.pos[b] * 64 + j0 + i];
      float *dst = a.qk + ((size_t)b * (a.H + a.Hkv) + head) * 128;
      dst[j0 + i] = lo * cs.x - hi * cs.y;
      dst[j0 + 64 + i] = hi * cs.x + lo * cs.y;
    } else if (s.valid[b]) {
      bf16 *dst = a.vc + lay + (((size_t)b * a.max_seq + s.pos[b]) * a.Hkv + (head - a.H - a.Hkv)) * 128;
      dst[j0 + i] = __float2bfloat16_rn(lo);
      dst[j0 + 64 + i] = __float2bfloat16_rn(hi);
    }
  }
}

// Residual: xout = xin + sum over the unit's rows (row r of the layer is
// column r of the residual), bf16(xout), and this CTA's sums of squares.
// The residual inputs of the rows this thread finishes, loaded at the start
// of the phase (element i: index e + 256 i of the unit's [32][R] block).
constexpr int XR = MAXB * MAX_R / (32 * NCW);
__device__ __forceinline__ void load_resid(const StepArgs &a, const Unit &u, const float *xin, int e, float (&xr)[XR]) {
#pragma unroll
  for (int i = 0; i < XR; i++) {
    const int idx = e + 32 * NCW * i, b = idx / u.R, col = u.r0 + idx % u.R;
    xr[i] = (idx < MAXB * u.R && b < a.B && col < u.N) ? __ldcg(xin + (size_t)b * a.d + col) : 0.f;
  }
}

__device__ void resid_epilogue(const StepArgs &a, const float *sum, const Unit &u, const float (&xr)[XR],
                               float *xout, bf16 *xbout, int e) {
#pragma unroll
  for (int i = 0; i < XR; i++) {
    const int idx = e + 32 * NCW * i;
    if (idx >= MAXB * u.R) break;
    const int b = idx / u.R, r = idx % u.R, col = u.r0 + r;
    if (b < a.B && col < u.N) {
      const float v = xr[i] + sum[idx];
      xout[(size_t)b * a.d + col] = v;
      xbout[(size_t)b * a.d + col] = __float2bfloat16_rn(v);
    }
  }
}

// lm_head rows [row0, row0 + 64): softcap, logits, and the running
// per-sequence winners of this thread (best[2 * m + h]: sequence m*16 + g + 8h).
template <int MT>
__device__ void head_group(const StepArgs &a, const Smem &s, const float (&acc)[MT][2][4], int row0, int warp,
                           int lane, ArgMax (&best)[4]) {
  const int g = lane >> 2, t4 = lane & 3;
  const float inv_cap = 1.0f / a.cap;
#pragma unroll
  for (int m = 0; m < MT; m++) {
#pragma unroll
    for (int hh = 0; hh < 2; hh++) {
      const int b = m * 16 + g + 8 * hh;
      if (b >= a.B) continue;
#pragma unroll
      for (int nt = 0; nt < 2; nt++) {
        const int col = row0 + warp * 16 + nt * 8 + 2 * t4;
        if (col >= a.V) continue;
        const float z0 = a.cap * tanhf(acc[m][nt][2 * hh] * s.inv[b] * inv_cap);
        const float z1 = a.cap * tanhf(acc[m][nt][2 * hh + 1] * s.inv[b] * inv_cap);
        if (s.valid[b]) *reinterpret_cast<float2 *>(a.logits + (size_t)b * a.V + col) = make_float2(z0, z1);
        float n0 = 0.f, n1 = 0.f;
        if (a.noise) {
          const float2 nz = *reinterpret_cast<const float2 *>(a.noise + (size_t)b * a.V + col);
          n0 = nz.x;
          n1 = nz.y;
        }
        best[2 * m + hh] = argmax_merge(best[2 * m + hh], ArgMax{z0 + n0, col});
        best[2 * m + hh] = argmax_merge(best[2 * m + hh], ArgMax{z1 + n1, col + 1});
      }
    }
  }
}

// The lm_head rows of this CTA, 64 at a time: warp w of group g takes rows
// 16 (w % 4) .. +15 of the 64 and k-block g of every slot (a slot holds two),
// full K from the ring. The halves are added in the group's last slot, which
// is released only afterwards; group 0 then writes the group's logits and
// keeps its winners.
template <int MT>
__device__ void head_rows(const StepArgs &a, const Smem &s, uint8_t *ring, const uint8_t *xs, const Unit &u,
                          uint32_t &t, int warp, int lane, ArgMax (&best)[4]) {
  const int grp = warp >> 2, wq = warp & 3;
  const int rows = min(u.R, a.V - u.r0);
  for (int g0 = 0; g0 < rows; g0 += HG) {
    float acc[MT][2][4];
#pragma unroll
    for (int m = 0; m < MT; m++)
#pragma unroll
      for (int n = 0; n < 2; n++) acc[m][n][0] = acc[m][n][1] = acc[m][n][2] = acc[m][n][3] = 0.f;
    uint32_t last_slot = 0;
    for (int kb2 = 0; kb2 < u.nkb; kb2 += HKB) {
      const uint32_t slot = ring_slot(t), ph = ring_ph(t);
      t = ring_next(t, a.slots);
      mbar_wait(&s.full[slot], ph, s.abort_flag, a.status);  // a timeout is raised at the next grid barrier
      const int n = min(HKB, u.nkb - kb2);
      for (int q = grp; q < n; q += 2) {  // warp group g takes the slot's k-blocks g, g + 2, ...
        const uint32_t wb = smem_u32(ring + slot * SLOT + q * HG * 128);
        const uint32_t xb = smem_u32(xs + (kb2 + q) * a.rb * 128);
        uint32_t af[4][MT][4], bf[4][4];
#pragma unroll
        for (int ks = 0; ks < 4; ks++) {
#pragma unroll
          for (int m = 0; m < MT; m++)
            ldsm_x4(xb + swz(m * 16 + (lane & 15), 2 * ks + (lane >> 4)), af[ks][m][0], af[ks][m][1], af[ks][m][2],
                    af[ks][m][3]);
          ldsm_x4(wb + swz(wq * 16 + (lane & 7) + ((lane >> 4) << 3), 2 * ks + ((lane >> 3) & 1)), bf[ks][0],
                  bf[ks][1], bf[ks][2], bf[ks][3]);
        }
#pragma unroll
        for (int ks = 0; ks < 4; ks++)
#pragma unroll
          for (int m = 0; m < MT; m++) {
            mma16816(acc[m][0], af[ks][m], bf[ks][0], bf[ks][1]);
            mma16816(acc[m][1], af[ks][m], bf[ks][2], bf[ks][3]);
          }
      }
      if (kb2 + HKB < u.nkb) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.empty[slot]);
      } else {
        last_slot = slot;
      }
    }
    // group 1's half into group 0 through the last slot (every warp is done
    // with its weights first)
    float *scr = reinterpret_cast<float *>(ring + last_slot * SLOT) + (wq * 32 + lane) * (MT * 8);
    csync();
    if (grp == 1) {
#pragma unroll
      for (int m = 0; m < MT; m++)
#pragma unroll
        for (int n = 0; n < 2; n++)
          *reinterpret_cast<float4 *>(scr + (m * 2 + n) * 4) = make_float4(acc[m][n][0], acc[m][n][1], acc[m][n][2], acc[m][n][3]);
    }
    csync();
    if (grp == 0) {
#pragma unroll
      for (int m = 0; m < MT; m++)
#pragma unroll
        for (int n = 0; n < 2; n++) {
          const float4 h = *reinterpret_cast<const float4 *>(scr + (m * 2 + n) * 4);
          acc[m][n][0] += h.x;
          acc[m][n][1] += h.y;
          acc[m][n][2] += h.z;
          acc[m][n][3] += h.w;
        }
      head_group<MT>(a, s, acc, u.r0 + g0, wq, lane, best);
    }
    csync();
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.empty[last_slot]);
  }
}

// ------------------------------------------------------------ the kernel
// Activation region of the kernel's shared memory for width d: the staged
// rows, the attention scratch or the warp partials of the widest unit.
__host__ __device__ constexpr int xreg_bytes(int d) {
  return ((MAXB * d * 2 > ATT_SCRATCH ? MAXB * d * 2 : ATT_SCRATCH) > (NCW + 1) * MAXB * MAX_R * 4
              ? (MAXB * d * 2 > ATT_SCRATCH ? MAXB * d * 2 : ATT_SCRATCH)
              : (NCW + 1) * MAXB * MAX_R * 4);
}

// 9 warps: registers are allocated to warps in groups of four (one per SM
// sub-partition), so the block is charged for 12 warps and must stay within
// 168 registers a thread
__global__ void __launch_bounds__(THREADS, 1) decode_step_kernel(StepArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint32_t raw = smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw + 1023) & ~1023u) - raw);
  uint8_t *ring = smem;
  uint8_t *xs = smem + a.slots * SLOT;
  Smem s;
  {
    uint64_t *bb = reinterpret_cast<uint64_t *>(xs + ((xreg_bytes(a.d) + 1023) & ~1023));
    s.full = bb;
    s.empty = bb + a.slots;
    s.x_bar = bb + 2 * a.slots;
    s.abort_flag = reinterpret_cast<int *>(s.x_bar + 1);
    s.pos = s.abort_flag + 1;
    s.valid = s.pos + 32;
    s.inv = reinterpret_cast<float *>(s.valid + 32);
    s.red_ss = s.inv + 32;
    s.flag = reinterpret_cast<int *>(s.red_ss + NCW * 32);
    s.nseg = s.flag + 1;
    s.seg = s.nseg + 1;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < a.slots; i++) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], NCW);
    }
    mbar_init(s.x_bar, 1);
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
  __syncthreads();
  if (warp == 0) tile_deal(a, s, lane);
  __syncthreads();

  if (warp == 0) {
    if (lane == 0) producer(a, s, ring);
  } else {
    const int e = threadIdx.x - 32;
    const int cw = warp - 1;  // compute warp 0..7
    const int MT = a.B > 16 ? 2 : 1;
    uint32_t t = 0;           // ring position (slot, parity), in the producer's order
    uint32_t xph = 0;         // staging barrier phase
    const int P = n_phases(a);
    bool ok = true;
    float *red = reinterpret_cast<float *>(xs);
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
          for (int i = e; i < a.d; i += 32 * NCW) {
            const float v = __bfloat162float(row[i]);
            sq += v * v;
          }
          sq = warp_sum(sq);
          if (lane == 0) red[cw] = sq;
          csync();
          float tot = 0.f;
          for (int w = 0; w < NCW; w++) tot += red[w];
          const float inv = rsqrtf(tot / a.d + a.eps);
          for (int i = e; i < a.d; i += 32 * NCW) {
            const float v = __bfloat162float(row[i]) * inv;
            a.x0[(size_t)b * a.d + i] = v;
            a.xb0[(size_t)b * a.d + i] = __float2bfloat16_rn(v);
          }
          csync();
        }
      } else if (type == P_ATTN) {
        ok = attention_phase(a, s, ring, xs, layer, e, t, xph, p);
      } else if (type == P_MERGE) {
        for (int b = blockIdx.x; b < a.B; b += gridDim.x) {
          if (!s.valid[b]) continue;
          ArgMax best{-INFINITY, 0x7fffffff};
          for (int i = e; i < a.n_h; i += 32 * NCW)
            best = argmax_merge(best, ArgMax{__ldcg(&a.cand_v[(size_t)i * 32 + b]), __ldcg(&a.cand_i[(size_t)i * 32 + b])});
          best = warp_argmax(best);
          if (lane == 0) {
            red[2 * cw] = best.v;
            reinterpret_cast<int *>(red)[2 * cw + 1] = best.i;
          }
          csync();
          if (e == 0) {
            ArgMax r{red[0], reinterpret_cast<int *>(red)[1]};
            for (int q = 1; q < NCW; q++) r = argmax_merge(r, ArgMax{red[2 * q], reinterpret_cast<int *>(red)[2 * q + 1]});
            if (a.next) a.next[b] = r.i;
            a.len[b] = s.pos[b] + 1;
          }
          csync();
        }
        for (int b = blockIdx.x; b < a.B; b += gridDim.x)
          if (!s.valid[b] && e == 0) atomicOr(a.status, (unsigned)NC_DEV_BAD_POSITION);
      } else {
        // linear layer
        const Unit u = unit_of(a, type, layer, blockIdx.x);
        if (u.active) {
          if (e == 0) stage_issue(s, xs, u.amap, u.kb0, u.sbox, a.rb);
          float xr[XR];  // residual inputs of the rows this thread finishes
          if (type == P_OPROJ) load_resid(a, u, a.x0, e, xr);
          else if (type == P_PROJ) load_resid(a, u, a.x1, e, xr);
          mbar_wait(s.x_bar, xph & 1, s.abort_flag, a.status);
          xph++;
          // the row factors of a normed input (QKV, MLP fc, lm_head)
          if (type == P_QKV || type == P_FC || type == P_HEAD) smem_inv(a, s, xs, u.nkb, cw, lane, e);
          if (e == 0) trace_mark(a, p, 1);
          if (ok && type == P_HEAD) {
            ArgMax best[4];
#pragma unroll
            for (int i = 0; i < 4; i++) best[i] = ArgMax{-INFINITY, 0x7fffffff};
            if (MT == 2) head_rows<2>(a, s, ring, xs, u, t, cw, lane, best);
            else head_rows<1>(a, s, ring, xs, u, t, cw, lane, best);
            if (e == 0) trace_mark(a, p, 2);
            // this CTA's winner per sequence: over the 4 lanes of a row group,
            // then over the warps
#pragma unroll
            for (int i = 0; i < 4; i++) {
              ArgMax o1{__shfl_xor_sync(0xffffffffu, best[i].v, 1), __shfl_xor_sync(0xffffffffu, best[i].i, 1)};
              best[i] = argmax_merge(best[i], o1);
              ArgMax o2{__shfl_xor_sync(0xffffffffu, best[i].v, 2), __shfl_xor_sync(0xffffffffu, best[i].i, 2)};
              best[i] = argmax_merge(best[i], o2);
            }
            csync();  // every warp is done with the staged rows: red may overlay them
            if ((lane & 3) == 0) {
              const int g = lane >> 2;
#pragma unroll
              for (int i = 0; i < 4; i++) {
                const int b = (i >> 1) * 16 + g + 8 * (i & 1);
                red[(cw * 32 + b) * 2] = best[i].v;
                reinterpret_cast<int *>(red)[(cw * 32 + b) * 2 + 1] = best[i].i;
              }
            }
            csync();
            if (e < 32) {
              ArgMax r{red[e * 2], reinterpret_cast<int *>(red)[e * 2 + 1]};
              for (int w = 1; w < NCW; w++)
                r = argmax_merge(r, ArgMax{red[(w * 32 + e) * 2], reinterpret_cast<int *>(red)[(w * 32 + e) * 2 + 1]});
              a.cand_v[(size_t)blockIdx.x * 32 + e] = r.v;
              a.cand_i[(size_t)blockIdx.x * 32 + e] = r.i;
            }
          } else if (ok) {
            ok = MT == 2 ? gemv_mt<2>(a, s, ring, xs, u, t, red, cw, lane) : gemv_mt<1>(a, s, ring, xs, u, t, red, cw, lane);
            if (e == 0) trace_mark(a, p, 2);
            if (ok) {
              float *sum = reduce_warps(red, u.R, MT, e);  // [32][R]
              if (e == 0) trace_mark(a, p, 3);
              if (type == P_QKV) {
                qkv_epilogue(a, s, sum, u, layer, e);
              } else if (type == P_OPROJ) {
                resid_epilogue(a, sum, u, xr, a.x1, a.xb1, e);
              } else if (type == P_FC) {
                for (int idx = e; idx < a.B * u.R; idx += 32 * NCW) {
                  const int b = idx / u.R, r = idx % u.R, col = u.r0 + r;
                  if (col < u.N) {
                    const float v = fmaxf(sum[idx] * s.inv[b], 0.f);
                    a.f[(size_t)b * a.F + col] = __float2bfloat16_rn(v * v);
                  }
                }
              } else {  // P_PROJ: publish this split, the last of the splits finishes the rows
                float *part = a.ppart + ((size_t)u.u * a.s_p + u.split) * MAXB * u.R;
                for (int idx = e; idx < a.B * u.R; idx += 32 * NCW) part[idx] = sum[idx];
                csync();
                if (e == 0) {
                  unsigned old;
                  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                               : "=r"(old)
                               : "l"(a.pcnt + u.u)
                               : "memory");
                  *s.flag = old == (unsigned)((layer + 1) * a.s_p - 1) ? 1 : 0;
                }
                csync();
                if (*s.flag) {
                  // every split's partial in one bulk copy, into the warp
                  // partials' space (free now), then added in split order
                  float *all = red;  // [s_p][32][R]
                  const uint32_t bytes = (uint32_t)(a.s_p * MAXB * u.R * 4);
                  if (e == 0) {
                    asm volatile("fence.proxy.async.global;" ::: "memory");
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    mbar_arrive_expect_tx(s.x_bar, bytes);
                    bulk_copy(all, a.ppart + (size_t)u.u * a.s_p * MAXB * u.R, bytes, s.x_bar);
                  }
                  mbar_wait(s.x_bar, xph & 1, s.abort_flag, a.status);
                  xph++;
                  for (int idx = e; idx < a.B * u.R; idx += 32 * NCW) {
                    float v = 0.f;
                    for (int q = 0; q < a.s_p; q++) v += all[(size_t)q * MAXB * u.R + idx];
                    sum[idx] = v;
                  }
                  csync();
                  resid_epilogue(a, sum, u, xr, a.x0, a.xb0, e);
                }
                csync();  // s.flag is rewritten by the next use
              }
            }
          }
        }
      }
      if (e == 0) trace_mark(a, p, 4);
      if (ok && p + 1 < P) ok = grid_sync(a, s.abort_flag, e, p);
    }
  }
  __syncthreads();
}

int round8(int v) { return (v + 7) / 8 * 8; }

}  // namespace

bool make_map_bf16(CUtensorMap *map, const void *ptr, int rank, const uint64_t *dims, const uint64_t *strides,
                   const uint32_t *box);

bool decode_step_plan(const nc_config &c, int num_sms, StepPlan *pl) {
  *pl = StepPlan{};
  if (!decode_step_supported(c, 1) || num_sms < 8) return false;
  const int d = c.d_model, F = c.mlp_hidden, V = c.vocab, H = c.n_head, Hkv = c.n_kv_head, Gq = H / Hkv;
  const int G = num_sms;
  StepPlan p;
  p.grid = G;
  // QKV units: 8, 16 or 32 RoPE pairs of one head, the smallest that fits the grid
  for (p.r_q = 16; p.r_q <= 64 && (H + 2 * Hkv) * (128 / p.r_q) > G; p.r_q *= 2) {
  }
  if (p.r_q > 64) return false;
  p.n_qkv = (H + 2 * Hkv) * (128 / p.r_q);
  p.r_o = round8((d + G - 1) / G);
  p.r_f = round8((F + G - 1) / G);
  p.s_p = (F + d - 1) / d;  // K splits of the MLP projection: K per split <= d
  const int sp_units = G / p.s_p;
  p.r_p = round8((d + sp_units - 1) / sp_units);
  p.r_h = ((V + G - 1) / G + HG - 1) / HG * HG;
  p.n_o = (d + p.r_o - 1) / p.r_o;
  p.n_f = (F + p.r_f - 1) / p.r_f;
  p.n_p = (d + p.r_p - 1) / p.r_p;
  p.n_h = (V + p.r_h - 1) / p.r_h;
  if (p.n_qkv > G || p.r_o > MAX_R || p.r_f > MAX_R || p.r_p > MAX_R || p.n_p * p.s_p > G || p.n_p > 256 ||
      p.n_o > G || p.n_f > G || p.n_h > G || p.s_p > NCW)
    return false;
  // the attention merge stages every split's G state rows in the activation region
  if (MAX_SPLIT * Gq * AROW * 4 > xreg_bytes(d)) return false;
  // the projection's K per split must fit the staged rows like the others
  const int kbt = F / 64, kbs = (kbt + p.s_p - 1) / p.s_p;
  if (kbs * 64 > d) return false;
  const int xreg = (xreg_bytes(d) + 1023) & ~1023;
  const int fixed = 1024 /*alignment*/ + xreg + MISC;
  p.slots = (SMEM_CAP - fixed) / SLOT;
  if (p.slots > 10) p.slots = 10;
  if (p.slots < 3) return false;
  p.smem = (size_t)fixed + (size_t)p.slots * SLOT;
  // workspace layout
  auto take = [&](size_t bytes) {
    const size_t off = p.ws_bytes;
    p.ws_bytes += (bytes + 255) & ~(size_t)255;
    return off;
  };
  p.ws_bytes = 0;
  p.off_ctr = take(CTR_BYTES);
  p.off_x0 = take(sizeof(float) * MAXB * d);
  p.off_x1 = take(sizeof(float) * MAXB * d);
  p.off_xb0 = take(2 * MAXB * d);
  p.off_xb1 = take(2 * MAXB * d);
  p.off_y = take(2 * MAXB * d);
  p.off_f = take(2 * MAXB * (size_t)F);
  p.off_qk = take(sizeof(float) * MAXB * (H + Hkv) * 128);
  p.off_cv = take(sizeof(float) * (size_t)G * 32);
  p.off_ci = take(sizeof(int) * (size_t)G * 32);
  p.off_ap = take(sizeof(float) * MAXB * Hkv * MAX_SPLIT * Gq * AROW);
  p.off_pp = take(sizeof(float) * (size_t)p.n_p * p.s_p * MAXB * p.r_p);
  *pl = p;
  return true;
}

// bf16, head_dim 128, G = H / Hkv <= 16 query heads per KV head (the rows of
// one attention unit's MMAs), H * 128 = d, at most 32 sequences
bool decode_step_supported(const nc_config &c, int B) {
  return decode_head_supported(c) && c.n_head % c.n_kv_head == 0 && c.n_head / c.n_kv_head <= 16 &&
         c.n_kv_head <= MAX_HKV && c.n_head * 128 == c.d_model && c.mlp_hidden % 64 == 0 && c.vocab % 8 == 0 &&
         B >= 1 && B <= MAXB;
}

int decode_step_maps_count(const nc_config &c) { return 4 * c.depth + 1 + 4 + 8; }

int decode_step_prefix_map_index(const nc_config &c) { return 4 * c.depth + 3; }

namespace {
// [rows, K] bf16 weights (row pitch K) as (64 columns, rows, K / 64 k-blocks):
// a box of (64, box_rows, box_kb) lands as [kb][row][128 B]
bool weight_map(CUtensorMap *m, const void *w, int rows, int K, int box_rows, int box_kb) {
  const uint64_t dims[3] = {64, (uint64_t)rows, (uint64_t)(K / 64)};
  const uint64_t strides[2] = {(uint64_t)K * 2, 128};
  const uint32_t box[3] = {64, (uint32_t)box_rows, (uint32_t)box_kb};
  return make_map_bf16(m, w, 3, dims, strides, box);
}

// the K or V cache, [rows][Hkv][128] bf16, as (64 dims, rows, 2 halves, Hkv
// heads): a box of (64, 64 keys, 2, 1) lands as [half][key][128 B]
bool cache_map(CUtensorMap *m, const void *cache, int rows, int Hkv) {
  const uint64_t dims[4] = {64, (uint64_t)rows, 2, (uint64_t)Hkv};
  const uint64_t strides[3] = {(uint64_t)Hkv * 256, 128, 256};
  const uint32_t box[4] = {64, (uint32_t)KT, 2, 1};
  return make_map_bf16(m, cache, 4, dims, strides, box);
}
}  // namespace

// The two maps through which the step kernel reads shared-prefix rows: the
// prefix cache's K and V viewed as [depth * max_batch * max_seq, Hkv, 128].
bool decode_step_prefix_maps(const void *kcache, const void *vcache, const nc_config &c, int max_batch, int max_seq,
                             CUtensorMap *out) {
  const int rows = c.depth * max_batch * max_seq;
  return cache_map(&out[0], kcache, rows, c.n_kv_head) && cache_map(&out[1], vcache, rows, c.n_kv_head);
}

// Tensor maps of the step kernel, written to host memory `out` (to be copied
// to the device): per layer the QKV weights as (64 columns, rows, 2 RoPE
// halves 64 rows apart, k-blocks) so that a unit's r_q/2 + r_q/2 paired rows
// arrive in one copy, then the O, fc, proj weights (boxes of the unit's rows and a
// slot's k-blocks), the lm_head (64 rows x HKB k-blocks); the K and V caches
// (this cache, then the prefix cache, initially this one); the activations
// the linear phases stage (bf16(x0), y, bf16(x1), f) as (64 columns, 32 rows,
// k-blocks) with a box of the phase's k-blocks and 32 rows, then the same
// four with boxes of 16 rows (batches of up to 16).
bool decode_step_build_maps(const nc_model *m, const void *kcache, const void *vcache, int max_batch, int max_seq,
                            const StepPlan &p, void *ws, CUtensorMap *out) {
  const nc_config &c = m->cfg;
  const int d = c.d_model, F = c.mlp_hidden, H = c.n_head, Hkv = c.n_kv_head;
  for (int l = 0; l < c.depth; l++) {
    const nc_layer_w &w = m->layers[l];
    {
      const uint64_t dims[4] = {64, (uint64_t)((H + 2 * Hkv) * 128 - 64), 2, (uint64_t)(d / 64)};
      const uint64_t strides[3] = {(uint64_t)d * 2, (uint64_t)64 * d * 2, 128};
      const uint32_t box[4] = {64, (uint32_t)(p.r_q / 2), 2, (uint32_t)kps_of(p.r_q)};
      if (!make_map_bf16(&out[4 * l + 0], w.wqkv, 4, dims, strides, box)) return false;
    }
    if (!weight_map(&out[4 * l + 1], w.wo, d, H * 128, p.r_o, kps_of(p.r_o))) return false;
    if (!weight_map(&out[4 * l + 2], w.wfc, F, d, p.r_f, kps_of(p.r_f))) return false;
    if (!weight_map(&out[4 * l + 3], w.wproj, d, F, p.r_p, kps_of(p.r_p))) return false;
  }
  if (!weight_map(&out[4 * c.depth], m->wlm, c.vocab, d, HG, HKB)) return false;
  const int rows = c.depth * max_batch * max_seq;
  if (!cache_map(&out[4 * c.depth + 1], kcache, rows, Hkv) || !cache_map(&out[4 * c.depth + 2], vcache, rows, Hkv))
    return false;
  // no shared prefixes yet: the prefix maps view this cache
  out[4 * c.depth + 3] = out[4 * c.depth + 1];
  out[4 * c.depth + 4] = out[4 * c.depth + 2];
  uint8_t *base = static_cast<uint8_t *>(ws);
  CUtensorMap *am = out + 4 * c.depth + 5;
  auto act_map = [&](CUtensorMap *mp, size_t off, int K, int box_kb, int rows) {
    const uint64_t dims[3] = {64, (uint64_t)MAXB, (uint64_t)(K / 64)};
    const uint64_t strides[2] = {(uint64_t)K * 2, 128};
    const uint32_t box[3] = {64, (uint32_t)rows, (uint32_t)box_kb};
    return make_map_bf16(mp, base + off, 3, dims, strides, box);
  };
  const int kbs = (F / 64 + p.s_p - 1) / p.s_p;
  // boxes of 32 rows (any batch), then of 16 rows (batches of up to 16)
  for (int h = 0; h < 2; h++) {
    const int rows = h ? 16 : MAXB;
    CUtensorMap *m4 = am + 4 * h;
    if (!act_map(&m4[0], p.off_xb0, d, d / 64, rows) || !act_map(&m4[1], p.off_y, d, d / 64, rows) ||
        !act_map(&m4[2], p.off_xb1, d, d / 64, rows) || !act_map(&m4[3], p.off_f, F, kbs, rows))
      return false;
  }
  return true;
}

// CTAs of the step kernel: one per SM, all co-resident (cooperative launch);
// 0 if the kernel cannot be placed that way.
int decode_step_grid(const StepPlan &p, int num_sms) {
  if (ensure_smem_attr((const void *)decode_step_kernel, p.smem) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_step_kernel, THREADS, p.smem) != cudaSuccess ||
      per_sm < 1) {
    cudaGetLastError();
    return 0;
  }
  return p.grid <= num_sms ? p.grid : 0;
}

cudaError_t k_decode_step(const nc_model *m, const StepPlan &pl, int B, int max_batch, int max_seq,
                          const CUtensorMap *maps_dev, void *ws, const int32_t *tokens, const int32_t *positions,
                          int32_t *len, void *kc, void *vc, const float2 *rope, float *logits, const float *noise,
                          int32_t *next, unsigned long long *trace, uint8_t *valid_out, const int32_t *pre_seq,
                          const int32_t *pre_len, int pmax_batch, int pmax_seq, cudaStream_t s) {
  const nc_config &c = m->cfg;
  uint8_t *base = static_cast<uint8_t *>(ws);
  StepArgs a;
  a.L = c.depth;
  a.d = c.d_model;
  a.H = c.n_head;
  a.Hkv = c.n_kv_head;
  a.G = c.n_head / c.n_kv_head;
  a.r_q = pl.r_q;
  a.F = c.mlp_hidden;
  a.V = c.vocab;
  a.B = B;
  a.max_batch = max_batch;
  a.max_seq = max_seq;
  a.grid = pl.grid;
  a.r_o = pl.r_o;
  a.r_f = pl.r_f;
  a.r_p = pl.r_p;
  a.s_p = pl.s_p;
  a.r_h = pl.r_h;
  a.n_o = pl.n_o;
  a.n_f = pl.n_f;
  a.n_p = pl.n_p;
  a.n_h = pl.n_h;
  a.n_qkv = pl.n_qkv;
  a.slots = pl.slots;
  {
    // key splits per (sequence, KV head): the units (pair, split) are dealt
    // to the CTAs in rounds, so a CTA streams ceil(units / grid) splits of
    // 1/s of a pair's keys and pays a unit's fixed cost (QK norm, merges:
    // measured at about a third of streaming a whole 2048-key pair) per
    // round. B = 32 with one KV head: 4 splits in one round; with ten KV
    // heads: one split, 3 rounds
    const int pairs = B * c.n_kv_head;
    int best = 1;
    double best_cost = 1e30;
    for (int sp = 1; sp <= MAX_SPLIT; sp++) {
      const int rounds = (pairs * sp + pl.grid - 1) / pl.grid;
      const double cost = (double)rounds / sp + 0.35 * rounds;
      if (cost < best_cost - 1e-9) {
        best_cost = cost;
        best = sp;
      }
    }
    a.splits = best;
    // more units than CTAs: deal the key tiles evenly instead (the kernel
    // falls back to the rounds when the deal does not fit its tables);
    // NC_DECODE_TILE_DEAL=0 keeps the rounds
    static const bool deal_on = [] {
      const char *env = getenv("NC_DECODE_TILE_DEAL");
      return !(env && atoi(env) == 0);
    }();
    a.stream = deal_on && pairs > pl.grid ? 1 : 0;
  }
  a.eps = c.norm_eps;
  a.cap = c.softcap;
  a.scale_log2 = 1.4426950408889634f / sqrtf(128.f);
  a.wte = (const bf16 *)m->wte;
  a.wmaps = maps_dev;
  a.kvmaps = maps_dev + 4 * c.depth + 1;
  a.rb = B <= 16 ? 16 : MAXB;
  a.amaps = maps_dev + 4 * c.depth + 5 + (B <= 16 ? 4 : 0);
  a.pre_seq = pre_seq;
  a.pre_len = pre_len;
  a.pmax_batch = pmax_batch;
  a.pmax_seq = pmax_seq;
  a.tokens = tokens;
  a.positions = positions;
  a.len = len;
  a.x0 = reinterpret_cast<float *>(base + pl.off_x0);
  a.x1 = reinterpret_cast<float *>(base + pl.off_x1);
  a.xb0 = reinterpret_cast<bf16 *>(base + pl.off_xb0);
  a.xb1 = reinterpret_cast<bf16 *>(base + pl.off_xb1);
  a.y = reinterpret_cast<bf16 *>(base + pl.off_y);
  a.f = reinterpret_cast<bf16 *>(base + pl.off_f);
  a.qk = reinterpret_cast<float *>(base + pl.off_qk);
  a.kc = (bf16 *)kc;
  a.vc = (bf16 *)vc;
  a.rope = rope;
  a.logits = logits;
  a.noise = noise;
  a.next = next;
  a.cand_v = reinterpret_cast<float *>(base + pl.off_cv);
  a.cand_i = reinterpret_cast<int *>(base + pl.off_ci);
  a.apart = reinterpret_cast<float *>(base + pl.off_ap);
  a.ppart = reinterpret_cast<float *>(base + pl.off_pp);
  a.bar = reinterpret_cast<unsigned long long *>(base + pl.off_ctr);
  a.acnt = reinterpret_cast<unsigned *>(base + pl.off_ctr + 64);
  a.pcnt = reinterpret_cast<unsigned *>(base + pl.off_ctr + 64 + 4 * MAXB * MAX_HKV);
  a.status = m->status;
  a.trace = trace;
  a.valid_out = valid_out;
  // grid-barrier and arrival counters from zero for every step
  cudaError_t e = cudaMemsetAsync(base + pl.off_ctr, 0, CTR_BYTES, s);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.grid);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  count_launch();
  return cudaLaunchKernelEx(&cfg, decode_step_kernel, a);
}

}  // namespace nc
