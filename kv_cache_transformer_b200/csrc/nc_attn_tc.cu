// nc_attn_tc.cu — causal multi-query / grouped-query prefill attention on
// tcgen05.
//
// The H query heads form Hkv groups of G = H/Hkv heads, and the G heads of a
// group read the same keys and values (one KV head: the feature list's
// multi-query attention, Hkv = 1; multi-head attention, G = 1). For one
// sequence and KV head j, the queries of group j at positions 0..T-1 are one
// [T*G, hd] matrix whose row r = t*G + g is head j*G + g at position t. A
// work item is 256 consecutive rows of one (sequence, KV head), two 128-row Q
// tiles (A and B) that share every K/V tile:
//   S_t  = Q_t K_j^T       (tcgen05, M=128 rows, N=128 keys, K=hd) -> TMEM
//   P_t  = 2^(S_t*scale*log2e - m) with the causal mask key <= t(row), online
//          max/sum, bf16 pairs written back into the upper half of S_t's
//          TMEM columns
//   O_t += P_t V_j         (tcgen05 with A read from TMEM, B = V read
//                           MN-major straight from the cache layout) -> TMEM
// and finally y = O_t / l in bf16. For a chunk appended to sequences that
// already hold off[b] tokens, query t sits at position off[b] + t and its
// keys are the cached rows 0 .. off[b] + t.
// Warp roles (320 threads): warp 0 TMA (one thread: the Q tiles of each item,
// then K_j and V_j alternately through a 4-slot ring), warp 1 TMEM
// allocator + MMA issuer, warps 2-5 softmax of tile A and warps 6-9 of tile B,
// one thread per row. Per key tile the MMA issuer runs PV_A(j), S_A(j+1),
// PV_B(j), S_B(j+1): while one warpgroup exponentiates, the tensor core works
// for the other. S_t(j+1) overwrites the TMEM columns PV_t(j) reads P from;
// tcgen05.mma operations of one CTA run in issue order, so it is issued right
// after PV_t(j) with no wait in between. PV_t(j) goes in two halves: the
// first 64 keys as soon as the softmax threads have stored their P, while
// they exponentiate the other 64. O is rescaled only when a row's
// running max grows by more than 2^8 (the probabilities of a tile are then at
// most 256, exact in fp32 and bf16). Items are ordered heaviest first and dealt
// to the CTAs in zig-zag rounds, which evens out the causal work per CTA.
// Every wait is bounded as in the GEMM.
#include "nc_internal.h"
#include "nc_sm100.cuh"

namespace nc {
using namespace sm100;

bool make_map_bf16_k64(CUtensorMap *map, const void *ptr, int rows, int cols, int ld, int box_rows);

namespace {

constexpr int HD = 128;            // head dim handled here
constexpr int BR = 128;            // rows (position, head) per Q tile
constexpr int ITEM = 2 * BR;       // rows per work item: Q tiles A and B
constexpr int BKV = 128;           // keys per K/V tile
constexpr int NSLOT = 4;           // K/V ring slots (K_j and V_j alternate)
constexpr int SUB = 128 * 64 * 2;  // one 128-row x 64-column swizzled box: 16 KB
constexpr int TILE = 2 * SUB;      // 128 x 128 bf16: 32 KB
constexpr int OFF_Q = 0;           // Q_A, Q_B
constexpr int OFF_KV = 2 * TILE;   // NSLOT tiles
constexpr int OFF_BAR = OFF_KV + NSLOT * TILE;
constexpr int SMEM_USED = OFF_BAR + 256;
constexpr int SMEM_BYTES = SMEM_USED + 1024;  // slack for 1024-byte alignment
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
constexpr float RESCALE_LOG2 = 8.0f;         // rescale O when the max grows by more than 2^8
constexpr int THREADS = 320;
// TMEM columns: S of tile t at 128t (P of tile t at 128t + 64, bf16 pairs),
// O of tile t at 256 + 128t
constexpr uint32_t TMEM_COLS = 512;

struct AttnArgs {
  int T, H, B, max_seq;
  int Hkv, G;        // KV heads, query heads per KV head
  int rows_per_seq;  // T*G rows of one (sequence, KV head)
  const int32_t *off;  // [B] position of row t = 0 of each sequence (appended chunks), or null
  float scale_log2;  // log2(e) / sqrt(hd)
  bf16 *y;           // [B*T*H, 128]
  uint32_t *status;
};

// Shared-memory descriptors split into 32-bit words: the low word holds the
// start address (>> 4) and the leading byte offset, the high word the stride
// byte offset, version and swizzle mode, the same for every tile here, so an
// MMA's operands cost one add each (the MMA warp shares its issue slots with
// two softmax warps).
constexpr uint32_t DESC_HI = (1024u >> 4) | (1u << 14) | (2u << 29);  // bits 32..63
__device__ __forceinline__ uint32_t desc_lo_k(uint32_t smem_addr) { return ((smem_addr >> 4) & 0x3FFF) | (1u << 16); }
__device__ __forceinline__ uint32_t desc_lo_mn(uint32_t smem_addr) {
  return ((smem_addr >> 4) & 0x3FFF) | ((uint32_t)(SUB >> 4) << 16);
}

// D (TMEM) (+)= A (shared) * B (shared), descriptors given as low words
__device__ __forceinline__ void mma_ss(uint32_t tmem_d, uint32_t alo, uint32_t blo, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n .reg .b64 da, db;\n setp.ne.b32 p, %4, 0;\n mov.b64 da, {%1, %5};\n"
      " mov.b64 db, {%2, %5};\n tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, p;\n}" ::"r"(tmem_d),
      "r"(alo), "r"(blo), "r"(idesc), "r"(accumulate), "n"(DESC_HI)
      : "memory");
}

// D (TMEM) (+)= A (TMEM, bf16 pairs per 32-bit column, K-major) * B (shared)
__device__ __forceinline__ void mma_ts(uint32_t tmem_d, uint32_t tmem_a, uint32_t blo, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n .reg .b64 db;\n setp.ne.b32 p, %4, 0;\n mov.b64 db, {%2, %5};\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %3, p;\n}" ::"r"(tmem_d),
      "r"(tmem_a), "r"(blo), "r"(idesc), "r"(accumulate), "n"(DESC_HI)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),
      "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
      "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 2^x (PTX ex2.approx.ftz: relative error ~2^-22, 2^-inf = 0)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// max(a, b, c) in one instruction (sm_100)
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

// round r of the zig-zag deal of items to G CTAs: CTA c takes item
// r*G + c in even rounds and r*G + G-1-c in odd ones
__device__ __forceinline__ int item_at(int r, int c, int G) { return r * G + ((r & 1) ? G - 1 - c : c); }

__global__ void __launch_bounds__(THREADS, 1)
    attn_prefill_tc_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                           const __grid_constant__ CUtensorMap mapV, AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint32_t raw = smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw + 1023) & ~1023u) - raw);
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  uint64_t *q_full = bar;               // 1
  uint64_t *q_empty = bar + 1;          // 1: Q tiles free once the item's last S is done
  uint64_t *kv_full = bar + 2;          // NSLOT
  uint64_t *kv_empty = kv_full + NSLOT; // NSLOT
  uint64_t *s_full = kv_empty + NSLOT;  // 2, per Q tile
  uint64_t *p_full = s_full + 2;        // 2 (128 arrivals)
  uint64_t *o_done = p_full + 2;        // 2: every P V of the tile so far is done
  uint64_t *o_free = o_done + 2;        // 2 (128 arrivals): the item's O has been read
  uint64_t *p_half = o_free + 2;        // 2 (128 arrivals): P of the tile's first 64 keys is in TMEM
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(p_half + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_pairs = (a.rows_per_seq + ITEM - 1) / ITEM;
  const int nvs = a.B * a.Hkv;  // (sequence, KV head) pairs
  const int n_items = n_pairs * nvs;
  const int G = gridDim.x, c = blockIdx.x;

  // item i: rows 256*pp .. of sequence b and KV head j, pp heaviest first;
  // n_kv key tiles, of which Q tile A needs the first n_kv_a (one fewer when
  // its last position ends a key tile earlier than tile B's, as with one
  // query head per KV head)
  auto item_of = [&](int i, int &b, int &j, int &row0, int &n_kv, int &n_kv_a) {
    const int pp = n_pairs - 1 - i / nvs;
    b = (i % nvs) / a.Hkv;
    j = i % a.Hkv;
    row0 = pp * ITEM;
    const int off = a.off ? a.off[b] : 0;
    const int last = min(row0 + ITEM, a.rows_per_seq) - 1, last_a = min(row0 + BR, a.rows_per_seq) - 1;
    n_kv = (off + last / a.G) / BKV + 1;
    n_kv_a = (off + last_a / a.G) / BKV + 1;
  };

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < NSLOT; s++) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int t = 0; t < 2; t++) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
      mbar_init(&o_done[t], 1);
      mbar_init(&o_free[t], 128);
      mbar_init(&p_half[t], 128);
    }
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&mapQ);
    tma_prefetch_desc(&mapK);
    tma_prefetch_desc(&mapV);
  }
  if (warp == 1) tmem_alloc(tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // one thread issues every load in consumption order: the item's Q tiles
    // (once its predecessor's last S is done), then K_j, V_j, K_{j+1}, ...
    // through the ring (a second lane with its own waits would share this
    // warp's issue slot and stall behind the first)
    if (lane == 0) {
      uint32_t n = 0;
      bool ok = true;
      for (int r = 0, it = 0; ok; r++, it++) {
        const int i = item_at(r, c, G);
        if (i >= n_items) break;
        int b, j, row0, n_kv, n_kv_a;
        item_of(i, b, j, row0, n_kv, n_kv_a);
        if (!mbar_wait(q_empty, (it & 1) ^ 1, abort_flag, a.status)) break;
        mbar_arrive_expect_tx(q_full, 2 * TILE);
        // Q map (128 dims, G heads, Hkv groups, rows): with one KV head the
        // rows are (position, head) pairs, else positions with G heads each
        const int qz = a.Hkv == 1 ? 0 : j;
        const int qw = a.Hkv == 1 ? b * a.rows_per_seq + row0 : b * a.T + row0 / a.G;
        const int qstep = a.Hkv == 1 ? BR : BR / a.G;
        tma_load_4d(smem + OFF_Q, &mapQ, 0, 0, qz, qw, q_full);
        tma_load_4d(smem + OFF_Q + SUB, &mapQ, 64, 0, qz, qw, q_full);
        tma_load_4d(smem + OFF_Q + TILE, &mapQ, 0, 0, qz, qw + qstep, q_full);
        tma_load_4d(smem + OFF_Q + TILE + SUB, &mapQ, 64, 0, qz, qw + qstep, q_full);
        const int krow = b * a.max_seq, kx = j * HD;
        for (int kt = 0; kt < n_kv && ok; kt++)
          for (int w = 0; w < 2; w++, n++) {
            const int s = n % NSLOT;
            if (!mbar_wait(&kv_empty[s], ((n / NSLOT) & 1) ^ 1, abort_flag, a.status)) { ok = false; break; }
            mbar_arrive_expect_tx(&kv_full[s], TILE);
            const CUtensorMap *map = w ? &mapV : &mapK;
            tma_load_2d(smem + OFF_KV + s * TILE, map, kx, krow + kt * BKV, &kv_full[s]);
            tma_load_2d(smem + OFF_KV + s * TILE + SUB, map, kx + 64, krow + kt * BKV, &kv_full[s]);
          }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16_f32(BR, BKV);
      const uint32_t id_o = idesc_bf16_f32(BR, HD) | (1u << 16);  // B (V) is MN-major
      const uint32_t qlo = desc_lo_k(smem_u32(smem + OFF_Q));
      uint32_t n = 0;          // K/V ring position
      int gt[2] = {0, 0};      // key tiles of each Q tile done so far, over all items
      bool ok = true;
      auto take = [&](uint32_t &addr, int &slot) -> bool {
        slot = n % NSLOT;
        if (!mbar_wait(&kv_full[slot], (n / NSLOT) & 1, abort_flag, a.status)) return false;
        n++;
        addr = smem_u32(smem + OFF_KV + slot * TILE);
        tc_fence_after();
        return true;
      };
      auto issue_s = [&](int t, uint32_t k0) {  // S_t = Q_t K^T
        const uint32_t qa = qlo + ((t * TILE) >> 4), kb = desc_lo_k(k0);
#pragma unroll
        for (int k = 0; k < HD / 16; k++) {
          const uint32_t off = ((k >> 2) * SUB + (k & 3) * 32) >> 4;
          mma_ss(tmem + t * 128, qa + off, kb + off, id_s, k != 0);
        }
        mma_commit(&s_full[t]);
      };
      for (int r = 0, it = 0; ok; r++, it++) {
        const int i = item_at(r, c, G);
        if (i >= n_items) break;
        int b, j_kv, row0, n_kv, n_kv_a;
        item_of(i, b, j_kv, row0, n_kv, n_kv_a);
        const int nkt[2] = {n_kv_a, n_kv};
        if (!mbar_wait(q_full, it & 1, abort_flag, a.status)) break;
        uint32_t kaddr, vaddr;
        int kslot, vslot;
        if (!take(kaddr, kslot)) break;
        issue_s(0, kaddr);
        issue_s(1, kaddr);
        mma_commit(&kv_empty[kslot]);
        if (n_kv == 1) mma_commit(q_empty);
        for (int j = 0; j < n_kv && ok; j++) {
          if (!take(vaddr, vslot)) { ok = false; break; }
          for (int t = 0; t < 2 && ok; t++) {
            if (j < nkt[t]) {  // key tile j reaches some row of Q tile t
              // P of keys 0..63 first: its MMAs run while the softmax
              // threads exponentiate keys 64..127
              if (!mbar_wait(&p_half[t], gt[t] & 1, abort_flag, a.status)) { ok = false; break; }
              // the epilogue of the previous item must have read O_t
              if (j == 0 && !mbar_wait(&o_free[t], (it & 1) ^ 1, abort_flag, a.status)) { ok = false; break; }
              tc_fence_after();
              const uint32_t pa = tmem + t * 128 + 64, vb = desc_lo_mn(vaddr);
#pragma unroll
              for (int k = 0; k < BKV / 32; k++)
                mma_ts(tmem + 256 + t * 128, pa + k * 8, vb + ((k * 2048) >> 4), id_o, (j | k) != 0);
              if (!mbar_wait(&p_full[t], gt[t] & 1, abort_flag, a.status)) { ok = false; break; }
              gt[t]++;
              tc_fence_after();
#pragma unroll
              for (int k = BKV / 32; k < BKV / 16; k++)
                mma_ts(tmem + 256 + t * 128, pa + k * 8, vb + ((k * 2048) >> 4), id_o, 1);
              mma_commit(&o_done[t]);
            }
            if (t == 1) mma_commit(&kv_empty[vslot]);
            if (j + 1 < n_kv) {
              if (t == 0 && !take(kaddr, kslot)) { ok = false; break; }
              if (j + 1 < nkt[t]) issue_s(t, kaddr);
              if (t == 1) {
                mma_commit(&kv_empty[kslot]);
                if (j + 2 == n_kv) mma_commit(q_empty);  // the item's last S
              }
            }
          }
        }
      }
    }
  } else {
    // softmax of Q tile t, one thread per row; then the item's epilogue
    const int t = (warp - 2) >> 2;
    const int quarter = warp & 3;  // this warp's TMEM lane quarter
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + t * 128 + lane_off, tO = tmem + 256 + t * 128 + lane_off;
    bool ok = true;
    int g = 0;
    for (int rr = 0;; rr++) {
      const int i = item_at(rr, c, G);
      if (i >= n_items) break;
      int b, j_kv, row0, n_kv, n_kv_a;
      item_of(i, b, j_kv, row0, n_kv, n_kv_a);
      const int nk = t == 0 ? n_kv_a : n_kv;  // key tiles this Q tile takes
      const int row = row0 + t * BR + r;  // row inside the (sequence, KV head)
      const int t_loc = row < a.rows_per_seq ? row / a.G : 0;  // its query among the T
      // its position: the causal limit of its keys
      const int t_row = row < a.rows_per_seq ? (a.off ? a.off[b] : 0) + t_loc : 0x3fffffff;
      float m = -INFINITY, l = 0.f;  // running max (scaled, log2 units) and sum
      for (int j = 0; j < nk; j++, g++) {
        ok = ok && mbar_wait(&s_full[t], g & 1, abort_flag, a.status);
        tc_fence_after();
        // the tile's 128 raw scores of this row, read from TMEM once; the
        // causal mask only matters on a tile that reaches past the row's
        // position (masked scores become -inf)
        const int kbase = j * BKV;
        const bool masked = kbase + BKV - 1 > t_row;
        uint32_t v[BKV];
        tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(v));
        tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
        tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(v + 64));
        tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(v + 96));
        tmem_ld_wait();
        if (masked) {  // a tile on the diagonal
#pragma unroll
          for (int q = 0; q < BKV; q++)
            if (kbase + q > t_row) v[q] = __float_as_uint(-INFINITY);
        }
        // row max (the scale is positive)
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int q = 0; q < BKV; q += 8) {
          mx[0] = max3(mx[0], __uint_as_float(v[q]), __uint_as_float(v[q + 1]));
          mx[1] = max3(mx[1], __uint_as_float(v[q + 2]), __uint_as_float(v[q + 3]));
          mx[2] = max3(mx[2], __uint_as_float(v[q + 4]), __uint_as_float(v[q + 5]));
          mx[3] = max3(mx[3], __uint_as_float(v[q + 6]), __uint_as_float(v[q + 7]));
        }
        const float tmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * a.scale_log2;
        const bool need = (m == -INFINITY) ? (tmax != -INFINITY) : (tmax > m + RESCALE_LOG2);
        const float m_new = need ? tmax : m;
        const float alpha = (need && m != -INFINITY) ? exp2f(m - m_new) : 1.f;
        if (j > 0 && __any_sync(0xffffffffu, need)) {
          // O must hold every earlier P V of this item before it is rescaled
          ok = ok && mbar_wait(&o_done[t], (g - 1) & 1, abort_flag, a.status);
          tc_fence_after();
#pragma unroll 1
          for (int cc = 0; cc < HD; cc += 32) {
            uint32_t o[32];
            tmem_ld32(tO + cc, o);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; q++) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
            tmem_st32(tO + cc, o);
          }
        }
        // p = 2^(s*scale - m), one FMA and one ex2 per score (masked scores
        // give 0), bf16 pairs into the P columns 64..127 of this S buffer
        // (keys 0..63 on columns 64..95, keys 64..127 on 96..127: every score
        // was read above)
        const float nm = -m_new;
        float sum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c8 = 0; c8 < BKV / 16; c8++) {  // 16 keys -> 8 columns of bf16 pairs
          uint32_t pk[8];
#pragma unroll
          for (int q = 0; q < 8; q++) {
            const float p0 = ex2(fmaf(__uint_as_float(v[c8 * 16 + 2 * q]), a.scale_log2, nm));
            const float p1 = ex2(fmaf(__uint_as_float(v[c8 * 16 + 2 * q + 1]), a.scale_log2, nm));
            sum[(2 * q) & 3] += p0;
            sum[(2 * q + 1) & 3] += p1;
            pk[q] = pack2(p0, p1);
          }
          tmem_st8(tS + 64 + c8 * 8, pk);
          if (c8 == BKV / 32 - 1) {  // keys 0..63 are in TMEM: their P V can start
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&p_half[t]);
          }
        }
        l = l * alpha + ((sum[0] + sum[1]) + (sum[2] + sum[3]));
        m = m_new;
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[t]);
      }
      // epilogue: y = O / l
      ok = ok && mbar_wait(&o_done[t], (g - 1) & 1, abort_flag, a.status);
      tc_fence_after();
      const float inv = 1.f / l;
      // y row of (position t_row, head j*G + g) in [B*T, H, 128]
      bf16 *dst = a.y + (((size_t)b * a.T + t_loc) * a.H + j_kv * a.G + row % a.G) * HD;
#pragma unroll 1
      for (int cc = 0; cc < HD; cc += 32) {
        uint32_t o[32];
        tmem_ld32(tO + cc, o);
        tmem_ld_wait();
        if (ok && row < a.rows_per_seq) {
          uint4 *d4 = reinterpret_cast<uint4 *>(dst + cc);
#pragma unroll
          for (int q = 0; q < 4; q++) {
            float f[8];
#pragma unroll
            for (int z = 0; z < 8; z++) f[z] = __uint_as_float(o[q * 8 + z]) * inv;
            d4[q] = make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]), pack2(f[6], f[7]));
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&o_free[t]);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

// A Q tile of 128 rows holds whole positions of one group unless there is a
// single KV head (then it holds (position, head) rows in order).
bool attn_prefill_tc_supported(int H, int Hkv, int hd) {
  return hd == HD && H >= 1 && Hkv >= 1 && H % Hkv == 0 && (Hkv == 1 || BR % (H / Hkv) == 0);
}

bool make_map_bf16(CUtensorMap *map, const void *ptr, int rank, const uint64_t *dims, const uint64_t *strides,
                   const uint32_t *box);

// q: [B*T, H, 128] bf16 (rotated + normed), kc/vc: layer cache
// [max_batch*max_seq, Hkv*128], y: [B*T, H, 128] bf16.
cudaError_t k_attn_prefill_tc(const void *q, const void *kc, const void *vc, int B, int T, int H, int Hkv,
                              int max_batch, int max_seq, void *y, uint32_t *status, cudaStream_t s,
                              const int32_t *off) {
  if (!attn_prefill_tc_supported(H, Hkv, HD)) return cudaErrorInvalidValue;
  CUtensorMap mq, mk, mv;
  const int G = H / Hkv, rows = T * G;
  bool ok;
  if (Hkv == 1) {  // rows (position, head) in order: (128 dims, 1, 1, B*T*H rows)
    const uint64_t dims[4] = {HD, 1, 1, (uint64_t)B * T * H};
    const uint64_t strides[3] = {HD * 2, HD * 2, HD * 2};
    const uint32_t box[4] = {64, 1, 1, BR};
    ok = make_map_bf16(&mq, q, 4, dims, strides, box);
  } else {  // (128 dims, G heads, Hkv groups, B*T positions), a box of 128/G positions
    const uint64_t dims[4] = {HD, (uint64_t)G, (uint64_t)Hkv, (uint64_t)B * T};
    const uint64_t strides[3] = {HD * 2, (uint64_t)G * HD * 2, (uint64_t)H * HD * 2};
    const uint32_t box[4] = {64, (uint32_t)G, 1, (uint32_t)(BR / G)};
    ok = make_map_bf16(&mq, q, 4, dims, strides, box);
  }
  if (!ok || !make_map_bf16_k64(&mk, kc, max_batch * max_seq, Hkv * HD, Hkv * HD, BKV) ||
      !make_map_bf16_k64(&mv, vc, max_batch * max_seq, Hkv * HD, Hkv * HD, BKV))
    return cudaErrorInvalidValue;
  {
    const cudaError_t e = ensure_smem_attr((const void *)attn_prefill_tc_kernel, SMEM_BYTES);
    if (e != cudaSuccess) return e;
  }
  AttnArgs a;
  a.T = T;
  a.H = H;
  a.B = B;
  a.max_seq = max_seq;
  a.Hkv = Hkv;
  a.G = G;
  a.rows_per_seq = rows;
  a.off = off;
  a.scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
  a.y = (bf16 *)y;
  a.status = status;
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  }
  const int items = ((rows + ITEM - 1) / ITEM) * B * Hkv;
  dim3 grid(items < sms ? items : sms);
  count_launch();
  attn_prefill_tc_kernel<<<grid, THREADS, SMEM_BYTES, s>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

}  // namespace nc
