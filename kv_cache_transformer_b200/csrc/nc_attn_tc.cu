// nc_attn_tc.cu — causal multi-query prefill attention on tcgen05.
//
// With one KV head, the H query heads of a position all read the same keys
// and values (the feature list's multi-query attention). The queries of a
// sequence, stored [T, H, hd], are therefore one [T*H, hd] matrix whose row
// r = t*H + h belongs to position t. A CTA takes 128 consecutive rows
// (about 128/H positions, every head) and streams the sequence's K/V tiles
// once for all of them:
//   S  = Q K^T          (tcgen05, M=128 rows, N=128 keys, K=hd=128) -> TMEM
//   P  = exp(S*scale - m) with the causal mask key <= t(row), online max/sum
//   O += P V            (tcgen05, A = P from shared memory, B = V read
//                        MN-major straight from the cache layout)  -> TMEM
// and finally y = O / l in bf16.
// Warp roles (192 threads): warp 0 TMA producer (Q once, K/V tiles through a
// 2-stage ring), warp 1 TMEM allocator + MMA issuer (S_{j+1} is issued before
// P_j is consumed), warps 2-5 softmax / O rescale / epilogue, one thread per
// row. P is double-buffered, so the softmax of tile j+1 overlaps P_j V_j, and
// O is rescaled only when a row's running max grows by more than 2^8 (the
// probabilities of a tile are then at most 256, exact in fp32 and bf16).
// Waits are bounded as in the GEMM.
#include "nc_internal.h"
#include "nc_sm100.cuh"

namespace nc {
using namespace sm100;

bool make_map_bf16_k64(CUtensorMap *map, const void *ptr, int rows, int cols, int ld, int box_rows);

namespace {

constexpr int HD = 128;           // head dim handled here
constexpr int BR = 128;           // rows (position, head) per CTA
constexpr int BKV = 128;          // keys per tile
constexpr int ST = 2;             // K/V stages
constexpr int SUB = 128 * 64 * 2; // one 128-row x 64-column swizzled box: 16 KB
constexpr int TILE = 2 * SUB;     // 128 x 128 bf16: 32 KB
constexpr int OFF_Q = 0;
constexpr int OFF_P = TILE;                  // 2 tiles (double-buffered P)
constexpr int OFF_K = 3 * TILE;              // ST tiles
constexpr int OFF_V = 3 * TILE + ST * TILE;  // ST tiles
constexpr int OFF_BAR = 3 * TILE + 2 * ST * TILE;
constexpr int OFF_XCH = OFF_BAR + 160;       // [2][2][128] fp32: row-max halves (x2); then the row-sum halves
constexpr float RESCALE_LOG2 = 8.0f;         // rescale O when the max grows by more than 2^8
constexpr int SMEM_USED = OFF_XCH + 2 * 2 * 128 * 4;
static_assert(SMEM_USED + 256 <= 227 * 1024, "shared memory budget");
constexpr int SMEM_BYTES = 227 * 1024;       // the rest is slack for 1024-byte alignment
constexpr int MAX_PAD = SMEM_BYTES - SMEM_USED;
constexpr int THREADS = 320;                 // warp 0 TMA, warp 1 MMA, warps 2-9 softmax (2 per row)
constexpr uint32_t TMEM_COLS = 512;  // O accumulators: cols 0..255, S buffers: 256..511

struct AttnArgs {
  int T, H, B, max_seq;
  int rows_per_seq;  // T*H
  float scale_log2;  // log2(e) / sqrt(hd)
  bf16 *y;           // [B*T*H, 128]
  uint32_t *status;
};

// Shared-memory descriptor for an MN-major operand (V: keys x dims, dims
// contiguous) written by TMA with 128-byte swizzle as two boxes of 64 dims:
// 8-key groups 1024 B apart (stride byte offset), the second 64-dim box 16 KB
// further (leading byte offset).
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFF);
  d |= (uint64_t)(SUB >> 4) << 16;   // leading byte offset: next 64-element MN chunk
  d |= (uint64_t)(1024 >> 4) << 32;  // stride byte offset: next 8-row K group
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
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

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 2^x (PTX ex2.approx.ftz: relative error ~2^-22, 2^-inf = 0)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

__global__ void __launch_bounds__(THREADS, 1)
    attn_prefill_tc_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                           const __grid_constant__ CUtensorMap mapV, AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = ((raw + 1023) & ~1023u) - raw;
  if (pad > (uint32_t)MAX_PAD) {  // shared memory window not aligned as expected: report, do nothing
    if (threadIdx.x == 0) atomicOr(a.status, (unsigned)NC_DEV_TIMEOUT);
    return;
  }
  uint8_t *smem = smem_raw + pad;
  float *xch = reinterpret_cast<float *>(smem + OFF_XCH);
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  uint64_t *q_full = bar;             // 1
  uint64_t *q_empty = bar + 1;        // 1: Q free once the item's last S is done
  uint64_t *k_full = bar + 2;         // ST
  uint64_t *v_full = k_full + ST;     // ST
  uint64_t *k_empty = v_full + ST;    // ST: K stage free once S = Q K^T is done
  uint64_t *v_empty = k_empty + ST;   // ST: V stage free once P V is done
  uint64_t *s_full = v_empty + ST;    // 2
  uint64_t *p_full = s_full + 2;      // 2 (256 arrivals), one per P buffer
  uint64_t *o_done = p_full + 2;      // 2, one per P buffer
  uint64_t *o_empty = o_done + 2;     // 2 (256 arrivals), one per O accumulator
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(o_empty + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_rt = (a.rows_per_seq + BR - 1) / BR;
  const int n_items = n_rt * a.B;

  // work item i: row tile n_rt-1 - i/B of sequence i%B (heaviest first), the
  // CTA takes items blockIdx.x, +gridDim.x, ...
  auto item_of = [&](int i, int &b, int &row0, int &n_kv) {
    const int rt = n_rt - 1 - i / a.B;
    b = i % a.B;
    row0 = rt * BR;
    int t_max = (row0 + BR - 1) / a.H;
    if (t_max > a.T - 1) t_max = a.T - 1;
    n_kv = t_max / BKV + 1;
  };

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < ST; s++) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int i = 0; i < 2; i++) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 256);
      mbar_init(&o_done[i], 1);
      mbar_init(&o_empty[i], 256);
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
  const uint32_t tO0 = tmem, tS = tmem + 256;  // O accumulators at columns 0 and 128, S buffers at 256 and 384

  if (warp == 0) {
    // lane 0 streams Q and K, lane 1 streams V, item after item
    if (lane == 0) {
      int j = 0, it = 0;
      bool ok = true;
      for (int i = blockIdx.x; i < n_items && ok; i += gridDim.x, it++) {
        int b, row0, n_kv;
        item_of(i, b, row0, n_kv);
        const int krow = b * a.max_seq;
        if (!mbar_wait(q_empty, (it & 1) ^ 1, abort_flag, a.status)) break;
        mbar_arrive_expect_tx(q_full, TILE);
        tma_load_2d(smem + OFF_Q, &mapQ, 0, b * a.rows_per_seq + row0, q_full);
        tma_load_2d(smem + OFF_Q + SUB, &mapQ, 64, b * a.rows_per_seq + row0, q_full);
        for (int jj = 0; jj < n_kv; jj++, j++) {
          const int s = j % ST;
          if (!mbar_wait(&k_empty[s], ((j / ST) & 1) ^ 1, abort_flag, a.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&k_full[s], TILE);
          tma_load_2d(smem + OFF_K + s * TILE, &mapK, 0, krow + jj * BKV, &k_full[s]);
          tma_load_2d(smem + OFF_K + s * TILE + SUB, &mapK, 64, krow + jj * BKV, &k_full[s]);
        }
      }
    } else if (lane == 1) {
      int j = 0;
      bool ok = true;
      for (int i = blockIdx.x; i < n_items && ok; i += gridDim.x) {
        int b, row0, n_kv;
        item_of(i, b, row0, n_kv);
        const int krow = b * a.max_seq;
        for (int jj = 0; jj < n_kv; jj++, j++) {
          const int s = j % ST;
          if (!mbar_wait(&v_empty[s], ((j / ST) & 1) ^ 1, abort_flag, a.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&v_full[s], TILE);
          tma_load_2d(smem + OFF_V + s * TILE, &mapV, 0, krow + jj * BKV, &v_full[s]);
          tma_load_2d(smem + OFF_V + s * TILE + SUB, &mapV, 64, krow + jj * BKV, &v_full[s]);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16_f32(BR, BKV);
      const uint32_t id_o = idesc_bf16_f32(BR, HD) | (1u << 16);  // B (V) is MN-major
      const uint32_t q0 = smem_u32(smem + OFF_Q), p0 = smem_u32(smem + OFF_P);
      // tile counters run across items; J indexes K/V stages, S and P buffers
      int J = 0, it = 0;
      bool ok = true;
      auto issue_s = [&](int jg) -> bool {  // S_jg = Q K_jg^T into S buffer jg % 2
        const int s = jg % ST;
        if (!mbar_wait(&k_full[s], (jg / ST) & 1, abort_flag, a.status)) return false;
        tc_fence_after();
        const uint32_t k0 = smem_u32(smem + OFF_K + s * TILE);
        const uint32_t d = tS + (jg & 1) * 128;
#pragma unroll
        for (int k = 0; k < HD / 16; k++) {
          const uint32_t off = (k >> 2) * SUB + (k & 3) * 32;
          mma_bf16(d, desc_k_sw128(q0 + off), desc_k_sw128(k0 + off), id_s, k != 0);
        }
        mma_commit(&s_full[jg & 1]);
        mma_commit(&k_empty[s]);
        return true;
      };
      for (int i = blockIdx.x; i < n_items && ok; i += gridDim.x, it++) {
        int b, row0, n_kv;
        item_of(i, b, row0, n_kv);
        const int ob = it & 1;
        const uint32_t tO = tO0 + ob * 128;
        if (!mbar_wait(q_full, it & 1, abort_flag, a.status)) break;
        // the epilogue of item it-2 must have read this O accumulator
        if (!mbar_wait(&o_empty[ob], ((it >> 1) & 1) ^ 1, abort_flag, a.status)) break;
        tc_fence_after();
        if (!issue_s(J)) break;
        for (int jj = 0; jj < n_kv && ok; jj++) {
          const int jg = J + jj;
          if (jj + 1 < n_kv) {
            if (!issue_s(jg + 1)) { ok = false; break; }
          } else {
            mma_commit(q_empty);  // the last S of the item: Q may be reloaded
          }
          if (!mbar_wait(&p_full[jg & 1], (jg >> 1) & 1, abort_flag, a.status)) { ok = false; break; }
          const int s = jg % ST;
          if (!mbar_wait(&v_full[s], (jg / ST) & 1, abort_flag, a.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t v0 = smem_u32(smem + OFF_V + s * TILE), pb = p0 + (jg & 1) * TILE;
#pragma unroll
          for (int k = 0; k < BKV / 16; k++) {
            const uint32_t poff = (k >> 2) * SUB + (k & 3) * 32;
            mma_bf16(tO, desc_k_sw128(pb + poff), desc_mn_sw128(v0 + k * 2048), id_o, (jj | k) != 0);
          }
          mma_commit(&o_done[jg & 1]);
          mma_commit(&v_empty[s]);
        }
        J += n_kv;
      }
    }
  } else {
    // softmax / correction / epilogue: two threads per row, each owning 64 of
    // the tile's 128 keys (and 64 of the 128 output dims)
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    bool ok = true;
    int J = 0, it = 0;
    // every thread runs every iteration (a failed wait only clears `ok`), so
    // the named-barrier syncs always pair up
    for (int i = blockIdx.x; i < n_items; i += gridDim.x, it++) {
      int b, row0, n_kv;
      item_of(i, b, row0, n_kv);
      const int ob = it & 1;
      const uint32_t tO = tO0 + ob * 128;
      const int row = row0 + r;  // row inside the sequence
      const int t_row = row < a.rows_per_seq ? row / a.H : 0x3fffffff;
      float m = -INFINITY, l = 0.f;  // reference max (scaled, log2 units) and this half's running sum
      for (int jj = 0; jj < n_kv; jj++) {
        const int jg = J + jj;
        ok = ok && mbar_wait(&s_full[jg & 1], (jg >> 1) & 1, abort_flag, a.status);
        tc_fence_after();
        const uint32_t sbase = tS + (jg & 1) * 128 + lane_off + half * 64;
        const int kbase = jj * BKV + half * 64;
        uint32_t v[64];
        tmem_ld32(sbase + 0, *reinterpret_cast<uint32_t(*)[32]>(v + 0));
        tmem_ld32(sbase + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
        tmem_ld_wait();
        // raw max of this half (the scale is positive); the causal mask only
        // matters on tiles that reach past the row's position
        const bool masked = kbase + 63 > t_row;
        float mx0 = -INFINITY, mx1 = -INFINITY;
        if (masked) {
#pragma unroll
          for (int q = 0; q < 64; q++) {
            if (kbase + q > t_row) v[q] = __float_as_uint(-INFINITY);
            if (q & 1) mx1 = fmaxf(mx1, __uint_as_float(v[q]));
            else mx0 = fmaxf(mx0, __uint_as_float(v[q]));
          }
        } else {
#pragma unroll
          for (int q = 0; q < 64; q += 2) {
            mx0 = fmaxf(mx0, __uint_as_float(v[q]));
            mx1 = fmaxf(mx1, __uint_as_float(v[q + 1]));
          }
        }
        // the two halves of the row agree on the row max (buffer jg&1: the
        // partner has read the previous use of it before arriving here again)
        float *xm = xch + (jg & 1) * 256;
        xm[half * 128 + r] = fmaxf(mx0, mx1);
        asm volatile("bar.sync 1, 256;" ::: "memory");
        const float tmax = fmaxf(xm[r], xm[128 + r]) * a.scale_log2;
        const bool need = (m == -INFINITY) ? (tmax != -INFINITY) : (tmax > m + RESCALE_LOG2);
        const float m_new = need ? tmax : m;
        const float alpha = (need && m != -INFINITY) ? exp2f(m - m_new) : 1.f;
        // P buffer jg&1 is free once P_{jg-2} V_{jg-2} is done (any item)
        if (jg >= 2) ok = ok && mbar_wait(&o_done[jg & 1], ((jg - 2) >> 1) & 1, abort_flag, a.status);
        if (jj > 0 && __any_sync(0xffffffffu, need)) {
          // O must hold every earlier P V of this item before it is rescaled;
          // this half rescales output dims half*64 .. +63
          ok = ok && mbar_wait(&o_done[(jg - 1) & 1], ((jg - 1) >> 1) & 1, abort_flag, a.status);
          tc_fence_after();
#pragma unroll 1
          for (int c = half * 64; c < half * 64 + 64; c += 32) {
            uint32_t o[32];
            tmem_ld32(tO + lane_off + c, o);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; q++) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
            tmem_st32(tO + lane_off + c, o);
          }
          tmem_st_wait();
        }
        // p = 2^(s*scale - m): one FMA and one ex2 per score (masked scores
        // are -inf and give 0), bf16 into box `half` of the swizzled P tile
        uint8_t *prow = smem + OFF_P + (jg & 1) * TILE + half * SUB + r * 128;
        const float nm = -m_new;
        float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
        for (int c = 0; c < 64; c += 8) {
          float pv[8];
#pragma unroll
          for (int q = 0; q < 8; q++) pv[q] = ex2(fmaf(__uint_as_float(v[c + q]), a.scale_log2, nm));
          sum0 += (pv[0] + pv[2]) + (pv[4] + pv[6]);
          sum1 += (pv[1] + pv[3]) + (pv[5] + pv[7]);
          const int chunk = c >> 3;
          *reinterpret_cast<uint4 *>(prow + ((chunk ^ (r & 7)) << 4)) =
              make_uint4(pack2(pv[0], pv[1]), pack2(pv[2], pv[3]), pack2(pv[4], pv[5]), pack2(pv[6], pv[7]));
        }
        l = l * alpha + (sum0 + sum1);
        m = m_new;
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        mbar_arrive(&p_full[jg & 1]);
      }
      // row sum = both halves (the exchange slot is free: every max above has
      // been read before this barrier)
      asm volatile("bar.sync 1, 256;" ::: "memory");
      float *xl = xch;  // both row-max slots have been read by now
      xl[half * 128 + r] = l;
      asm volatile("bar.sync 1, 256;" ::: "memory");
      const float lsum = xl[r] + xl[128 + r];
      const int jl = J + n_kv - 1;
      ok = ok && mbar_wait(&o_done[jl & 1], (jl >> 1) & 1, abort_flag, a.status);
      tc_fence_after();
      const float inv = 1.f / lsum;
      bf16 *dst = a.y + ((size_t)b * a.rows_per_seq + row) * HD;
#pragma unroll 1
      for (int c = half * 64; c < half * 64 + 64; c += 32) {
        uint32_t o[32];
        tmem_ld32(tO + lane_off + c, o);
        tmem_ld_wait();
        if (ok && row < a.rows_per_seq) {
          uint4 *d4 = reinterpret_cast<uint4 *>(dst + c);
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
      mbar_arrive(&o_empty[ob]);
      // keep the l exchange slot from being overwritten before the partner read it
      asm volatile("bar.sync 1, 256;" ::: "memory");
      J += n_kv;
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

bool attn_prefill_tc_supported(int H, int Hkv, int hd) { return hd == HD && Hkv == 1 && H >= 1; }

// q: [B*T*H, 128] bf16 (rotated + normed), kc/vc: layer cache [max_batch*max_seq, 128],
// y: [B*T*H, 128] bf16.
cudaError_t k_attn_prefill_tc(const void *q, const void *kc, const void *vc, int B, int T, int H, int max_batch,
                              int max_seq, void *y, uint32_t *status, cudaStream_t s) {
  CUtensorMap mq, mk, mv;
  const int rows = T * H;
  if (!make_map_bf16_k64(&mq, q, B * rows, HD, HD, BR) ||
      !make_map_bf16_k64(&mk, kc, max_batch * max_seq, HD, HD, BKV) ||
      !make_map_bf16_k64(&mv, vc, max_batch * max_seq, HD, HD, BKV))
    return cudaErrorInvalidValue;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(attn_prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  AttnArgs a;
  a.T = T;
  a.H = H;
  a.B = B;
  a.max_seq = max_seq;
  a.rows_per_seq = rows;
  a.scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
  a.y = (bf16 *)y;
  a.status = status;
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  }
  const int items = ((rows + BR - 1) / BR) * B;
  dim3 grid(items < sms ? items : sms);
  count_launch();
  attn_prefill_tc_kernel<<<grid, THREADS, SMEM_BYTES, s>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

}  // namespace nc
