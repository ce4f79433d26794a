// nc_gemm_tc.cu — tcgen05 tensor-core GEMM for the prefill linear layers.
//
// C[M, N] (epilogue) acc, acc = A[M, K] * W[N, K]^T, A and W bf16 with K
// contiguous (activations row-major, weights row-major [out, in]), fp32
// accumulation in tensor memory (TMEM).
//
// Persistent kernel, one CTA per SM. With more than 128 rows the CTAs run
// as clusters of two on an SM pair: a pair walks 256 x 256 output tiles with
// a static stride, its even CTA issues tcgen05.mma.cta_group::2 (M=256), and
// each CTA loads its own 128 A rows and 128 of the 256 W rows of every
// k-block (no multicast), so a stage is 32 KB and six fit. Otherwise one CTA
// walks 128 x 256 tiles with 48 KB stages, four of them. Either way each CTA
// finishes 128 x 256 outputs per tile. Warp roles (320 threads):
//   warp 0      TMA producer: A and W tiles of 64 K-columns (128-byte
//               swizzle) into the shared-memory ring; in a pair both CTAs'
//               bytes are counted on the even CTA's barrier;
//   warp 1      TMEM allocator and MMA issuer: 4 x tcgen05.mma (K=16) per
//               stage into one of two TMEM accumulators (2 x 256 fp32
//               columns), tcgen05.commit frees the stage (in both CTAs of a
//               pair);
//   warps 2-9   epilogue: tcgen05.ld of the finished accumulator (each warp
//               its 32-lane TMEM quarter = 32 rows, and one 128-column half),
//               epilogue math, stores, then release the accumulator so the
//               next tile's MMAs run while this one drains (a pair's
//               accumulator is free once all 16 epilogue warps released it).
// The environment variable NC_GEMM_PAIR=0 selects the one-CTA kernel for
// every shape.
// Fused prefill epilogues (GemmFuse): the RMS factor of un-normed bf16(x)
// rows applied to the accumulator; RoPE + QK norm + cache append of the qkv
// projection; bf16(x) and per-tile sums of squares written beside the
// residual update.
// Every mbarrier wait is bounded (nc_sm100.cuh); a timeout sets
// NC_DEV_TIMEOUT and all roles drain to the common exit, where TMEM is freed.
#include <stdlib.h>

#include <atomic>
#include <mutex>

#include "nc_internal.h"
#include "nc_sm100.cuh"

namespace nc {
using namespace sm100;

namespace {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int A_BYTES = BM * BK * 2;  // 16 KB
constexpr int EPI_WARPS = 8;   // two per TMEM lane quarter, one per 128-column half of the tile
constexpr int HC = BN / 2;      // columns per epilogue warp
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int EPI_BUF = EPI_WARPS * 32 * 32 * 4;  // per epilogue warp: a 32 x 32 fp32 transpose buffer
constexpr uint32_t TMEM_COLS = 2 * BN;

// Per-CTA tiling. A single CTA loads all BN = 256 W rows of a k-block into a
// 4-stage ring (48 KB stages). A CTA pair (PAIR) computes a 256 x 256 tile
// with tcgen05.mma.cta_group::2: each CTA loads its 128 A rows and 128 of the
// 256 W rows, so a stage is 32 KB and the same shared memory holds 6 stages;
// each CTA's TMEM still receives a 128 x 256 accumulator.
template <bool PAIR>
struct Tiling {
  static constexpr int BNL = PAIR ? BN / 2 : BN;  // W rows this CTA loads per k-block
  static constexpr int B_BYTES = BNL * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = PAIR ? 6 : 4;
  static constexpr int TM = PAIR ? 2 * BM : BM;   // output rows per tile
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256 + EPI_BUF;
};
static_assert(Tiling<false>::SMEM_BYTES <= 227 * 1024 && Tiling<true>::SMEM_BYTES <= 227 * 1024, "shared memory");

struct GemmArgs {
  int M, N, K;
  void *out;
  int ldo;
  float cap;
  uint32_t *status;
  GemmFuse fz;
};

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

// Apply the STORE / RELU2 / SOFTCAP epilogue to 32 consecutive columns of one
// row; `scale` is the row's RMS factor (1 when A is already normed).
template <int EPI>
__device__ __forceinline__ void epilogue32(const GemmArgs &g, int row, int col, const uint32_t (&r)[32], float scale,
                                           float &) {
  size_t o = (size_t)row * g.ldo + col;
  if (EPI == EPI_STORE || EPI == EPI_RELU2) {
    uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<bf16 *>(g.out) + o);
#pragma unroll
    for (int q = 0; q < 4; q++) {
      float v[8];
#pragma unroll
      for (int j = 0; j < 8; j++) {
        float x = u2f(r[q * 8 + j]) * scale;
        if (EPI == EPI_RELU2) {
          x = fmaxf(x, 0.f);
          x = x * x;
        }
        v[j] = x;
      }
      dst[q] = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                          pack_bf16(v[6], v[7]));
    }
  } else {  // EPI_SOFTCAP
    float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(g.out) + o);
    float cap = g.cap, inv = 1.0f / g.cap;
#pragma unroll
    for (int q = 0; q < 8; q++) {
      float4 x;
      x.x = cap * tanhf(u2f(r[q * 4 + 0]) * inv);
      x.y = cap * tanhf(u2f(r[q * 4 + 1]) * inv);
      x.z = cap * tanhf(u2f(r[q * 4 + 2]) * inv);
      x.w = cap * tanhf(u2f(r[q * 4 + 3]) * inv);
      dst[q] = x;
    }
  }
}

// TMEM columns [col, col+32) of the warp's 32 rows -> registers (lane = row)
// -> the warp's swizzled 32 x 32 shared buffer -> out[i] = float4 column
// (lane & 7) of row 4i + (lane >> 3).
__device__ __forceinline__ void transpose_chunk(uint32_t taddr, float *ebuf, int lane, float4 (&out)[8]) {
  uint32_t r[32];
  tmem_ld32(taddr, r);
  tmem_ld_wait();
#pragma unroll
  for (int j = 0; j < 8; j++)
    *reinterpret_cast<float4 *>(ebuf + lane * 32 + ((j ^ (lane & 7)) << 2)) =
        make_float4(u2f(r[4 * j]), u2f(r[4 * j + 1]), u2f(r[4 * j + 2]), u2f(r[4 * j + 3]));
  __syncwarp();
  const int q = lane & 7, rsub = lane >> 3;
#pragma unroll
  for (int i = 0; i < 8; i++) {
    const int rr = 4 * i + rsub;
    out[i] = *reinterpret_cast<const float4 *>(ebuf + rr * 32 + ((q ^ (rr & 7)) << 2));
  }
  __syncwarp();
}

// Per-row metadata of EPI_QKV for the lane's 8 transposed rows rbase + 4i +
// (lane >> 3): the position, and the cache row b*max_seq + position (-1: no
// cache write). It reads only kernel inputs, so it runs before the
// accumulator is ready.
__device__ __forceinline__ void qkv_rows(const GemmArgs &g, int rbase, int lane, int (&pos)[8], int (&crow)[8]) {
  const GemmFuse &f = g.fz;
  const int rsub = lane >> 3;
#pragma unroll
  for (int i = 0; i < 8; i++) {
    const int row = rbase + 4 * i + rsub;
    const int b = row / f.T;
    pos[i] = row < g.M ? (f.off ? f.off[b] : 0) + row - b * f.T : 0;
    crow[i] = row < g.M && (!f.valid || f.valid[b]) ? b * f.max_seq + pos[i] : -1;
  }
}

// EPI_QKV for one 128-column head of the warp's 32 rows (rbase + lane); the
// head's accumulator columns start at TMEM address tcol, `scale` is the RMS
// factor of this lane's row, pos / crow come from qkv_rows. Heads 0..H-1
// are q, heads H..H+Hkv-1 the keys and H+Hkv..H+2Hkv-1 the values of the Hkv
// KV heads; KV head j occupies elements [128j, 128j + 128) of a cache row.
// RoPE pairs element e with element e+64 and rotates by the angle of
// (e, position); q and k are then RMS normed over their 128 elements. A
// rotation keeps each pair's sum of squares, so the norm factor is taken from
// the unrotated accumulator row (lane = row); the rotation, scaling and
// stores then run on transposed chunks, lane = (row group, 4 columns).
__device__ __forceinline__ void qkv_head(const GemmArgs &g, int rbase, int lane, int head, uint32_t tcol, float scale,
                                         float *ebuf, const int (&pos)[8], const int (&crow)[8]) {
  const GemmFuse &f = g.fz;
  const bool isv = head >= f.H + f.Hkv;
  const int kvh = head < f.H ? 0 : (isv ? head - f.H - f.Hkv : head - f.H);  // KV head of a k or v head
  float fac = scale;
  if (!isv) {
    float ss = 0.f;
#pragma unroll 1
    for (int j = 0; j < 4; j++) {
      uint32_t r[32];
      tmem_ld32(tcol + 32 * j, r);
      tmem_ld_wait();
#pragma unroll
      for (int k = 0; k < 32; k++) ss += u2f(r[k]) * u2f(r[k]);
    }
    fac = scale * rsqrtf(scale * scale * ss * (1.0f / 128) + f.eps);
  }
  const int q = lane & 7, rsub = lane >> 3;
  float facr[8];
#pragma unroll
  for (int i = 0; i < 8; i++) facr[i] = __shfl_sync(0xffffffffu, fac, 4 * i + rsub);
  auto dst_of = [&](int i) -> bf16 * {
    const int row = rbase + 4 * i + rsub;
    return (head < f.H ? reinterpret_cast<bf16 *>(f.q) + ((size_t)row * f.H + head) * 128
                       : reinterpret_cast<bf16 *>(isv ? f.vc : f.kc) + ((size_t)crow[i] * f.Hkv + kvh) * 128) +
           4 * q;
  };
  if (isv) {
#pragma unroll 1
    for (int c = 0; c < 4; c++) {
      float4 v[8];
      transpose_chunk(tcol + 32 * c, ebuf, lane, v);
#pragma unroll
      for (int i = 0; i < 8; i++)
        if (rbase + 4 * i + rsub < g.M && crow[i] >= 0)
          *reinterpret_cast<uint2 *>(dst_of(i) + 32 * c) =
              make_uint2(pack_bf16(v[i].x * facr[i], v[i].y * facr[i]), pack_bf16(v[i].z * facr[i], v[i].w * facr[i]));
    }
    return;
  }
#pragma unroll 1
  for (int c = 0; c < 2; c++) {  // elements 32c + 4q .. +3 and their partners 64 + 32c + 4q .. +3
    float4 lo[8], hi[8];
    transpose_chunk(tcol + 32 * c, ebuf, lane, lo);
    transpose_chunk(tcol + 64 + 32 * c, ebuf, lane, hi);
    // the (cos, sin) of 4 rows' 4 pairs at a time, requested before any of
    // their stores, so the L2 round trips of a group overlap
#pragma unroll
    for (int i0 = 0; i0 < 8; i0 += 4) {
      float4 cu[4], cw[4];
#pragma unroll
      for (int k = 0; k < 4; k++) {
        const float4 *cs = reinterpret_cast<const float4 *>(f.rope + (size_t)pos[i0 + k] * 64) + 16 * c + 2 * q;
        cu[k] = __ldg(cs);
        cw[k] = __ldg(cs + 1);
      }
#pragma unroll
      for (int k = 0; k < 4; k++) {
        const int i = i0 + k;
        if (rbase + 4 * i + rsub >= g.M || (head >= f.H && crow[i] < 0)) continue;
        const float4 a = lo[i], h = hi[i], u = cu[k], w = cw[k];  // (cos, sin) of the 4 pairs
        const float F = facr[i];
        const float l0 = a.x * u.x - h.x * u.y, h0 = a.x * u.y + h.x * u.x;
        const float l1 = a.y * u.z - h.y * u.w, h1 = a.y * u.w + h.y * u.z;
        const float l2 = a.z * w.x - h.z * w.y, h2 = a.z * w.y + h.z * w.x;
        const float l3 = a.w * w.z - h.w * w.w, h3 = a.w * w.w + h.w * w.z;
        bf16 *d = dst_of(i);
        *reinterpret_cast<uint2 *>(d + 32 * c) = make_uint2(pack_bf16(l0 * F, l1 * F), pack_bf16(l2 * F, l3 * F));
        *reinterpret_cast<uint2 *>(d + 64 + 32 * c) = make_uint2(pack_bf16(h0 * F, h1 * F), pack_bf16(h2 * F, h3 * F));
      }
    }
  }
}

template <int EPI, bool PAIR>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapW, GemmArgs g) {
  using TL = Tiling<PAIR>;
  constexpr int STAGES = TL::STAGES, B_BYTES = TL::B_BYTES, STAGE_BYTES = TL::STAGE_BYTES, TM = TL::TM;
  extern __shared__ uint8_t smem_raw[];
  uint32_t raw = smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw + 1023) & ~1023u) - raw);
  uint8_t *sA = smem;
  uint8_t *sW = smem + STAGES * A_BYTES;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
  uint64_t *empty = full + STAGES;
  uint64_t *tfull = empty + STAGES;
  uint64_t *tempty = tfull + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_n = (g.N + BN - 1) / BN;
  const int tiles = ((g.M + TM - 1) / TM) * tiles_n;
  const int kblocks = g.K / BK;
  // tiles are walked by CTA (or by pair) with a static stride
  const uint32_t rank = PAIR ? cluster_rank() : 0u;
  const int walker = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int walkers = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; s++) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; a++) {
      mbar_init(&tfull[a], 1);
      // a pair's accumulator is released by each epilogue warp of both CTAs
      mbar_init(&tempty[a], PAIR ? 2 * EPI_WARPS : 32 * EPI_WARPS);
    }
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&mapA);
    tma_prefetch_desc(&mapW);
  }
  if (warp == 1) {
    if constexpr (PAIR) tmem_alloc_pair(tmem_slot, TMEM_COLS);
    else tmem_alloc(tmem_slot, TMEM_COLS);
  }
  tc_fence_before();
  // a pair: the peer's barriers are initialised before any remote arrival
  if constexpr (PAIR) cluster_sync();
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = walker; tile < tiles && ok; tile += walkers) {
        // this CTA's A rows and W rows of the tile
        const int m0 = (tile / tiles_n) * TM + (int)rank * BM, n0 = (tile % tiles_n) * BN + (int)rank * TL::BNL;
        for (int kb = 0; kb < kblocks; kb++) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, g.status)) {
            ok = false;
            break;
          }
          if constexpr (PAIR) {
            // both CTAs' bytes are counted on the rank-0 CTA's barrier, whose
            // MMA thread reads both CTAs' stages
            if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * STAGE_BYTES);
            const uint32_t fb = cluster_addr(smem_u32(&full[stage]), 0);
            tma_load_2d_pair(sA + stage * A_BYTES, &mapA, kb * BK, m0, fb);
            tma_load_2d_pair(sW + stage * B_BYTES, &mapW, kb * BK, n0, fb);
          } else {
            mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
            tma_load_2d(sA + stage * A_BYTES, &mapA, kb * BK, m0, &full[stage]);
            tma_load_2d(sW + stage * B_BYTES, &mapW, kb * BK, n0, &full[stage]);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {  // a pair's MMAs are issued by its rank-0 CTA
      const uint32_t idesc = idesc_bf16_f32(TM, BN);
      int stage = 0, local = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = walker; tile < tiles && ok; tile += walkers, local++) {
        const int acc = local & 1;
        const uint32_t accphase = (local >> 1) & 1;
        if (PAIR ? !mbar_wait_cluster(&tempty[acc], accphase ^ 1, abort_flag, g.status)
                 : !mbar_wait(&tempty[acc], accphase ^ 1, abort_flag, g.status))
          break;
        tc_fence_after();
        const uint32_t d = tmem + acc * BN;
        // a wait's result takes ~160 cycles even when the stage is full, so
        // the next stage is probed before this stage's MMAs are issued and
        // its answer is read after them
        bool ready = mbar_try_wait(smem_u32(&full[stage]), phase);
        for (int kb = 0; kb < kblocks; kb++) {
          if (!ready && !mbar_wait(&full[stage], phase, abort_flag, g.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int nstage = stage + 1 == STAGES ? 0 : stage + 1;
          const uint32_t nphase = stage + 1 == STAGES ? phase ^ 1 : phase;
          const bool next_ready = kb + 1 < kblocks && mbar_try_wait(smem_u32(&full[nstage]), nphase);
          const uint32_t a0 = smem_u32(sA + stage * A_BYTES), w0 = smem_u32(sW + stage * B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; k++) {
            if constexpr (PAIR)
              mma_bf16_pair(d, desc_k_sw128(a0 + 32 * k), desc_k_sw128(w0 + 32 * k), idesc, (kb | k) != 0);
            else
              mma_bf16(d, desc_k_sw128(a0 + 32 * k), desc_k_sw128(w0 + 32 * k), idesc, (kb | k) != 0);
          }
          // the stage is free in both CTAs of a pair once these MMAs are done
          if constexpr (PAIR) mma_commit_pair(&empty[stage]);
          else mma_commit(&empty[stage]);
          stage = nstage;
          phase = nphase;
          ready = next_ready;
        }
        if constexpr (PAIR) mma_commit_pair(&tfull[acc]);
        else mma_commit(&tfull[acc]);
      }
    }
  } else {
    const int ew = warp - 2;       // epilogue warp 0..7
    const int quarter = warp & 3;  // its TMEM lane quarter (a warp reaches lanes 32*(warp%4) .. +31)
    const int half = ew >> 2;      // its 128-column half of the tile
    float *ebuf = reinterpret_cast<float *>(smem + STAGES * STAGE_BYTES + 256) + ew * 1024;
    int local = 0;
    for (int tile = walker; tile < tiles; tile += walkers, local++) {
      const int acc = local & 1;
      const uint32_t accphase = (local >> 1) & 1;
      // this CTA's 128 rows of the tile, all of its 256 columns
      const int m0 = (tile / tiles_n) * TM + (int)rank * BM, n0 = (tile % tiles_n) * BN;
      const int nh = n0 + half * HC;  // first column of this warp's half
      const int row = m0 + quarter * 32 + lane;
      const bool rok = row < g.M;
      const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + acc * BN + half * HC;
      if constexpr (EPI == EPI_RESID || EPI == EPI_RESID_X) {
        // x += acc over the half's 4 chunks of 32 columns. Each chunk goes
        // TMEM -> registers (lane = row) -> a swizzled shared buffer, and is
        // read back with lane = (row group, float4 column), so that every
        // global access of a warp covers 4 rows x 128 contiguous bytes. The
        // residual is read 2 chunks ahead (cur / nxt), the first 2 before the
        // accumulator is ready.
        const int q = lane & 7, rsub = lane >> 3;
        const int rbase = m0 + quarter * 32;
        float *xt = reinterpret_cast<float *>(g.out) + (size_t)rbase * g.ldo + nh + 4 * q;
        bf16 *xbt = reinterpret_cast<bf16 *>(g.fz.xb) + (size_t)rbase * g.ldo + nh + 4 * q;
        float4 cur[8], nxt[8];
        auto load_chunk = [&](int c, float4 (&dst)[8]) {
#pragma unroll
          for (int i = 0; i < 8; i++)
            if (rbase + 4 * i + rsub < g.M && nh + 32 * c < g.N)
              dst[i] = *reinterpret_cast<const float4 *>(xt + (size_t)(4 * i + rsub) * g.ldo + 32 * c);
        };
        load_chunk(0, cur);
        load_chunk(1, nxt);
        if (!mbar_wait(&tfull[acc], accphase, abort_flag, g.status)) break;
        tc_fence_after();
        float ssl[8];
#pragma unroll
        for (int i = 0; i < 8; i++) ssl[i] = 0.f;
#pragma unroll 1
        for (int c = 0; c < HC / 32; c++) {
          uint32_t r[32];
          tmem_ld32(tbase + 32 * c, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 8; j++)
            *reinterpret_cast<float4 *>(ebuf + lane * 32 + ((j ^ (lane & 7)) << 2)) =
                make_float4(u2f(r[4 * j]), u2f(r[4 * j + 1]), u2f(r[4 * j + 2]), u2f(r[4 * j + 3]));
          __syncwarp();
          if (nh + 32 * c < g.N) {
#pragma unroll
            for (int i = 0; i < 8; i++) {
              const int rr = 4 * i + rsub;
              const float4 a = *reinterpret_cast<const float4 *>(ebuf + rr * 32 + ((q ^ (rr & 7)) << 2));
              if (rbase + rr < g.M) {
                float4 x = cur[i];
                x.x += a.x;
                x.y += a.y;
                x.z += a.z;
                x.w += a.w;
                *reinterpret_cast<float4 *>(xt + (size_t)rr * g.ldo + 32 * c) = x;
                if (EPI == EPI_RESID_X) {
                  *reinterpret_cast<uint2 *>(xbt + (size_t)rr * g.ldo + 32 * c) =
                      make_uint2(pack_bf16(x.x, x.y), pack_bf16(x.z, x.w));
                  ssl[i] += x.x * x.x + x.y * x.y + x.z * x.z + x.w * x.w;
                }
              }
            }
          }
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 8; i++) cur[i] = nxt[i];
          if (c + 2 < HC / 32) load_chunk(c + 2, nxt);
        }
        if (EPI == EPI_RESID_X && nh < g.N) {
          // row sums over the half: the 8 lanes of a row group hold its 8 float4 columns
#pragma unroll
          for (int i = 0; i < 8; i++) {
            float v = ssl[i];
            v += __shfl_xor_sync(0xffffffffu, v, 1);
            v += __shfl_xor_sync(0xffffffffu, v, 2);
            v += __shfl_xor_sync(0xffffffffu, v, 4);
            if (q == 0 && rbase + 4 * i + rsub < g.M)
              g.fz.ss_out[(size_t)(nh / HC) * g.M + rbase + 4 * i + rsub] = v;
          }
        }
      } else {
        float scale = 1.f;
        if (EPI == EPI_STORE || EPI == EPI_RELU2 || EPI == EPI_QKV) {
          if (g.fz.nss > 0 && rok) {
            float t = 0.f;
            for (int j = 0; j < g.fz.nss; j++) t += g.fz.ss_in[(size_t)j * g.M + row];  // fixed order
            scale = rsqrtf(t / g.K + g.fz.eps);
          }
        }
        int qpos[8], qcrow[8];
        if constexpr (EPI == EPI_QKV) qkv_rows(g, m0 + quarter * 32, lane, qpos, qcrow);
        if (!mbar_wait(&tfull[acc], accphase, abort_flag, g.status)) break;
        tc_fence_after();
        if constexpr (EPI == EPI_QKV) {
          const int head = nh / 128;  // one head per half
          if (head < g.fz.H + 2 * g.fz.Hkv)
            qkv_head(g, m0 + quarter * 32, lane, head, tbase, scale, ebuf, qpos, qcrow);
        } else {
          float ss = 0.f;
#pragma unroll 1
          for (int c = 0; c < HC; c += 32) {
            uint32_t r[32];
            tmem_ld32(tbase + c, r);
            tmem_ld_wait();
            if (rok && nh + c < g.N) epilogue32<EPI>(g, row, nh + c, r, scale, ss);
          }
        }
      }
      tc_fence_before();
      if constexpr (PAIR) {
        // one arrival per warp, on the rank-0 CTA's barrier
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(cluster_addr(smem_u32(&tempty[acc]), 0));
      } else {
        mbar_arrive(&tempty[acc]);
      }
    }
  }
  __syncwarp();
  if constexpr (PAIR) {
    // neither CTA leaves while the other may still read its shared memory
    // (the MMAs read both CTAs' stages) or arrive on its barriers
    tc_fence_before();
    cluster_sync();
  } else {
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem, TMEM_COLS);
    else tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

}  // namespace

// 2-D bf16 tensor map over a row-major [rows, cols] matrix with row pitch
// ld elements; boxes of box_rows x 64 columns, 128-byte swizzle, zero fill
// outside the matrix.
bool make_map_bf16_k64(CUtensorMap *map, const void *ptr, int rows, int cols, int ld, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// bf16 tensor map of rank 2..5 over `ptr`: dims[0] is the contiguous
// dimension (64 elements = the 128-byte swizzle span), strides[i] the byte
// stride of dims[i + 1] (any order, multiples of 16), box[i] the box extent
// in each dimension; 128-byte swizzle, zero fill outside the tensor.
bool make_map_bf16(CUtensorMap *map, const void *ptr, int rank, const uint64_t *dims, const uint64_t *strides,
                   const uint32_t *box) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || rank < 2 || rank > 5) return false;
  cuuint64_t d[5], st[4];
  cuuint32_t bx[5], estr[5];
  for (int i = 0; i < rank; i++) {
    d[i] = dims[i];
    bx[i] = box[i];
    estr[i] = 1;
    if (i + 1 < rank) st[i] = strides[i];
  }
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(ptr), d, st, bx, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool gemm_tc_supported(int M, int N, int K, int lda) {
  return M > 0 && N > 0 && K > 0 && K % BK == 0 && N % 32 == 0 && lda % 8 == 0;
}

template <int EPI, bool PAIR>
static cudaError_t launch_tc(const CUtensorMap &ma, const CUtensorMap &mw, const GemmArgs &g, int grid,
                             cudaStream_t s) {
  constexpr int SMEM = Tiling<PAIR>::SMEM_BYTES;
  {
    const cudaError_t e = ensure_smem_attr((const void *)gemm_tc_kernel<EPI, PAIR>, SMEM);
    if (e != cudaSuccess) return e;
  }
  count_launch();
  if constexpr (!PAIR) {
    gemm_tc_kernel<EPI, false><<<grid, THREADS, SMEM, s>>>(ma, mw, g);
    return cudaGetLastError();
  } else {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<EPI, true>, ma, mw, g);
  }
}

// How many CTA pairs of the pair kernel can be resident at once on the
// current device (0 if none, or when the environment sets NC_GEMM_PAIR=0,
// which selects the one-CTA kernel for every shape). Computed once per device.
static int pair_slots() {
  static std::atomic<int> cache[64];
  static std::once_flag init;
  std::call_once(init, [] {
    for (auto &c : cache) c.store(-1);
  });
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  const int have = cache[dev].load();
  if (have >= 0) return have;
  int n = 0;
  const char *env = getenv("NC_GEMM_PAIR");
  if (!(env && atoi(env) == 0)) {
    const void *fn = (const void *)gemm_tc_kernel<EPI_STORE, true>;
    if (ensure_smem_attr(fn, Tiling<true>::SMEM_BYTES) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2);
      cfg.blockDim = dim3(THREADS);
      cfg.dynamicSmemBytes = Tiling<true>::SMEM_BYTES;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
      }
    }
  }
  cache[dev].store(n);
  return n;
}

template <bool PAIR>
static cudaError_t dispatch_tc(int epi, const CUtensorMap &ma, const CUtensorMap &mw, const GemmArgs &g, int grid,
                               cudaStream_t s) {
  switch (epi) {
    case EPI_STORE: return launch_tc<EPI_STORE, PAIR>(ma, mw, g, grid, s);
    case EPI_RELU2: return launch_tc<EPI_RELU2, PAIR>(ma, mw, g, grid, s);
    case EPI_RESID: return launch_tc<EPI_RESID, PAIR>(ma, mw, g, grid, s);
    case EPI_QKV: return launch_tc<EPI_QKV, PAIR>(ma, mw, g, grid, s);
    case EPI_RESID_X: return launch_tc<EPI_RESID_X, PAIR>(ma, mw, g, grid, s);
    default: return launch_tc<EPI_SOFTCAP, PAIR>(ma, mw, g, grid, s);
  }
}

cudaError_t k_gemm_tc(int epi, const void *A, int lda, const void *W, int M, int N, int K, void *out, int ldo,
                      float cap, uint32_t *status, int num_sms, cudaStream_t s, const GemmFuse *fz) {
  if (!gemm_tc_supported(M, N, K, lda)) return cudaErrorInvalidValue;
  if ((epi == EPI_QKV || epi == EPI_RESID_X) && !fz) return cudaErrorInvalidValue;
  if (epi == EPI_QKV && N != (fz->H + 2 * fz->Hkv) * 128) return cudaErrorInvalidValue;
  GemmArgs g{M, N, K, out, ldo, cap, status, fz ? *fz : GemmFuse{}};
  const int tiles_n = (N + BN - 1) / BN;
  // CTA pairs once there are two 128-row blocks to pair up
  const int pairs = M > BM ? pair_slots() : 0;
  CUtensorMap ma, mw;
  if (!make_map_bf16_k64(&ma, A, M, K, lda, BM) || !make_map_bf16_k64(&mw, W, N, K, K, pairs > 0 ? BN / 2 : BN))
    return cudaErrorInvalidValue;
  if (pairs > 0) {
    const int tiles = ((M + 2 * BM - 1) / (2 * BM)) * tiles_n;
    return dispatch_tc<true>(epi, ma, mw, g, 2 * (tiles < pairs ? tiles : pairs), s);
  }
  const int tiles = ((M + BM - 1) / BM) * tiles_n;
  return dispatch_tc<false>(epi, ma, mw, g, tiles < num_sms ? tiles : num_sms, s);
}

}  // namespace nc
