// nc_gemm_tc.cu — tcgen05 tensor-core GEMM for the prefill linear layers.
//
// C[M, N] (epilogue) acc, acc = A[M, K] * W[N, K]^T, A and W bf16 with K
// contiguous (activations row-major, weights row-major [out, in]), fp32
// accumulation in tensor memory (TMEM).
//
// Persistent kernel, one CTA per SM, 128 x 256 output tiles walked with a
// static stride of gridDim.x. Warp roles (320 threads):
//   warp 0      TMA producer: A and W tiles of 64 K-columns (128-byte
//               swizzle) into a 4-stage shared-memory ring;
//   warp 1      TMEM allocator and MMA issuer: 4 x tcgen05.mma (M=128,
//               N=256, K=16) per stage into one of two TMEM accumulators
//               (2 x 256 fp32 columns), tcgen05.commit frees the stage;
//   warps 2-9   epilogue: tcgen05.ld of the finished accumulator (each warp
//               its 32-lane TMEM quarter = 32 rows, and one 128-column half),
//               epilogue math, stores, then release the accumulator so the
//               next tile's MMAs run while this one drains.
// Fused prefill epilogues (GemmFuse): the RMS factor of un-normed bf16(x)
// rows applied to the accumulator; RoPE + QK norm + cache append of the qkv
// projection; bf16(x) and per-tile sums of squares written beside the
// residual update.
// Every mbarrier wait is bounded (nc_sm100.cuh); a timeout sets
// NC_DEV_TIMEOUT and all roles drain to the common exit, where TMEM is freed.
#include "nc_internal.h"
#include "nc_sm100.cuh"

namespace nc {
using namespace sm100;

namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;  // 16 KB
constexpr int B_BYTES = BN * BK * 2;  // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int EPI_WARPS = 8;   // two per TMEM lane quarter, one per 128-column half of the tile
constexpr int HC = BN / 2;      // columns per epilogue warp
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int EPI_BUF = EPI_WARPS * 32 * 32 * 4;  // per epilogue warp: a 32 x 32 fp32 transpose buffer
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256 + EPI_BUF;
constexpr uint32_t TMEM_COLS = 2 * BN;

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

// EPI_QKV for one 128-column head of the warp's 32 rows (rbase + lane); the
// head's accumulator columns start at TMEM address tcol, `scale` is the RMS
// factor of this lane's row. Heads 0..H-1 are q, heads H..H+Hkv-1 the keys
// and H+Hkv..H+2Hkv-1 the values of the Hkv KV heads; KV head j occupies
// elements [128j, 128j + 128) of a cache row.
// RoPE pairs element e with element e+64 and rotates by the angle of
// (e, position); q and k are then RMS normed over their 128 elements. A
// rotation keeps each pair's sum of squares, so the norm factor is taken from
// the unrotated accumulator row (lane = row); the rotation, scaling and
// stores then run on transposed chunks, lane = (row group, 4 columns).
__device__ __forceinline__ void qkv_head(const GemmArgs &g, int rbase, int lane, int head, uint32_t tcol, float scale,
                                         float *ebuf) {
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
  int pos[8], crow[8];  // position, and cache row b*max_seq + position (-1: no cache write)
#pragma unroll
  for (int i = 0; i < 8; i++) {
    const int row = rbase + 4 * i + rsub;
    facr[i] = __shfl_sync(0xffffffffu, fac, 4 * i + rsub);
    const int b = row / f.T;
    pos[i] = row < g.M ? (f.off ? f.off[b] : 0) + row - b * f.T : 0;
    crow[i] = row < g.M && (!f.valid || f.valid[b]) ? b * f.max_seq + pos[i] : -1;
  }
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
#pragma unroll
    for (int i = 0; i < 8; i++) {
      if (rbase + 4 * i + rsub >= g.M || (head >= f.H && crow[i] < 0)) continue;
      const float4 *cs = reinterpret_cast<const float4 *>(f.rope + (size_t)pos[i] * 64) + 16 * c + 2 * q;
      const float4 a = lo[i], h = hi[i], u = cs[0], w = cs[1];  // (cos, sin) of the 4 pairs
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

template <int EPI>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapW, GemmArgs g) {
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
  const int tiles = ((g.M + BM - 1) / BM) * tiles_n;
  const int kblocks = g.K / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; s++) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; a++) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 32 * EPI_WARPS);
    }
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&mapA);
    tma_prefetch_desc(&mapW);
  }
  if (warp == 1) tmem_alloc(tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
        const int m0 = (tile / tiles_n) * BM, n0 = (tile % tiles_n) * BN;
        for (int kb = 0; kb < kblocks; kb++) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, g.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
          tma_load_2d(sA + stage * A_BYTES, &mapA, kb * BK, m0, &full[stage]);
          tma_load_2d(sW + stage * B_BYTES, &mapW, kb * BK, n0, &full[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(BM, BN);
      int stage = 0, local = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, local++) {
        const int acc = local & 1;
        const uint32_t accphase = (local >> 1) & 1;
        if (!mbar_wait(&tempty[acc], accphase ^ 1, abort_flag, g.status)) break;
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
          for (int k = 0; k < BK / 16; k++)
            mma_bf16(d, desc_k_sw128(a0 + 32 * k), desc_k_sw128(w0 + 32 * k), idesc, (kb | k) != 0);
          mma_commit(&empty[stage]);
          stage = nstage;
          phase = nphase;
          ready = next_ready;
        }
        mma_commit(&tfull[acc]);
      }
    }
  } else {
    const int ew = warp - 2;       // epilogue warp 0..7
    const int quarter = warp & 3;  // its TMEM lane quarter (a warp reaches lanes 32*(warp%4) .. +31)
    const int half = ew >> 2;      // its 128-column half of the tile
    float *ebuf = reinterpret_cast<float *>(smem + STAGES * STAGE_BYTES + 256) + ew * 1024;
    int local = 0;
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, local++) {
      const int acc = local & 1;
      const uint32_t accphase = (local >> 1) & 1;
      const int m0 = (tile / tiles_n) * BM, n0 = (tile % tiles_n) * BN;
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
        if (!mbar_wait(&tfull[acc], accphase, abort_flag, g.status)) break;
        tc_fence_after();
        if constexpr (EPI == EPI_QKV) {
          const int head = nh / 128;  // one head per half
          if (head < g.fz.H + 2 * g.fz.Hkv) qkv_head(g, m0 + quarter * 32, lane, head, tbase, scale, ebuf);
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
      mbar_arrive(&tempty[acc]);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
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

template <int EPI>
static cudaError_t launch_tc(const CUtensorMap &ma, const CUtensorMap &mw, const GemmArgs &g, int grid,
                             cudaStream_t s) {
  {
    const cudaError_t e = ensure_smem_attr((const void *)gemm_tc_kernel<EPI>, SMEM_BYTES);
    if (e != cudaSuccess) return e;
  }
  count_launch();
  gemm_tc_kernel<EPI><<<grid, THREADS, SMEM_BYTES, s>>>(ma, mw, g);
  return cudaGetLastError();
}

cudaError_t k_gemm_tc(int epi, const void *A, int lda, const void *W, int M, int N, int K, void *out, int ldo,
                      float cap, uint32_t *status, int num_sms, cudaStream_t s, const GemmFuse *fz) {
  if (!gemm_tc_supported(M, N, K, lda)) return cudaErrorInvalidValue;
  if ((epi == EPI_QKV || epi == EPI_RESID_X) && !fz) return cudaErrorInvalidValue;
  if (epi == EPI_QKV && N != (fz->H + 2 * fz->Hkv) * 128) return cudaErrorInvalidValue;
  CUtensorMap ma, mw;
  if (!make_map_bf16_k64(&ma, A, M, K, lda, BM) || !make_map_bf16_k64(&mw, W, N, K, K, BN))
    return cudaErrorInvalidValue;
  GemmArgs g{M, N, K, out, ldo, cap, status, fz ? *fz : GemmFuse{}};
  int tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  int grid = tiles < num_sms ? tiles : num_sms;
  switch (epi) {
    case EPI_STORE: return launch_tc<EPI_STORE>(ma, mw, g, grid, s);
    case EPI_RELU2: return launch_tc<EPI_RELU2>(ma, mw, g, grid, s);
    case EPI_RESID: return launch_tc<EPI_RESID>(ma, mw, g, grid, s);
    case EPI_QKV: return launch_tc<EPI_QKV>(ma, mw, g, grid, s);
    case EPI_RESID_X: return launch_tc<EPI_RESID_X>(ma, mw, g, grid, s);
    default: return launch_tc<EPI_SOFTCAP>(ma, mw, g, grid, s);
  }
}

}  // namespace nc
