// nc_gemm_tc.cu — tcgen05 tensor-core GEMM for the prefill linear layers.
//
// C[M, N] (epilogue) acc, acc = A[M, K] * W[N, K]^T, A and W bf16 with K
// contiguous (activations row-major, weights row-major [out, in]), fp32
// accumulation in tensor memory (TMEM).
//
// Persistent kernel, one CTA per SM, 128 x 256 output tiles walked with a
// static stride of gridDim.x. Warp roles (192 threads):
//   warp 0      TMA producer: A and W tiles of 64 K-columns (128-byte
//               swizzle) into a 4-stage shared-memory ring;
//   warp 1      TMEM allocator and MMA issuer: 4 x tcgen05.mma (M=128,
//               N=256, K=16) per stage into one of two TMEM accumulators
//               (2 x 256 fp32 columns), tcgen05.commit frees the stage;
//   warps 2-5   epilogue: tcgen05.ld of the finished accumulator (each warp
//               its 32-lane TMEM quarter = 32 rows), epilogue math, stores,
//               then release the accumulator so the next tile's MMAs run
//               while this one drains.
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
constexpr int THREADS = 192;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
constexpr uint32_t TMEM_COLS = 2 * BN;

struct GemmArgs {
  int M, N, K;
  void *out;
  int ldo;
  float cap;
  uint32_t *status;
};

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

// Apply the epilogue to 32 consecutive columns of one row.
template <int EPI>
__device__ __forceinline__ void epilogue32(const GemmArgs &g, int row, int col, const uint32_t (&r)[32]) {
  size_t o = (size_t)row * g.ldo + col;
  if (EPI == EPI_STORE || EPI == EPI_RELU2) {
    uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<bf16 *>(g.out) + o);
#pragma unroll
    for (int q = 0; q < 4; q++) {
      float v[8];
#pragma unroll
      for (int j = 0; j < 8; j++) {
        float x = u2f(r[q * 8 + j]);
        if (EPI == EPI_RELU2) {
          x = fmaxf(x, 0.f);
          x = x * x;
        }
        v[j] = x;
      }
      dst[q] = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                          pack_bf16(v[6], v[7]));
    }
  } else if (EPI == EPI_RESID) {
    float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(g.out) + o);
#pragma unroll
    for (int q = 0; q < 8; q++) {
      float4 x = dst[q];
      x.x += u2f(r[q * 4 + 0]);
      x.y += u2f(r[q * 4 + 1]);
      x.z += u2f(r[q * 4 + 2]);
      x.w += u2f(r[q * 4 + 3]);
      dst[q] = x;
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
      mbar_init(&tempty[a], 128);
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
        for (int kb = 0; kb < kblocks; kb++) {
          if (!mbar_wait(&full[stage], phase, abort_flag, g.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * A_BYTES), w0 = smem_u32(sW + stage * B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; k++)
            mma_bf16(d, desc_k_sw128(a0 + 32 * k), desc_k_sw128(w0 + 32 * k), idesc, (kb | k) != 0);
          mma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        mma_commit(&tfull[acc]);
      }
    }
  } else {
    const int quarter = warp & 3;  // this warp's TMEM lane quarter
    int local = 0;
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, local++) {
      const int acc = local & 1;
      const uint32_t accphase = (local >> 1) & 1;
      if (!mbar_wait(&tfull[acc], accphase, abort_flag, g.status)) break;
      tc_fence_after();
      const int m0 = (tile / tiles_n) * BM, n0 = (tile % tiles_n) * BN;
      const int row = m0 + quarter * 32 + lane;
      const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + acc * BN;
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        uint32_t r[32];
        tmem_ld32(tbase + c, r);
        tmem_ld_wait();
        if (row < g.M && n0 + c < g.N) epilogue32<EPI>(g, row, n0 + c, r);
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

bool gemm_tc_supported(int M, int N, int K, int lda) {
  return M > 0 && N > 0 && K > 0 && K % BK == 0 && N % 32 == 0 && lda % 8 == 0;
}

template <int EPI>
static cudaError_t launch_tc(const CUtensorMap &ma, const CUtensorMap &mw, const GemmArgs &g, int grid,
                             cudaStream_t s) {
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  count_launch();
  gemm_tc_kernel<EPI><<<grid, THREADS, SMEM_BYTES, s>>>(ma, mw, g);
  return cudaGetLastError();
}

cudaError_t k_gemm_tc(int epi, const void *A, int lda, const void *W, int M, int N, int K, void *out, int ldo,
                      float cap, uint32_t *status, int num_sms, cudaStream_t s) {
  if (!gemm_tc_supported(M, N, K, lda)) return cudaErrorInvalidValue;
  CUtensorMap ma, mw;
  if (!make_map_bf16_k64(&ma, A, M, K, lda, BM) || !make_map_bf16_k64(&mw, W, N, K, K, BN))
    return cudaErrorInvalidValue;
  GemmArgs g{M, N, K, out, ldo, cap, status};
  int tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  int grid = tiles < num_sms ? tiles : num_sms;
  switch (epi) {
    case EPI_STORE: return launch_tc<EPI_STORE>(ma, mw, g, grid, s);
    case EPI_RELU2: return launch_tc<EPI_RELU2>(ma, mw, g, grid, s);
    case EPI_RESID: return launch_tc<EPI_RESID>(ma, mw, g, grid, s);
    default: return launch_tc<EPI_SOFTCAP>(ma, mw, g, grid, s);
  }
}

}  // namespace nc
