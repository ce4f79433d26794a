// nc_rowops.cu — bandwidth kernels for the row-wise prefill steps of bf16
// models with head_dim 128 (d_model a multiple of 128).
//
//   rows_norm_bf16     h = bf16(x / sqrt(mean(x^2) + eps)), one warp per row,
//                      16-byte loads / 8-byte stores
//   rope_qk_bf16       one warp per row: RoPE on split-half pairs, RMS norm
//                      of every q head and the k head, q out, k and v
//                      appended to the row's sequence in the cache (the
//                      unfused prefill path; the fused one does this in the
//                      QKV GEMM epilogue)
//   gather_rows_ss     copy selected rows of x (the last position of each
//                      prompt) and their per-128-column sums of squares, the
//                      input the fused lm_head + softcap + argmax kernel of
//                      the decode path consumes
#include "nc_internal.h"

namespace nc {

namespace {

__device__ __forceinline__ uint32_t pack_bf(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ float2 unpack_bf(uint32_t u) {
  __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162 *>(&u);
  return __bfloat1622float2(h);
}

// d = 128 * C: lane l holds columns 4l..4l+3 of each 128-column chunk.
template <int C>
__global__ void __launch_bounds__(256) rows_norm_kernel(const float *x, int rows, float eps, bf16 *h) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= rows) return;
  const float4 *src = reinterpret_cast<const float4 *>(x + (size_t)warp * C * 128);
  float4 v[C];
  float ss = 0.f;
#pragma unroll
  for (int c = 0; c < C; c++) {
    v[c] = src[c * 32 + lane];
    ss += v[c].x * v[c].x + v[c].y * v[c].y + v[c].z * v[c].z + v[c].w * v[c].w;
  }
  ss = warp_sum(ss);
  const float inv = rsqrtf(ss / (C * 128) + eps);
  uint2 *dst = reinterpret_cast<uint2 *>(h + (size_t)warp * C * 128);
#pragma unroll
  for (int c = 0; c < C; c++)
    dst[c * 32 + lane] = make_uint2(pack_bf(v[c].x * inv, v[c].y * inv), pack_bf(v[c].z * inv, v[c].w * inv));
}

// One warp per row of qkv [M][(H+2)*128]: every head's loads are issued
// before any is used, the RoPE (cos, sin) of the row's position is read once;
// lane l owns the pairs (2l, 64+2l) and (2l+1, 65+2l) of each head.
template <int NH>
__global__ void __launch_bounds__(256) rope_qk_kernel(const bf16 *qkv, int M, int T, const float2 *rope, bf16 *q_out,
                                                      bf16 *kc, bf16 *vc, int max_seq, float eps) {
  constexpr int H = NH - 2;
  const int m = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (m >= M) return;
  const int b = m / T, pos = m % T;
  const uint32_t *src = reinterpret_cast<const uint32_t *>(qkv + (size_t)m * NH * 128);
  uint32_t lo[NH], hi[NH];
#pragma unroll
  for (int h = 0; h < NH; h++) {
    lo[h] = src[h * 64 + lane];       // elements 2l, 2l+1 of head h
    hi[h] = src[h * 64 + 32 + lane];  // elements 64+2l, 65+2l
  }
  const float4 cs = reinterpret_cast<const float4 *>(rope + (size_t)pos * 64)[lane];  // pairs 2l and 2l+1
  const size_t crow = ((size_t)b * max_seq + pos) * 128;
#pragma unroll
  for (int h = 0; h < NH - 1; h++) {  // q heads and the k head: RoPE + RMS norm
    const float2 a = unpack_bf(lo[h]), c = unpack_bf(hi[h]);
    const float r0 = a.x * cs.x - c.x * cs.y, r64 = a.x * cs.y + c.x * cs.x;
    const float r1 = a.y * cs.z - c.y * cs.w, r65 = a.y * cs.w + c.y * cs.z;
    const float ss = warp_sum(r0 * r0 + r1 * r1 + r64 * r64 + r65 * r65);
    const float inv = rsqrtf(ss * (1.0f / 128) + eps);
    uint32_t *dst = h < H ? reinterpret_cast<uint32_t *>(q_out + ((size_t)m * H + h) * 128)
                          : reinterpret_cast<uint32_t *>(kc + crow);
    dst[lane] = pack_bf(r0 * inv, r1 * inv);
    dst[32 + lane] = pack_bf(r64 * inv, r65 * inv);
  }
  uint32_t *dv = reinterpret_cast<uint32_t *>(vc + crow);  // v: copied unchanged
  dv[lane] = lo[NH - 1];
  dv[32 + lane] = hi[NH - 1];
}

// Row r of xl = row r*stride + offset of x; ss[j][r] = sum of squares of its
// 128-column chunk j. One block of 128 threads per row.
__global__ void gather_rows_ss_kernel(const float *x, int d, int stride, int offset, float *xl, float *ss, int ssb) {
  __shared__ float part[4];
  const int r = blockIdx.x;
  const float *src = x + ((size_t)r * stride + offset) * d;
  for (int j = 0; j < d / 128; j++) {
    const float v = src[j * 128 + threadIdx.x];
    xl[(size_t)r * d + j * 128 + threadIdx.x] = v;
    const float q = warp_sum(v * v);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = q;
    __syncthreads();
    if (threadIdx.x == 0) ss[(size_t)j * ssb + r] = part[0] + part[1] + part[2] + part[3];
    __syncthreads();
  }
}

}  // namespace

bool rowops_supported(const nc_config &c) {
  return c.dtype == NC_BF16 && c.head_dim == 128 && c.d_model % 128 == 0 && c.d_model / 128 <= 16 &&
         c.n_head <= 16;
}

cudaError_t k_rows_norm_bf16(const float *x, int rows, int d, float eps, void *h, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  const int grid = (rows + 7) / 8;
  count_launch();
  switch (d / 128) {
#define NC_NORM_CASE(C) \
  case C: rows_norm_kernel<C><<<grid, 256, 0, s>>>(x, rows, eps, (bf16 *)h); break;
    NC_NORM_CASE(1) NC_NORM_CASE(2) NC_NORM_CASE(3) NC_NORM_CASE(4) NC_NORM_CASE(5) NC_NORM_CASE(6)
    NC_NORM_CASE(7) NC_NORM_CASE(8) NC_NORM_CASE(9) NC_NORM_CASE(10) NC_NORM_CASE(11) NC_NORM_CASE(12)
    NC_NORM_CASE(13) NC_NORM_CASE(14) NC_NORM_CASE(15) NC_NORM_CASE(16)
#undef NC_NORM_CASE
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t k_rope_qk_bf16(const void *qkv, int M, int T, int H, const float2 *rope, void *q_out, void *kc, void *vc,
                           int max_seq, float eps, cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  const unsigned grid = (unsigned)((M + 7) / 8);
  count_launch();
  switch (H + 2) {
#define NC_ROPE_CASE(NH)                                                                                        \
  case NH:                                                                                                       \
    rope_qk_kernel<NH><<<grid, 256, 0, s>>>((const bf16 *)qkv, M, T, rope, (bf16 *)q_out, (bf16 *)kc, (bf16 *)vc, \
                                            max_seq, eps);                                                      \
    break;
    NC_ROPE_CASE(3) NC_ROPE_CASE(4) NC_ROPE_CASE(5) NC_ROPE_CASE(6) NC_ROPE_CASE(7) NC_ROPE_CASE(8)
    NC_ROPE_CASE(9) NC_ROPE_CASE(10) NC_ROPE_CASE(11) NC_ROPE_CASE(12) NC_ROPE_CASE(13) NC_ROPE_CASE(14)
    NC_ROPE_CASE(15) NC_ROPE_CASE(16) NC_ROPE_CASE(17) NC_ROPE_CASE(18)
#undef NC_ROPE_CASE
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t k_gather_rows_ss(const float *x, int rows, int d, int stride, int offset, float *xl, float *ss, int ssb,
                             cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  count_launch();
  gather_rows_ss_kernel<<<rows, 128, 0, s>>>(x, d, stride, offset, xl, ss, ssb);
  return cudaGetLastError();
}

}  // namespace nc
