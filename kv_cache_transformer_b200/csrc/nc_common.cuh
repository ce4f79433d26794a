// nc_common.cuh — device helpers shared by the engine's kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace nc {

using bf16 = __nv_bfloat16;

// Storage <-> fp32 conversions for the two storage types.
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(bf16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float v) { return __float2bfloat16_rn(v); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide sum for blockDim.x a multiple of 32 (<= 1024). `red` holds >= 32
// floats of shared memory. Every thread gets the total.
__device__ __forceinline__ float block_sum(float v, float *red) {
  int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float t = lane < nw ? red[lane] : 0.f;
  return warp_sum(t);
}

__device__ __forceinline__ float block_max(float v, float *red) {
  int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float t = lane < nw ? red[lane] : -INFINITY;
  return warp_max(t);
}

// (value, index) argmax with the lowest index winning ties.
struct ArgMax {
  float v;
  int i;
};
__device__ __forceinline__ ArgMax argmax_merge(ArgMax a, ArgMax b) {
  if (b.v > a.v || (b.v == a.v && b.i < a.i)) return b;
  return a;
}
__device__ __forceinline__ ArgMax warp_argmax(ArgMax a) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ArgMax b;
    b.v = __shfl_xor_sync(0xffffffffu, a.v, o);
    b.i = __shfl_xor_sync(0xffffffffu, a.i, o);
    a = argmax_merge(a, b);
  }
  return a;
}

// Which sequence / position a row of activations belongs to. Prefill rows
// are m = b*T + t (position t, or off[b] + t when a chunk is appended to
// sequences already holding off[b] tokens); decode rows are m = b with
// position pos[b].
struct RowMap {
  int T;                         // prefill prompt / chunk length (ignored for decode)
  const int32_t *pos;            // decode positions [B], or nullptr for prefill
  const int32_t *off = nullptr;  // chunk start of each sequence [B], or nullptr (from position 0)
  __device__ __forceinline__ int seq(int m) const { return pos ? m : m / T; }
  __device__ __forceinline__ int position(int m) const {
    return pos ? pos[m] : (off ? off[m / T] : 0) + m % T;
  }
};

}  // namespace nc
