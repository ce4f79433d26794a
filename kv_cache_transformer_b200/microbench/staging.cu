// staging.cu — costs of the steps of one linear phase of the decode step.
//
//   * staging a [32][1280] bf16 activation block into shared memory right
//     after a grid barrier, with every CTA (one per SM) doing it at once:
//     thread loads, an fp32 quarter converted, and bulk asynchronous copies;
//   * a GEMV of R weight rows x 1280 x 32 sequences with mma.sync out of
//     shared memory (eight warps splitting K, partials added in order);
//   * how many thread-block clusters of 2, 4 and 8 CTAs the GPU places.
// Every wait is bounded; a timeout sets a flag that is printed.
#include <cstdio>
#include <cstdlib>
#include <cstdint>
#include <vector>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include "nc_sm100.cuh"
using namespace nc::sm100;
#define CK(x) do { cudaError_t e_ = (x); if (e_ != cudaSuccess) { printf("CUDA %s at %d: %s\n", #x, __LINE__, cudaGetErrorString(e_)); exit(1);} } while (0)

constexpr int KD = 1280, NBATCH = 32;
constexpr int XBYTES = NBATCH * KD * 2;  // 80 KB bf16

__device__ __forceinline__ bool poll_ge(unsigned long long *p, unsigned long long target) {
  for (uint32_t it = 0; it < (1u << 22); it++) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    if (v >= target) return true;
  }
  return false;
}

// mode 0: thread loads of the whole 80 KB bf16 block; 1: fp32 quarter (40 KB) converted;
// 2: cp.async.bulk of 80 KB in 5 chunks
__global__ void stage_probe(uint4 *xb, float4 *xf, unsigned long long *ctr, int iters, int mode, long long *out,
                            int *err) {
  extern __shared__ __align__(1024) uint8_t sm[];
  __shared__ uint64_t bar;
  __shared__ int bad;
  const int t = threadIdx.x;
  if (t == 0) { mbar_init(&bar, 1); fence_barrier_init(); bad = 0; }
  __syncthreads();
  long long acc = 0, accb = 0;
  uint32_t phase = 0;
  for (int it = 0; it < iters; it++) {
    // fresh data: each CTA rewrites its share of both buffers
    const int nb16 = XBYTES / 16;
    for (int i = blockIdx.x * blockDim.x + t; i < nb16; i += gridDim.x * blockDim.x) xb[i] = make_uint4(it, i, 1, 2);
    for (int i = blockIdx.x * blockDim.x + t; i < nb16 * 2; i += gridDim.x * blockDim.x) xf[i] = make_float4(it, 1, 2, 3);
    __syncthreads();
    const uint64_t tb = global_ns();
    if (t == 0) {
      asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(ctr) : "memory");
      if (!poll_ge(ctr, (unsigned long long)(it + 1) * gridDim.x)) { atomicOr(err, 1); bad = 1; }
    }
    __syncthreads();
    if (bad) break;
    const uint64_t t0 = global_ns();
    if (mode == 0) {
      uint4 v[20];
#pragma unroll
      for (int u = 0; u < 20; u++) {
        const int i = t + u * 256;
        v[u] = i < nb16 ? __ldcg(xb + i) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 20; u++) {
        const int i = t + u * 256;
        if (i < nb16) reinterpret_cast<uint4 *>(sm)[i ^ ((i >> 3) & 7)] = v[u];
      }
    } else if (mode == 1) {
      // quarter of K (320 columns) in fp32: 32 rows x 80 float4
      float4 v[10];
#pragma unroll
      for (int u = 0; u < 10; u++) {
        const int i = t + u * 256;  // 0..2559
        const int row = i / 80, c = i % 80;
        v[u] = __ldcg(xf + row * (KD / 4) + c);
      }
#pragma unroll
      for (int u = 0; u < 10; u++) {
        const int i = t + u * 256;
        __nv_bfloat162 a = __floats2bfloat162_rn(v[u].x, v[u].y), b = __floats2bfloat162_rn(v[u].z, v[u].w);
        uint2 w = make_uint2(*reinterpret_cast<uint32_t *>(&a), *reinterpret_cast<uint32_t *>(&b));
        reinterpret_cast<uint2 *>(sm)[i] = w;
      }
    } else {
      if (t == 0) {
        asm volatile("fence.proxy.async.global;" ::: "memory");
        mbar_arrive_expect_tx(&bar, XBYTES);
        for (int c = 0; c < 5; c++)
          asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                           smem_u32(sm + c * 16384)),
                       "l"(reinterpret_cast<const uint8_t *>(xb) + c * 16384), "r"(16384), "r"(smem_u32(&bar))
                       : "memory");
      }
      volatile int ab = 0;
      uint32_t st = 0;
      mbar_wait(&bar, phase, &ab, &st);
      phase ^= 1;
    }
    __syncthreads();
    const uint64_t t1 = global_ns();
    acc += (long long)(t1 - t0);
    accb += (long long)(t0 - tb);
    __syncthreads();
  }
  if (t == 0) {
    out[2 * blockIdx.x] = acc / iters;
    out[2 * blockIdx.x + 1] = accb / iters;
  }
}

// ---- mma.sync GEMV: R weight rows x 1280 K x 32 batch, both operands in smem (128B-swizzled k-blocks)
__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];" : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3]) : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// swizzled offset of (row r, 16-byte chunk c) inside a k-block of `rows` rows
__device__ __forceinline__ uint32_t swz(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

template <int MT>
__global__ void gemv_probe(int reps, float *out, long long *cyc) {
  extern __shared__ __align__(1024) uint8_t sm[];
  const int R = MT * 16;
  uint8_t *W = sm, *X = sm + R * KD * 2;  // W: [20 kb][R][128 B], X: [20 kb][32][128 B]
  float *red = reinterpret_cast<float *>(X + XBYTES);  // [8 warps][R][32]
  for (int i = threadIdx.x; i < (R * KD * 2 + XBYTES) / 4; i += blockDim.x)
    reinterpret_cast<uint32_t *>(sm)[i] = 0x3c003c00u ^ (i * 2654435761u & 0x00010001u);
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  long long t0 = clock64();
  for (int rep = 0; rep < reps; rep++) {
    float acc[MT][4][4];
#pragma unroll
    for (int m = 0; m < MT; m++)
#pragma unroll
      for (int n = 0; n < 4; n++) acc[m][n][0] = acc[m][n][1] = acc[m][n][2] = acc[m][n][3] = 0.f;
    for (int ks = warp * 10; ks < warp * 10 + 10; ks++) {  // 80 k-steps of 16 over 8 warps
      const int kb = ks >> 2, kk = (ks & 3) * 2;           // k-block, 16-byte chunk pair inside it
      // B (X): rows = batch; matrices (b0-7,k0-7) (b0-7,k8-15) (b8-15,k0-7) (b8-15,k8-15)
      uint32_t b[4][2];
#pragma unroll
      for (int np = 0; np < 2; np++) {
        const int r = np * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int c = kk + ((lane >> 3) & 1);
        ldsm4(smem_u32(X + kb * 4096 + swz(r, c)), b[2 * np][0], b[2 * np][1], b[2 * np + 1][0], b[2 * np + 1][1]);
      }
#pragma unroll
      for (int m = 0; m < MT; m++) {
        const int r = m * 16 + (lane & 15);
        const int c = kk + (lane >> 4);
        uint32_t a0, a1, a2, a3;
        ldsm4(smem_u32(W + kb * R * 128 + swz(r, c)), a0, a1, a2, a3);
#pragma unroll
        for (int n = 0; n < 4; n++) mma16816(acc[m][n], a0, a1, a2, a3, b[n][0], b[n][1]);
      }
    }
    // cross-warp reduction through smem
    const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int m = 0; m < MT; m++)
#pragma unroll
      for (int n = 0; n < 4; n++) {
        float *p = red + (warp * R + m * 16 + g) * 32 + n * 8 + 2 * t4;
        p[0] = acc[m][n][0]; p[1] = acc[m][n][1];
        p[8 * 32] = acc[m][n][2]; p[8 * 32 + 1] = acc[m][n][3];
      }
    __syncthreads();
    for (int i = threadIdx.x; i < R * 32; i += blockDim.x) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < 8; w++) s += red[w * R * 32 + i];
      if (rep == reps - 1) out[blockIdx.x * R * 32 + i] = s;
    }
    __syncthreads();
  }
  long long t1 = clock64();
  if (threadIdx.x == 0) cyc[blockIdx.x] = (t1 - t0) / reps;
}

__global__ void cl_kernel(int *p) { if (p) p[0] = 1; }

int main() {
  int sms = 0;
  CK(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0));
  uint4 *xb; float4 *xf; unsigned long long *ctr; long long *out; int *err;
  CK(cudaMalloc(&xb, XBYTES)); CK(cudaMalloc(&xf, XBYTES * 2)); CK(cudaMalloc(&ctr, 64));
  CK(cudaMalloc(&out, 16 * 1024)); CK(cudaMalloc(&err, 4)); CK(cudaMemset(err, 0, 4));
  const int smem = 200 * 1024;
  CK(cudaFuncSetAttribute(stage_probe, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  const char *names[3] = {"thread loads, 80 KB bf16", "thread loads, 40 KB fp32 quarter -> bf16", "cp.async.bulk, 80 KB bf16"};
  for (int mode = 0; mode < 3; mode++) {
    CK(cudaMemset(ctr, 0, 64));
    const int iters = 200;
    stage_probe<<<sms, 256, smem>>>(xb, xf, ctr, iters, mode, out, err);
    CK(cudaDeviceSynchronize());
    std::vector<long long> o(2 * sms);
    CK(cudaMemcpy(o.data(), out, 16 * sms, cudaMemcpyDeviceToHost));
    long long mx = 0, mn = 1LL << 60, sum = 0, bmx = 0;
    for (int i = 0; i < sms; i++) { mx = std::max(mx, o[2 * i]); mn = std::min(mn, o[2 * i]); sum += o[2 * i]; bmx = std::max(bmx, o[2 * i + 1]); }
    printf("staging (%s), %d CTAs: mean %lld ns, min %lld, max %lld; barrier %lld ns\n", names[mode], sms, sum / sms, mn, mx, bmx);
  }
  float *gout; long long *gcyc;
  CK(cudaMalloc(&gout, sms * 64 * 32 * 4 * 4)); CK(cudaMalloc(&gcyc, 8 * sms));
  {
    const int s16 = 16 * KD * 2 + XBYTES + 8 * 16 * 32 * 4;
    CK(cudaFuncSetAttribute(gemv_probe<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, s16));
    gemv_probe<1><<<sms, 256, s16>>>(50, gout, gcyc);
    CK(cudaDeviceSynchronize());
    long long c; CK(cudaMemcpy(&c, gcyc, 8, cudaMemcpyDeviceToHost));
    printf("mma.sync GEMV 16 rows x 1280 x 32: %lld cycles (%.2f us at 1.9 GHz)\n", c, c / 1900.0);
    const int s32 = 32 * KD * 2 + XBYTES + 8 * 32 * 32 * 4;
    CK(cudaFuncSetAttribute(gemv_probe<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, s32));
    gemv_probe<2><<<sms, 256, s32>>>(50, gout, gcyc);
    CK(cudaDeviceSynchronize());
    CK(cudaMemcpy(&c, gcyc, 8, cudaMemcpyDeviceToHost));
    printf("mma.sync GEMV 32 rows x 1280 x 32: %lld cycles (%.2f us)\n", c, c / 1900.0);
    const int s48 = 48 * KD * 2 + XBYTES + 8 * 48 * 32 * 4;
    if (s48 <= 227 * 1024) {
      CK(cudaFuncSetAttribute(gemv_probe<3>, cudaFuncAttributeMaxDynamicSharedMemorySize, s48));
      gemv_probe<3><<<sms, 256, s48>>>(50, gout, gcyc);
      CK(cudaDeviceSynchronize());
      CK(cudaMemcpy(&c, gcyc, 8, cudaMemcpyDeviceToHost));
      printf("mma.sync GEMV 48 rows x 1280 x 32: %lld cycles (%.2f us)\n", c, c / 1900.0);
    } else printf("48-row probe needs %d B smem, skipped\n", s48);
  }
  for (int cs : {2, 4, 8}) {
    for (int sm_kb : {100, 160, 200, 220}) {
      CK(cudaFuncSetAttribute(cl_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, sm_kb * 1024));
      CK(cudaFuncSetAttribute(cl_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(cs * 64);
      cfg.blockDim = dim3(256);
      cfg.dynamicSmemBytes = sm_kb * 1024;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = cs; attr[0].val.clusterDim.y = 1; attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr; cfg.numAttrs = 1;
      int n = 0;
      cudaError_t e = cudaOccupancyMaxActiveClusters(&n, cl_kernel, &cfg);
      printf("cluster size %d, %d KB smem: %d clusters (%d CTAs) %s\n", cs, sm_kb, n, n * cs, e == cudaSuccess ? "" : cudaGetErrorString(e));
    }
  }
  int e = 0;
  CK(cudaMemcpy(&e, err, 4, cudaMemcpyDeviceToHost));
  printf("err %d\n", e);
  return 0;
}
