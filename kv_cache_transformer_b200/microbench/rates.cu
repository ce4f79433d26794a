// rates.cu — costs of the sm_100a operations the decode step is built from.
//
// Measured on one GPU, printed as text:
//   * mma.sync m16n8k16 bf16 throughput per SM (4, 8, 16 warps, operands in
//     registers);
//   * tcgen05.mma issue cost by (M, N), K = 16, with the A and B shared-memory
//     tiles held or rotated every four instructions;
//   * a grid barrier of one CTA per SM (release add, acquire polling);
//   * the round trip of a flag between two CTAs;
//   * the latency of a dependent L2 load.
// Every wait is bounded; a timeout sets a flag that is printed.
#include <cstdio>
#include <cstdlib>
#include <cstdint>
#include <vector>
#include <cuda_runtime.h>
#include "nc_sm100.cuh"
using namespace nc::sm100;

#define CK(x) do { cudaError_t e_ = (x); if (e_ != cudaSuccess) { printf("CUDA %s at %d: %s\n", #x, __LINE__, cudaGetErrorString(e_)); exit(1);} } while (0)

// ---------------------------------------------------------------- mma.sync
__global__ void mma_sync_tput(int iters, float *out, long long *cyc) {
  uint32_t a[4] = {threadIdx.x, threadIdx.x * 3u, threadIdx.x * 5u, threadIdx.x * 7u};
  uint32_t b0 = threadIdx.x * 11u, b1 = threadIdx.x * 13u;
  float d[8][4];
  for (int i = 0; i < 8; i++) for (int j = 0; j < 4; j++) d[i][j] = 0.f;
  __syncthreads();
  long long t0 = clock64();
  for (int it = 0; it < iters; it++) {
#pragma unroll
    for (int i = 0; i < 8; i++)
      asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                   : "+f"(d[i][0]), "+f"(d[i][1]), "+f"(d[i][2]), "+f"(d[i][3])
                   : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
  __syncthreads();
  long long t1 = clock64();
  float s = 0.f;
  for (int i = 0; i < 8; i++) for (int j = 0; j < 4; j++) s += d[i][j];
  out[blockIdx.x * blockDim.x + threadIdx.x] = s;
  if (threadIdx.x == 0) cyc[blockIdx.x] = t1 - t0;
}

// ---------------------------------------------------------------- tcgen05 issue rate
// smem: NSLOT A tiles of 128 rows x 128 B (16 KB) then NSLOT B tiles of 256 rows x 128 B (32 KB)
constexpr int NSLOT = 3;
__global__ void tc_rate(int M, int N, int n_mma, int rotate_a, int rotate_b, long long *cyc) {
  extern __shared__ __align__(1024) uint8_t sm[];
  uint8_t *base = sm + ((1024 - (smem_u32(sm) & 1023)) & 1023);
  uint8_t *A = base, *Bt = base + NSLOT * 16384;
  __shared__ uint64_t bar;
  __shared__ uint32_t tslot;
  for (int i = threadIdx.x; i < NSLOT * (16384 + 32768) / 4; i += blockDim.x) reinterpret_cast<uint32_t *>(base)[i] = 0x3c003c00u;
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (threadIdx.x == 0) { mbar_init(&bar, 1); fence_barrier_init(); }
  if (threadIdx.x < 32) tmem_alloc(&tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tslot;
  if (threadIdx.x == 0) {
    const uint32_t idesc = idesc_bf16_f32(M, N);
    // warm
    for (int i = 0; i < 8; i++) mma_bf16(tmem, desc_k_sw128(smem_u32(A)), desc_k_sw128(smem_u32(Bt)), idesc, 0);
    mma_commit(&bar);
    volatile int ab = 0; uint32_t st = 0;
    mbar_wait(&bar, 0, &ab, &st);
    long long t0 = clock64();
    for (int i = 0; i < n_mma; i++) {
      const int sa = rotate_a ? (i / 4) % NSLOT : 0, sb = rotate_b ? (i / 4) % NSLOT : 0;
      const uint32_t a = smem_u32(A + sa * 16384) + 32 * (i & 3), b = smem_u32(Bt + sb * 32768) + 32 * (i & 3);
      mma_bf16(tmem + (uint32_t)((i & 1) * 256 * 0), desc_k_sw128(a), desc_k_sw128(b), idesc, 1);
    }
    mma_commit(&bar);
    mbar_wait(&bar, 1, &ab, &st);
    long long t1 = clock64();
    cyc[0] = t1 - t0;
    cyc[1] = st;
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) { tc_fence_after(); tmem_dealloc(tmem, 512); }
}

// ---------------------------------------------------------------- grid barrier
__device__ __forceinline__ bool poll_ge(unsigned long long *p, unsigned long long target) {
  for (uint32_t it = 0; it < (1u << 22); it++) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    if (v >= target) return true;
  }
  return false;
}

__global__ void grid_bar(unsigned long long *ctr, int n, long long *ns, int *err) {
  __syncthreads();
  uint64_t t0 = global_ns();
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  for (int i = 0; i < n; i++) {
    __syncthreads();
    if (bad) break;
    if (threadIdx.x == 0) {
      asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(ctr) : "memory");
      if (!poll_ge(ctr, (unsigned long long)(i + 1) * gridDim.x)) { atomicOr(err, 1); bad = 1; }
    }
    __syncthreads();
  }
  uint64_t t1 = global_ns();
  if (threadIdx.x == 0) ns[blockIdx.x] = (long long)(t1 - t0);
}

// ping-pong between block 0 and block `peer` through a global flag
__global__ void ping(unsigned long long *flag, int n, int peer, long long *ns, int *err) {
  if (threadIdx.x != 0) return;
  if (blockIdx.x != 0 && blockIdx.x != peer) return;
  const bool me0 = blockIdx.x == 0;
  uint64_t t0 = global_ns();
  for (int i = 0; i < n; i++) {
    if (me0) {
      asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(flag), "l"((unsigned long long)(2 * i + 1)) : "memory");
      if (!poll_ge(flag, 2ull * i + 2)) { atomicOr(err, 2); return; }
    } else {
      if (!poll_ge(flag, 2ull * i + 1)) { atomicOr(err, 4); return; }
      asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(flag), "l"((unsigned long long)(2 * i + 2)) : "memory");
    }
  }
  uint64_t t1 = global_ns();
  if (me0) ns[0] = (long long)(t1 - t0);
}

// dependent L2 load latency: pointer chase
__global__ void chase(const unsigned *next, int hops, long long *ns, unsigned *sink) {
  if (threadIdx.x) return;
  unsigned j = 0;
  uint64_t t0 = global_ns();
  for (int i = 0; i < hops; i++) j = __ldcg(next + j);
  uint64_t t1 = global_ns();
  ns[0] = (long long)(t1 - t0);
  sink[0] = j;
}

int main() {
  int sms = 0;
  CK(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0));
  int clk = 0;
  CK(cudaDeviceGetAttribute(&clk, cudaDevAttrClockRate, 0));
  printf("sms %d clock %d kHz\n", sms, clk);
  long long *dcyc; float *dout; int *derr;
  CK(cudaMalloc(&dcyc, 4096 * 8)); CK(cudaMalloc(&dout, 1 << 22)); CK(cudaMalloc(&derr, 4));
  CK(cudaMemset(derr, 0, 4));
  // mma.sync
  for (int warps : {4, 8, 16}) {
    const int iters = 4096;
    mma_sync_tput<<<sms, 32 * warps>>>(iters, dout, dcyc);
    CK(cudaDeviceSynchronize());
    std::vector<long long> c(sms);
    CK(cudaMemcpy(c.data(), dcyc, 8 * sms, cudaMemcpyDeviceToHost));
    double mx = 0; for (auto v : c) mx = v > mx ? v : mx;
    double macs = (double)warps * iters * 8 * 2048;
    printf("mma.sync m16n8k16 bf16: %d warps/SM: %.0f MAC/cycle/SM (%.1f cycles per mma per SMSP)\n", warps, macs / mx,
           mx / ((double)warps * iters * 8 / 4));
  }
  // tcgen05 rates
  CK(cudaFuncSetAttribute(tc_rate, cudaFuncAttributeMaxDynamicSharedMemorySize, NSLOT * 49152 + 1024));
  int shapes[][2] = {{128, 256}, {128, 128}, {128, 64}, {128, 32}, {128, 16}, {64, 256}, {64, 128}, {64, 64}, {64, 32}};
  for (auto &sh : shapes) {
    for (int rot = 0; rot < 4; rot++) {
      const int n_mma = 4096;
      tc_rate<<<1, 128, NSLOT * 49152 + 1024>>>(sh[0], sh[1], n_mma, rot & 1, (rot >> 1) & 1, dcyc);
      CK(cudaDeviceSynchronize());
      long long c[2];
      CK(cudaMemcpy(c, dcyc, 16, cudaMemcpyDeviceToHost));
      printf("tcgen05 M=%d N=%d rotA=%d rotB=%d: %.1f cycles/mma (status %lld)\n", sh[0], sh[1], rot & 1, (rot >> 1) & 1,
             (double)c[0] / n_mma, c[1]);
    }
  }
  // grid barrier, one CTA per SM (big smem request keeps one per SM)
  unsigned long long *ctr;
  CK(cudaMalloc(&ctr, 64));
  CK(cudaFuncSetAttribute(grid_bar, cudaFuncAttributeMaxDynamicSharedMemorySize, 150000));
  for (int grid : {sms, 132, 64}) {
    CK(cudaMemset(ctr, 0, 64));
    const int n = 2000;
    grid_bar<<<grid, 128, 150000>>>(ctr, n, dcyc, derr);
    CK(cudaDeviceSynchronize());
    std::vector<long long> c(grid);
    CK(cudaMemcpy(c.data(), dcyc, 8 * grid, cudaMemcpyDeviceToHost));
    long long mx = 0; for (auto v : c) mx = v > mx ? v : mx;
    printf("grid barrier, %d CTAs: %.0f ns per barrier\n", grid, (double)mx / n);
  }
  CK(cudaFuncSetAttribute(ping, cudaFuncAttributeMaxDynamicSharedMemorySize, 150000));
  for (int peer : {1, 2, 8, 37, 74, 100, 147}) {
    if (peer >= sms) continue;
    CK(cudaMemset(ctr, 0, 64));
    const int n = 2000;
    ping<<<sms, 32, 150000>>>(ctr, n, peer, dcyc, derr);
    CK(cudaDeviceSynchronize());
    long long c;
    CK(cudaMemcpy(&c, dcyc, 8, cudaMemcpyDeviceToHost));
    printf("ping-pong CTA 0 <-> CTA %d: %.0f ns round trip\n", peer, (double)c / n);
  }
  // pointer chase in L2 (4 MB, random cycle)
  {
    const int n = 1 << 20;
    std::vector<unsigned> perm(n), nxt(n);
    for (int i = 0; i < n; i++) perm[i] = i;
    srand(1);
    for (int i = n - 1; i > 0; i--) { int j = rand() % (i + 1); std::swap(perm[i], perm[j]); }
    for (int i = 0; i < n; i++) nxt[perm[i]] = perm[(i + 1) % n];
    unsigned *dn, *sink;
    CK(cudaMalloc(&dn, 4 * n)); CK(cudaMalloc(&sink, 4));
    CK(cudaMemcpy(dn, nxt.data(), 4 * n, cudaMemcpyHostToDevice));
    chase<<<1, 32>>>(dn, 20000, dcyc, sink);  // warm L2
    CK(cudaDeviceSynchronize());
    chase<<<1, 32>>>(dn, 20000, dcyc, sink);
    CK(cudaDeviceSynchronize());
    long long c;
    CK(cudaMemcpy(&c, dcyc, 8, cudaMemcpyDeviceToHost));
    printf("dependent L2 load (4 MB working set): %.0f ns per hop\n", (double)c / 20000);
  }
  int err = 0;
  CK(cudaMemcpy(&err, derr, 4, cudaMemcpyDeviceToHost));
  printf("err flags %d\n", err);
  return 0;
}
