// nc_noalloc.cu — decode attention that allocates nothing.
//
// nc_attention_decode_bf16 needs a scratch workspace for its split-KV
// partial results, and someone has to allocate it. Some callers cannot: an
// inference server whose memory manager owns all device memory and gives
// kernels no way to request more, a plugin loaded into a host framework
// that exposes no workspace hook, or a deployment that must keep a fixed,
// known device footprint. For them this file keeps the scratch in a
// file-scope __device__ array that is part of the library image: every GPU
// that loads the library holds it (about 4.3 MB) until the process exits,
// and no call here allocates or frees device memory.
#include <stdio.h>

#include "nc_internal.h"
#include "nc_kernels.h"

namespace {

constexpr int kStaticMaxBatch = 32;   // sequences per call
constexpr int kStaticMaxSplits = 16;  // the planning rule never uses more
constexpr size_t kPartFloats = (size_t)kStaticMaxBatch * kStaticMaxSplits * 16 * 130;

// Split-KV partials (m, l, O per head row), then one counter per sequence.
static __device__ __align__(256) float g_decode_scratch[kPartFloats + kStaticMaxBatch];

// Device address of g_decode_scratch on the current device. In host code the
// array's name is only a host-side handle, so the kernel must be given this
// address instead. It is looked up on every call (a host-side query, cheap):
// a cached address would dangle after cudaDeviceReset unloads the module.
// The first lookup on a device loads the library's module there, which is
// why the first call on each device belongs before any stream capture.
int scratch_address(void **out) {
  void *p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
  if (e != cudaSuccess || !p) {
    char msg[160];
    snprintf(msg, sizeof msg, "cudaGetSymbolAddress of the static scratch failed: %s", cudaGetErrorString(e));
    return nc::set_error(NC_ECUDA, msg);
  }
  *out = p;
  return NC_OK;
}

}  // namespace

extern "C" int nc_attention_decode_bf16_static(const void *d_q, const void *d_k, const void *d_v, const int32_t *d_pos,
                                               int B, int H, int max_seq, void *d_y, void *stream) {
  if (!d_q || !d_k || !d_v || !d_pos || !d_y) return nc::set_error(NC_EINVAL, "null pointer");
  if (B <= 0 || H <= 0 || H > 16 || max_seq <= 0) return nc::set_error(NC_EINVAL, "bad decode attention shape");
  if (B > kStaticMaxBatch) {
    char msg[128];
    snprintf(msg, sizeof msg, "B=%d exceeds the static scratch limit of %d sequences", B, kStaticMaxBatch);
    return nc::set_error(NC_EINVAL, msg);
  }
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return nc::set_error(NC_ECUDA, "no CUDA device");
  int chunk = 0, splits = 0;
  nc::attn_decode_plan(B, max_seq, sms, &chunk, &splits);
  if (splits > kStaticMaxSplits || nc::attn_decode_partial_floats(B, splits) > kPartFloats)
    return nc::set_error(NC_EINVAL, "max_seq needs more key splits than the static scratch holds");
  void *base = nullptr;
  int rc = scratch_address(&base);
  if (rc != NC_OK) return rc;
  float *part = static_cast<float *>(base);
  unsigned *counters = reinterpret_cast<unsigned *>(part + kPartFloats);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The array keeps whatever the last call left; the per-sequence counters
  // must start at zero, so clear them (the partials are always overwritten).
  cudaError_t e = cudaMemsetAsync(counters, 0, sizeof(unsigned) * (size_t)B, s);
  if (e == cudaSuccess)
    e = nc::k_dec_attn(d_q, d_k, d_v, d_pos, nullptr, B, H, max_seq, chunk, splits, part, counters, d_y, s);
  if (e != cudaSuccess) return nc::set_error(NC_ECUDA, cudaGetErrorString(e));
  return NC_OK;
}
