/*
 * ncgen.c — seeded synthetic inputs for the KV-cache Transformer engine.
 *
 * This file holds NO arithmetic of the model. It only draws random numbers:
 * weight tensors N(0, std), Zipf(s) and uniform token ids, and Gumbel noise.
 * Both the CUDA engine's tests/benchmarks and the CPU oracle consume its
 * output; neither side's arithmetic lives here.
 *
 * Generator: splitmix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014; the 64-bit finaliser constants are the
 * published "Mix13/variant 13" ones). splitmix64's state advances by the
 * golden-ratio gamma, so output i of a stream is mix64(base + (i+1)*gamma):
 * any index can be computed directly, which lets OpenMP threads fill one
 * stream in parallel and still produce the same sequence.
 *
 * Streams: every tensor/token array gets its own stream id, and
 *   base(seed, stream) = mix64(seed * GAMMA ^ (stream + STREAM_SALT)).
 */
#include <stdint.h>
#include <stddef.h>
#include <stdlib.h>
#include <math.h>

#define NCG_GAMMA 0x9E3779B97F4A7C15ULL
#define NCG_STREAM_SALT 0x632BE59BD9B4E019ULL

static inline uint64_t ncg_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* Output i (0-based) of the splitmix64 sequence whose state starts at `state`. */
uint64_t ncg_splitmix64_at(uint64_t state, uint64_t i) {
  return ncg_mix64(state + (i + 1) * NCG_GAMMA);
}

uint64_t ncg_stream_base(uint64_t seed, uint64_t stream) {
  return ncg_mix64((seed * NCG_GAMMA) ^ (stream + NCG_STREAM_SALT));
}

/* Uniform on the open interval (0,1): top 53 bits, offset by half an ulp. */
static inline double ncg_u01(uint64_t base, uint64_t i) {
  return ((double)(ncg_splitmix64_at(base, i) >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

void ncg_uniform01(uint64_t seed, uint64_t stream, int64_t n, double *out) {
  uint64_t base = ncg_stream_base(seed, stream);
#pragma omp parallel for schedule(static) if (n > 65536)
  for (int64_t i = 0; i < n; i++) out[i] = ncg_u01(base, (uint64_t)i);
}

/* Standard-normal draw for element i: Box-Muller on the pair (2j, 2j+1),
 * j = i/2; even i takes the cosine branch, odd i the sine branch. */
static inline double ncg_normal_at(uint64_t base, uint64_t i) {
  uint64_t j = i >> 1;
  double u1 = ncg_u01(base, 2 * j), u2 = ncg_u01(base, 2 * j + 1);
  double r = sqrt(-2.0 * log(u1));
  double a = 6.283185307179586476925286766559 * u2;
  return (i & 1) ? r * sin(a) : r * cos(a);
}

/* fp32 -> bf16 bits, round to nearest, ties to even (inputs are finite). */
static inline uint16_t ncg_f32_to_bf16_rne(float f) {
  union { float f; uint32_t u; } v;
  v.f = f;
  uint32_t lsb = (v.u >> 16) & 1u;
  return (uint16_t)((v.u + 0x7FFFu + lsb) >> 16);
}

void ncg_round_bf16(const float *in, int64_t n, uint16_t *out) {
#pragma omp parallel for schedule(static) if (n > 65536)
  for (int64_t i = 0; i < n; i++) out[i] = ncg_f32_to_bf16_rne(in[i]);
}

/* n draws of N(0, std^2): as fp32 (out_f32) or rounded fp32->bf16 (out_bf16).
 * Exactly one of the outputs is non-null. The fp32 value is formed first,
 * then rounded, so the bf16 blob is the RNE image of the fp32 one. */
void ncg_normal(uint64_t seed, uint64_t stream, int64_t n, double std,
                float *out_f32, uint16_t *out_bf16) {
  uint64_t base = ncg_stream_base(seed, stream);
#pragma omp parallel for schedule(static) if (n > 65536)
  for (int64_t i = 0; i < n; i++) {
    float v = (float)(std * ncg_normal_at(base, (uint64_t)i));
    if (out_f32) out_f32[i] = v;
    else out_bf16[i] = ncg_f32_to_bf16_rne(v);
  }
}

/* Token ids uniform in [0, vocab): floor(u * vocab). */
void ncg_tokens_uniform(uint64_t seed, uint64_t stream, int64_t n, int vocab, int32_t *out) {
  uint64_t base = ncg_stream_base(seed, stream);
  for (int64_t i = 0; i < n; i++) {
    int64_t t = (int64_t)(ncg_u01(base, (uint64_t)i) * (double)vocab);
    out[i] = (int32_t)(t >= vocab ? vocab - 1 : t);
  }
}

/* Token ids Zipf(s) over ranks 1..vocab (p(r) proportional to r^-s), token =
 * rank-1, by inverse CDF in double: smallest r with CDF(r) >= u * CDF(vocab). */
int ncg_tokens_zipf(uint64_t seed, uint64_t stream, int64_t n, int vocab, double s, int32_t *out) {
  double *cdf = (double *)malloc(sizeof(double) * (size_t)vocab);
  if (!cdf) return -1;
  double acc = 0.0;
  for (int r = 1; r <= vocab; r++) { acc += pow((double)r, -s); cdf[r - 1] = acc; }
  uint64_t base = ncg_stream_base(seed, stream);
#pragma omp parallel for schedule(static) if (n > 65536)
  for (int64_t i = 0; i < n; i++) {
    double target = ncg_u01(base, (uint64_t)i) * acc;
    int lo = 0, hi = vocab - 1;
    while (lo < hi) {
      int mid = (lo + hi) >> 1;
      if (cdf[mid] >= target) hi = mid; else lo = mid + 1;
    }
    out[i] = lo;
  }
  free(cdf);
  return 0;
}

/* Standard Gumbel noise g = -ln(-ln u), u uniform on (0,1), as fp32. */
void ncg_gumbel(uint64_t seed, uint64_t stream, int64_t n, float *out) {
  uint64_t base = ncg_stream_base(seed, stream);
#pragma omp parallel for schedule(static) if (n > 65536)
  for (int64_t i = 0; i < n; i++) out[i] = (float)(-log(-log(ncg_u01(base, (uint64_t)i))));
}
