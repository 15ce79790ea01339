/*
 * Seeded synthetic inputs for the BitLinear W1.58A8 forward.
 *
 * This file draws random numbers and nothing else: it holds none of the
 * BitLinear arithmetic (no absmean, no ternarisation, no packing, no
 * activation quantisation, no product, no dequantisation).  Both the CPU
 * oracle tests and the CUDA path consume the arrays it writes, so the two
 * sides see byte-identical inputs.
 *
 * Generator: SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast Splittable
 * Pseudorandom Number Generators", OOPSLA 2014), used as a counter-based
 * generator: value i of stream s under seed S is mix64(key(S, s) + (i+1)*G)
 * with G the golden-ratio increment.  Normals come from the Box-Muller
 * transform (cosine branch only, one normal per pair of uniforms) in double
 * precision, rounded once to fp32.  Because every element depends only on
 * (seed, stream, index), results do not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define SYNTH_GOLDEN 0x9e3779b97f4a7c15ULL

static inline uint64_t synth_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
  return z ^ (z >> 31);
}

static inline uint64_t synth_key(uint64_t seed, uint64_t stream) {
  return synth_mix64(synth_mix64(seed + SYNTH_GOLDEN) ^ (stream * 0xd1342543de82ef95ULL + 1));
}

static inline uint64_t synth_draw(uint64_t key, uint64_t counter) {
  return synth_mix64(key + (counter + 1) * SYNTH_GOLDEN);
}

/* One standard normal from counter pair (2i, 2i+1). */
static inline double synth_std_normal(uint64_t key, uint64_t i) {
  uint64_t a = synth_draw(key, 2 * i);
  uint64_t b = synth_draw(key, 2 * i + 1);
  double u1 = ((double)(a >> 11) + 1.0) * 0x1.0p-53; /* (0, 1] */
  double u2 = (double)(b >> 11) * 0x1.0p-53;         /* [0, 1) */
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925286766559 * u2);
}

/* out[j] = fp32(mean + std * z_{offset+j}), j in [0, n). */
void synth_normal_f32(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n,
                      double mean, double std, float* out) {
  uint64_t key = synth_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < n; ++j) {
    out[j] = (float)(mean + std * synth_std_normal(key, offset + (uint64_t)j));
  }
}

/* Uniform integer in [0, range) by the multiply-shift map of a 64-bit draw. */
static inline uint64_t synth_below(uint64_t key, uint64_t counter, uint64_t range) {
  unsigned __int128 p = (unsigned __int128)synth_draw(key, counter) * range;
  return (uint64_t)(p >> 64);
}

/*
 * The first `count` entries of a seeded Fisher-Yates shuffle of [0, K):
 * `count` distinct channel indices, in selection order.  Returns 0, or -1
 * when count is outside [0, K].
 */
int synth_choose_channels(uint64_t seed, uint64_t stream, int32_t K, int32_t count,
                          int32_t* out) {
  if (K < 0 || count < 0 || count > K) return -1;
  uint64_t key = synth_key(seed, stream);
  int32_t* perm = out; /* uses out[0..K) as scratch: caller passes K slots */
  for (int32_t i = 0; i < K; ++i) perm[i] = i;
  for (int32_t i = 0; i < count; ++i) {
    int32_t j = i + (int32_t)synth_below(key, (uint64_t)i, (uint64_t)(K - i));
    int32_t t = perm[i];
    perm[i] = perm[j];
    perm[j] = t;
  }
  return 0;
}

/*
 * Activations: x[m][k] = fp32(z * (k is an outlier channel ? outlier_scale : 1)),
 * z ~ N(0, 1) from stream `stream`, element index m*K + k.  The outlier mask
 * has K bytes (nonzero = outlier).
 */
void synth_activations_f32(uint64_t seed, uint64_t stream, int64_t M, int64_t K,
                           const uint8_t* outlier_mask, double outlier_scale, float* out) {
  uint64_t key = synth_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < M * K; ++i) {
    double z = synth_std_normal(key, (uint64_t)i);
    if (outlier_mask && outlier_mask[i % K]) z *= outlier_scale;
    out[i] = (float)z;
  }
}

/* fp32 -> bf16 bit pattern, round to nearest even (inputs are finite). */
void synth_f32_to_bf16(const float* in, int64_t n, uint16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    uint32_t u;
    memcpy(&u, &in[i], 4);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    out[i] = (uint16_t)(u >> 16);
  }
}

/* bf16 bit pattern -> fp32 (exact). */
void synth_bf16_to_f32(const uint16_t* in, int64_t n, float* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    uint32_t u = (uint32_t)in[i] << 16;
    memcpy(&out[i], &u, 4);
  }
}
