/*
 * Seeded, counter-based synthetic input generator.
 *
 * This file holds no arithmetic of the MoE method itself: it only turns
 * (seed, stream, index) into reproducible pseudo-random numbers.  Both the
 * CUDA path and the CPU oracle read the buffers it fills, so they see
 * identical inputs.
 *
 * Definition (stated so that any implementation can reproduce it):
 *   mix(z)       = SplitMix64 output function (Steele, Lea & Flood, OOPSLA
 *                  2014): z += 0x9E3779B97F4A7C15;
 *                  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9;
 *                  z = (z ^ (z >> 27)) * 0x94D049BB133111EB;
 *                  return z ^ (z >> 31)
 *   key(seed,s)  = mix((seed << 32) ^ s)
 *   bits(i)      = mix(key + i)
 *   unif(i)      = ((bits(i) >> 11) + 0.5) * 2^-53            in (0, 1)
 *   normal(i)    : pair p = i / 2, u1 = unif(2p), u2 = unif(2p + 1),
 *                  r = sqrt(-2 ln u1); element 2p is r cos(2 pi u2),
 *                  element 2p+1 is r sin(2 pi u2)              (Box-Muller)
 *   f32 value    = (float)(std * normal(i))     (round to nearest)
 *   bf16 value   = f32 value rounded to nearest-even bfloat16
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static inline uint64_t sg_mix(uint64_t z) {
  z += 0x9E3779B97F4A7C15ULL;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t sg_key(uint64_t seed, uint64_t stream) {
  return sg_mix((seed << 32) ^ stream);
}

static inline double sg_unif(uint64_t key, uint64_t i) {
  return ((double)(sg_mix(key + i) >> 11) + 0.5) * 0x1.0p-53;
}

static inline double sg_normal(uint64_t key, uint64_t i) {
  uint64_t p = i >> 1;
  double u1 = sg_unif(key, 2 * p);
  double u2 = sg_unif(key, 2 * p + 1);
  double r = sqrt(-2.0 * log(u1));
  double a = 6.283185307179586476925286766559 * u2;
  return (i & 1) ? r * sin(a) : r * cos(a);
}

static inline uint16_t sg_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)(u >> 16); /* inf/nan: truncate */
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* Fill out[0..n) with normal values of indices [first, first + n). */
void synth_normal_f32(uint64_t seed, uint64_t stream, uint64_t first, uint64_t n,
                      double std, float* out) {
  uint64_t key = sg_key(seed, stream);
  int64_t nn = (int64_t)n;
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < nn; ++j) out[j] = (float)(std * sg_normal(key, first + (uint64_t)j));
}

void synth_normal_bf16(uint64_t seed, uint64_t stream, uint64_t first, uint64_t n,
                       double std, uint16_t* out) {
  uint64_t key = sg_key(seed, stream);
  int64_t nn = (int64_t)n;
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < nn; ++j)
    out[j] = sg_f32_to_bf16((float)(std * sg_normal(key, first + (uint64_t)j)));
}

/* Raw 64-bit draws, for tests of the generator itself. */
void synth_bits(uint64_t seed, uint64_t stream, uint64_t first, uint64_t n, uint64_t* out) {
  uint64_t key = sg_key(seed, stream);
  for (uint64_t j = 0; j < n; ++j) out[j] = sg_mix(key + first + j);
}
