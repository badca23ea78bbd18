/*
 * Seeded synthetic inputs for the Llama-style decode workloads.
 *
 * This file holds no arithmetic of the decode step itself: it only turns
 * (key, element index) into bytes.  Both the CPU oracle's tests and the GPU
 * engine consume the bytes it writes, so the bytes -- not any library PRNG
 * -- are the contract.
 *
 * Generator (counter based, so any element can be produced independently and
 * in parallel):
 *   gamma      = 0x9E3779B97F4A7C15
 *   mix(z)     = SplitMix64 finaliser:
 *                  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9
 *                  z = (z ^ (z >> 27)) * 0x94D049BB133111EB
 *                  z =  z ^ (z >> 31)
 *   word(k, c) = mix(k + (c + 1) * gamma)          (all arithmetic mod 2^64)
 *
 * Normal values (Box-Muller, one pair per pair index i):
 *   a  = word(k, 2i), b = word(k, 2i + 1)
 *   u1 = ((a >> 11) + 1) * 2^-53      in (0, 1]
 *   u2 =  (b >> 11)      * 2^-53      in [0, 1)
 *   r  = sqrt(-2 ln u1),  t = 2 pi u2
 *   element 2i   = (float)(sigma * r * cos t)
 *   element 2i+1 = (float)(sigma * r * sin t)
 *   then rounded float -> bf16 with round-to-nearest-even.
 *
 * Uniform integers in [lo, hi):  lo + ((word(k, i) >> 32) * (hi - lo)) >> 32.
 *
 * Stream keys: key(seed, a, b, c) = mix(mix(mix(mix(seed) ^ a) ^ b) ^ c) with
 * every component shifted by one so that zero ids still change the key.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <string.h>

#define SYN_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t syn_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t syn_word(uint64_t key, uint64_t c) {
  return syn_mix(key + (c + 1ULL) * SYN_GAMMA);
}

static inline uint16_t syn_f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

uint64_t syn_key(uint64_t seed, uint64_t a, uint64_t b, uint64_t c) {
  uint64_t k = syn_mix(seed + SYN_GAMMA);
  k = syn_mix(k ^ (a + 1ULL));
  k = syn_mix(k ^ ((b + 1ULL) * 0x100000001B3ULL));
  k = syn_mix(k ^ ((c + 1ULL) * 0xC2B2AE3D27D4EB4FULL));
  return k;
}

/* Normal pair i of stream `key`, as two floats. */
static inline void syn_normal_pair(uint64_t key, uint64_t i, double sigma,
                                   float *z0, float *z1) {
  const double two_pi = 6.283185307179586476925286766559;
  uint64_t a = syn_word(key, 2 * i), b = syn_word(key, 2 * i + 1);
  double u1 = (double)((a >> 11) + 1ULL) * 0x1.0p-53;
  double u2 = (double)(b >> 11) * 0x1.0p-53;
  double r = sqrt(-2.0 * log(u1)), t = two_pi * u2;
  *z0 = (float)(sigma * r * cos(t));
  *z1 = (float)(sigma * r * sin(t));
}

/*
 * out[j] = bf16 of element (first + j) of the normal stream `key`, j < n.
 * Elements are indexed globally so a tensor can be filled in pieces.
 */
void syn_normal_bf16(uint16_t *out, uint64_t n, uint64_t key, double sigma,
                     uint64_t first) {
  if (n == 0) return;
  int64_t lo = (int64_t)(first / 2), hi = (int64_t)((first + n - 1) / 2);
#pragma omp parallel for schedule(static)
  for (int64_t i = lo; i <= hi; ++i) {
    float z0, z1;
    syn_normal_pair(key, (uint64_t)i, sigma, &z0, &z1);
    uint64_t e0 = 2 * (uint64_t)i, e1 = e0 + 1;
    if (e0 >= first && e0 < first + n) out[e0 - first] = syn_f32_to_bf16_rne(z0);
    if (e1 >= first && e1 < first + n) out[e1 - first] = syn_f32_to_bf16_rne(z1);
  }
}

/*
 * out[j] = bf16 of (mean + element (first + j)) of the normal stream `key`:
 * the same Box-Muller value as syn_normal_bf16, offset by `mean` in float
 * before the rounding (norm weights around 1).
 */
void syn_normal_bf16_mean(uint16_t *out, uint64_t n, uint64_t key, double mean,
                          double sigma, uint64_t first) {
  if (n == 0) return;
  int64_t lo = (int64_t)(first / 2), hi = (int64_t)((first + n - 1) / 2);
#pragma omp parallel for schedule(static)
  for (int64_t i = lo; i <= hi; ++i) {
    float z0, z1;
    syn_normal_pair(key, (uint64_t)i, sigma, &z0, &z1);
    uint64_t e0 = 2 * (uint64_t)i, e1 = e0 + 1;
    if (e0 >= first && e0 < first + n) out[e0 - first] = syn_f32_to_bf16_rne((float)mean + z0);
    if (e1 >= first && e1 < first + n) out[e1 - first] = syn_f32_to_bf16_rne((float)mean + z1);
  }
}

/* Same stream as syn_normal_bf16 but kept as float (used by the tests of the
 * generator itself). */
void syn_normal_f32(float *out, uint64_t n, uint64_t key, double sigma) {
  int64_t pairs = (int64_t)((n + 1) / 2);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < pairs; ++i) {
    float z0, z1;
    syn_normal_pair(key, (uint64_t)i, sigma, &z0, &z1);
    out[2 * i] = z0;
    if ((uint64_t)(2 * i + 1) < n) out[2 * i + 1] = z1;
  }
}

/* out[i] uniform in [lo, hi), i < n. */
void syn_uniform_i32(int32_t *out, uint64_t n, uint64_t key, int32_t lo,
                     int32_t hi) {
  uint64_t span = (uint64_t)((int64_t)hi - (int64_t)lo);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < (int64_t)n; ++i) {
    uint64_t w = syn_word(key, (uint64_t)i) >> 32;
    out[i] = (int32_t)((int64_t)lo + (int64_t)((w * span) >> 32));
  }
}

/* Fill a bf16 tensor with one value (norm weights). */
void syn_fill_bf16(uint16_t *out, uint64_t n, float value) {
  uint16_t v = syn_f32_to_bf16_rne(value);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < (int64_t)n; ++i) out[i] = v;
}
