/*
 * Seeded synthetic inputs for the temporal-module workloads.
 *
 * This file is shared input infrastructure: both the fp64 oracle's tests and
 * the CUDA path's tests and benchmark draw their inputs from it.  It holds no
 * arithmetic of the temporal modules themselves, only a counter-based random
 * number generator:
 *
 *   - SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast splittable pseudorandom
 *     number generators", OOPSLA 2014): state advances by the golden-ratio
 *     increment 0x9E3779B97F4A7C15 and each output is the finaliser
 *     z ^= z>>30; z *= 0xBF58476D1CE4E5B9; z ^= z>>27; z *= 0x94D049BB133111EB;
 *     z ^= z>>31.  Output n of a stream seeded with s is therefore
 *     mix(s + (n+1) * increment), which lets any element be drawn on its own.
 *   - Box-Muller (G. Box, M. Muller, Ann. Math. Stat. 29, 1958), cosine
 *     branch only: n = sqrt(-2 ln u1) cos(2 pi u2) with u1 in (0,1].
 *
 * Element i of tensor `tid` under seed `seed` is
 *   key = splitmix64_at(seed, tid)
 *   u1  = 1 - top53(splitmix64_at(key, 2i))      (in (0,1])
 *   u2  =     top53(splitmix64_at(key, 2i + 1))  (in [0,1))
 *   x   = mean + std * sqrt(-2 ln u1) * cos(2 pi u2)
 * rounded to float (round to nearest even) and, for bf16 tensors, from float
 * to bf16 (round to nearest even).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define SM64_INC 0x9E3779B97F4A7C15ULL

static inline uint64_t sm64_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* Output number n (0-based) of a SplitMix64 stream seeded with s. */
uint64_t synth_splitmix64_at(uint64_t s, uint64_t n) {
  return sm64_mix(s + (n + 1) * SM64_INC);
}

static inline double top53(uint64_t z) { return (double)(z >> 11) * 0x1.0p-53; }

static inline double normal_at(uint64_t key, uint64_t i) {
  const double u1 = 1.0 - top53(synth_splitmix64_at(key, 2 * i));
  const double u2 = top53(synth_splitmix64_at(key, 2 * i + 1));
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925286766559 * u2);
}

/* float -> bf16 bit pattern, round to nearest even (NaN kept quiet). */
static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

uint64_t synth_stream_key(uint64_t seed, uint64_t tid) { return synth_splitmix64_at(seed, tid); }

/* Standard normals (fp64, unrounded) for elements [first, first+n). */
void synth_normal_f64(double* out, int64_t n, int64_t first, uint64_t seed, uint64_t tid,
                      double mean, double std) {
  const uint64_t key = synth_stream_key(seed, tid);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = mean + std * normal_at(key, (uint64_t)(first + i));
}

void synth_normal_f32(float* out, int64_t n, int64_t first, uint64_t seed, uint64_t tid,
                      double mean, double std) {
  const uint64_t key = synth_stream_key(seed, tid);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = (float)(mean + std * normal_at(key, (uint64_t)(first + i)));
}

void synth_normal_bf16(uint16_t* out, int64_t n, int64_t first, uint64_t seed, uint64_t tid,
                       double mean, double std) {
  const uint64_t key = synth_stream_key(seed, tid);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i)
    out[i] = f32_to_bf16_rne((float)(mean + std * normal_at(key, (uint64_t)(first + i))));
}

/* Round an fp32 array to bf16 bit patterns (round to nearest even). */
void synth_f32_to_bf16(const float* in, uint16_t* out, int64_t n) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16_rne(in[i]);
}

/* Widen bf16 bit patterns to fp32 (exact). */
void synth_bf16_to_f32(const uint16_t* in, float* out, int64_t n) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    uint32_t u = (uint32_t)in[i] << 16;
    memcpy(&out[i], &u, 4);
  }
}
