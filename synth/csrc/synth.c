/*
 * Seeded synthetic tensor generator shared by the CUDA path's tests/bench and
 * the oracle's tests.  It holds none of the attention arithmetic: it only
 * turns (seed, tensor id, flat index) into an N(0,1) sample.
 *
 * Generator (stated so either side could re-derive it):
 *   SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
 *   generators", OOPSLA 2014) used as a counter-based hash:
 *     mix(x): z = x + 0x9E3779B97F4A7C15;
 *             z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9;
 *             z = (z ^ (z >> 27)) * 0x94D049BB133111EB;
 *             return z ^ (z >> 31);
 *   stream base  = mix(mix(seed) + tensor_id)
 *   element k    : a = mix(base + 2k), b = mix(base + 2k + 1)
 *                  u1 = ((a >> 11) + 1) * 2^-53   in (0, 1]
 *                  u2 = (b >> 11) * 2^-53         in [0, 1)
 *   Box-Muller (Box and Muller, 1958), cosine branch, in double:
 *                  z = sqrt(-2 ln u1) * cos(2 pi u2)
 *   then rounded to fp32 (and optionally to bf16, round-to-nearest-even).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static inline uint64_t sm_mix(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ULL;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

uint64_t synth_splitmix64(uint64_t x) { return sm_mix(x); }

static inline float normal_at(uint64_t base, uint64_t k) {
  const double two_pi = 6.283185307179586476925286766559;
  uint64_t a = sm_mix(base + 2 * k);
  uint64_t b = sm_mix(base + 2 * k + 1);
  double u1 = (double)((a >> 11) + 1) * (1.0 / 9007199254740992.0);
  double u2 = (double)(b >> 11) * (1.0 / 9007199254740992.0);
  return (float)(sqrt(-2.0 * log(u1)) * cos(two_pi * u2));
}

/* round-to-nearest-even fp32 -> bf16 bit pattern (NaN kept quiet) */
static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x0040u);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* out[k] = N(0,1) sample k of stream (seed, tensor_id), k in [offset, offset+count) */
void synth_normal_f32(uint64_t seed, uint64_t tensor_id, uint64_t offset, int64_t count, float* out) {
  uint64_t base = sm_mix(sm_mix(seed) + tensor_id);
#pragma omp parallel for schedule(static)
  for (int64_t k = 0; k < count; ++k) out[k] = normal_at(base, offset + (uint64_t)k);
}

/* same stream, rounded to bf16 (bit patterns) */
void synth_normal_bf16(uint64_t seed, uint64_t tensor_id, uint64_t offset, int64_t count, uint16_t* out) {
  uint64_t base = sm_mix(sm_mix(seed) + tensor_id);
#pragma omp parallel for schedule(static)
  for (int64_t k = 0; k < count; ++k) out[k] = f32_to_bf16_rne(normal_at(base, offset + (uint64_t)k));
}

/* bf16 bit patterns -> fp32 (exact) */
void synth_bf16_to_f32(const uint16_t* in, int64_t count, float* out) {
#pragma omp parallel for schedule(static)
  for (int64_t k = 0; k < count; ++k) {
    uint32_t u = (uint32_t)in[k] << 16;
    memcpy(&out[k], &u, 4);
  }
}

/* fp32 -> bf16 bit patterns (RNE) */
void synth_f32_to_bf16(const float* in, int64_t count, uint16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t k = 0; k < count; ++k) out[k] = f32_to_bf16_rne(in[k]);
}
