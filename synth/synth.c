/*
 * Seeded, counter-based random draws for synthetic LatentMoE inputs.
 *
 * This module holds random-number generation only: no step of the layer's
 * arithmetic.  Both the CUDA path's tests/benchmark and the oracle take their
 * inputs from here.
 *
 * Stream: key = mix64(seed * GOLDEN ^ mix64(tag)).
 * Element i (a global counter, so any slice can be drawn on its own):
 *   w1 = mix64(key + (2i + 1) * GOLDEN),  w2 = mix64(key + (2i + 2) * GOLDEN)
 *   u1 = ((w1 >> 11) + 1) * 2^-53  in (0, 1]
 *   u2 = (w2 >> 11) * 2^-53        in [0, 1)
 *   normal  = sqrt(-2 ln u1) * cos(2 pi u2)        (Box-Muller, one output)
 *   uniform = u2
 * mix64 is the SplitMix64 output function (Steele, Lea, Flood 2014).
 * Outputs: float32 = (float)(mean + std * normal) (round to nearest even), and
 * bf16 = that float rounded to nearest even on its upper 16 bits.
 */
#include <math.h>
#include <stdint.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static uint64_t stream_key(uint64_t seed, uint64_t tag) { return mix64(seed * GOLDEN ^ mix64(tag)); }

static void draw(uint64_t key, int64_t i, double* normal, double* uniform) {
  uint64_t w1 = mix64(key + (uint64_t)(2 * i + 1) * GOLDEN);
  uint64_t w2 = mix64(key + (uint64_t)(2 * i + 2) * GOLDEN);
  double u1 = (double)((w1 >> 11) + 1) * 0x1.0p-53;
  double u2 = (double)(w2 >> 11) * 0x1.0p-53;
  if (normal) *normal = sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925 * u2);
  if (uniform) *uniform = u2;
}

static uint16_t f32_to_bf16_rne(float f) {
  union { float f; uint32_t u; } v = {f};
  uint32_t bias = 0x7FFFu + ((v.u >> 16) & 1u);
  return (uint16_t)((v.u + bias) >> 16);
}

/* out[j] = mean + std * normal(offset + j), j < n, as float32. */
void synth_normal_f32(uint64_t seed, uint64_t tag, int64_t offset, int64_t n, double mean,
                      double std, float* out) {
  uint64_t key = stream_key(seed, tag);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < n; ++j) {
    double z;
    draw(key, offset + j, &z, 0);
    out[j] = (float)(mean + std * z);
  }
}

/* Same draws, rounded on to bf16 (stored as raw uint16). */
void synth_normal_bf16(uint64_t seed, uint64_t tag, int64_t offset, int64_t n, double mean,
                       double std, uint16_t* out) {
  uint64_t key = stream_key(seed, tag);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < n; ++j) {
    double z;
    draw(key, offset + j, &z, 0);
    out[j] = f32_to_bf16_rne((float)(mean + std * z));
  }
}

/* out[j] = lo + (hi - lo) * uniform(offset + j), as float32. */
void synth_uniform_f32(uint64_t seed, uint64_t tag, int64_t offset, int64_t n, double lo,
                       double hi, float* out) {
  uint64_t key = stream_key(seed, tag);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < n; ++j) {
    double u;
    draw(key, offset + j, 0, &u);
    out[j] = (float)(lo + (hi - lo) * u);
  }
}

/* bf16 (raw uint16) -> float32, exact. */
void synth_bf16_to_f32(int64_t n, const uint16_t* in, float* out) {
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < n; ++j) {
    union { uint32_t u; float f; } v;
    v.u = (uint32_t)in[j] << 16;
    out[j] = v.f;
  }
}

/* float32 -> bf16 (raw uint16), round to nearest even. */
void synth_f32_to_bf16(int64_t n, const float* in, uint16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < n; ++j) out[j] = f32_to_bf16_rne(in[j]);
}
