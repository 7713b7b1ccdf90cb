/*
 * rocs_gen.c - seeded, counter-based synthetic input generator.
 *
 * This file holds no arithmetic of the method under test: it only draws
 * random numbers and rounds them to the storage type.  Both the CUDA path and
 * the CPU oracle consume the buffers it fills, so the two sides always see
 * bit-identical inputs.
 *
 * Random stream: SplitMix64 (Steele, Lea, Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014).  Output i of the stream with
 * key k is mix(k + (i + 1) * GAMMA), so any element can be drawn on its own and
 * the fill is embarrassingly parallel and independent of the thread count.
 *
 * Normals: Box-Muller transform (Box & Muller 1958), one 64-bit draw per
 * normal (upper 32 bits -> u1 in (0,1), lower 32 bits -> u2 in [0,1)).
 *
 * bf16 storage: round-to-nearest-even of the fp32 value (IEEE 754 rule applied
 * to the upper 16 bits of the binary32 encoding).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GAMMA 0x9E3779B97F4A7C15ull

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

/* Key of stream `stream` under `seed`: two SplitMix64 steps, so that nearby
 * (seed, stream) pairs give unrelated keys. */
static inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
  return mix64(mix64(seed + GAMMA) ^ (stream * 0xD1B54A32D192ED03ull + 1ull));
}

static inline uint64_t draw(uint64_t key, uint64_t i) { return mix64(key + (i + 1ull) * GAMMA); }

static inline double normal_of(uint64_t x) {
  const double two_pi = 6.283185307179586476925286766559;
  double u1 = ((double)(x >> 32) + 0.5) * (1.0 / 4294967296.0); /* (0,1) */
  double u2 = (double)(x & 0xffffffffull) * (1.0 / 4294967296.0); /* [0,1) */
  return sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return (uint16_t)((u >> 16) | 0x40u);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

uint64_t rocs_gen_u64(uint64_t seed, uint64_t stream, uint64_t i) { return draw(stream_key(seed, stream), i); }

/* out[j] = fp32(std * N(0,1)) for j in [0,n), element j drawn from index (offset + j). */
void rocs_gen_normal_f32(uint64_t seed, uint64_t stream, uint64_t offset, double std, float* out, int64_t n) {
  const uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < n; ++j) out[j] = (float)(std * normal_of(draw(key, offset + (uint64_t)j)));
}

/* Same values as rocs_gen_normal_f32, stored as bf16 bit patterns (RNE from the fp32 value). */
void rocs_gen_normal_bf16(uint64_t seed, uint64_t stream, uint64_t offset, double std, uint16_t* out, int64_t n) {
  const uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < n; ++j) out[j] = f32_to_bf16_rne((float)(std * normal_of(draw(key, offset + (uint64_t)j))));
}

/* Integers uniform on [lo, hi] (inclusive), by the multiply-high range map of a 64-bit draw. */
void rocs_gen_uniform_int(uint64_t seed, uint64_t stream, int64_t lo, int64_t hi, int64_t* out, int64_t n) {
  const uint64_t key = stream_key(seed, stream);
  const uint64_t span = (uint64_t)(hi - lo) + 1ull;
  for (int64_t j = 0; j < n; ++j) {
    unsigned __int128 p = (unsigned __int128)draw(key, (uint64_t)j) * span;
    out[j] = lo + (int64_t)(uint64_t)(p >> 64);
  }
}

/* Integers round(exp(mu + sigma * N(0,1))) clipped to [lo, hi]. */
void rocs_gen_lognormal_int(uint64_t seed, uint64_t stream, double mu, double sigma, int64_t lo, int64_t hi,
                            int64_t* out, int64_t n) {
  const uint64_t key = stream_key(seed, stream);
  for (int64_t j = 0; j < n; ++j) {
    double v = floor(exp(mu + sigma * normal_of(draw(key, (uint64_t)j))) + 0.5);
    if (v < (double)lo) v = (double)lo;
    if (v > (double)hi) v = (double)hi;
    out[j] = (int64_t)v;
  }
}
