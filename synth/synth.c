/*
 * synth.c -- seeded synthetic inputs shared by the tests and the benchmark.
 * It holds none of the GEMM or quantiser arithmetic: only a counter-based
 * SplitMix64 stream (Steele, Lea & Flood, "Fast splittable pseudorandom number
 * generators", OOPSLA 2014; constants as published by Vigna) and the
 * Box-Muller transform (Box & Muller, Ann. Math. Statist. 29, 1958).
 *
 * Output i of stream `seed` is mix(seed + (i + 1) * 0x9E3779B97F4A7C15), so any
 * sub-range can be produced independently (and in parallel).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t sm64(uint64_t seed, uint64_t i) {
  return mix64(seed + (i + 1) * 0x9E3779B97F4A7C15ULL);
}

/* uniform double in [0, 1) from the top 53 bits */
static inline double u01(uint64_t seed, uint64_t i) {
  return (double)(sm64(seed, i) >> 11) * (1.0 / 9007199254740992.0);
}

void synth_u64(uint64_t seed, uint64_t offset, uint64_t* out, size_t n) {
  #pragma omp parallel for schedule(static)
  for (size_t i = 0; i < n; ++i) out[i] = sm64(seed, offset + i);
}

/* N(0,1) float32: element j pairs counters 2*(j/2) and 2*(j/2)+1; even j takes
 * the cosine branch, odd j the sine branch. */
void synth_normal_f32(uint64_t seed, uint64_t offset, float* out, size_t n) {
  const double two_pi = 6.283185307179586476925286766559;
  #pragma omp parallel for schedule(static)
  for (size_t i = 0; i < n; ++i) {
    uint64_t j = offset + i;
    uint64_t p = j >> 1;
    double u1 = 1.0 - u01(seed, 2 * p);     /* (0, 1] */
    double u2 = u01(seed, 2 * p + 1);
    double r = sqrt(-2.0 * log(u1));
    double z = (j & 1) ? r * sin(two_pi * u2) : r * cos(two_pi * u2);
    out[i] = (float)z;
  }
}

/* integers uniform in [lo, hi]: lo + floor(u * (hi - lo + 1)) */
void synth_randint(uint64_t seed, uint64_t offset, int64_t lo, int64_t hi, int64_t* out, size_t n) {
  double span = (double)(hi - lo + 1);
  for (size_t i = 0; i < n; ++i) {
    int64_t v = lo + (int64_t)floor(u01(seed, offset + i) * span);
    out[i] = v > hi ? hi : v;
  }
}
