/* Counter-based seeded normals: the C implementation of synth/gen.py's generator.
 *
 * splitmix64 (Steele, Lea & Flood, OOPSLA 2014): state_i = key + (i + 1) * gamma, value_i =
 * mix64(state_i).  Uniform = top 53 bits * 2^-53.  Box-Muller on element pairs.  The numpy
 * implementation in gen.py is the definition; this file reproduces it element for element
 * (same integer stream, same double-precision transform) and is only faster.
 */
#include <math.h>
#include <stdint.h>

#define GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint16_t to_bf16(float f) {
  union { float f; uint32_t u; } v;
  v.f = f;
  uint32_t lsb = (v.u >> 16) & 1u;
  return (uint16_t)((v.u + 0x7FFFu + lsb) >> 16);
}

static inline void pair(uint64_t key, int64_t p, double stdv, double *z0, double *z1) {
  uint64_t a = mix64(key + (uint64_t)(2 * p + 1) * GAMMA);
  uint64_t b = mix64(key + (uint64_t)(2 * p + 2) * GAMMA);
  double u1 = (double)(a >> 11) * 0x1.0p-53;
  double u2 = (double)(b >> 11) * 0x1.0p-53;
  double r = sqrt(-2.0 * log1p(-u1));
  double ang = 2.0 * M_PI * u2;
  *z0 = r * cos(ang) * stdv;
  *z1 = r * sin(ang) * stdv;
}

void synth_normal_f32(uint64_t key, int64_t n, double stdv, float *out) {
  int64_t m = (n + 1) / 2;
#pragma omp parallel for schedule(static)
  for (int64_t p = 0; p < m; p++) {
    double z0, z1;
    pair(key, p, stdv, &z0, &z1);
    out[2 * p] = (float)z0;
    if (2 * p + 1 < n) out[2 * p + 1] = (float)z1;
  }
}

void synth_normal_bf16(uint64_t key, int64_t n, double stdv, uint16_t *out) {
  int64_t m = (n + 1) / 2;
#pragma omp parallel for schedule(static)
  for (int64_t p = 0; p < m; p++) {
    double z0, z1;
    pair(key, p, stdv, &z0, &z1);
    out[2 * p] = to_bf16((float)z0);
    if (2 * p + 1 < n) out[2 * p + 1] = to_bf16((float)z1);
  }
}
