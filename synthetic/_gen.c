/* Counter-based SplitMix64 draws for the synthetic encoder inputs.
 * Same definitions as the module docstring of synthetic/__init__.py:
 * element i of stream key k is mix(k + (i+1) * 0x9E3779B97F4A7C15);
 * uniform = (x >> 11) * 2^-53; normals by Box-Muller on pairs (u1, u2). */
#include <math.h>
#include <stdint.h>

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}
static inline double unif(uint64_t key, uint64_t i) {
  return (double)(mix64(key + (i + 1) * 0x9E3779B97F4A7C15ULL) >> 11) * 0x1.0p-53;
}

void synth_uniform(uint64_t key, int64_t start, int64_t n, double scale, double shift, float *out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = (float)(unif(key, (uint64_t)(start + i)) * scale + shift);
}

/* out[i] = (float)(normal_i * std + mean), i in [0, n). */
void synth_normal(uint64_t key, int64_t n, double std, double mean, float *out) {
  const int64_t npairs = (n + 1) / 2;
#pragma omp parallel for schedule(static)
  for (int64_t p = 0; p < npairs; ++p) {
    double u1 = unif(key, (uint64_t)(2 * p)), u2 = unif(key, (uint64_t)(2 * p + 1));
    double r = sqrt(-2.0 * log1p(-u1));
    double th = 6.283185307179586476925286766559 * u2;
    out[2 * p] = (float)(r * cos(th) * std + mean);
    if (2 * p + 1 < n) out[2 * p + 1] = (float)(r * sin(th) * std + mean);
  }
}

/* Round float32 to bfloat16 (nearest, ties to even) in place, keeping float32 storage. */
void synth_round_bf16(float *x, int64_t n) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    union { float f; uint32_t u; } v; v.f = x[i];
    if ((v.u & 0x7F800000u) == 0x7F800000u && (v.u & 0x7FFFFFu)) continue;   /* NaN */
    uint32_t lsb = (v.u >> 16) & 1u;
    v.u = (v.u + 0x7FFFu + lsb) & 0xFFFF0000u;
    x[i] = v.f;
  }
}
