/* Host-side fill of the synthetic streams (same definition as synth/gen.py):
 * element i of stream `key` is table[mix64(key + (i+1)*GOLDEN) >> 48].
 * Integer hashing plus a table gather; no floating-point arithmetic. */
#include <stdint.h>

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

void synth_host_fill_f32(float* out, uint64_t key, int64_t start, int64_t n, const float* table) {
  const uint64_t golden = 0x9E3779B97F4A7C15ull;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    out[i] = table[mix64(key + (uint64_t)(start + i + 1) * golden) >> 48];
  }
}

void synth_host_fill_f64(double* out, uint64_t key, int64_t start, int64_t n, const double* table) {
  const uint64_t golden = 0x9E3779B97F4A7C15ull;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    out[i] = table[mix64(key + (uint64_t)(start + i + 1) * golden) >> 48];
  }
}
