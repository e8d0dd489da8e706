/* Oracle-side weight generator (test infrastructure only): the same
 * SplitMix64 + four-term Irwin-Hall construction as oracle/rng.py, in plain C
 * with OpenMP, so that full-size layers can be drawn in well under a second.
 * It is checked bit-exact against the numpy implementation by the tests.
 *
 * out[i] = float32(z_i) * scale, z_i = (sum of the four 16-bit fields of
 * mix64(key + (start + i + 1) * GAMMA)) - 131070, optionally rounded to bf16
 * (nearest, ties to even) and returned as float32. */
#include <stdint.h>

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

static inline float round_bf16(float x) {
  union { float f; uint32_t u; } v;
  v.f = x;
  v.u = (v.u + 0x7FFFu + ((v.u >> 16) & 1u)) & 0xFFFF0000u;
  return v.f;
}

void oracle_weight_normal(uint64_t key, uint64_t start, int64_t count, float scale, int bf16,
                          float* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < count; ++i) {
    const uint64_t u = mix64(key + ((uint64_t)start + (uint64_t)i + 1ull) * 0x9E3779B97F4A7C15ull);
    const int32_t s = (int32_t)(u & 0xFFFFu) + (int32_t)((u >> 16) & 0xFFFFu) +
                      (int32_t)((u >> 32) & 0xFFFFu) + (int32_t)(u >> 48);
    const float x = (float)(s - 131070) * scale;
    out[i] = bf16 ? round_bf16(x) : x;
  }
}
