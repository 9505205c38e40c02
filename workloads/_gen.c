/* Host-side counter-hash generator; bit-identical to the torch version in
 * workloads/gen.py (same hash, same float32 operations, no FMA contraction).
 * Built with: gcc -O2 -fopenmp -ffp-contract=off -shared -fPIC. */
#include <stdint.h>

static inline uint32_t mix32(uint32_t h) {
  h ^= h >> 16;
  h *= 0x7FEB352Du;
  h ^= h >> 15;
  h *= 0x846CA68Bu;
  h ^= h >> 16;
  return h;
}

static inline uint32_t hash_index(uint64_t i, uint32_t key) {
  uint32_t h = mix32((uint32_t)(i & 0xFFFFFFFFu) ^ key);
  uint32_t hi = (uint32_t)(i >> 32);
  if (hi) h = mix32(h ^ mix32(hi + 0x68E31DA4u));
  return h;
}

static inline float sample(uint64_t i, uint32_t key, const float* pool,
                           float inv_sqrt2, float std) {
  uint32_t h = hash_index(i, key);
  uint32_t i1 = h & 0xFFFFFFu;
  uint32_t i2 = mix32(h ^ 0x9E3779B9u) & 0xFFFFFFu;
  float v = pool[i1] + pool[i2];
  v = v * inv_sqrt2;
  v = v * std;
  return v;
}

void gen_normal_range(int64_t start, int64_t n, uint32_t key,
                      const float* pool, float inv_sqrt2, float std,
                      float* out) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < n; ++t)
    out[t] = sample((uint64_t)(start + t), key, pool, inv_sqrt2, std);
}

void gen_normal_at(const int64_t* idx, int64_t n, uint32_t key,
                   const float* pool, float inv_sqrt2, float std, float* out) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < n; ++t)
    out[t] = sample((uint64_t)idx[t], key, pool, inv_sqrt2, std);
}
