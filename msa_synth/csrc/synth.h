// Counter-based synthetic input generator (host + device), mirroring msa_synth/__init__.py.
// Draws numbers only: no step of the attention method lives here.
#pragma once
#include <stdint.h>

#if defined(__CUDACC__)
#define SYNTH_HD __host__ __device__ __forceinline__
#else
#define SYNTH_HD static inline
#endif

#define SYNTH_GOLDEN 0x9E3779B97F4A7C15ull
#define SYNTH_LAYER_MUL 0xD1B54A32D192ED03ull
#define SYNTH_IH_SCALE_BITS 0x37ddb3d7u  // fp32 nearest to sqrt(3)/65536

SYNTH_HD uint64_t synth_mix64(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ull;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBull;
  z ^= z >> 31;
  return z;
}

SYNTH_HD uint64_t synth_tensor_key(uint64_t seed, uint32_t stream, uint32_t layer, uint32_t sub) {
  uint64_t k = synth_mix64(seed * SYNTH_GOLDEN + (uint64_t)stream + ((uint64_t)sub << 32));
  return synth_mix64(k + ((uint64_t)layer + 1ull) * SYNTH_LAYER_MUL);
}

SYNTH_HD uint64_t synth_hash(uint64_t key, uint64_t idx) {
  return synth_mix64(key + (idx + 1ull) * SYNTH_GOLDEN);
}

// Irwin-Hall(4) integer sum minus its mean, in [-131070, 131070].
SYNTH_HD int32_t synth_ih_centered(uint64_t h) {
  return (int32_t)((h & 0xFFFFull) + ((h >> 16) & 0xFFFFull) + ((h >> 32) & 0xFFFFull) + (h >> 48)) -
         131070;
}
