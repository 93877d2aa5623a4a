// Temperature sampling of the token decoder's output by the Gumbel-max rule.
//
// The PHOTON explainer (quality section) closes the single-query quality gap
// with several varied queries per prompt; that needs a stochastic decoder.
// A token is drawn from softmax(logits / T): with G_v independent standard
// Gumbel variables, argmax_v (logit_v / T + G_v) has exactly that law, so
// the draw fuses into the same packed-key maximum as greedy decoding (ties
// to the lowest id).  The noise is counter-based, a pure function of
// (seed, sequence, token index, vocabulary id):
//   row key  K = mix64(mix64(seed + g*(b+1)) + g*(t+1))
//            (mix64: the SplitMix64 output function, g = 0x9E3779B97F4A7C15);
//   element  h = MurmurHash3_x86_32, seed 0, of the 12-byte message K (8
//            bytes, little-endian) followed by v (4 bytes, little-endian);
//   uniform  u = (floor(h / 256) + 1/2) / 2^24;  G = -ln(-ln u).
// The message's first two blocks depend on the row only: the row key below
// is the hash state after them, and each vocabulary id adds its block, the
// length and the finaliser.
// b = the sequence's batch row, t = chunk * C1*C2 + sub-chunk * C1 + position
// (the chunk count is read on the device, so captured steps replay).
#pragma once

#include <stdint.h>

#include "kernels.h"  // SampleArgs

namespace photon {

__device__ __forceinline__ uint64_t sample_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ uint32_t sample_fmix32(uint32_t h) {
  h ^= h >> 16;
  h *= 0x85EBCA6Bu;
  h ^= h >> 13;
  h *= 0xC2B2AE35u;
  h ^= h >> 16;
  return h;
}

// One 4-byte block of MurmurHash3_x86_32 folded into the hash state h.
__device__ __forceinline__ uint32_t sample_mm3_block(uint32_t h, uint32_t k) {
  k *= 0xCC9E2D51u;
  k = (k << 15) | (k >> 17);
  k *= 0x1B873593u;
  h ^= k;
  h = (h << 13) | (h >> 19);
  return h * 5u + 0xE6546B64u;
}

// Hash state of head row `row`'s draw after the row key's two blocks.
__device__ __forceinline__ uint32_t sample_row_key(const SampleArgs& sa, long long row) {
  constexpr uint64_t kG = 0x9E3779B97F4A7C15ull;
  const long long b = row / sa.C2;
  const int j = (int)(row - b * sa.C2);
  const long long t = (long long)(*sa.chunk) * sa.C1 * sa.C2 + (long long)j * sa.C1 + sa.i;
  uint64_t k = sample_mix64(sa.seed + kG * (uint64_t)(b + 1));
  k = sample_mix64(k + kG * (uint64_t)(t + 1));
  return sample_mm3_block(sample_mm3_block(0u, (uint32_t)k), (uint32_t)(k >> 32));
}

// Standard Gumbel variable of vocabulary id v under `key`.  -ln u is taken
// from whichever of u and 1 - u is exact in fp32 on its half of the grid
// (u = (2m + 1) / 2^25 has at most 24 significant bits when u < 1/2, and so
// has 1 - u when u >= 1/2), so draws near u = 1 keep their precision.
static __device__ __noinline__ float sample_gumbel(uint32_t key, int v) {
  const uint32_t m = sample_fmix32(sample_mm3_block(key, (uint32_t)v) ^ 12u) >> 8;
  float e;  // -ln u > 0
  if (m < (1u << 23))
    e = -logf((float)(2u * m + 1u) * 2.98023223876953125e-08f);  // u exactly
  else
    e = -log1pf(-(float)((1u << 25) - 2u * m - 1u) * 2.98023223876953125e-08f);  // 1 - u exactly
  return -logf(e);
}

// Perturbed value a head logit competes with when sampling.  Callers branch
// once per row between this and the plain logit, so the greedy loops carry
// no sampling code (the noise is kept out of line for the same reason).
__device__ __forceinline__ float sample_value(float inv_t, uint32_t key, float logit, int v) {
  return logit * inv_t + sample_gumbel(key, v);
}

}  // namespace photon
