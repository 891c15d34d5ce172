// Counter-hash dropout decision, the library's reading of the optional elementwise dropout
// step of "FlashAttention 的第一原则", section 2 (the sources fix no generator).
//
//   ctr  = ((b*H + h)*N + i)*N + j                 i = query row, j = key column (uint64)
//   z    = seed + (ctr + 1) * 0x9E3779B97F4A7C15    (mod 2^64)
//   z    = SplitMix64 output mix (Steele, Lea & Flood, OOPSLA 2014)
//   keep = (z >> 32) >= thr,   thr = min(floor(p * 2^32), 2^32 - 1), computed on the host
//
// Kept probabilities are scaled by 1/(1-p); the row sum and lse use the undropped values.
#pragma once
#include <cstdint>

namespace fa {

__device__ __forceinline__ uint32_t dropout_bits(uint64_t seed, uint64_t ctr) {
  uint64_t z = seed + (ctr + 1ull) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  z ^= z >> 31;
  return uint32_t(z >> 32);
}

__device__ __forceinline__ bool dropout_keep(uint64_t seed, uint64_t ctr, uint32_t thr) {
  return dropout_bits(seed, ctr) >= thr;
}

// The same draw from z = seed + (ctr + 1) * gamma already formed, for runs of counters with a fixed
// stride s: z(ctr + s) = z(ctr) + s * gamma (mod 2^64), one 64-bit add per element.  Only the high
// word of the last product is needed: (z ^ (z >> 31)) >> 32 = hi ^ (hi >> 31).
constexpr uint64_t kDropGamma = 0x9E3779B97F4A7C15ull;
__device__ __forceinline__ uint64_t dropout_z(uint64_t seed, uint64_t ctr) { return seed + (ctr + 1ull) * kDropGamma; }
__device__ __forceinline__ uint32_t dropout_bits_z(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  const uint32_t hi = uint32_t(z >> 32);
  return hi ^ (hi >> 31);
}

}  // namespace fa
