// Counter-hash dropout decision, the library's reading of the optional elementwise dropout step of
// "FlashAttention 的第一原则", section 2 (the sources fix no generator).  One 64-bit draw serves four
// consecutive key columns of a query row:
//
//   W    = ceil(N / 4)                                  draws per query row
//   g    = ((b*H + h)*N + i)*W + (j >> 2)               i = query row, j = key column (uint64)
//   z    = seed + (g + 1) * 0x9E3779B97F4A7C15          (mod 2^64)
//   x    = SplitMix64 output mix of z (Steele, Lea & Flood, OOPSLA 2014)
//   u    = (x >> 16 (j & 3)) & 0x7fff                   the 15-bit draw of column j
//   keep = u >= thr,  thr = min(floor(p * 2^15), 2^15 - 1), computed on the host
//
// Kept probabilities are scaled by 1/(1-p); the row sum and lse use the undropped values.
// Two columns are decided by one add: with c = (2^15 - thr) * 0x00010001, the word
// (half & 0x7fff7fff) + c carries nothing from one 16-bit lane into the next (each lane stays
// below 2^16) and has bit 15 (lane 0) and bit 31 (lane 1) set exactly where u >= thr.
#pragma once
#include <cstdint>

namespace fa {

constexpr uint64_t kDropGamma = 0x9E3779B97F4A7C15ull;

__device__ __forceinline__ uint64_t dropout_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Draws per query row.
__host__ __device__ __forceinline__ uint64_t dropout_row_draws(int N) { return (uint64_t(N) + 3ull) >> 2; }

// z of draw g; the draws of a run g, g + s, g + 2s, ... step by s * gamma (one 64-bit add).
__device__ __forceinline__ uint64_t dropout_z(uint64_t seed, uint64_t g) { return seed + (g + 1ull) * kDropGamma; }

// The per-lane constant c of the two-column test.
__device__ __forceinline__ uint32_t dropout_lane_c(uint32_t thr) { return (0x8000u - thr) * 0x00010001u; }

// Keep flags of the two columns held by a 32-bit half of a draw: bit 15 and bit 31.
__device__ __forceinline__ uint32_t dropout_flags(uint32_t half, uint32_t c) { return (half & 0x7fff7fffu) + c; }

// 0xffff over each kept 16-bit lane (each lane's top bit replicated over its two bytes): the mask of
// a packed bf16 pair.
__device__ __forceinline__ uint32_t dropout_mask2(uint32_t flags) {
  uint32_t m;
  asm("prmt.b32 %0, %1, 0, 0xBB99;" : "=r"(m) : "r"(flags));
  return m;
}

// One decision: query row `row` = (b*H + h)*N + i, key column j.
__device__ __forceinline__ bool dropout_keep(uint64_t seed, uint64_t row, uint64_t W, int j, uint32_t thr) {
  const uint64_t x = dropout_mix(dropout_z(seed, row * W + uint64_t(j >> 2)));
  return uint32_t((x >> (16 * (j & 3))) & 0x7fffu) >= thr;
}

}  // namespace fa
