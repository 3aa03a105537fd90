// Counter-based random numbers for the LoRA dropout mask (device side).
//
// Philox4x64 with ten rounds, as published by Salmon, Moraes, Dror and Shaw
// ("Parallel Random Numbers: As Easy as 1, 2, 3", SC 2011): a counter of four
// 64-bit words is scrambled by ten rounds; each round multiplies words 0 and
// 2 by two fixed odd constants (full 128-bit products), swaps and mixes the
// halves with words 1 and 3 and the key, and the two key words are bumped by
// two Weyl constants (the fractional parts of the golden ratio and of
// sqrt(3) - 1, scaled to 64 bits).
//
// The dropout mask draws one 16-bit value per element: element e (row-major
// flat index) takes 16-bit lane e % 16 of the block for counter
// (e / 16, offset, 0, 0) under key (seed, 0), lane i being bits 16 (i % 4) of
// word i / 4, and is kept when that value is >= the call's threshold.
#pragma once

#include <cstdint>

namespace qlora {

struct PhiloxBlock {
  uint64_t w[4];
};

__device__ __forceinline__ PhiloxBlock philox4x64_10(uint64_t c0, uint64_t c1, uint64_t c2, uint64_t c3,
                                                     uint64_t k0, uint64_t k1) {
  constexpr uint64_t kMul0 = 0xD2E7470EE14C6C93ull, kMul1 = 0xCA5A826395121157ull;
  constexpr uint64_t kWeyl0 = 0x9E3779B97F4A7C15ull, kWeyl1 = 0xBB67AE8584CAA73Bull;
#pragma unroll
  for (int round = 0; round < 10; ++round) {
    const uint64_t hi0 = __umul64hi(kMul0, c0), lo0 = kMul0 * c0;
    const uint64_t hi1 = __umul64hi(kMul1, c2), lo1 = kMul1 * c2;
    const uint64_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
    k0 += kWeyl0;
    k1 += kWeyl1;
  }
  PhiloxBlock b;
  b.w[0] = c0;
  b.w[1] = c1;
  b.w[2] = c2;
  b.w[3] = c3;
  return b;
}

// The 16 keep bits (bit i: element 16 * block + i is kept) of one block.
__device__ __forceinline__ uint32_t dropout_keep_bits(uint64_t block, uint64_t seed, uint64_t offset,
                                                      uint32_t threshold) {
  const PhiloxBlock b = philox4x64_10(block, offset, 0ull, 0ull, seed, 0ull);
  uint32_t bits = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t u = static_cast<uint32_t>(b.w[i >> 2] >> (16 * (i & 3))) & 0xFFFFu;
    bits |= (u >= threshold ? 1u : 0u) << i;
  }
  return bits;
}

}  // namespace qlora
