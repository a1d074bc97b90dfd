// Shared-memory operand layout of the block-ALS tensor-core contractions
// (tcgen05.mma, no swizzle, K-major): the ternary B operand of one 32-wide K
// chunk holds 64 components x 32 K entries of bf16, in core matrices of
// 8 components x 8 K entries (16 bytes per component row); K-adjacent core
// matrices lie 128 bytes apart (leading byte offset) and 8-component groups
// 512 bytes apart (stride byte offset).  One chunk is 4 KB.  The ternary
// codes are written in this layout once per half-step (one chunk per 32
// entries) and copied into shared memory as they are.
#pragma once

#include <cstdint>

namespace externd {
namespace umma {

constexpr int kM = 128;                 // accumulator rows (TMEM lanes)
constexpr int kN = 64;                  // components (TMEM columns)
constexpr int kKc = 32;                 // K chunk
constexpr int kBBytes = kN * kKc * 2;   // B chunk: 4 KB
constexpr int kSboK = 8 * kKc * 2;      // bytes between 8-row groups (K-major)

// byte offset of element (row, k) of a [rows x kKc] K-major bf16 tile
__host__ __device__ __forceinline__ uint32_t kmaj_off(int row, int k) {
  return (uint32_t)((row >> 3) * kSboK + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2);
}

// bf16 codes of -1, 0, +1 for 8 consecutive entries (bit e of m8 = entry e
// nonzero, bit e of s8 = entry e negative), packed little-endian into 16 bytes
__device__ __forceinline__ uint4 bf16_codes8(uint32_t m8, uint32_t s8) {
  uint32_t w[4];
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    uint32_t v = 0u;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int e = 2 * h + t;
      const uint32_t bits = ((m8 >> e) & 1u) ? (((s8 >> e) & 1u) ? 0xBF80u : 0x3F80u) : 0u;
      v |= bits << (16 * t);
    }
    w[h] = v;
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

}  // namespace umma
}  // namespace externd
