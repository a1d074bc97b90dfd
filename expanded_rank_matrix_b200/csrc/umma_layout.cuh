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

namespace externd {
namespace umma {

// Stream-K partition of a contraction: the (tile, K-chunk) units u = t C + c
// (T tiles of 128 output rows, C chunks of 32 along K) are split into G
// contiguous ranges [u0(b), u0(b+1)), one per CTA.  A CTA's range covers a
// run of tiles; its part of tile t is one "segment" with its own partial
// result.  The segments of a tile belong to consecutive CTAs
// first(t) .. last(t), and CTA b's partial of tile t goes to slot
// b - first(t) of that tile: Xp[(t * S + slot) * 128 + row][64] (S = most
// segments of any tile).  A tile's partials are summed in slot order.
__host__ __device__ __forceinline__ long long sk_u0(int b, long long U, int G) {
  return (long long)b * U / G;
}
__host__ __device__ __forceinline__ int sk_owner(long long u, long long U, int G) {
  int b = (int)((u * G) / U);
  while (b + 1 < G && sk_u0(b + 1, U, G) <= u) ++b;
  while (b > 0 && sk_u0(b, U, G) > u) --b;
  return b;
}
__host__ __device__ __forceinline__ int sk_first(int t, int C, long long U, int G) {
  return sk_owner((long long)t * C, U, G);
}
__host__ __device__ __forceinline__ int sk_nseg(int t, int C, long long U, int G) {
  return sk_owner((long long)(t + 1) * C - 1, U, G) - sk_first(t, C, U, G) + 1;
}

// CTA count of a contraction with T tiles and C chunks on nsm SMs: one CTA
// per SM but one (that SM runs the kernels beside the contraction), at most
// one per unit, and few enough that no tile has more than max_segs segments
// (G <= (max_segs - 1) T gives at least C / (max_segs - 1) units per CTA).
inline int sk_ctas(int T, int C, int nsm, int max_segs) {
  long long g = (long long)T * C;
  const long long cap = nsm > 1 ? nsm - 1 : 1;
  if (cap < g) g = cap;
  if ((long long)(max_segs - 1) * T < g) g = (long long)(max_segs - 1) * T;
  return g < 1 ? 1 : (int)g;
}

}  // namespace umma
}  // namespace externd
