// Shared device helpers for the ExTernD kernels (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/externd.h"

namespace externd {

// threads per CTA of the persistent sequential kernel: twelve warps, so the
// kernel may hold 168 registers per thread (at sixteen warps the 128-register
// cap spills its loop state, and with the residual filling shared memory the
// spills miss L1)
constexpr int kThreads = 384;
constexpr int kWarps = kThreads / 32;
constexpr long long kDefaultWaitBudget = 2000000000LL;  // SM cycles, about 1 s

// ---------------------------------------------------------------------------
// Flag-tagged exchange words.  A 64-bit word carries a 32-bit payload in its
// low half and the exchange's epoch in its high half; it is written and read
// with single 64-bit accesses, so a reader that sees the epoch also sees the
// payload and no separate fence or barrier is needed.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void xw_store(uint64_t* p, uint32_t epoch, uint32_t payload) {
  uint64_t v = ((uint64_t)epoch << 32) | (uint64_t)payload;
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ uint64_t xw_load(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ int ld_flag(const int* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Waits until *p carries `epoch` and returns its payload.  The wait is
// bounded by `budget` SM cycles; when it runs out (or another CTA has
// already given up, which it announces through *abort_word) the caller's
// `ab` is set, the first error is recorded, and 0 is returned.  Once `ab` is
// set no further waiting happens.
__device__ __forceinline__ uint32_t xw_wait(const uint64_t* p, uint32_t epoch, bool& ab,
                                            long long budget, int* abort_word) {
  if (ab) return 0u;
  uint64_t v = xw_load(p);
  if ((uint32_t)(v >> 32) == epoch) return (uint32_t)v;
  const long long t0 = clock64();
  unsigned spins = 0;
  while (true) {
    v = xw_load(p);
    if ((uint32_t)(v >> 32) == epoch) return (uint32_t)v;
    if (((++spins) & 63u) == 0u) {
      if (ld_flag(abort_word) != 0) { ab = true; return 0u; }
    }
    if (clock64() - t0 > budget) {
      atomicCAS(abort_word, 0, EXTERND_ERR_TIMEOUT);
      ab = true;
      return 0u;
    }
  }
}

// Waits for `count` (<= N) words base[t * stride], t < count, all tagged with
// `epoch`, and writes their payloads to out[].  All words are loaded back to
// back; every later round re-loads all words still stale together, so each
// round costs one memory round trip however many words it covers.  Bounded
// like xw_wait.
template <int N>
__device__ __forceinline__ void xw_wait_n(const uint64_t* base, long long stride, int count,
                                          uint32_t epoch, uint32_t (&out)[N], bool& ab,
                                          long long budget, int* abort_word) {
  uint64_t v[N];
  unsigned pending = 0u;
#pragma unroll
  for (int t = 0; t < N; ++t)
    if (t < count) v[t] = xw_load(base + t * stride);
#pragma unroll
  for (int t = 0; t < N; ++t)
    if (t < count && (uint32_t)(v[t] >> 32) != epoch) pending |= 1u << t;
  if (pending && !ab) {
    const long long t0 = clock64();
    unsigned spins = 0;
    while (pending) {
#pragma unroll
      for (int t = 0; t < N; ++t)
        if ((pending >> t) & 1u) v[t] = xw_load(base + t * stride);
#pragma unroll
      for (int t = 0; t < N; ++t)
        if (((pending >> t) & 1u) && (uint32_t)(v[t] >> 32) == epoch) pending &= ~(1u << t);
      if (!pending) break;
      if (((++spins) & 63u) == 0u && ld_flag(abort_word) != 0) {
        ab = true;
        break;
      }
      if (clock64() - t0 > budget) {
        atomicCAS(abort_word, 0, EXTERND_ERR_TIMEOUT);
        ab = true;
        break;
      }
    }
  }
#pragma unroll
  for (int t = 0; t < N; ++t) out[t] = (t < count && !ab) ? (uint32_t)v[t] : 0u;
}

__device__ __forceinline__ uint32_t f2u(float x) { return __float_as_uint(x); }
__device__ __forceinline__ float u2f(uint32_t x) { return __uint_as_float(x); }
__device__ __forceinline__ uint32_t dlo(double x) { return (uint32_t)__double_as_longlong(x); }
__device__ __forceinline__ uint32_t dhi(double x) {
  return (uint32_t)((unsigned long long)__double_as_longlong(x) >> 32);
}
__device__ __forceinline__ double u2d(uint32_t lo, uint32_t hi) {
  return __longlong_as_double((long long)(((unsigned long long)hi << 32) | lo));
}

// Deterministic block-wide fp64 sum: fixed per-thread order, fixed shuffle
// tree, warp partials summed by thread 0 in warp order.  All threads get the
// result.  `red` holds kWarps + 1 doubles of shared memory.
__device__ __forceinline__ double block_sum(double x, double* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  __syncthreads();
  if (lane == 0) red[wid] = x;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int i = 0; i < kWarps; ++i) s += red[i];
    red[kWarps] = s;
  }
  __syncthreads();
  return red[kWarps];
}

__device__ __forceinline__ int block_sum_int(int x, int* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  __syncthreads();
  if (lane == 0) red[wid] = x;
  __syncthreads();
  if (threadIdx.x == 0) {
    int s = 0;
    for (int i = 0; i < kWarps; ++i) s += red[i];
    red[kWarps] = s;
  }
  __syncthreads();
  return red[kWarps];
}

}  // namespace externd
