// Inference with the packed factors: Y = X (B diag(D) C)^T, straight from the
// bitplanes, without forming the dense matrix.
//
// The pages note that ExTernD keeps inference multiplication-free -- ternary
// additions and subtractions plus one real scale per component (the
// romaanj.github.io review, "Significance") -- and that no fused inference
// kernel exists yet ("Limitations", "Future work").  For each input vector x
// (a row of X):
//   t_c = sum_j C_cj x_j             (add/subtract over the bits of row c of C)
//   s_c = D_c t_c
//   y_i = sum_c B_ic s_c             (add/subtract over the bits of column c of B)
//
// One persistent launch, one CTA per SM, three phases separated by grid
// barriers (bounded waits; the launch is cooperative, so every CTA is
// resident):
//  1. t: a warp per component, lanes over the packed words of C; x is staged
//     in shared memory with the 32 entries of word w rotated by w, so that
//     the lanes (one word each) read distinct banks at every bit.
//  2. partial y: CTA g takes a contiguous run of components; its threads own
//     packed row words of B (coalesced loads, lanes over words) and keep the
//     32 rows of their word in registers; the streams of the CTA are summed
//     in shared memory and the CTA's partial goes to global memory.
//  3. y_i = sum over the CTAs' partials, in CTA order.
// Every sum runs in a fixed order, so results are reproducible run to run.

#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/externd.h"
#include "common.cuh"
#include "internal.h"

namespace externd {
namespace {

constexpr int kApThreads = 512;
constexpr int kApWarps = kApThreads / 32;
constexpr int kXChunk = 4096;  // columns of x staged per pass of phase 1

struct ApArgs {
  const uint32_t* pB;  // [k][2][Wm]
  const uint32_t* pC;  // [k][2][Wn]
  const float* D;
  const float* X;      // [nb][n] (this launch's vectors)
  float* Y;            // [nb][m]
  float* S;            // [k][NB] scratch: s_c
  float* P;            // [G][m][NB] scratch: per-CTA partial y
  unsigned* bar;       // grid barrier counter
  int m, n, k, nb;
  long long budget;
  int* status;
};

// Grid barrier number `phase` (1, 2): release my CTA's writes, count in,
// wait (bounded) until every CTA has, acquire theirs.
__device__ __forceinline__ void grid_barrier(const ApArgs& a, unsigned phase) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(a.bar, 1u);
    const unsigned want = phase * gridDim.x;
    const long long t0 = clock64();
    while (true) {
      unsigned v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a.bar) : "memory");
      if (v >= want) break;
      if (clock64() - t0 > a.budget) {
        atomicCAS(a.status, 0, EXTERND_ERR_TIMEOUT);
        break;
      }
    }
    __threadfence();
  }
  __syncthreads();
}

template <int NB>
__global__ void __launch_bounds__(kApThreads, 1) apply_kernel(const ApArgs a) {
  extern __shared__ __align__(16) float ash[];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int m = a.m, n = a.n, k = a.k;
  const int Wm = (m + 31) >> 5, Wn = (n + 31) >> 5;

  // ---- phase 1: s_c = D_c sum_j C_cj x_j ----
  {
    float* xs = ash;  // [kXChunk][NB], entry 32 w + b of a chunk at 32 w + ((b + w) & 31)
    const int gw = blockIdx.x * kApWarps + wid, nw = gridDim.x * kApWarps;
    float acc[NB];
    // components are visited in the same order in every chunk, so each warp
    // keeps its running sums for at most one component at a time: loop the
    // components outermost and the chunks inside
    const int nchunks = (n + kXChunk - 1) / kXChunk;
    for (int cbase = 0; cbase < k; cbase += nw) {
      const int c = cbase + gw;
#pragma unroll
      for (int b = 0; b < NB; ++b) acc[b] = 0.f;
      for (int ch = 0; ch < nchunks; ++ch) {
        const int j0 = ch * kXChunk, jn = min(kXChunk, n - j0);
        if (nchunks > 1 || cbase == 0) {
          __syncthreads();
          for (int e = tid; e < jn; e += kApThreads) {
            const int w = e >> 5, r = e & 31;
#pragma unroll
            for (int b = 0; b < NB; ++b)
              xs[((w << 5) + ((r + w) & 31)) * NB + b] = b < a.nb ? a.X[(size_t)b * n + j0 + e] : 0.f;
          }
          __syncthreads();
        }
        if (c < k) {
          const uint32_t* mk = a.pC + (size_t)c * 2 * Wn + (j0 >> 5);
          const uint32_t* sg = mk + Wn;
          const int nwords = (jn + 31) >> 5;
          for (int w = lane; w < nwords; w += 32) {
            const uint32_t pos = __ldg(mk + w) & ~__ldg(sg + w);
            const uint32_t neg = __ldg(mk + w) & __ldg(sg + w);
            const float* xw = xs + (size_t)(w << 5) * NB;
#pragma unroll
            for (int r = 0; r < 32; ++r) {
              const int slot = (r + w) & 31;
#pragma unroll
              for (int b = 0; b < NB; ++b) {
                const float xv = xw[slot * NB + b];
                if ((pos >> r) & 1u) acc[b] += xv;
                if ((neg >> r) & 1u) acc[b] -= xv;
              }
            }
          }
        }
      }
      if (c < k) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          float v = acc[b];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          if (lane == 0) a.S[(size_t)c * NB + b] = a.D[c] * v;
        }
      }
    }
  }
  grid_barrier(a, 1u);

  // ---- phase 2: this CTA's partial y over its run of components ----
  {
    const int G = gridDim.x, g = blockIdx.x;
    const int cb = (int)((long long)g * k / G), ce = (int)((long long)(g + 1) * k / G);
    const int WG = (Wm + 31) >> 5;                 // warps per set of all row words
    const int NSt = max(1, kApWarps / WG);         // component streams in the CTA
    const int s = wid / WG, t = (wid % WG) * 32 + lane;
    float acc[32][NB];
#pragma unroll
    for (int r = 0; r < 32; ++r)
#pragma unroll
      for (int b = 0; b < NB; ++b) acc[r][b] = 0.f;
    const bool active = s < NSt && t < Wm;
    if (s < NSt) {
      for (int c = cb + s; c < ce; c += NSt) {
        uint32_t pos = 0u, neg = 0u;
        if (t < Wm) {
          const uint32_t mk = __ldg(a.pB + (size_t)c * 2 * Wm + t);
          const uint32_t sg = __ldg(a.pB + (size_t)c * 2 * Wm + Wm + t);
          pos = mk & ~sg;
          neg = mk & sg;
        }
        float sv[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) sv[b] = __ldcg(a.S + (size_t)c * NB + b);
#pragma unroll
        for (int r = 0; r < 32; ++r)
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            if ((pos >> r) & 1u) acc[r][b] += sv[b];
            if ((neg >> r) & 1u) acc[r][b] -= sv[b];
          }
      }
    }
    // sum the streams in stream order: stream 0 writes, the others add in turn
    float* ys = ash;  // [Wm * 32][NB]
    for (int st = 0; st < NSt; ++st) {
      if (s == st && active) {
#pragma unroll
        for (int r = 0; r < 32; ++r)
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            float* p = ys + (size_t)(t * 32 + r) * NB + b;
            *p = st == 0 ? acc[r][b] : *p + acc[r][b];
          }
      }
      __syncthreads();
    }
    float* Pg = a.P + (size_t)g * m * NB;
    for (int e = tid; e < m * NB; e += kApThreads) Pg[e] = ys[e];
  }
  grid_barrier(a, 2u);

  // ---- phase 3: y_i = sum of the CTAs' partials, CTA order ----
  {
    const int G = gridDim.x;
    for (int e = blockIdx.x * kApThreads + tid; e < m * NB; e += G * kApThreads) {
      float y = 0.f;
      for (int g = 0; g < G; ++g) y += __ldcg(a.P + (size_t)g * m * NB + e);
      const int i = e / NB, b = e - i * NB;
      if (b < a.nb) a.Y[(size_t)b * m + i] = y;
    }
  }
}

template <int NB>
int launch_apply(ApArgs a, int G, size_t smem, cudaStream_t st) {
  auto kern = apply_kernel<NB>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return EXTERND_ERR_CUDA;
  void* params[] = {&a};
  if (cudaLaunchCooperativeKernel((const void*)kern, dim3(G), dim3(kApThreads), params, smem,
                                  st) != cudaSuccess) {
    cudaGetLastError();
    return EXTERND_ERR_CUDA;
  }
  return EXTERND_OK;
}

}  // namespace

int ternary_apply(const uint32_t* pB, const uint32_t* pC, const float* D, int64_t m, int64_t n,
                  int64_t k, const float* X, int64_t nb, float* Y, cudaStream_t st) {
  int dev = 0, nsm = 0, optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return EXTERND_ERR_CUDA;
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const int NB = nb >= 2 ? 2 : 1;
  const int Wm = (int)((m + 31) / 32);
  const size_t smem1 = sizeof(float) * (size_t)kXChunk * NB;
  const size_t smem2 = sizeof(float) * (size_t)Wm * 32 * NB;
  const size_t smem = smem1 > smem2 ? smem1 : smem2;
  if (smem > (size_t)optin) return EXTERND_ERR_INVALID_ARG;
  int per_sm = 0;
  cudaError_t e = NB == 2
                      ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, apply_kernel<2>,
                                                                      kApThreads, smem)
                      : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, apply_kernel<1>,
                                                                      kApThreads, smem);
  if (e != cudaSuccess || per_sm < 1) {
    cudaGetLastError();
    return EXTERND_ERR_NO_COOP;
  }
  const int G = nsm;  // one CTA per SM
  const size_t oS = 0;
  const size_t oP = (sizeof(float) * (size_t)k * NB + 255) & ~(size_t)255;
  const size_t oBar = (oP + sizeof(float) * (size_t)G * m * NB + 255) & ~(size_t)255;
  void* ws = nullptr;
  if (cudaMallocAsync(&ws, oBar + 256, st) != cudaSuccess) {
    cudaGetLastError();
    return EXTERND_ERR_OOM;
  }
  int rc = EXTERND_OK;
  ApArgs a = {};
  a.pB = pB; a.pC = pC; a.D = D;
  a.S = (float*)((char*)ws + oS);
  a.P = (float*)((char*)ws + oP);
  a.bar = (unsigned*)((char*)ws + oBar);
  a.m = (int)m; a.n = (int)n; a.k = (int)k;
  a.budget = kDefaultWaitBudget;
  a.status = status_word_ptr();
  if (!a.status) rc = EXTERND_ERR_CUDA;
  // vectors in launches of NB
  for (int64_t b0 = 0; rc == EXTERND_OK && b0 < nb; b0 += NB) {
    a.X = X + (size_t)b0 * n;
    a.Y = Y + (size_t)b0 * m;
    a.nb = (int)((nb - b0) < NB ? (nb - b0) : NB);
    if (cudaMemsetAsync(a.bar, 0, sizeof(unsigned), st) != cudaSuccess) {
      rc = EXTERND_ERR_CUDA;
      break;
    }
    rc = NB == 2 ? launch_apply<2>(a, G, smem, st) : launch_apply<1>(a, G, smem, st);
  }
  if (cudaFreeAsync(ws, st) != cudaSuccess && rc == EXTERND_OK) rc = EXTERND_ERR_CUDA;
  return rc;
}

}  // namespace externd
