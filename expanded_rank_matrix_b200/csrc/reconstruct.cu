// A_hat = B diag(D) C from packed bitplanes (the factor form of the ExTernD
// abstract).  Each CTA owns a 32 x 256 tile of A_hat; thread t owns column t
// of the tile and keeps its 32 entries as fp64 accumulators, adding +-d_c in
// component order, so the sum is the same sequence of fp64 additions a plain
// per-entry loop over c would make.  Verification kernel, not the hot path.

#include <cuda_runtime.h>

#include <cstdint>

#include "common.cuh"
#include "internal.h"

namespace externd {

constexpr int kRecCols = 256;
constexpr int kRecChunk = 64;  // components staged in shared memory at a time

__global__ void __launch_bounds__(kRecCols) reconstruct_kernel(const uint32_t* __restrict__ pB,
                                                               const uint32_t* __restrict__ pC,
                                                               const float* __restrict__ D, int m,
                                                               int n, int k, float* __restrict__ out) {
  __shared__ uint32_t su[kRecChunk][2];
  __shared__ float sd[kRecChunk];
  const int Wm = (m + 31) >> 5, Wn = (n + 31) >> 5;
  const int rw = blockIdx.y;                  // row word: rows 32*rw .. 32*rw+31
  const int j = blockIdx.x * kRecCols + threadIdx.x;
  const int jw = j >> 5, jb = j & 31;
  double acc[32];
#pragma unroll
  for (int r = 0; r < 32; ++r) acc[r] = 0.0;
  for (int c0 = 0; c0 < k; c0 += kRecChunk) {
    const int nc = min(kRecChunk, k - c0);
    __syncthreads();
    for (int t = threadIdx.x; t < nc; t += kRecCols) {
      su[t][0] = pB[(size_t)(c0 + t) * 2 * Wm + rw];
      su[t][1] = pB[(size_t)(c0 + t) * 2 * Wm + Wm + rw];
      sd[t] = D[c0 + t];
    }
    __syncthreads();
    if (j < n) {
      for (int t = 0; t < nc; ++t) {
        const uint32_t vm = pC[(size_t)(c0 + t) * 2 * Wn + jw];
        if (!((vm >> jb) & 1u)) continue;
        const uint32_t vs = pC[(size_t)(c0 + t) * 2 * Wn + Wn + jw];
        const double d = (double)sd[t];
        const double dv = ((vs >> jb) & 1u) ? -d : d;
        const uint32_t um = su[t][0], us = su[t][1];
#pragma unroll
        for (int r = 0; r < 32; ++r)
          if ((um >> r) & 1u) acc[r] += ((us >> r) & 1u) ? -dv : dv;
      }
    }
  }
  if (j < n) {
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      const int i = rw * 32 + r;
      if (i < m) out[(size_t)i * n + j] = (float)acc[r];
    }
  }
}

int reconstruct(const uint32_t* pB, const uint32_t* pC, const float* D, int64_t m, int64_t n,
                int64_t k, float* out, cudaStream_t st) {
  dim3 grid((unsigned)((n + kRecCols - 1) / kRecCols), (unsigned)((m + 31) / 32));
  reconstruct_kernel<<<grid, kRecCols, 0, st>>>(pB, pC, D, (int)m, (int)n, (int)k, out);
  if (cudaGetLastError() != cudaSuccess) return EXTERND_ERR_CUDA;
  return EXTERND_OK;
}

}  // namespace externd
