// Per-matrix rank allocation to an energy target, on the device.
//
// The pages tune the rank multiplier per matrix so that each matrix reaches
// a reference quantiser's energy (romaanj.github.io review, "Results"; the
// Pith review's "Assumptions & free parameters" lists mu = 1.97 .. 3.43 per
// matrix).  Greedy sequential deflation fixes component c from the residual
// of components 0 .. c-1 alone, so a decomposition at rank k holds every
// shorter one as its prefix: the rank a target needs is read off one run's
// energy trace as the first c with energy[c] >= target, plus one.

#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "../../include/externd.h"

namespace {

constexpr int kScanThreads = 256;

// One block: scans the trace in chunks of kScanThreads and stops at the first
// chunk holding a hit; the lowest hit index wins.
__global__ void __launch_bounds__(kScanThreads) rank_for_energy_kernel(const double* e,
                                                                         long long k,
                                                                         double target,
                                                                         long long* out) {
  __shared__ unsigned long long first;
  if (threadIdx.x == 0) first = ~0ull;
  __syncthreads();
  for (long long base = 0; base < k; base += kScanThreads) {
    const long long c = base + threadIdx.x;
    if (c < k && e[c] >= target) atomicMin(&first, (unsigned long long)c);
    __syncthreads();
    const bool done = first != ~0ull;  // the same value in every thread
    __syncthreads();                   // nobody writes before everyone has read
    if (done) break;
  }
  if (threadIdx.x == 0) *out = first == ~0ull ? 0 : (long long)first + 1;
}

}  // namespace

extern "C" int externd_rank_for_energy(const double* energy_trace, int64_t k, double target,
                                       int64_t* rank, externd_stream_t stream) {
  if (!energy_trace || !rank || k < 1 || !std::isfinite(target)) return EXTERND_ERR_INVALID_ARG;
  if (((uintptr_t)energy_trace & 7u) || ((uintptr_t)rank & 7u)) return EXTERND_ERR_INVALID_ARG;
  rank_for_energy_kernel<<<1, kScanThreads, 0, (cudaStream_t)stream>>>(
      energy_trace, (long long)k, target, (long long*)rank);
  if (cudaGetLastError() != cudaSuccess) return EXTERND_ERR_CUDA;
  return EXTERND_OK;
}
