// externd_decompose_noalloc: the sequential decomposition with its scratch
// memory in a fixed array inside this library instead of a per-call
// allocation (see the entry point's description in include/externd.h).

#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/externd.h"
#include "internal.h"

namespace {

// The scratch every externd_decompose_noalloc call on a device uses: the
// cross-CTA exchange ring and the abort word.  Each device that loads the
// library holds EXTERND_NOALLOC_SCRATCH_BYTES of it until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[EXTERND_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device.  In host code
// the array's name only stands in for the device object, so the address is
// looked up once per device, with that device current, and cached.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return EXTERND_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return EXTERND_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return EXTERND_OK;
}

bool aligned4(const void* p) { return ((uintptr_t)p & 3u) == 0; }

}  // namespace

extern "C" int externd_decompose_noalloc(const float* A, int64_t m, int64_t n, float mu,
                                         float tau, int iters, const float* w,
                                         uint32_t* packed_B, uint32_t* packed_C, float* D,
                                         double* energy_trace, externd_stream_t stream) {
  if (!A || !packed_B || !packed_C || !D || !energy_trace) return EXTERND_ERR_INVALID_ARG;
  if (!aligned4(A) || !aligned4(packed_B) || !aligned4(packed_C) || !aligned4(D) ||
      ((uintptr_t)energy_trace & 7u) || (w && !aligned4(w)))
    return EXTERND_ERR_INVALID_ARG;
  const int64_t k = externd_rank(m, n, mu);
  if (k < 1) return EXTERND_ERR_INVALID_ARG;
  if (!(tau >= 0.0f) || !std::isfinite(tau)) return EXTERND_ERR_INVALID_ARG;
  if (iters < 1 || iters > 1000) return EXTERND_ERR_INVALID_ARG;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != EXTERND_OK) return rc;
  externd::SeqHostArgs h = {};
  h.A = A; h.m = m; h.n = n; h.k = k; h.tau = tau; h.iters = iters; h.w = w;
  h.packed_B = packed_B; h.packed_C = packed_C; h.D = D; h.energy = energy_trace;
  return externd::seq_decompose_with_scratch(h, scratch, EXTERND_NOALLOC_SCRATCH_BYTES,
                                             (cudaStream_t)stream);
}
