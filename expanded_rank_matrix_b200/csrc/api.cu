// C ABI of libexternd.so: argument checks and dispatch (declarations and the
// contract of every entry point are in include/externd.h).

#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "../../include/externd.h"
#include "internal.h"

namespace {

bool aligned4(const void* p) { return ((uintptr_t)p & 3u) == 0; }

bool sizes_ok(int64_t m, int64_t n) {
  return m >= 1 && n >= 1 && m <= (int64_t)1 << 30 && n <= (int64_t)1 << 30 &&
         m * n < ((int64_t)1 << 31);
}

}  // namespace

extern "C" {

int64_t externd_rank(int64_t m, int64_t n, float mu) {
  if (!sizes_ok(m, n) || !(mu > 0.0f) || !std::isfinite(mu)) return 0;
  const double k = std::floor((double)mu * (double)(m < n ? m : n) + 1e-9);
  if (k < 1.0 || k > 2147483647.0) return 0;
  return (int64_t)k;
}

int externd_decompose_traced(const float* A, int64_t m, int64_t n, float mu, float tau, int iters,
                             const float* w, int block, unsigned flags, int sweeps,
                             uint32_t* packed_B, uint32_t* packed_C, float* D,
                             double* energy_trace, double* sweep_energy, int64_t ntrace,
                             const int64_t* trace_comp, uint32_t* trace_bits, int32_t* trace_row,
                             uint8_t* trace_flags, int64_t* stats, int64_t wait_budget,
                             externd_stream_t stream) {
  if (!A || !packed_B || !packed_C || !D || !energy_trace) return EXTERND_ERR_INVALID_ARG;
  if (!aligned4(A) || !aligned4(packed_B) || !aligned4(packed_C) || !aligned4(D) ||
      ((uintptr_t)energy_trace & 7u) || (w && !aligned4(w)))
    return EXTERND_ERR_INVALID_ARG;
  if (!sizes_ok(m, n)) return EXTERND_ERR_INVALID_ARG;
  const int64_t k = externd_rank(m, n, mu);
  if (k < 1) return EXTERND_ERR_INVALID_ARG;
  if (!(tau >= 0.0f) || !std::isfinite(tau)) return EXTERND_ERR_INVALID_ARG;
  if (iters < 1 || iters > 1000) return EXTERND_ERR_INVALID_ARG;
  if (block < 1 || block > 64 || block > k || block > (m < n ? m : n)) return EXTERND_ERR_INVALID_ARG;
  if (flags & ~(unsigned)(EXTERND_TSTAT_MEAN_ABS | EXTERND_VSTEP_NAIVE)) return EXTERND_ERR_INVALID_ARG;
  if (sweeps < 0 || sweeps > EXTERND_MAX_SWEEPS || (sweeps > 0 && block != 1))
    return EXTERND_ERR_INVALID_ARG;
  if (sweeps > 0 && (!sweep_energy || ((uintptr_t)sweep_energy & 7u))) return EXTERND_ERR_INVALID_ARG;
  if (k * (1 + (int64_t)sweeps) > 2147483647LL) return EXTERND_ERR_INVALID_ARG;
  if (ntrace < 0 || wait_budget < 0) return EXTERND_ERR_INVALID_ARG;
  if (ntrace > 0 && (!trace_comp || !trace_bits || !trace_row || !trace_flags || block != 1))
    return EXTERND_ERR_INVALID_ARG;
  if (stats && ((uintptr_t)stats & 7u)) return EXTERND_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (block == 1) {
    externd::SeqHostArgs h = {};
    h.A = A; h.m = m; h.n = n; h.k = k; h.tau = tau; h.iters = iters; h.w = w;
    h.packed_B = packed_B; h.packed_C = packed_C; h.D = D; h.energy = energy_trace;
    h.ntrace = ntrace; h.trace_comp = trace_comp; h.trace_bits = trace_bits;
    h.trace_row = trace_row; h.trace_flags = trace_flags; h.stats = stats;
    h.wait_budget = wait_budget; h.flags = flags; h.sweeps = sweeps;
    h.sweep_energy = sweep_energy;
    return externd::seq_decompose(h, st);
  }
  externd::BlockHostArgs b = {};
  b.A = A; b.m = m; b.n = n; b.k = k; b.tau = tau; b.iters = iters; b.w = w; b.block = block;
  b.packed_B = packed_B; b.packed_C = packed_C; b.D = D; b.energy = energy_trace; b.stats = stats;
  b.flags = flags;
  return externd::block_decompose(b, st);
}

int externd_decompose_block_traced(const float* A, int64_t m, int64_t n, float mu, float tau,
                                   int iters, const float* w, int block, unsigned flags,
                                   uint32_t* packed_B,
                                   uint32_t* packed_C, float* D, double* energy_trace,
                                   int64_t ntrace, const int64_t* trace_block, uint64_t* trace_uv,
                                   int32_t* trace_rows, int64_t wait_budget,
                                   externd_stream_t stream) {
  if (block < 2 || wait_budget < 0) return EXTERND_ERR_INVALID_ARG;
  if (ntrace < 0 || (ntrace > 0 && (!trace_block || !trace_uv || !trace_rows)))
    return EXTERND_ERR_INVALID_ARG;
  if (!A || !packed_B || !packed_C || !D || !energy_trace) return EXTERND_ERR_INVALID_ARG;
  if (!aligned4(A) || !aligned4(packed_B) || !aligned4(packed_C) || !aligned4(D) ||
      ((uintptr_t)energy_trace & 7u) || (w && !aligned4(w)) || ((uintptr_t)trace_uv & 7u))
    return EXTERND_ERR_INVALID_ARG;
  if (!sizes_ok(m, n)) return EXTERND_ERR_INVALID_ARG;
  const int64_t k = externd_rank(m, n, mu);
  if (k < 1) return EXTERND_ERR_INVALID_ARG;
  if (!(tau >= 0.0f) || !std::isfinite(tau)) return EXTERND_ERR_INVALID_ARG;
  if (iters < 1 || iters > 1000) return EXTERND_ERR_INVALID_ARG;
  if (block > 64 || block > k || block > (m < n ? m : n)) return EXTERND_ERR_INVALID_ARG;
  if (flags & ~(unsigned)(EXTERND_TSTAT_MEAN_ABS | EXTERND_VSTEP_NAIVE)) return EXTERND_ERR_INVALID_ARG;
  externd::BlockHostArgs b = {};
  b.A = A; b.m = m; b.n = n; b.k = k; b.tau = tau; b.iters = iters; b.w = w; b.block = block;
  b.packed_B = packed_B; b.packed_C = packed_C; b.D = D; b.energy = energy_trace;
  b.ntrace = ntrace; b.trace_block = trace_block; b.trace_uv = trace_uv; b.trace_rows = trace_rows;
  b.flags = flags; b.wait_budget = wait_budget;
  return externd::block_decompose(b, (cudaStream_t)stream);
}

int externd_decompose_ex(const float* A, int64_t m, int64_t n, float mu, float tau, int iters,
                         const float* w, int block, unsigned flags, int sweeps,
                         uint32_t* packed_B, uint32_t* packed_C, float* D, double* energy_trace,
                         double* sweep_energy, externd_stream_t stream) {
  return externd_decompose_traced(A, m, n, mu, tau, iters, w, block, flags, sweeps, packed_B,
                                  packed_C, D, energy_trace, sweep_energy, 0, nullptr, nullptr,
                                  nullptr, nullptr, nullptr, 0, stream);
}

int externd_decompose(const float* A, int64_t m, int64_t n, float mu, float tau, int iters,
                      const float* w, int block, uint32_t* packed_B, uint32_t* packed_C,
                      float* D, double* energy_trace, externd_stream_t stream) {
  return externd_decompose_ex(A, m, n, mu, tau, iters, w, block, 0u, 0, packed_B, packed_C, D,
                              energy_trace, nullptr, stream);
}

int externd_reconstruct(const uint32_t* packed_B, const uint32_t* packed_C, const float* D,
                        int64_t m, int64_t n, int64_t k, float* A_hat, externd_stream_t stream) {
  if (!packed_B || !packed_C || !D || !A_hat) return EXTERND_ERR_INVALID_ARG;
  if (!aligned4(packed_B) || !aligned4(packed_C) || !aligned4(D) || !aligned4(A_hat))
    return EXTERND_ERR_INVALID_ARG;
  if (!sizes_ok(m, n) || k < 1 || k > 2147483647LL) return EXTERND_ERR_INVALID_ARG;
  return externd::reconstruct(packed_B, packed_C, D, m, n, k, A_hat, (cudaStream_t)stream);
}

int externd_ternary_apply(const uint32_t* packed_B, const uint32_t* packed_C, const float* D,
                          int64_t m, int64_t n, int64_t k, const float* X, int64_t nb, float* Y,
                          externd_stream_t stream) {
  if (!packed_B || !packed_C || !D || !X || !Y) return EXTERND_ERR_INVALID_ARG;
  if (!aligned4(packed_B) || !aligned4(packed_C) || !aligned4(D) || !aligned4(X) || !aligned4(Y))
    return EXTERND_ERR_INVALID_ARG;
  if (!sizes_ok(m, n) || m > EXTERND_APPLY_MAX_ROWS || k < 1 || k > 2147483647LL)
    return EXTERND_ERR_INVALID_ARG;
  if (nb < 1 || nb > 65536 || nb * (m > n ? m : n) >= ((int64_t)1 << 31))
    return EXTERND_ERR_INVALID_ARG;
  return externd::ternary_apply(packed_B, packed_C, D, m, n, k, X, nb, Y, (cudaStream_t)stream);
}

int externd_release_cache(void) {
  const int a = externd::block_release_graphs();
  const int b = externd::apply_trim_pools();
  return a != EXTERND_OK ? a : b;
}

int externd_sync_status(externd_stream_t stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return EXTERND_ERR_CUDA;
  int* p = externd::status_word_ptr();
  if (!p) return EXTERND_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return EXTERND_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
    return EXTERND_ERR_CUDA;
  return v;
}

}  // extern "C"
