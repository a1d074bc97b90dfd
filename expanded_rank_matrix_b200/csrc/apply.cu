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
// One persistent launch, one CTA per SM.  CTA g owns a contiguous run of
// components; it needs only that run's rows of C and columns of B, which
// are contiguous in the component-major packed layout, so at launch it
// starts asynchronous copies (cp.async) of the whole run into shared memory
// -- every SM's share of the factor traffic is in flight at once -- and then
//  1. sums s_c for its components (a warp per component, lanes over words;
//     x sits in shared memory with the entries of word w rotated by w, so the
//     lanes read distinct banks at every bit);
//  2. adds its components' contributions to every y_i (threads own packed row
//     words of B and keep their 32 rows in registers; the CTA's component
//     streams are summed in shared memory) and writes its partial y;
//  3. after one grid barrier (a bounded wait; the launch is cooperative, so
//     every CTA is resident), sums the CTAs' partials: eight threads per
//     output take a slice of CTAs each, loads in flight together, and their
//     sums are combined by a fixed butterfly.
// Runs longer than the shared-memory budget are processed in chunks.  Every
// sum has a fixed order, so results are reproducible run to run.

#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/externd.h"
#include "common.cuh"
#include "internal.h"

namespace externd {
namespace {

constexpr int kApThreads = 512;
constexpr int kApWarps = kApThreads / 32;
constexpr int kRedThreads = 8;  // threads per output in the final sum
constexpr int kRedSlice = 32;   // CTA partials one such thread loads at once (at most)

struct ApArgs {
  const uint32_t* pB;  // [k][2][Wm]
  const uint32_t* pC;  // [k][2][Wn]
  const float* D;
  const float* X;      // [nb][n] (this launch's vectors)
  float* Y;            // [nb][m]
  float* P;            // [G][m][NB] scratch: per-CTA partial y
  unsigned* bar;       // grid barrier counter
  int m, n, k, nb;
  int CC;              // components per chunk of a CTA's run
  long long budget;
  int* status;
};

__device__ __forceinline__ void cp_async4(uint32_t* sdst, const uint32_t* gsrc) {
  const unsigned s = (unsigned)__cvta_generic_to_shared(sdst);
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(s), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_all;" ::: "memory");
}

template <int NB>
__global__ void __launch_bounds__(kApThreads, 1) apply_kernel(const ApArgs a) {
  extern __shared__ __align__(16) unsigned char asm_[];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int m = a.m, n = a.n, k = a.k;
  const int Wm = (m + 31) >> 5, Wn = (n + 31) >> 5;
  const int G = gridDim.x, g = blockIdx.x;
  const int cb = (int)((long long)g * k / G), ce = (int)((long long)(g + 1) * k / G);
  // shared memory: x [Wn*32][NB] (rotated), y [32][Wm+1][NB] (row 32 tw + r
  // of word tw at [r][tw]: the lanes of a warp, one word each, write
  // consecutive slots), s [CC][NB], C run [CC][2][Wn], B run [CC][2][Wm]
  const int YW = Wm + 1;
  float* xs = (float*)asm_;
  float* ys = xs + (size_t)Wn * 32 * NB;
  float* ss = ys + (size_t)32 * YW * NB;
  uint32_t* Cs = (uint32_t*)(ss + (size_t)a.CC * NB);
  uint32_t* Bs = Cs + (size_t)a.CC * 2 * Wn;

  const int WG = (Wm + 31) >> 5;              // warps per set of all row words
  const int NSt = max(1, kApWarps / WG);      // component streams
  const int st = wid / WG;
  float acc[32][NB];
#pragma unroll
  for (int r = 0; r < 32; ++r)
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[r][b] = 0.f;

  for (int c0 = cb; c0 < ce; c0 += a.CC) {
    const int cn = min(a.CC, ce - c0);
    // ---- this chunk's rows of C and columns of B, copied asynchronously ----
    {
      const uint32_t* srcC = a.pC + (size_t)c0 * 2 * Wn;
      const uint32_t* srcB = a.pB + (size_t)c0 * 2 * Wm;
      const int nC = cn * 2 * Wn, nB = cn * 2 * Wm;
      for (int e = tid; e < nC; e += kApThreads) cp_async4(Cs + e, srcC + e);
      for (int e = tid; e < nB; e += kApThreads) cp_async4(Bs + e, srcB + e);
    }
    if (c0 == cb) {
      // x, rotated within each word (while the copies are in flight)
      for (int e = tid; e < Wn * 32; e += kApThreads) {
        const int w = e >> 5, r = e & 31;
#pragma unroll
        for (int b = 0; b < NB; ++b)
          xs[((w << 5) + ((r + w) & 31)) * NB + b] =
              (b < a.nb && e < n) ? __ldg(a.X + (size_t)b * n + e) : 0.f;
      }
    }
    cp_async_wait_all();
    __syncthreads();

    // ---- 1. s_c = D_c sum_j C_cj x_j for the chunk's components ----
    for (int cl = wid; cl < cn; cl += kApWarps) {
      const uint32_t* mk = Cs + (size_t)cl * 2 * Wn;
      float t[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) t[b] = 0.f;
      for (int w = lane; w < Wn; w += 32) {
        const uint32_t mw = mk[w], sw = mk[Wn + w];
        const uint32_t pos = mw & ~sw, neg = mw & sw;
        const float* xw = xs + (size_t)(w << 5) * NB;
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          // the word's 32 entries loaded together, summed in four chains
          float xv[32];
#pragma unroll
          for (int r = 0; r < 32; ++r) xv[r] = xw[((r + w) & 31) * NB + b];
          float c4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int r = 0; r < 32; ++r) {
            if ((pos >> r) & 1u) c4[r & 3] += xv[r];
            if ((neg >> r) & 1u) c4[r & 3] -= xv[r];
          }
          t[b] += (c4[0] + c4[1]) + (c4[2] + c4[3]);
        }
      }
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        float v = t[b];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) ss[cl * NB + b] = __ldg(a.D + c0 + cl) * v;
      }
    }
    __syncthreads();

    // ---- 2. the chunk's contributions to every y_i ----
    if (st < NSt) {
      const int tw = (wid % WG) * 32 + lane;  // my row word
      if (tw < Wm) {
        for (int cl = st; cl < cn; cl += NSt) {
          const uint32_t mw = Bs[(size_t)cl * 2 * Wm + tw], sw = Bs[(size_t)cl * 2 * Wm + Wm + tw];
          const uint32_t pos = mw & ~sw, neg = mw & sw;
          float sv[NB];
#pragma unroll
          for (int b = 0; b < NB; ++b) sv[b] = ss[cl * NB + b];
#pragma unroll
          for (int r = 0; r < 32; ++r)
#pragma unroll
            for (int b = 0; b < NB; ++b) {
              if ((pos >> r) & 1u) acc[r][b] += sv[b];
              if ((neg >> r) & 1u) acc[r][b] -= sv[b];
            }
        }
      }
    }
    __syncthreads();  // the next chunk's copies overwrite Cs, Bs and ss
  }

  // ---- the CTA's partial y: its streams summed in stream order ----
  {
    const int tw = (wid % WG) * 32 + lane;
    const bool active = st < NSt && tw < Wm;
    for (int s2 = 0; s2 < NSt; ++s2) {
      if (st == s2 && active) {
#pragma unroll
        for (int r = 0; r < 32; ++r)
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            float* p = ys + ((size_t)r * YW + tw) * NB + b;
            *p = s2 == 0 ? acc[r][b] : *p + acc[r][b];
          }
      }
      __syncthreads();
    }
    float* Pg = a.P + (size_t)g * m * NB;
    for (int e = tid; e < m * NB; e += kApThreads) {
      const int i = e / NB, b = e - i * NB;
      Pg[e] = ys[((size_t)(i & 31) * YW + (i >> 5)) * NB + b];
    }
  }

  // ---- grid barrier: every CTA's partial written and visible ----
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    atomicAdd(a.bar, 1u);
    const long long t0 = clock64();
    while (true) {
      unsigned v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a.bar) : "memory");
      if (v >= (unsigned)G) break;
      if (clock64() - t0 > a.budget) {
        atomicCAS(a.status, 0, EXTERND_ERR_TIMEOUT);
        break;
      }
    }
    __threadfence();
  }
  __syncthreads();

  // ---- 3. y = sum of the CTAs' partials ----
  {
    const int per = (G + kRedThreads - 1) / kRedThreads;  // CTAs per thread (<= kRedSlice)
    const long long nout = (long long)m * NB, ntot = nout * kRedThreads;
    // whole warps step together (the butterfly below needs every lane)
    for (long long w0 = (long long)g * kApThreads + wid * 32; w0 < ntot;
         w0 += (long long)G * kApThreads) {
      const long long e8 = w0 + lane;
      const bool ok = e8 < ntot;
      const long long e = ok ? e8 / kRedThreads : 0;
      const int h = (int)(e8 % kRedThreads);
      const int g0 = h * per, g1 = ok ? min(G, g0 + per) : g0;
      float v[kRedSlice];
#pragma unroll
      for (int u = 0; u < kRedSlice; ++u)
        v[u] = (g0 + u < g1) ? __ldcg(a.P + (size_t)(g0 + u) * m * NB + e) : 0.f;
      float sacc = 0.f;
#pragma unroll
      for (int u = 0; u < kRedSlice; ++u) sacc += v[u];
      // the eight slices of one output sit in eight adjacent lanes
      sacc += __shfl_xor_sync(0xffffffffu, sacc, 1);
      sacc += __shfl_xor_sync(0xffffffffu, sacc, 2);
      sacc += __shfl_xor_sync(0xffffffffu, sacc, 4);
      if (ok && h == 0) {
        const int i = (int)(e / NB), b = (int)(e % NB);
        if (b < a.nb) a.Y[(size_t)b * m + i] = sacc;
      }
    }
  }
}

template <int NB>
int launch_apply(ApArgs a, int G, size_t smem, cudaStream_t st) {
  auto kern = apply_kernel<NB>;
  void* params[] = {&a};
  if (cudaLaunchCooperativeKernel((const void*)kern, dim3(G), dim3(kApThreads), params, smem,
                                  st) != cudaSuccess) {
    cudaGetLastError();
    return EXTERND_ERR_CUDA;
  }
  return EXTERND_OK;
}

// The scratch of every call comes from a pool this library owns on each
// device, which keeps its memory mapped between calls (the default pool
// returns freed memory at every synchronisation, and mapping it again costs
// more than the kernel).
std::mutex g_pool_mu;
cudaMemPool_t g_pools[64] = {};

cudaMemPool_t apply_pool(int dev) {
  cudaMemPool_t* const pools = g_pools;
  if (dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_pool_mu);
  if (!pools[dev]) {
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t p = nullptr;
    if (cudaMemPoolCreate(&p, &props) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    unsigned long long keep = ~0ull;
    cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &keep);
    pools[dev] = p;
  }
  return pools[dev];
}

}  // namespace

// Returns the memory the pools hold beyond what queued calls still use.
int apply_trim_pools() {
  std::lock_guard<std::mutex> lk(g_pool_mu);
  int rc = EXTERND_OK;
  for (cudaMemPool_t p : g_pools)
    if (p && cudaMemPoolTrimTo(p, 0) != cudaSuccess) {
      cudaGetLastError();
      rc = EXTERND_ERR_CUDA;
    }
  return rc;
}

int ternary_apply(const uint32_t* pB, const uint32_t* pC, const float* D, int64_t m, int64_t n,
                  int64_t k, const float* X, int64_t nb, float* Y, cudaStream_t st) {
  int dev = 0, nsm = 0, optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return EXTERND_ERR_CUDA;
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const int NB = nb >= 2 ? 2 : 1;
  const int Wm = (int)((m + 31) / 32), Wn = (int)((n + 31) / 32);
  const int G = nsm;  // one CTA per SM
  if ((G + kRedThreads - 1) / kRedThreads > kRedSlice) return EXTERND_ERR_INVALID_ARG;
  // shared memory: x and y (fixed), then per component of a chunk its C row,
  // its B column and its s
  const size_t fixed = sizeof(float) * ((size_t)Wn * 32 + (size_t)32 * (Wm + 1)) * NB;
  const size_t per_comp = sizeof(uint32_t) * 2 * ((size_t)Wm + Wn) + sizeof(float) * NB;
  if (fixed + per_comp > (size_t)optin) return EXTERND_ERR_INVALID_ARG;
  const int run = (int)((k + G - 1) / G);
  int CC = (int)(((size_t)optin - fixed) / per_comp);
  if (CC > run) CC = run;
  const size_t smem = fixed + per_comp * (size_t)CC;
  // The kernel attribute and the co-residency check are done once per device
  // and launch shape (they cost far more than the launch itself).
  struct Ready {
    int dev, NB;
    size_t smem;
  };
  static std::mutex mu;
  static Ready ready[16];
  static int nready = 0;
  bool known = false;
  {
    std::lock_guard<std::mutex> lk(mu);
    for (int i = 0; i < nready; ++i)
      known = known || (ready[i].dev == dev && ready[i].NB == NB && ready[i].smem == smem);
  }
  if (!known) {
    // (the dynamic shared-memory limit first: the occupancy query honours it)
    cudaError_t e = NB == 2 ? cudaFuncSetAttribute(apply_kernel<2>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   (int)smem)
                            : cudaFuncSetAttribute(apply_kernel<1>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   (int)smem);
    int per_sm = 0;
    if (e == cudaSuccess)
      e = NB == 2 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, apply_kernel<2>,
                                                                  kApThreads, smem)
                  : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, apply_kernel<1>,
                                                                  kApThreads, smem);
    if (e != cudaSuccess || per_sm < 1) {
      cudaGetLastError();
      return EXTERND_ERR_NO_COOP;
    }
    std::lock_guard<std::mutex> lk(mu);
    if (nready < 16) ready[nready++] = Ready{dev, NB, smem};
  }
  const size_t oP = 0;
  const size_t oBar = (sizeof(float) * (size_t)G * m * NB + 255) & ~(size_t)255;
  void* ws = nullptr;
  cudaMemPool_t pool = apply_pool(dev);
  if (!pool || cudaMallocFromPoolAsync(&ws, oBar + 256, pool, st) != cudaSuccess) {
    cudaGetLastError();
    return EXTERND_ERR_OOM;
  }
  int rc = EXTERND_OK;
  ApArgs a = {};
  a.pB = pB; a.pC = pC; a.D = D;
  a.P = (float*)((char*)ws + oP);
  a.bar = (unsigned*)((char*)ws + oBar);
  a.m = (int)m; a.n = (int)n; a.k = (int)k; a.CC = CC;
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
