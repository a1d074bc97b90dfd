// Greedy sequential-deflation ALS for ExTernD, as one persistent kernel.
//
// Method (arXiv:2607.13511 as summarised by the Pith review's referee report,
// paper Sec. 2.3, and the romaanj.github.io review's "Method"): for each
// component, start from the ternarised largest-energy residual row, run
// `iters` rounds of u = T_tau(R W v), v = T_tau(R^T u), take the closed-form
// scale d = u^T R W v / (|u|^2 v^T W v), fall back to the best single entry
// when that gain is below it (Appendix A, Prop. 2), and deflate
// R <- R - d u v^T before the next component.
//
// Layout.  The grid is NC clusters of CS CTAs, one CTA per SM.  Cluster c
// owns a band of rows, CTA q of the cluster owns a band of columns (a run of
// 32-column chunks), so every CTA holds one TR x TC tile of the residual --
// in shared memory when the whole matrix fits in the grid's shared memory,
// otherwise in a private global-memory (L2/HBM) region that the CTA streams.
// The tile never moves; only vectors do:
//  * R W v: partial row sums per CTA, all-gathered inside the cluster through
//    distributed shared memory; the cluster's sum of y^2 crosses clusters.
//  * R^T u: partial column sums per cluster cross clusters; each CTA sums the
//    NC partials of its own columns in a fixed order, so every cluster holds
//    the same z; sum z^2 is combined inside the cluster.
// Cross-cluster data moves through flag-tagged 64-bit words (payload +
// epoch), so the arrival of the data is the synchronisation; independent
// words are loaded back to back before any of them is waited on.  Every wait
// is bounded; a wait that runs out raises EXTERND_ERR_TIMEOUT and the kernel
// winds down without further waits.  All reductions run in a fixed order,
// so results are bit-reproducible run to run.

#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <cstdlib>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace externd {

__device__ int g_status = 0;  // per-device sticky status (first error wins)

int* status_word_ptr() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
  return (int*)p;
}

struct SeqArgs {
  const float* A;
  int m, n, k;
  float tau;
  int iters;
  const float* w;
  uint32_t* pB;
  uint32_t* pC;
  float* D;
  double* energy;
  int NC, CS, nchc;
  int TRmax, TCp, recw;
  int SR;        // leading rows of each CTA's tile held in shared memory
  float* gtile;  // the remaining TRmax - SR rows of each CTA, in global memory
  uint64_t* xbuf;
  long long slot_words;
  const int64_t* trace_comp;
  int ntrace;
  uint32_t* trace_bits;
  int32_t* trace_row;
  uint8_t* trace_flags;
  int64_t* stats;
  long long budget;
  int* abort_word;
  int* dev_status;
};

// phases timed (SM cycles, CTA 0) into stats[kStatPhase0 + p]
enum {
  PH_SETUP = 0,
  PH_YPASS,
  PH_YGATHER,
  PH_YXCHG,
  PH_ZPASS,
  PH_ZXCHG,
  PH_ZSYNC,
  PH_SCALE,
  PH_DEFLATE,
  PH_STATS,
  PH_N
};
constexpr int kStatPhase0 = 6;

// Shared-memory carve-up, identical on host and device.
//  gat   [CS][TRp]  row partials pushed by every CTA of the cluster (R W v
//                   partials, or the row energies in the statistics step)
//  zall  [CS][TCp]  z of every column of the cluster (pushed by each CTA)
//  wall  [CS][TCp]  weight of every column of the cluster
//  zred  [RG][TCp]  R^T u partials per row group; also holds y after the
//                   gather (their lifetimes are disjoint)
struct SeqSmem {
  size_t wp, wpi, misc, rss, xd, xu, erec, abg, tile, uval, ypart, gat, rho_p, rmax, rmaxj, zred,
      zall, wall, wcol, vval, nnzu, total;
  __host__ __device__ SeqSmem(int TRmax, int TCp, int NC, int CS, int NQL, int SR, bool weighted) {
    const int TRp = (TRmax + 31) & ~31;
    const int RG = kWarps / NQL;
    size_t o = 0;
    auto take = [&](size_t bytes) {
      size_t r = o;
      o += (bytes + 15) & ~(size_t)15;
      return r;
    };
    wp = take(sizeof(double) * 2 * kWarps * 4);  // block-reduction partials
    wpi = take(sizeof(int) * 2 * kWarps);
    misc = take(sizeof(double) * 32);
    rss = take(sizeof(double) * 16);       // row sums of squares of the start row
    xd = take(sizeof(double) * 2 * NC);    // per-cluster fp64 records
    xu = take(sizeof(uint32_t) * 6 * NC);  // per-cluster 32-bit records
    erec = take(sizeof(double) * 4 * CS);  // per-CTA best entry (pushed)
    abg = take(sizeof(int) * CS);          // per-CTA abort flags (pushed)
    uval = take(sizeof(float) * TRp);
    gat = take(sizeof(float) * (size_t)CS * TRp);
    rho_p = take(sizeof(float) * TRp);
    rmax = take(sizeof(float) * TRp);
    rmaxj = take(sizeof(int) * TRp);
    const size_t zb = sizeof(float) * (size_t)RG * TCp;
    const size_t yb = sizeof(float) * TRp;
    zred = take(zb > yb ? zb : yb);
    ypart = zred;
    zall = take(sizeof(float) * (size_t)CS * TCp);
    wall = take(weighted ? sizeof(float) * (size_t)CS * TCp : 0);
    wcol = take(sizeof(float) * TCp);
    vval = take(sizeof(float) * TCp);
    nnzu = take(sizeof(int) * NC);
    tile = take(sizeof(float) * (size_t)SR * TCp);
    total = o;
  }
};

// misc[] slots (doubles)
enum {
  MS_E0 = 0,
  MS_R2,
  MS_M,      // entry score of the best single entry (as fp64)
  MS_MVAL,   // its signed value
  MS_MI,     // its row
  MS_MJ,     // its column
  MS_ISTAR,  // starting row of the component
  MS_BAD,
  MS_ABORT,  // cluster-wide abort decision of the last decision point
  MS_PH = 16 // phase timers (long long, CTA 0 thread 0 only)
};

__device__ __forceinline__ float tern(float x, double thr) {
  double a = fabs((double)x);
  return a > thr ? (x > 0.f ? 1.f : -1.f) : 0.f;
}

// Packed bitplanes of the ternary values vals[0..len) (floats in {-1,0,1})
// that stand for global entries [g0, g0+len), g0 % 32 == 0: plain stores into
// plane0[g0/32 ..] and plane0[W + g0/32 ..].  One warp per word.
__device__ __forceinline__ void pack_planes(const float* vals, int len, int g0, uint32_t* plane0,
                                            int W) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nw = (len + 31) >> 5;
  for (int t = wid; t < nw; t += kWarps) {
    const int e = t * 32 + lane;
    const float x = e < len ? vals[e] : 0.f;
    const uint32_t mk = __ballot_sync(0xffffffffu, x != 0.f);
    const uint32_t sg = __ballot_sync(0xffffffffu, x < 0.f);
    if (lane == 0) {
      plane0[(g0 >> 5) + t] = mk;
      plane0[W + (g0 >> 5) + t] = sg;
    }
  }
}

// Same for an arbitrary start g0: words are shared with the neighbouring
// bands, so the bits are OR-ed into zero-initialised planes.
__device__ __forceinline__ void pack_planes_or(const float* vals, int len, int g0,
                                               uint32_t* plane0, int W) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int w0 = g0 >> 5, w1 = (g0 + len + 31) >> 5;
  for (int t = w0 + wid; t < w1; t += kWarps) {
    const int e = t * 32 + lane - g0;
    const float x = (e >= 0 && e < len) ? vals[e] : 0.f;
    const uint32_t mk = __ballot_sync(0xffffffffu, x != 0.f);
    const uint32_t sg = __ballot_sync(0xffffffffu, x < 0.f);
    if (lane == 0) {
      if (mk) atomicOr(plane0 + t, mk);
      if (sg) atomicOr(plane0 + W + t, sg);
    }
  }
}

__device__ __forceinline__ long long tick() { return clock64(); }

// Split cluster barrier: arrive (release) now, wait (acquire) later.
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Two flag-tagged words at once (16-byte aligned pair).
__device__ __forceinline__ void xw_store2(uint64_t* p, uint32_t epoch, uint32_t a, uint32_t b) {
  const uint64_t va = ((uint64_t)epoch << 32) | a, vb = ((uint64_t)epoch << 32) | b;
  asm volatile("st.relaxed.gpu.global.v2.b64 [%0], {%1, %2};" ::"l"(p), "l"(va), "l"(vb)
               : "memory");
}
__device__ __forceinline__ void xw_load2(const uint64_t* p, uint64_t& a, uint64_t& b) {
  asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "l"(p)
               : "memory");
}

// Deterministic block reductions with a single barrier: warp trees, then
// every thread adds the kWarps warp partials in warp order itself.  `wp`
// holds two alternating [kWarps][4] buffers selected by `ph`.
template <int NV>
__device__ __forceinline__ void bsum(double (&x)[NV], double* wp, int& ph) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int v = 0; v < NV; ++v)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x[v] += __shfl_xor_sync(0xffffffffu, x[v], o);
  double* b = wp + (size_t)ph * kWarps * 4;
  if (lane == 0)
#pragma unroll
    for (int v = 0; v < NV; ++v) b[wid * 4 + v] = x[v];
  __syncthreads();
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    double s = 0.0;
    for (int w = 0; w < kWarps; ++w) s += b[w * 4 + v];
    x[v] = s;
  }
  ph ^= 1;
}

// Block argmax of (val, idx): largest val, lowest idx on ties; plus a sum.
__device__ __forceinline__ void bargmax_sum(double& val, int& idx, double& sum, double* wp,
                                            int* wpi, int& ph) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double ov = __shfl_xor_sync(0xffffffffu, val, o);
    const int oi = __shfl_xor_sync(0xffffffffu, idx, o);
    if (ov > val || (ov == val && oi < idx)) { val = ov; idx = oi; }
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
  }
  double* b = wp + (size_t)ph * kWarps * 4;
  int* bi = wpi + ph * kWarps;
  if (lane == 0) {
    b[wid * 4 + 0] = val;
    b[wid * 4 + 1] = sum;
    bi[wid] = idx;
  }
  __syncthreads();
  val = b[0];
  idx = bi[0];
  sum = b[1];
  for (int w = 1; w < kWarps; ++w) {
    const double ov = b[w * 4 + 0];
    const int oi = bi[w];
    if (ov > val || (ov == val && oi < idx)) { val = ov; idx = oi; }
    sum += b[w * 4 + 1];
  }
  ph ^= 1;
}

template <int NQL, bool HYB>
__global__ void __launch_bounds__(kThreads, 1) seq_als_kernel(const SeqArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  cg::cluster_group cl = cg::this_cluster();
  const int q = (int)cl.block_rank();
  const int CS = a.CS;
  const int c = (int)blockIdx.x / CS;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int m = a.m, n = a.n;

  // ---- partition: rows split evenly over clusters, 32-column chunks over CTAs
  const int r0 = (int)((long long)c * m / a.NC), r1 = (int)((long long)(c + 1) * m / a.NC);
  const int TR = r1 - r0;
  auto col0 = [&](int qq) { return (qq * a.nchc / CS) * 32; };
  auto col1 = [&](int qq) { return min(((qq + 1) * a.nchc / CS) * 32, n); };
  const int c0 = col0(q), c1 = col1(q), TC = c1 - c0;
  const int TCp = a.TCp;
  const int NQ = (TC + 3) >> 2;
  const int Wm = (m + 31) >> 5, Wn = (n + 31) >> 5;
  constexpr int RG = kWarps / NQL;  // row groups of the z pass
  // contiguous row block of this warp (y pass, deflation)
  const int rpw = (TR + kWarps - 1) / kWarps;
  const int wr0 = min(TR, wid * rpw), wr1 = min(TR, wr0 + rpw);

  const bool weighted = a.w != nullptr;
  const SeqSmem L(a.TRmax, TCp, a.NC, CS, NQL, a.SR, weighted);
  double* wp = (double*)(smem + L.wp);
  int* wpi = (int*)(smem + L.wpi);
  double* misc = (double*)(smem + L.misc);
  double* xd = (double*)(smem + L.xd);
  uint32_t* xu = (uint32_t*)(smem + L.xu);
  double* erec = (double*)(smem + L.erec);
  int* abg = (int*)(smem + L.abg);
  float* uval = (float*)(smem + L.uval);
  float* ypart = (float*)(smem + L.ypart);  // shares the zred region (disjoint lifetimes)
  float* gat = (float*)(smem + L.gat);
  float* rho_p = (float*)(smem + L.rho_p);
  float* rmax = (float*)(smem + L.rmax);
  int* rmaxj = (int*)(smem + L.rmaxj);
  float* zred = (float*)(smem + L.zred);
  float* yfull = (float*)(smem + L.gat);  // summed in place over gat's first row block
  float* zall = (float*)(smem + L.zall);
  float* wall = (float*)(smem + L.wall);  // all cluster columns' weights (weighted runs)
  float* wcol = (float*)(smem + L.wcol);
  float* vval = (float*)(smem + L.vval);
  int* nnzu = (int*)(smem + L.nnzu);
  float* const Ts = (float*)(smem + L.tile);
  float* const Tg = a.gtile + (size_t)blockIdx.x * (size_t)(a.TRmax - a.SR) * (size_t)TCp;
  const int SR = a.SR;
  // row i of this CTA's tile: shared memory for the first SR rows, else global
  // (the two cases are kept apart so that shared accesses stay shared loads)
  // (HYB == false: every row is in shared memory, SR == TRmax)
  auto ld4 = [&](int i, int quad) -> float4 {
    if (!HYB || i < SR) return ((const float4*)(Ts + (size_t)i * TCp))[quad];
    return ((const float4*)(Tg + (size_t)(i - SR) * TCp))[quad];
  };
  auto st4 = [&](int i, int quad, float4 x) {
    if (!HYB || i < SR)
      ((float4*)(Ts + (size_t)i * TCp))[quad] = x;
    else
      ((float4*)(Tg + (size_t)(i - SR) * TCp))[quad] = x;
  };
  auto ld1 = [&](int i, int j) -> float {
    return (!HYB || i < SR) ? Ts[(size_t)i * TCp + j] : Tg[(size_t)(i - SR) * TCp + j];
  };
  auto st1 = [&](int i, int j, float x) {
    if (!HYB || i < SR)
      Ts[(size_t)i * TCp + j] = x;
    else
      Tg[(size_t)(i - SR) * TCp + j] = x;
  };
  const int TRp = (a.TRmax + 31) & ~31;
  const double tau = (double)a.tau;
  int rph = 0;  // reduction buffer phase

  const bool timer = blockIdx.x == 0 && tid == 0;
  long long* phs = (long long*)(misc + MS_PH);
  if (timer) {
    for (int p = 0; p <= PH_N; ++p) phs[p] = 0;
    phs[PH_N] = tick();
  }
  auto mark = [&](int p) {
    if (timer) {
      const long long t = tick();
      phs[p] += t - phs[PH_N];
      phs[PH_N] = t;
    }
  };

  bool ab = false;  // gave up waiting (made block uniform at the syncs after waits)
  bool pending_wait = false;  // a split cluster barrier was arrived at, not yet waited on
  uint32_t ep = 0;  // exchange epoch (identical sequence in every CTA)
  auto slot = [&](uint32_t e) -> uint64_t* { return a.xbuf + (size_t)(e % 3u) * a.slot_words; };
  auto rec = [&](uint64_t* s, int cc, int qq) -> uint64_t* {
    return s + (size_t)(cc * CS + qq) * a.recw;
  };
  auto take = [&](uint64_t v, const uint64_t* p) -> uint32_t {
    return ((uint32_t)(v >> 32) == ep) ? (uint32_t)v : xw_wait(p, ep, ab, a.budget, a.abort_word);
  };

  // ---- setup: A -> tile, weights of every cluster column, validity ----
  int bad = 0;
  for (int e = tid; e < TR * TCp; e += kThreads) {
    const int i = e / TCp, j = e - i * TCp;
    float x = 0.f;
    if (j < TC) {
      x = a.A[(size_t)(r0 + i) * n + (c0 + j)];
      if (!isfinite(x)) bad = 1;
    }
    st1(i, j, x);
  }
  for (int e = tid; e < CS * TCp; e += kThreads) {
    const int qq = e / TCp, j = e - qq * TCp;
    const int j0 = col0(qq), tcq = col1(qq) - j0;
    float wv = 0.f;
    if (j < tcq) {
      wv = weighted ? a.w[j0 + j] : 1.f;
      if (qq == q && (!(wv > 0.f) || !isfinite(wv))) bad = 1;
    }
    if (weighted) wall[e] = wv;
    if (qq == q) wcol[j] = wv;
    zall[e] = 0.f;
  }
  for (int j = tid; j < TCp; j += kThreads) vval[j] = 0.f;
  for (int i = tid; i < TRp; i += kThreads) {
    uval[i] = 0.f;
    ypart[i] = 0.f;
    rho_p[i] = 0.f;
  }
  {
    double b1[1] = {(double)bad};
    bsum<1>(b1, wp, rph);
    bad = b1[0] > 0.0 ? 1 : 0;
  }

  // ---- deflation of a 4-row group with refreshed row statistics ----
  // Rows i0..i0+3 (< wr1); rows whose u is 0 are left as they are.  Per row:
  // rho_p = sum_j w_j R_ij^2 (fp32), rmax/rmaxj = largest score (|R_ij|, or
  // fp32 (R_ij*R_ij)*w_j when weighted) and its lowest local column.
  auto deflate_group = [&](int i0, float d) {
    float rh[4];
    unsigned long long key[4];
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const int i = i0 + rr;
      const bool live = i < wr1;
      const float sd = live ? uval[i] * d : 0.f;  // exact: +-d or 0
      rh[rr] = 0.f;
      key[rr] = 0ull;
#pragma unroll
      for (int qi = 0; qi < NQL; ++qi) {
        const int quad = lane + 32 * qi;
        if (live && quad < NQ) {
          float4 x = ld4(i, quad);
          if (sd != 0.f) {
            const float4 v4 = *(const float4*)(vval + 4 * quad);
            x.x = v4.x > 0.f ? __fsub_rn(x.x, sd) : (v4.x < 0.f ? __fadd_rn(x.x, sd) : x.x);
            x.y = v4.y > 0.f ? __fsub_rn(x.y, sd) : (v4.y < 0.f ? __fadd_rn(x.y, sd) : x.y);
            x.z = v4.z > 0.f ? __fsub_rn(x.z, sd) : (v4.z < 0.f ? __fadd_rn(x.z, sd) : x.z);
            x.w = v4.w > 0.f ? __fsub_rn(x.w, sd) : (v4.w < 0.f ? __fadd_rn(x.w, sd) : x.w);
            st4(i, quad, x);
          }
          const float4 w4 = *(const float4*)(wcol + 4 * quad);
          const float xs[4] = {x.x, x.y, x.z, x.w};
          const float ws[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = 4 * quad + e;
            if (j < TC) {
              const float sq = __fmul_rn(xs[e], xs[e]);
              rh[rr] = fmaf(ws[e], sq, rh[rr]);
              const float sc = weighted ? __fmul_rn(sq, ws[e]) : fabsf(xs[e]);
              const unsigned long long k =
                  ((unsigned long long)__float_as_uint(sc) << 32) | (0xffffffffu - (unsigned)j);
              key[rr] = k > key[rr] ? k : key[rr];
            }
          }
        }
      }
    }
    // butterflies: 4 row sums and 4 row maxima over the warp
    const bool b4 = lane & 16, b3 = lane & 8;
    {
      const float s0 = b4 ? rh[0] : rh[2], s1 = b4 ? rh[1] : rh[3];
      const float t0 = __shfl_xor_sync(0xffffffffu, s0, 16);
      const float t1 = __shfl_xor_sync(0xffffffffu, s1, 16);
      const float h0 = (b4 ? rh[2] : rh[0]) + t0, h1 = (b4 ? rh[3] : rh[1]) + t1;
      const float tx = __shfl_xor_sync(0xffffffffu, b3 ? h0 : h1, 8);
      float v = (b3 ? h1 : h0) + tx;
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      const unsigned long long k0 = b4 ? key[0] : key[2], k1 = b4 ? key[1] : key[3];
      const unsigned long long u0 = __shfl_xor_sync(0xffffffffu, k0, 16);
      const unsigned long long u1 = __shfl_xor_sync(0xffffffffu, k1, 16);
      const unsigned long long g0 = b4 ? key[2] : key[0], g1 = b4 ? key[3] : key[1];
      const unsigned long long m0 = g0 > u0 ? g0 : u0, m1 = g1 > u1 ? g1 : u1;
      const unsigned long long ux = __shfl_xor_sync(0xffffffffu, b3 ? m0 : m1, 8);
      unsigned long long kk = b3 ? m1 : m0;
      kk = ux > kk ? ux : kk;
#pragma unroll
      for (int o = 4; o > 0; o >>= 1) {
        const unsigned long long ok = __shfl_xor_sync(0xffffffffu, kk, o);
        kk = ok > kk ? ok : kk;
      }
      if ((lane & 7) == 0) {
        const int i = i0 + (b4 ? 2 : 0) + (b3 ? 1 : 0);
        if (i < wr1) {
          rho_p[i] = v;
          rmax[i] = __uint_as_float((unsigned)(kk >> 32));
          rmaxj[i] = (int)(0xffffffffu - (unsigned)(kk & 0xffffffffu));
        }
      }
    }
  };

  for (int i0 = wr0; i0 < wr1; i0 += 4) deflate_group(i0, 0.f);
  __syncthreads();

  // ---- statistics exchange: row energies, best row, best entry, |R|^2 ----
  // Leaves misc[MS_R2], misc[MS_M], misc[MS_MVAL], misc[MS_MI], misc[MS_MJ],
  // misc[MS_ISTAR], misc[MS_BAD] and the starting v (vval) for this CTA.
  auto stats_exchange = [&](int bad_in) {
    // this CTA's best entry (score, then lowest row-major index)
    double bs = -1.0;
    int bflat = 0x7fffffff;
    for (int i = tid; i < TR; i += kThreads) {
      const double s = (double)rmax[i];
      const int f = (r0 + i) * n + c0 + rmaxj[i];
      if (s > bs || (s == bs && f < bflat)) { bs = s; bflat = f; }
    }
    {
      double dummy = 0.0;
      bargmax_sum(bs, bflat, dummy, wp, wpi, rph);
    }
    // push row energies and the entry record to every CTA of the cluster
    for (int e = tid; e < CS * (TRp >> 2); e += kThreads) {
      const int qq = e / (TRp >> 2), i4 = e - qq * (TRp >> 2);
      float4* dst = (float4*)cl.map_shared_rank(gat, qq) + (size_t)q * (TRp >> 2) + i4;
      *dst = ((const float4*)rho_p)[i4];
    }
    if (tid < CS) {
      double* dst = cl.map_shared_rank(erec, tid) + 4 * q;
      const int li = bflat / n - r0, lj = bflat % n - c0;
      const float val = (li >= 0 && li < TR && lj >= 0 && lj < TC) ? ld1(li, lj) : 0.f;
      dst[0] = bs;
      dst[1] = (double)bflat;
      dst[2] = (double)val;
    }
    cl.sync();
    // cluster rows: energies, best row, |R|^2 over the cluster's rows
    double brho = -1.0, r2 = 0.0;
    int bi = 0x7fffffff;
    for (int i = tid; i < TR; i += kThreads) {
      double s = 0.0;
      for (int qq = 0; qq < CS; ++qq) s += (double)gat[(size_t)qq * TRp + i];
      r2 += s;
      if (s > brho) { brho = s; bi = i; }
    }
    bargmax_sum(brho, bi, r2, wp, wpi, rph);
    const double R2c = r2;
    // the row energies in gat are read: peers may refill gat once they have
    // waited on this arrival (just before their next push)
    cluster_arrive();
    pending_wait = true;
    // best entry of the cluster from the pushed records (same scan everywhere)
    double Ms = erec[0], Mf = erec[1], Mv = erec[2];
    for (int qq = 1; qq < CS; ++qq) {
      const double s = erec[4 * qq], f = erec[4 * qq + 1];
      if (s > Ms || (s == Ms && f < Mf)) { Ms = s; Mf = f; Mv = erec[4 * qq + 2]; }
    }
    const int ib = (bi >= 0 && bi < TR) ? bi : 0;
    ++ep;
    uint64_t* s = slot(ep);
    uint64_t* mine = rec(s, c, q);
    // my slice of the cluster's best row (pairs of words), then its sum of squares
    for (int j = 2 * tid; j < TC; j += 2 * kThreads) {
      const float x0 = ld1(ib, j), x1 = (j + 1 < TC) ? ld1(ib, j + 1) : 0.f;
      xw_store2(mine + j, ep, f2u(x0), f2u(x1));
    }
    if (wid == 0) {
      double ss = 0.0;
      for (int j = lane; j < TC; j += 32) {
        const double x = (double)ld1(ib, j);
        ss += x * x;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (lane == 0) xw_store2(mine + TCp, ep, dlo(ss), dhi(ss));
    }
    if (q == 0 && tid == 32) {
      uint64_t* r = mine + TCp + 2;
      xw_store2(r + 0, ep, dlo(brho), dhi(brho));
      xw_store2(r + 2, ep, (uint32_t)(r0 + ib), f2u((float)Ms));
      xw_store2(r + 4, ep, (uint32_t)(int)Mf, f2u((float)Mv));
      xw_store2(r + 6, ep, dlo(R2c), dhi(R2c));
      xw_store(r + 8, ep, (uint32_t)bad_in);
    }
    // One wait round fetches, in disjoint thread ranges: the cluster records
    // (one thread per cluster), every cluster's candidate-row slice for my
    // columns (one thread per column, kept in registers until the winner is
    // known) and every CTA's slice sum of squares.  Shapes where that does not
    // fit in one pass of the block fetch the winner's row in a second round.
    double* x_rho = xd;
    double* x_r2 = xd + a.NC;
    uint32_t* x_row = xu;
    uint32_t* x_flat = xu + a.NC;
    uint32_t* x_bad = xu + 2 * a.NC;
    float* x_bs = (float*)(xu + 3 * a.NC);
    float* x_bv = (float*)(xu + 4 * a.NC);
    double* rsa = (double*)zred;  // [NC][CS] slice sums of squares (one-round path)
    const int zred_floats = max(RG * TCp, TRp);
    const bool one_round = a.NC <= 16 && TC + a.NC + a.NC * CS <= kThreads &&
                           2 * a.NC * CS <= zred_floats;
    const long long cstride = (long long)CS * a.recw;
    const int rbase = one_round ? TC : 0;  // first thread of the record range
    uint32_t slice[16];
    if (tid >= rbase && tid < rbase + a.NC) {
      const int cc = tid - rbase;
      uint32_t p[9];
      xw_wait_n<9>(rec(s, cc, 0) + TCp + 2, 1, 9, ep, p, ab, a.budget, a.abort_word);
      x_rho[cc] = u2d(p[0], p[1]);
      x_row[cc] = p[2];
      x_bs[cc] = u2f(p[3]);
      x_flat[cc] = p[4];
      x_bv[cc] = u2f(p[5]);
      x_r2[cc] = u2d(p[6], p[7]);
      x_bad[cc] = p[8];
    } else if (one_round && tid >= TC + a.NC && tid < TC + a.NC + a.NC * CS) {
      const int t = tid - TC - a.NC, cc = t / CS, qq = t - cc * CS;
      uint32_t p[2];
      xw_wait_n<2>(rec(s, cc, qq) + TCp, 1, 2, ep, p, ab, a.budget, a.abort_word);
      rsa[t] = u2d(p[0], p[1]);
    } else if (one_round && tid < TC) {
      xw_wait_n<16>(rec(s, 0, q) + tid, cstride, a.NC, ep, slice, ab, a.budget, a.abort_word);
    }
    ab = __syncthreads_or(ab);
    // every thread derives the same global view
    int win = 0;
    double R2 = 0.0;
    int anybad = 0;
    float gMs = -1.f, gMv = 0.f;
    uint32_t gMf = 0xffffffffu;
    for (int cc = 0; cc < a.NC; ++cc) {
      R2 += x_r2[cc];
      anybad |= (x_bad[cc] != 0);
      if (x_rho[cc] > x_rho[win] || (x_rho[cc] == x_rho[win] && x_row[cc] < x_row[win])) win = cc;
      if (x_bs[cc] > gMs || (x_bs[cc] == gMs && x_flat[cc] < gMf)) {
        gMs = x_bs[cc]; gMv = x_bv[cc]; gMf = x_flat[cc];
      }
    }
    win = (win >= 0 && win < a.NC) ? win : 0;
    if (one_round) {
      double rs = 0.0;
      for (int qq = 0; qq < CS; ++qq) rs += rsa[win * CS + qq];
      const double thr0 = tau * sqrt(rs / (double)n);
      for (int j = tid; j < TCp; j += kThreads) {
        float x = 0.f;
        if (j < TC) {
#pragma unroll
          for (int t = 0; t < 16; ++t)
            if (t == win) x = u2f(slice[t]);
        }
        vval[j] = j < TC ? tern(x, thr0) : 0.f;
      }
    } else {
      // second round: the winner's slice and the row's sum of squares
      double* rss = (double*)(smem + L.rss);
      float* rowbuf = zred;
      const uint64_t* wr = rec(s, win, q);
      if (tid < CS) {
        uint32_t p[2];
        xw_wait_n<2>(rec(s, win, tid) + TCp, 1, 2, ep, p, ab, a.budget, a.abort_word);
        rss[tid] = u2d(p[0], p[1]);
      }
      for (int j = tid; j < TC; j += kThreads) {
        uint32_t p[1];
        xw_wait_n<1>(wr + j, 1, 1, ep, p, ab, a.budget, a.abort_word);
        rowbuf[j] = u2f(p[0]);
      }
      ab = __syncthreads_or(ab);
      double rs = 0.0;
      for (int qq = 0; qq < CS; ++qq) rs += rss[qq];
      const double thr0 = tau * sqrt(rs / (double)n);
      for (int j = tid; j < TCp; j += kThreads) vval[j] = j < TC ? tern(rowbuf[j], thr0) : 0.f;
    }
    if (tid == 0) {
      misc[MS_R2] = R2;
      misc[MS_BAD] = (double)anybad;
      misc[MS_ISTAR] = (double)x_row[win];
      misc[MS_M] = weighted ? (double)gMs : (double)gMs * (double)gMs;
      misc[MS_MVAL] = (double)gMv;
      misc[MS_MI] = (double)(gMf / (uint32_t)n);
      misc[MS_MJ] = (double)(gMf % (uint32_t)n);
    }
    ab = __syncthreads_or(ab);
  };

  stats_exchange(bad);
  const double E0 = misc[MS_R2];
  mark(PH_SETUP);

  long long n_fb = 0, n_zero = 0;
  int tpos = 0;
  const int S_tr = 2 * Wn + a.iters * 2 * (Wm + Wn);
  bool stop = false;

  for (int comp = 0; comp < a.k && !stop; ++comp) {
    const bool traced = tpos < a.ntrace && a.trace_comp[tpos] == (int64_t)comp;
    uint32_t* tb = traced ? a.trace_bits + (size_t)tpos * S_tr : nullptr;
    int nu_total = 0;
    double Sz = 0.0;
    for (int it = 0; it < a.iters; ++it) {
      // ---- y = R (w o v) over my columns: partial per row ----
      float4 vr[NQL];
#pragma unroll
      for (int qi = 0; qi < NQL; ++qi) {
        const int quad = lane + 32 * qi;
        if (quad < NQ) {
          const float4 v4 = *(const float4*)(vval + 4 * quad);
          const float4 w4 = *(const float4*)(wcol + 4 * quad);
          vr[qi] = make_float4(v4.x * w4.x, v4.y * w4.y, v4.z * w4.z, v4.w * w4.w);
        } else {
          vr[qi] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      for (int i0 = wr0; i0 < wr1; i0 += 4) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
          if (i0 + rr < wr1) {
#pragma unroll
            for (int qi = 0; qi < NQL; ++qi) {
              const int quad = lane + 32 * qi;
              if (quad < NQ) {
                const float4 r4 = ld4(i0 + rr, quad);
                acc[rr] = fmaf(r4.x, vr[qi].x, acc[rr]);
                acc[rr] = fmaf(r4.y, vr[qi].y, acc[rr]);
                acc[rr] = fmaf(r4.z, vr[qi].z, acc[rr]);
                acc[rr] = fmaf(r4.w, vr[qi].w, acc[rr]);
              }
            }
          }
        }
        const bool b4 = lane & 16, b3 = lane & 8;
        const float s0 = b4 ? acc[0] : acc[2], s1 = b4 ? acc[1] : acc[3];
        const float t0 = __shfl_xor_sync(0xffffffffu, s0, 16);
        const float t1 = __shfl_xor_sync(0xffffffffu, s1, 16);
        const float h0 = (b4 ? acc[2] : acc[0]) + t0;
        const float h1 = (b4 ? acc[3] : acc[1]) + t1;
        const float tx = __shfl_xor_sync(0xffffffffu, b3 ? h0 : h1, 8);
        float v = (b3 ? h1 : h0) + tx;
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        if ((lane & 7) == 0) {
          const int i = i0 + (b4 ? 2 : 0) + (b3 ? 1 : 0);
          if (i < wr1) ypart[i] = v;
        }
      }
      __syncthreads();
      mark(PH_YPASS);
      // push my row partials (and, once per component, my abort flag)
      if (pending_wait) {
        cluster_wait();
        pending_wait = false;
      }
      for (int e = tid; e < CS * (TRp >> 2); e += kThreads) {
        const int qq = e / (TRp >> 2), i4 = e - qq * (TRp >> 2);
        float4* dst = (float4*)cl.map_shared_rank(gat, qq) + (size_t)q * (TRp >> 2) + i4;
        *dst = ((const float4*)ypart)[i4];
      }
      if (it == 0 && tid < CS) cl.map_shared_rank(abg, tid)[q] = ab ? 1 : 0;
      cl.sync();
      if (it == 0) {
        // ---- cluster-uniform decision point ----
        int any_ab = 0;
        for (int qq = 0; qq < CS; ++qq) any_ab |= abg[qq];
        if (any_ab || misc[MS_BAD] != 0.0) {
          stop = true;
          break;
        }
        if (comp > 0 && blockIdx.x == 0 && tid == 0)
          a.energy[comp - 1] = E0 > 0.0 ? 1.0 - misc[MS_R2] / E0 : 1.0;
        if (misc[MS_M] <= 0.0) {
          // the residual vanished: the remaining components are empty
          // (packed_B was zeroed before the launch)
          for (int cc = comp; cc < a.k; ++cc) {
            for (int t = (c0 >> 5) + tid; t < (c1 + 31) >> 5; t += kThreads) {
              a.pC[(size_t)cc * 2 * Wn + t] = 0u;
              a.pC[(size_t)cc * 2 * Wn + Wn + t] = 0u;
            }
            if (blockIdx.x == 0 && tid == 0) {
              a.D[cc] = 0.f;
              a.energy[cc] = 1.0;
            }
          }
          n_zero = a.k - comp;
          stop = true;
          break;
        }
        if (traced) {
          pack_planes(vval, TC, c0, tb, Wn);
          if (blockIdx.x == 0 && tid == 0) a.trace_row[tpos] = (int32_t)misc[MS_ISTAR];
        }
      }
      // y over the cluster's rows (fixed order), sum of squares
      double ys[1] = {0.0};
      for (int i = tid; i < TR; i += kThreads) {
        float sy = 0.f;
        for (int qq = 0; qq < CS; ++qq) sy += gat[(size_t)qq * TRp + i];
        yfull[i] = sy;  // overwrites gat[i] after its last read, same thread
        ys[0] += (double)sy * (double)sy;
      }
      bsum<1>(ys, wp, rph);
      mark(PH_YGATHER);
      ++ep;
      {
        uint64_t* s = slot(ep);
        if (q == 0 && tid == 0) xw_store2(rec(s, c, 0), ep, dlo(ys[0]), dhi(ys[0]));
        double* ysum = xd;
        for (int cc = tid; cc < a.NC; cc += kThreads) {
          const uint64_t* r = rec(s, cc, 0);
          uint64_t v0, v1;
          xw_load2(r, v0, v1);
          ysum[cc] = u2d(take(v0, r), take(v1, r + 1));
        }
        ab = __syncthreads_or(ab);
      }
      double sy_all = 0.0;
      for (int cc = 0; cc < a.NC; ++cc) sy_all += xd[cc];
      const double thr_u = tau * sqrt(sy_all / (double)m);
      double cnt[1] = {0.0};
      for (int i = tid; i < TRp; i += kThreads) {
        const float uu = i < TR ? tern(yfull[i], thr_u) : 0.f;
        uval[i] = uu;
        cnt[0] += uu != 0.f ? 1.0 : 0.0;
      }
      bsum<1>(cnt, wp, rph);
      const int nnz_c = (int)cnt[0];
      if (traced && q == 0) pack_planes_or(uval, TR, r0, tb + 2 * Wn + it * 2 * (Wm + Wn), Wm);
      mark(PH_YXCHG);

      // ---- z = R^T u over the cluster's rows, my columns ----
      {
        const int strip = wid % NQL, rgrp = wid / NQL;
        const int quad = strip * 32 + lane;
        if (rgrp < RG && quad < NQ) {
          float4 za = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int i = rgrp; i < TR; i += 4 * RG) {
            float ui[4];
            float4 r4[4];
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              const int ii = i + k4 * RG;
              ui[k4] = ii < TR ? uval[ii] : 0.f;
              r4[k4] = ui[k4] != 0.f ? ld4(ii, quad) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              za.x = fmaf(ui[k4], r4[k4].x, za.x);
              za.y = fmaf(ui[k4], r4[k4].y, za.y);
              za.z = fmaf(ui[k4], r4[k4].z, za.z);
              za.w = fmaf(ui[k4], r4[k4].w, za.w);
            }
          }
          *(float4*)(zred + (size_t)rgrp * TCp + 4 * quad) = za;
        }
      }
      __syncthreads();
      mark(PH_ZPASS);
      ++ep;
      {
        uint64_t* s = slot(ep);
        uint64_t* mine = rec(s, c, q);
        for (int j = 2 * tid; j < TC; j += 2 * kThreads) {
          float z0 = 0.f, z1 = 0.f;
          for (int g = 0; g < RG; ++g) {
            z0 += zred[(size_t)g * TCp + j];
            z1 += zred[(size_t)g * TCp + j + 1];
          }
          xw_store2(mine + j, ep, f2u(z0), f2u(j + 1 < TC ? z1 : 0.f));
        }
        if (tid == 0) xw_store(mine + TCp, ep, (uint32_t)nnz_c);
        float* zmine = zall + (size_t)q * TCp;
        const long long cstride = (long long)CS * a.recw;
        for (int j = tid; j < TC; j += kThreads) {
          float z = 0.f;
          for (int cc0 = 0; cc0 < a.NC; cc0 += 16) {
            uint32_t pl[16];
            const int cnt = min(16, a.NC - cc0);
            xw_wait_n<16>(rec(s, cc0, q) + j, cstride, cnt, ep, pl, ab, a.budget, a.abort_word);
#pragma unroll
            for (int t = 0; t < 16; ++t)
              if (t < cnt) z += u2f(pl[t]);
          }
          zmine[j] = z;
        }
        for (int cc = tid; cc < a.NC; cc += kThreads) {
          const uint64_t* r = rec(s, cc, q) + TCp;
          nnzu[cc] = (int)take(xw_load(r), r);
        }
        ab = __syncthreads_or(ab);
        // all-gather z inside the cluster
        for (int e = tid; e < (CS - 1) * (TCp >> 2); e += kThreads) {
          const int k2 = e / (TCp >> 2), j4 = e - k2 * (TCp >> 2);
          const int qq = k2 < q ? k2 : k2 + 1;
          float4* dst = (float4*)cl.map_shared_rank(zall, qq) + (size_t)q * (TCp >> 2) + j4;
          *dst = ((const float4*)zmine)[j4];
        }
      }
      mark(PH_ZXCHG);
      cl.sync();
      {
        double zz[1] = {0.0};
        for (int e = tid; e < CS * TCp; e += kThreads) {
          const double z = (double)zall[e];
          zz[0] += z * z;
        }
        bsum<1>(zz, wp, rph);
        Sz = zz[0];
      }
      const double thr_v = tau * sqrt(Sz / (double)n);
      for (int j = tid; j < TCp; j += kThreads)
        vval[j] = j < TC ? tern(zall[(size_t)q * TCp + j], thr_v) : 0.f;
      nu_total = 0;
      for (int cc = 0; cc < a.NC; ++cc) nu_total += nnzu[cc];
      __syncthreads();
      if (traced) pack_planes(vval, TC, c0, tb + 2 * Wn + it * 2 * (Wm + Wn) + 2 * Wm, Wn);
      mark(PH_ZSYNC);
    }
    if (stop) break;

    // ---- scale, gain, safeguard (every CTA over all of the cluster's columns) ----
    const double thr_v = tau * sqrt(Sz / (double)n);
    double pv[3] = {0.0, 0.0, 0.0};
    for (int e = tid; e < CS * TCp; e += kThreads) {
      const float z = zall[e];
      if (tern(z, thr_v) != 0.f) {
        const double wv = weighted ? (double)wall[e] : 1.0;
        pv[0] += wv * fabs((double)z);
        pv[1] += wv;
        pv[2] += 1.0;
      }
    }
    bsum<3>(pv, wp, rph);
    const double P = pv[0], VW = pv[1];
    const double den = (double)nu_total * VW;
    const double gain = den > 0.0 ? P * P / den : 0.0;
    const bool fb = gain < misc[MS_M];
    float d;
    if (fb) {
      d = (float)misc[MS_MVAL];
      const int ip = (int)misc[MS_MI], jp = (int)misc[MS_MJ];
      for (int i = tid; i < TRp; i += kThreads) uval[i] = (r0 + i == ip && i < TR) ? 1.f : 0.f;
      for (int j = tid; j < TCp; j += kThreads) vval[j] = (c0 + j == jp && j < TC) ? 1.f : 0.f;
      ++n_fb;
    } else {
      d = den > 0.0 ? (float)(P / den) : 0.f;
    }
    __syncthreads();
    if (traced && blockIdx.x == 0 && tid == 0) a.trace_flags[tpos] = fb ? 1 : 0;
    if (traced) ++tpos;

    // ---- emit ----
    if (q == 0) pack_planes_or(uval, TR, r0, a.pB + (size_t)comp * 2 * Wm, Wm);
    pack_planes(vval, TC, c0, a.pC + (size_t)comp * 2 * Wn, Wn);
    if (blockIdx.x == 0 && tid == 0) a.D[comp] = d;
    mark(PH_SCALE);

    // ---- deflate R <- R - d u v^T, refresh touched rows' statistics ----
    for (int i0 = wr0; i0 < wr1; i0 += 4) {
      bool any = false;
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) any |= (i0 + rr < wr1) && uval[i0 + rr] != 0.f;
      if (any) deflate_group(i0, d);
    }
    __syncthreads();
    mark(PH_DEFLATE);
    stats_exchange(0);
    mark(PH_STATS);
  }

  // final energy entry, counters, status
  __syncthreads();
  if (blockIdx.x == 0 && tid == 0) {
    if (!stop && n_zero == 0 && a.k > 0)
      a.energy[a.k - 1] = E0 > 0.0 ? 1.0 - misc[MS_R2] / E0 : 1.0;
    if (a.stats) {
      a.stats[0] = n_fb;
      a.stats[1] = n_zero;
      a.stats[2] = a.NC;
      a.stats[3] = CS;
      a.stats[4] = SR;
      a.stats[5] = a.TRmax;
      for (int p = 0; p < PH_N; ++p) a.stats[kStatPhase0 + p] = phs[p];
    }
    if (misc[MS_BAD] != 0.0) atomicCAS(a.dev_status, 0, EXTERND_ERR_NONFINITE);
  }
  if (tid == 0) {
    const int aw = ld_flag(a.abort_word);
    if (aw != 0) atomicCAS(a.dev_status, 0, aw);
  }
  // no CTA may leave while a cluster peer can still access its shared memory
  if (pending_wait) cluster_wait();
  cl.sync();
}


// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

template <int NQL, bool HYB>
static cudaError_t launch_one(const SeqArgs& args, size_t smem, cudaStream_t st,
                              int* max_clusters_out, bool query_only) {
  auto kern = seq_als_kernel<NQL, HYB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (args.CS > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(args.NC * args.CS));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)args.CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (query_only) {
    int nc = 0;
    e = cudaOccupancyMaxActiveClusters(&nc, kern, &cfg);
    *max_clusters_out = nc;
    return e;
  }
  return cudaLaunchKernelEx(&cfg, kern, args);
}

template <bool HYB>
static cudaError_t dispatch_t(int NQL, const SeqArgs& args, size_t smem, cudaStream_t st, int* mc,
                              bool query_only) {
  switch (NQL) {
    case 1: return launch_one<1, HYB>(args, smem, st, mc, query_only);
    case 2: return launch_one<2, HYB>(args, smem, st, mc, query_only);
    case 3: return launch_one<3, HYB>(args, smem, st, mc, query_only);
    case 4: return launch_one<4, HYB>(args, smem, st, mc, query_only);
    case 5: return launch_one<5, HYB>(args, smem, st, mc, query_only);
    case 6: return launch_one<6, HYB>(args, smem, st, mc, query_only);
    case 8: return launch_one<8, HYB>(args, smem, st, mc, query_only);
    default: return cudaErrorInvalidValue;
  }
}

// HYB is chosen from the arguments: rows outside shared memory need the
// hybrid kernel.
static cudaError_t dispatch(int NQL, const SeqArgs& args, size_t smem, cudaStream_t st, int* mc,
                            bool query_only) {
  return args.SR < args.TRmax ? dispatch_t<true>(NQL, args, smem, st, mc, query_only)
                              : dispatch_t<false>(NQL, args, smem, st, mc, query_only);
}

template <bool HYB>
static size_t static_smem_t(int NQL) {
  cudaFuncAttributes fa = {};
  cudaError_t e = cudaErrorInvalidValue;
  switch (NQL) {
    case 1: e = cudaFuncGetAttributes(&fa, seq_als_kernel<1, HYB>); break;
    case 2: e = cudaFuncGetAttributes(&fa, seq_als_kernel<2, HYB>); break;
    case 3: e = cudaFuncGetAttributes(&fa, seq_als_kernel<3, HYB>); break;
    case 4: e = cudaFuncGetAttributes(&fa, seq_als_kernel<4, HYB>); break;
    case 5: e = cudaFuncGetAttributes(&fa, seq_als_kernel<5, HYB>); break;
    case 6: e = cudaFuncGetAttributes(&fa, seq_als_kernel<6, HYB>); break;
    case 8: e = cudaFuncGetAttributes(&fa, seq_als_kernel<8, HYB>); break;
    default: break;
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return (size_t)1 << 30;
  }
  return fa.sharedSizeBytes;
}

static size_t static_smem(int NQL) {
  return std::max(static_smem_t<true>(NQL), static_smem_t<false>(NQL));
}

static int nql_for(int TCp) {
  const int nq = TCp / 4;
  int v = (nq + 31) / 32;
  if (v == 7) v = 8;
  return v;
}

struct SeqPlan {
  int NC = 0, CS = 0, TRmax = 0, TCp = 0, NQL = 0, SR = 0;
  size_t smem = 0;
};

// Chooses cluster size, cluster count and how many rows of each CTA's tile
// stay in shared memory (the rest stream from global memory).  Candidates
// must be co-resident (occupancy query).  The estimated cost per half-step
// -- tile words read per CTA, global rows weighted 4x, plus the cross-cluster
// words each CTA polls -- is minimised.
static cudaError_t plan_seq(int m, int n, bool weighted, cudaStream_t st, SeqPlan* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int nsm = 0, optin = 0;
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const int nchc = (n + 31) / 32;
  int force_cs = 0;
  if (const char* s = getenv("EXTERND_CLUSTER")) force_cs = atoi(s);
  const int cands[] = {16, 12, 10, 9, 8, 6, 5, 4, 3, 2, 1};
  SeqPlan best;
  double best_cost = 1e300;
  for (int CS : cands) {
    if (force_cs > 0 && CS != force_cs) continue;
    if (CS > nchc) continue;
    const int colchunks = (nchc + CS - 1) / CS;
    const int TC = std::min(colchunks * 32, n);
    const int TCp = (TC + 3) & ~3;
    const int NQL = nql_for(TCp);
    if (NQL > 8) continue;
    const size_t stat = static_smem(NQL);
    int nc = std::min(std::min(m, 64), std::max(1, nsm / CS));
    for (int guard = 0; guard < 16 && nc >= 1; ++guard) {
      const int TRmax = (m + nc - 1) / nc;
      const SeqSmem L0(TRmax, TCp, nc, CS, NQL, 0, weighted);
      if (L0.total + stat > (size_t)optin) break;
      const size_t room = (size_t)optin - stat - L0.total;
      const int SR = (int)std::min((size_t)TRmax, room / (sizeof(float) * (size_t)TCp));
      const SeqSmem L(TRmax, TCp, nc, CS, NQL, SR, weighted);
      SeqArgs probe = {};
      probe.NC = nc;
      probe.CS = CS;
      probe.SR = SR;
      probe.TRmax = TRmax;
      int maxc = 0;
      cudaError_t qe = dispatch(NQL, probe, L.total, st, &maxc, true);
      if (qe != cudaSuccess) {
        cudaGetLastError();
        break;
      }
      if (maxc >= nc) {
        const double tile_w = (double)SR * TCp + 4.0 * (double)(TRmax - SR) * TCp;
        const double cost = tile_w + 8.0 * nc * TCp;
        if (cost < best_cost) {
          best_cost = cost;
          best.NC = nc;
          best.CS = CS;
          best.TRmax = TRmax;
          best.TCp = TCp;
          best.NQL = NQL;
          best.SR = SR;
          best.smem = L.total;
        }
        break;
      }
      if (maxc < 1) break;
      nc = std::min(nc - 1, maxc);
    }
  }
  if (best.NC == 0) return cudaErrorNotSupported;
  *out = best;
  return cudaSuccess;
}

static void fill_args(SeqArgs& a, const SeqHostArgs& h, const SeqPlan& pl, int recw,
                      long long slot_words) {
  a.A = h.A;
  a.m = (int)h.m;
  a.n = (int)h.n;
  a.k = (int)h.k;
  a.tau = h.tau;
  a.iters = h.iters;
  a.w = h.w;
  a.pB = h.packed_B;
  a.pC = h.packed_C;
  a.D = h.D;
  a.energy = h.energy;
  a.NC = pl.NC;
  a.CS = pl.CS;
  a.nchc = (a.n + 31) / 32;
  a.TRmax = pl.TRmax;
  a.TCp = pl.TCp;
  a.SR = pl.SR;
  a.recw = recw;
  a.slot_words = slot_words;
  a.trace_comp = h.trace_comp;
  a.ntrace = (int)h.ntrace;
  a.trace_bits = h.trace_bits;
  a.trace_row = h.trace_row;
  a.trace_flags = h.trace_flags;
  a.stats = h.stats;
  a.budget = h.wait_budget > 0 ? h.wait_budget : kDefaultWaitBudget;
}

// Zero-initialises what the kernel ORs into.
static cudaError_t clear_outputs(const SeqHostArgs& h, cudaStream_t st) {
  const size_t Wm = (size_t)((h.m + 31) / 32), Wn = (size_t)((h.n + 31) / 32);
  cudaError_t e = cudaMemsetAsync(h.packed_B, 0, sizeof(uint32_t) * 2 * Wm * (size_t)h.k, st);
  if (e == cudaSuccess && h.ntrace > 0 && h.trace_bits)
    e = cudaMemsetAsync(h.trace_bits, 0,
                        sizeof(uint32_t) * (size_t)h.ntrace * (2 * Wn + (size_t)h.iters * 2 * (Wm + Wn)),
                        st);
  return e;
}

int seq_decompose(const SeqHostArgs& h, cudaStream_t st) {
  SeqPlan pl;
  cudaError_t e = plan_seq((int)h.m, (int)h.n, h.w != nullptr, st, &pl);
  if (e == cudaErrorNotSupported) return EXTERND_ERR_NO_COOP;
  if (e != cudaSuccess) return EXTERND_ERR_CUDA;
  const int recw = pl.TCp + 16;
  const long long slot_words = (long long)pl.NC * pl.CS * recw;
  const size_t xbytes = sizeof(uint64_t) * 3 * (size_t)slot_words;
  const size_t abort_off = (xbytes + 255) & ~(size_t)255;
  const size_t tile_off = abort_off + 256;
  const size_t tile_bytes =
      sizeof(float) * (size_t)pl.NC * pl.CS * (size_t)(pl.TRmax - pl.SR) * (size_t)pl.TCp;
  void* ws = nullptr;
  e = cudaMallocAsync(&ws, tile_off + tile_bytes, st);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return EXTERND_ERR_OOM;
  }
  int rc = EXTERND_OK;
  if (cudaMemsetAsync(ws, 0, tile_off, st) != cudaSuccess) rc = EXTERND_ERR_CUDA;
  if (rc == EXTERND_OK && clear_outputs(h, st) != cudaSuccess) rc = EXTERND_ERR_CUDA;
  if (rc == EXTERND_OK) {
    SeqArgs a = {};
    fill_args(a, h, pl, recw, slot_words);
    a.gtile = tile_bytes ? (float*)((char*)ws + tile_off) : nullptr;
    a.xbuf = (uint64_t*)ws;
    a.abort_word = (int*)((char*)ws + abort_off);
    a.dev_status = status_word_ptr();
    if (!a.dev_status) rc = EXTERND_ERR_CUDA;
    if (rc == EXTERND_OK) {
      int dummy = 0;
      e = dispatch(pl.NQL, a, pl.smem, st, &dummy, false);
      if (e != cudaSuccess) {
        cudaGetLastError();
        rc = EXTERND_ERR_CUDA;
      }
    }
  }
  if (cudaFreeAsync(ws, st) != cudaSuccess && rc == EXTERND_OK) rc = EXTERND_ERR_CUDA;
  return rc;
}

// Same launch as seq_decompose, but the exchange ring and the abort word live
// in caller-provided device scratch instead of a cudaMallocAsync workspace,
// and only plans whose residual tiles stay in shared memory are accepted (a
// global tile store would need m*n*4 bytes of scratch).  No allocation.
int seq_decompose_with_scratch(const SeqHostArgs& h, void* scratch, size_t scratch_bytes,
                               cudaStream_t st) {
  SeqPlan pl;
  cudaError_t e = plan_seq((int)h.m, (int)h.n, h.w != nullptr, st, &pl);
  if (e == cudaErrorNotSupported) return EXTERND_ERR_NO_COOP;
  if (e != cudaSuccess) return EXTERND_ERR_CUDA;
  if (pl.SR < pl.TRmax) return EXTERND_ERR_SCRATCH_LIMIT;
  const int recw = pl.TCp + 16;
  const long long slot_words = (long long)pl.NC * pl.CS * recw;
  const size_t xbytes = sizeof(uint64_t) * 3 * (size_t)slot_words;
  const size_t abort_off = (xbytes + 255) & ~(size_t)255;
  const size_t need = abort_off + 256;
  if (need > scratch_bytes) return EXTERND_ERR_SCRATCH_LIMIT;
  if (cudaMemsetAsync(scratch, 0, need, st) != cudaSuccess) return EXTERND_ERR_CUDA;
  if (clear_outputs(h, st) != cudaSuccess) return EXTERND_ERR_CUDA;
  SeqArgs a = {};
  fill_args(a, h, pl, recw, slot_words);
  a.gtile = nullptr;
  a.xbuf = (uint64_t*)scratch;
  a.abort_word = (int*)((char*)scratch + abort_off);
  a.dev_status = status_word_ptr();
  if (!a.dev_status) return EXTERND_ERR_CUDA;
  int dummy = 0;
  e = dispatch(pl.NQL, a, pl.smem, st, &dummy, false);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return EXTERND_ERR_CUDA;
  }
  return EXTERND_OK;
}

}  // namespace externd
