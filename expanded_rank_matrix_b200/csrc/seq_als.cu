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
  float* gtile;
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

// Shared-memory carve-up, identical on host and device.  yfull lives in the
// zred region: their lifetimes (y gather..threshold, z reduction) are disjoint.
struct SeqSmem {
  size_t red, ired, cx, misc, xd, xu, tile, uval, ypart, yfull, rho_p, rmax, rmaxv, rmaxj, zred,
      wcol, vval, zfull, nnzu, total;
  __host__ __device__ SeqSmem(int TRmax, int TCp, int NC, int NQL, bool smem_tile) {
    const int TRp = (TRmax + 31) & ~31;
    const int RG = kWarps / NQL;
    size_t o = 0;
    auto take = [&](size_t bytes) {
      size_t r = o;
      o += (bytes + 15) & ~(size_t)15;
      return r;
    };
    red = take(sizeof(double) * (kWarps + 1));
    ired = take(sizeof(int) * (kWarps + 1));
    cx = take(sizeof(double) * 4 * 4);
    misc = take(sizeof(double) * 32);
    xd = take(sizeof(double) * 2 * NC);    // per-cluster fp64 records
    xu = take(sizeof(uint32_t) * 6 * NC);  // per-cluster 32-bit records
    tile = take(smem_tile ? sizeof(float) * (size_t)TRmax * TCp : 0);
    uval = take(sizeof(float) * TRp);
    ypart = take(sizeof(float) * 2 * TRp);
    rho_p = take(sizeof(float) * TRp);
    rmax = take(sizeof(float) * TRp);
    rmaxv = take(sizeof(float) * TRp);
    rmaxj = take(sizeof(int) * TRp);
    const size_t zb = sizeof(float) * (size_t)RG * TCp;
    const size_t yb = sizeof(float) * TRp;
    zred = take(zb > yb ? zb : yb);
    yfull = zred;
    wcol = take(sizeof(float) * TCp);
    vval = take(sizeof(float) * TCp);
    zfull = take(sizeof(float) * TCp);
    nnzu = take(sizeof(int) * NC);
    total = o;
  }
};

// misc[] slots (doubles)
enum {
  MS_E0 = 0,
  MS_R2,
  MS_M,      // entry score of the best single entry (as fp64)
  MS_MVAL,   // its signed value (fp32 held in fp64)
  MS_MI,     // its row
  MS_MJ,     // its column
  MS_ISTAR,  // starting row of the component
  MS_WIN,    // winning cluster
  MS_BAD,
  MS_SY,
  MS_ROWSS,
  MS_ABORT,  // cluster-wide abort decision
  MS_AB0,    // per-CTA abort flags, double buffered (read by cluster peers)
  MS_AB1,
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

template <int NQL, bool SMT>
__global__ void __launch_bounds__(kThreads, 1) seq_als_kernel(const SeqArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  cg::cluster_group cl = cg::this_cluster();
  const int q = (int)cl.block_rank();
  const int c = (int)blockIdx.x / a.CS;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int m = a.m, n = a.n;

  // ---- partition: rows split evenly over clusters, 32-column chunks over CTAs
  const int r0 = (int)((long long)c * m / a.NC), r1 = (int)((long long)(c + 1) * m / a.NC);
  const int TR = r1 - r0;
  const int ca = q * a.nchc / a.CS, cb = (q + 1) * a.nchc / a.CS;
  const int c0 = ca * 32, c1 = min(cb * 32, n), TC = c1 - c0;
  const int TCp = a.TCp;
  const int NQ = (TC + 3) >> 2;
  const int Wm = (m + 31) >> 5, Wn = (n + 31) >> 5;
  constexpr int RG = kWarps / NQL;  // row groups of the z pass

  const SeqSmem L(a.TRmax, TCp, a.NC, NQL, SMT);
  double* xd = (double*)(smem + L.xd);
  uint32_t* xu = (uint32_t*)(smem + L.xu);
  double* red = (double*)(smem + L.red);
  int* ired = (int*)(smem + L.ired);
  double* cx = (double*)(smem + L.cx);
  double* misc = (double*)(smem + L.misc);
  float* uval = (float*)(smem + L.uval);
  float* ypart = (float*)(smem + L.ypart);
  float* yfull = (float*)(smem + L.yfull);
  float* rho_p = (float*)(smem + L.rho_p);
  float* rmax = (float*)(smem + L.rmax);
  float* rmaxv = (float*)(smem + L.rmaxv);
  int* rmaxj = (int*)(smem + L.rmaxj);
  float* zred = (float*)(smem + L.zred);
  float* wcol = (float*)(smem + L.wcol);
  float* vval = (float*)(smem + L.vval);
  float* zfull = (float*)(smem + L.zfull);
  int* nnzu = (int*)(smem + L.nnzu);
  float* T = SMT ? (float*)(smem + L.tile)
                 : a.gtile + (size_t)blockIdx.x * (size_t)a.TRmax * (size_t)TCp;
  const int TRp = (a.TRmax + 31) & ~31;
  const bool weighted = a.w != nullptr;
  const double tau = (double)a.tau;
  const bool timer = blockIdx.x == 0 && tid == 0;
  // phase accumulators live in shared memory (misc[16..]): one thread uses them
  long long* ph = (long long*)(misc + 16);
  if (timer) {
    for (int p = 0; p < PH_N; ++p) ph[p] = 0;
    ph[PH_N] = tick();
  }
  auto mark = [&](int p) {
    if (timer) {
      const long long t = tick();
      ph[p] += t - ph[PH_N];
      ph[PH_N] = t;
    }
  };

  bool ab = false;  // this CTA gave up waiting (made block uniform at sync points)
  uint32_t ep = 0;  // exchange epoch (identical sequence in every CTA)
  auto slot = [&](uint32_t e) -> uint64_t* { return a.xbuf + (size_t)(e % 3u) * a.slot_words; };
  auto rec = [&](uint64_t* s, int cc, int qq) -> uint64_t* {
    return s + (size_t)(cc * a.CS + qq) * a.recw;
  };
  // payload of an already loaded word, or wait for it
  auto take = [&](uint64_t v, const uint64_t* p) -> uint32_t {
    return ((uint32_t)(v >> 32) == ep) ? (uint32_t)v : xw_wait(p, ep, ab, a.budget, a.abort_word);
  };

  // ---- setup: A -> tile, weights, validity ----
  int bad = 0;
  for (int e = tid; e < TR * TCp; e += kThreads) {
    const int i = e / TCp, j = e - i * TCp;
    float x = 0.f;
    if (j < TC) {
      x = a.A[(size_t)(r0 + i) * n + (c0 + j)];
      if (!isfinite(x)) bad = 1;
    }
    T[e] = x;
  }
  for (int j = tid; j < TCp; j += kThreads) {
    float wv = 0.f;
    if (j < TC) {
      wv = weighted ? a.w[c0 + j] : 1.f;
      if (!(wv > 0.f) || !isfinite(wv)) bad = 1;
    }
    wcol[j] = wv;
    vval[j] = 0.f;
  }
  for (int i = tid; i < TRp; i += kThreads) {
    uval[i] = 0.f;
    ypart[i] = 0.f;
    ypart[TRp + i] = 0.f;
  }
  bad = block_sum_int(bad, ired) > 0 ? 1 : 0;

  // Per-row statistics of this CTA's columns: rho_p[i] = sum_j w_j R_ij^2
  // (fp32), rmax/rmaxv/rmaxj = best entry score, its value and its local
  // column (lowest column on ties).  One warp per row.
  auto row_stats = [&](int i) {
    const float4* row = (const float4*)(T + (size_t)i * TCp);
    float rho = 0.f, bs = -1.f, bv = 0.f;
    int bj = 0x7fffffff;
#pragma unroll
    for (int qi = 0; qi < NQL; ++qi) {
      const int quad = lane + 32 * qi;
      if (quad < NQ) {
        const float4 r4 = row[quad];
        const float4 w4 = *(const float4*)(wcol + 4 * quad);
        const float rr[4] = {r4.x, r4.y, r4.z, r4.w};
        const float ww[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = 4 * quad + e;
          if (j < TC) {
            const float sq = __fmul_rn(rr[e], rr[e]);
            rho = fmaf(ww[e], sq, rho);
            const float s = weighted ? __fmul_rn(sq, ww[e]) : fabsf(rr[e]);
            if (s > bs) { bs = s; bv = rr[e]; bj = j; }
          }
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      rho += __shfl_xor_sync(0xffffffffu, rho, o);
      const float os = __shfl_xor_sync(0xffffffffu, bs, o);
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
      if (os > bs || (os == bs && oj < bj)) { bs = os; bv = ov; bj = oj; }
    }
    if (lane == 0) {
      rho_p[i] = rho;
      rmax[i] = bs;
      rmaxv[i] = bv;
      rmaxj[i] = bj;
    }
  };

  for (int i = wid; i < TR; i += kWarps) row_stats(i);

  // ---- statistics exchange: row energies, best row, best entry, |R|^2 ----
  // Leaves misc[MS_R2], misc[MS_M], misc[MS_MVAL], misc[MS_MI], misc[MS_MJ],
  // misc[MS_ISTAR], misc[MS_BAD] and the starting v (vval) for this CTA.
  auto stats_exchange = [&](int bad_in) {
    cl.sync();
    // cluster-wide row energies, best row (lowest index on ties)
    double r2 = 0.0, brho = -1.0;
    int bi = 0x7fffffff;
    for (int i = tid; i < TR; i += kThreads) {
      double s = 0.0;
      for (int qq = 0; qq < a.CS; ++qq) s += (double)cl.map_shared_rank(rho_p, qq)[i];
      r2 += s;
      if (s > brho) { brho = s; bi = i; }
    }
    // best entry over the cluster (lowest row-major index on ties)
    float bs = -1.f, bv = 0.f;
    long long bflat = 0x7fffffffffffffffLL;
    for (int e = tid; e < TR * a.CS; e += kThreads) {
      const int qq = e / TR, i = e - qq * TR;
      const float s = cl.map_shared_rank(rmax, qq)[i];
      const int jl = cl.map_shared_rank(rmaxj, qq)[i];
      const int cq0 = (qq * a.nchc / a.CS) * 32;
      const long long flat = (long long)(r0 + i) * n + (cq0 + jl);
      if (s > bs || (s == bs && flat < bflat)) {
        bs = s;
        bv = cl.map_shared_rank(rmaxv, qq)[i];
        bflat = flat;
      }
    }
    const double R2c = block_sum(r2, red);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double orho = __shfl_xor_sync(0xffffffffu, brho, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (orho > brho || (orho == brho && oi < bi)) { brho = orho; bi = oi; }
      const float os = __shfl_xor_sync(0xffffffffu, bs, o);
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const long long of = __shfl_xor_sync(0xffffffffu, bflat, o);
      if (os > bs || (os == bs && of < bflat)) { bs = os; bv = ov; bflat = of; }
    }
    __shared__ double s_rho[kWarps];
    __shared__ int s_i[kWarps];
    __shared__ float s_bs[kWarps], s_bv[kWarps];
    __shared__ long long s_bf[kWarps];
    if (lane == 0) {
      s_rho[wid] = brho; s_i[wid] = bi; s_bs[wid] = bs; s_bv[wid] = bv; s_bf[wid] = bflat;
    }
    __syncthreads();
    if (tid == 0) {
      for (int ww = 1; ww < kWarps; ++ww) {
        if (s_rho[ww] > brho || (s_rho[ww] == brho && s_i[ww] < bi)) { brho = s_rho[ww]; bi = s_i[ww]; }
        if (s_bs[ww] > bs || (s_bs[ww] == bs && s_bf[ww] < bflat)) {
          bs = s_bs[ww]; bv = s_bv[ww]; bflat = s_bf[ww];
        }
      }
      s_i[0] = bi;
      s_rho[0] = brho;
      s_bs[0] = bs;
      s_bv[0] = bv;
      s_bf[0] = bflat;
    }
    __syncthreads();
    bi = s_i[0];
    brho = s_rho[0];
    bs = s_bs[0];
    bv = s_bv[0];
    bflat = s_bf[0];
    const int ib = (bi >= 0 && bi < TR) ? bi : 0;
    // my slice of the cluster's best row, and its unweighted sum of squares
    double ss = 0.0;
    for (int j = tid; j < TC; j += kThreads) {
      const float x = T[(size_t)ib * TCp + j];
      ss += (double)x * (double)x;
    }
    ss = block_sum(ss, red);
    ++ep;
    uint64_t* s = slot(ep);
    uint64_t* mine = rec(s, c, q);
    for (int j = tid; j < TC; j += kThreads) xw_store(mine + j, ep, f2u(T[(size_t)ib * TCp + j]));
    if (tid == 0) {
      xw_store(mine + TCp + 0, ep, dlo(ss));
      xw_store(mine + TCp + 1, ep, dhi(ss));
      if (q == 0) {
        xw_store(mine + TCp + 2, ep, dlo(brho));
        xw_store(mine + TCp + 3, ep, dhi(brho));
        xw_store(mine + TCp + 4, ep, (uint32_t)(r0 + ib));
        xw_store(mine + TCp + 5, ep, f2u(bs));
        xw_store(mine + TCp + 6, ep, (uint32_t)bflat);
        xw_store(mine + TCp + 7, ep, f2u(bv));
        xw_store(mine + TCp + 8, ep, dlo(R2c));
        xw_store(mine + TCp + 9, ep, dhi(R2c));
        xw_store(mine + TCp + 10, ep, (uint32_t)bad_in);
      }
    }
    // cluster records: one thread per cluster, its 9 words loaded together
    double* x_rho = xd;
    double* x_r2 = xd + a.NC;
    uint32_t* x_row = xu;
    uint32_t* x_flat = xu + a.NC;
    uint32_t* x_bad = xu + 2 * a.NC;
    float* x_bs = (float*)(xu + 3 * a.NC);
    float* x_bv = (float*)(xu + 4 * a.NC);
    for (int cc = tid; cc < a.NC; cc += kThreads) {
      const uint64_t* r = rec(s, cc, 0) + TCp + 2;
      uint64_t v[9];
#pragma unroll
      for (int b = 0; b < 9; ++b) v[b] = xw_load(r + b);
      uint32_t p[9];
#pragma unroll
      for (int b = 0; b < 9; ++b) p[b] = take(v[b], r + b);
      x_rho[cc] = u2d(p[0], p[1]);
      x_row[cc] = p[2];
      x_bs[cc] = u2f(p[3]);
      x_flat[cc] = p[4];
      x_bv[cc] = u2f(p[5]);
      x_r2[cc] = u2d(p[6], p[7]);
      x_bad[cc] = p[8];
    }
    ab = __syncthreads_or(ab);
    if (tid == 0) {
      int win = 0;
      double R2 = 0.0;
      int anybad = 0;
      float Ms = -1.f, Mv = 0.f;
      uint32_t Mf = 0xffffffffu;
      for (int cc = 0; cc < a.NC; ++cc) {
        R2 += x_r2[cc];
        anybad |= (x_bad[cc] != 0);
        if (x_rho[cc] > x_rho[win] || (x_rho[cc] == x_rho[win] && x_row[cc] < x_row[win])) win = cc;
        if (x_bs[cc] > Ms || (x_bs[cc] == Ms && x_flat[cc] < Mf)) {
          Ms = x_bs[cc]; Mv = x_bv[cc]; Mf = x_flat[cc];
        }
      }
      misc[MS_R2] = R2;
      misc[MS_BAD] = (double)anybad;
      misc[MS_WIN] = (double)win;
      misc[MS_ISTAR] = (double)x_row[win];
      misc[MS_M] = weighted ? (double)Ms : (double)Ms * (double)Ms;
      misc[MS_MVAL] = (double)Mv;
      misc[MS_MI] = (double)(Mf / (uint32_t)n);
      misc[MS_MJ] = (double)(Mf % (uint32_t)n);
    }
    __syncthreads();
    int win = (int)misc[MS_WIN];
    win = (win >= 0 && win < a.NC) ? win : 0;
    // starting v for my columns: T_tau of the winning row
    if (tid < a.CS) {
      const uint64_t* r = rec(s, win, tid) + TCp;
      const uint64_t v0 = xw_load(r), v1 = xw_load(r + 1);
      const uint32_t lo = take(v0, r), hi = take(v1, r + 1);
      red[tid] = u2d(lo, hi);
    }
    ab = __syncthreads_or(ab);
    if (tid == 0) {
      double rs = 0.0;
      for (int qq = 0; qq < a.CS; ++qq) rs += red[qq];
      misc[MS_ROWSS] = rs;
    }
    __syncthreads();
    const double thr0 = tau * sqrt(misc[MS_ROWSS] / (double)n);
    const uint64_t* wr = rec(s, win, q);
    for (int j = tid; j < TCp; j += kThreads) {
      float x = 0.f;
      if (j < TC) x = u2f(xw_wait(wr + j, ep, ab, a.budget, a.abort_word));
      vval[j] = j < TC ? tern(x, thr0) : 0.f;
    }
    ab = __syncthreads_or(ab);
  };

  stats_exchange(bad);
  if (tid == 0) misc[MS_E0] = misc[MS_R2];
  __syncthreads();
  const double E0 = misc[MS_E0];
  mark(PH_SETUP);

  long long n_fb = 0, n_zero = 0;
  int tpos = 0;
  const int S_tr = 2 * Wn + a.iters * 2 * (Wm + Wn);

  for (int comp = 0; comp < a.k; ++comp) {
    // ---- cluster-uniform decision point ----
    if (tid == 0) misc[(comp & 1) ? MS_AB1 : MS_AB0] = ab ? 1.0 : 0.0;
    cl.sync();
    if (tid == 0) {
      int any_ab = 0;
      for (int qq = 0; qq < a.CS; ++qq)
        any_ab |= cl.map_shared_rank(misc, qq)[(comp & 1) ? MS_AB1 : MS_AB0] != 0.0;
      misc[MS_ABORT] = (double)any_ab;
    }
    __syncthreads();
    if (misc[MS_ABORT] != 0.0) break;
    if (misc[MS_BAD] != 0.0) break;
    if (comp > 0 && blockIdx.x == 0 && tid == 0)
      a.energy[comp - 1] = E0 > 0.0 ? 1.0 - misc[MS_R2] / E0 : 1.0;
    if (misc[MS_M] <= 0.0) {
      // the residual vanished: the remaining components are empty (packed_B
      // was zeroed before the launch)
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
      break;
    }
    const bool traced = tpos < a.ntrace && a.trace_comp[tpos] == (int64_t)comp;
    uint32_t* tb = traced ? a.trace_bits + (size_t)tpos * S_tr : nullptr;
    if (traced) {
      pack_planes(vval, TC, c0, tb, Wn);
      if (blockIdx.x == 0 && tid == 0) a.trace_row[tpos] = (int32_t)misc[MS_ISTAR];
    }
    mark(PH_STATS);

    int nu_total = 0;
    for (int it = 0; it < a.iters; ++it) {
      const int buf = it & 1;
      // ---- y = R (w o v) over my columns, partial per row ----
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
      float* yp = ypart + buf * TRp;
      for (int g = wid; 4 * g < TR; g += kWarps) {
        const int i0 = 4 * g;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
          if (i0 + rr < TR) {
            const float4* row = (const float4*)(T + (size_t)(i0 + rr) * TCp);
#pragma unroll
            for (int qi = 0; qi < NQL; ++qi) {
              const int quad = lane + 32 * qi;
              if (quad < NQ) {
                const float4 r4 = row[quad];
                acc[rr] = fmaf(r4.x, vr[qi].x, acc[rr]);
                acc[rr] = fmaf(r4.y, vr[qi].y, acc[rr]);
                acc[rr] = fmaf(r4.z, vr[qi].z, acc[rr]);
                acc[rr] = fmaf(r4.w, vr[qi].w, acc[rr]);
              }
            }
          }
        }
        // butterfly: 4 row sums over 32 lanes with 6 shuffles
        const bool b4 = lane & 16, b3 = lane & 8;
        const float s0 = b4 ? acc[0] : acc[2], s1 = b4 ? acc[1] : acc[3];
        const float t0 = __shfl_xor_sync(0xffffffffu, s0, 16);
        const float t1 = __shfl_xor_sync(0xffffffffu, s1, 16);
        const float h0 = (b4 ? acc[2] : acc[0]) + t0;
        const float h1 = (b4 ? acc[3] : acc[1]) + t1;
        const float sx = b3 ? h0 : h1;
        const float tx = __shfl_xor_sync(0xffffffffu, sx, 8);
        float v = (b3 ? h1 : h0) + tx;
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        if ((lane & 7) == 0) {
          const int rr = (b4 ? 2 : 0) + (b3 ? 1 : 0);
          if (i0 + rr < TR) yp[i0 + rr] = v;
        }
      }
      mark(PH_YPASS);
      cl.sync();
      // all-gather y over the cluster (fixed order), local sum of squares
      double ys = 0.0;
      for (int i = tid; i < TR; i += kThreads) {
        float s = 0.f;
        for (int qq = 0; qq < a.CS; ++qq) s += cl.map_shared_rank(yp, qq)[i];
        yfull[i] = s;
        ys += (double)s * (double)s;
      }
      const double Syc = block_sum(ys, red);
      mark(PH_YGATHER);
      ++ep;
      {
        uint64_t* s = slot(ep);
        if (q == 0 && tid == 0) {
          xw_store(rec(s, c, 0) + 0, ep, dlo(Syc));
          xw_store(rec(s, c, 0) + 1, ep, dhi(Syc));
        }
        double* ysum = xd;
        for (int cc = tid; cc < a.NC; cc += kThreads) {
          const uint64_t* r = rec(s, cc, 0);
          const uint64_t v0 = xw_load(r), v1 = xw_load(r + 1);
          const uint32_t lo = take(v0, r), hi = take(v1, r + 1);
          ysum[cc] = u2d(lo, hi);
        }
        ab = __syncthreads_or(ab);
        if (tid == 0) {
          double sy = 0.0;
          for (int cc = 0; cc < a.NC; ++cc) sy += ysum[cc];
          misc[MS_SY] = sy;
        }
        __syncthreads();
      }
      const double thr_u = tau * sqrt(misc[MS_SY] / (double)m);
      int cnt = 0;
      for (int i = tid; i < TRp; i += kThreads) {
        const float uu = i < TR ? tern(yfull[i], thr_u) : 0.f;
        uval[i] = uu;
        cnt += uu != 0.f;
      }
      const int nnz_c = block_sum_int(cnt, ired);  // includes __syncthreads
      if (traced && q == 0) pack_planes_or(uval, TR, r0, tb + 2 * Wn + it * 2 * (Wm + Wn), Wm);
      mark(PH_YXCHG);

      // ---- z = R^T u over the cluster's rows, my columns ----
      // warp wid covers 128-column strip (wid % NQL) over row group (wid / NQL)
      {
        const int strip = wid % NQL, rgrp = wid / NQL;
        const int quad = strip * 32 + lane;
        if (rgrp < RG) {
          float4 za = make_float4(0.f, 0.f, 0.f, 0.f);
          if (quad < NQ) {
            for (int i = rgrp; i < TR; i += RG) {
              const float ui = uval[i];
              if (ui == 0.f) continue;
              const float4 r4 = ((const float4*)(T + (size_t)i * TCp))[quad];
              za.x = fmaf(ui, r4.x, za.x);
              za.y = fmaf(ui, r4.y, za.y);
              za.z = fmaf(ui, r4.z, za.z);
              za.w = fmaf(ui, r4.w, za.w);
            }
            *(float4*)(zred + (size_t)rgrp * TCp + 4 * quad) = za;
          }
        }
      }
      __syncthreads();
      mark(PH_ZPASS);
      ++ep;
      {
        uint64_t* s = slot(ep);
        uint64_t* mine = rec(s, c, q);
        for (int j = tid; j < TC; j += kThreads) {
          float zs = 0.f;
          for (int g = 0; g < RG; ++g) zs += zred[(size_t)g * TCp + j];
          xw_store(mine + j, ep, f2u(zs));
        }
        if (tid == 0) xw_store(mine + TCp, ep, (uint32_t)nnz_c);
        double zz = 0.0;
        for (int j = tid; j < TC; j += kThreads) {
          float z = 0.f;
          for (int cc0 = 0; cc0 < a.NC; cc0 += 8) {
            uint64_t v[8];
#pragma unroll
            for (int b = 0; b < 8; ++b)
              if (cc0 + b < a.NC) v[b] = xw_load(rec(s, cc0 + b, q) + j);
#pragma unroll
            for (int b = 0; b < 8; ++b)
              if (cc0 + b < a.NC) z += u2f(take(v[b], rec(s, cc0 + b, q) + j));
          }
          zfull[j] = z;
          zz += (double)z * (double)z;
        }
        for (int cc = tid; cc < a.NC; cc += kThreads) {
          const uint64_t* r = rec(s, cc, q) + TCp;
          nnzu[cc] = (int)take(xw_load(r), r);
        }
        ab = __syncthreads_or(ab);
        const double Szq = block_sum(zz, red);
        if (tid == 0) cx[buf * 4 + 0] = Szq;
      }
      mark(PH_ZXCHG);
      cl.sync();
      double Sz = 0.0;
      for (int qq = 0; qq < a.CS; ++qq) Sz += cl.map_shared_rank(cx, qq)[buf * 4 + 0];
      const double thr_v = tau * sqrt(Sz / (double)n);
      for (int j = tid; j < TCp; j += kThreads) vval[j] = j < TC ? tern(zfull[j], thr_v) : 0.f;
      if (tid == 0) {
        int nt = 0;
        for (int cc = 0; cc < a.NC; ++cc) nt += nnzu[cc];
        ired[kWarps] = nt;
      }
      __syncthreads();
      nu_total = ired[kWarps];
      if (traced) pack_planes(vval, TC, c0, tb + 2 * Wn + it * 2 * (Wm + Wn) + 2 * Wm, Wn);
      mark(PH_ZSYNC);
    }

    // ---- scale, gain, safeguard ----
    double pp = 0.0, vw = 0.0;
    int nv = 0;
    for (int j = tid; j < TC; j += kThreads)
      if (vval[j] != 0.f) {
        pp += (double)wcol[j] * fabs((double)zfull[j]);
        vw += (double)wcol[j];
        ++nv;
      }
    pp = block_sum(pp, red);
    vw = block_sum(vw, red);
    nv = block_sum_int(nv, ired);
    if (tid == 0) {
      cx[2 * 4 + 0] = pp;
      cx[2 * 4 + 1] = vw;
      cx[2 * 4 + 2] = (double)nv;
    }
    cl.sync();
    double P = 0.0, VW = 0.0;
    for (int qq = 0; qq < a.CS; ++qq) {
      P += cl.map_shared_rank(cx, qq)[8];
      VW += cl.map_shared_rank(cx, qq)[9];
    }
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
    for (int i = wid; i < TR; i += kWarps) {
      const float ui = uval[i];
      if (ui == 0.f) continue;
      const float sd = ui * d;  // exact: +-d
      float4* row = (float4*)(T + (size_t)i * TCp);
#pragma unroll
      for (int qi = 0; qi < NQL; ++qi) {
        const int quad = lane + 32 * qi;
        if (quad < NQ) {
          float4 r4 = row[quad];
          const float4 v4 = *(const float4*)(vval + 4 * quad);
          r4.x = v4.x > 0.f ? __fsub_rn(r4.x, sd) : (v4.x < 0.f ? __fadd_rn(r4.x, sd) : r4.x);
          r4.y = v4.y > 0.f ? __fsub_rn(r4.y, sd) : (v4.y < 0.f ? __fadd_rn(r4.y, sd) : r4.y);
          r4.z = v4.z > 0.f ? __fsub_rn(r4.z, sd) : (v4.z < 0.f ? __fadd_rn(r4.z, sd) : r4.z);
          r4.w = v4.w > 0.f ? __fsub_rn(r4.w, sd) : (v4.w < 0.f ? __fadd_rn(r4.w, sd) : r4.w);
          row[quad] = r4;
        }
      }
      __syncwarp();
      row_stats(i);
    }
    __syncthreads();
    mark(PH_DEFLATE);
    stats_exchange(0);
    mark(PH_STATS);
  }

  // final energy entry, counters, status
  __syncthreads();
  if (blockIdx.x == 0 && tid == 0) {
    if (misc[MS_ABORT] == 0.0 && misc[MS_BAD] == 0.0 && n_zero == 0 && a.k > 0)
      a.energy[a.k - 1] = E0 > 0.0 ? 1.0 - misc[MS_R2] / E0 : 1.0;
    if (a.stats) {
      a.stats[0] = n_fb;
      a.stats[1] = n_zero;
      a.stats[2] = a.NC;
      a.stats[3] = a.CS;
      a.stats[4] = SMT ? 1 : 0;
      a.stats[5] = (long long)gridDim.x;
      for (int p = 0; p < PH_N; ++p) a.stats[kStatPhase0 + p] = ph[p];
    }
    if (misc[MS_BAD] != 0.0) atomicCAS(a.dev_status, 0, EXTERND_ERR_NONFINITE);
  }
  if (tid == 0) {
    const int aw = ld_flag(a.abort_word);
    if (aw != 0) atomicCAS(a.dev_status, 0, aw);
  }
  // no CTA may leave while a cluster peer can still read its shared memory
  cl.sync();
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

template <int NQL, bool SMT>
static cudaError_t launch_one(const SeqArgs& args, size_t smem, cudaStream_t st,
                              int* max_clusters_out, bool query_only) {
  auto kern = seq_als_kernel<NQL, SMT>;
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

template <bool SMT>
static cudaError_t dispatch(int NQL, const SeqArgs& args, size_t smem, cudaStream_t st, int* mc,
                            bool query_only) {
  switch (NQL) {
    case 1: return launch_one<1, SMT>(args, smem, st, mc, query_only);
    case 2: return launch_one<2, SMT>(args, smem, st, mc, query_only);
    case 3: return launch_one<3, SMT>(args, smem, st, mc, query_only);
    case 4: return launch_one<4, SMT>(args, smem, st, mc, query_only);
    case 5: return launch_one<5, SMT>(args, smem, st, mc, query_only);
    case 6: return launch_one<6, SMT>(args, smem, st, mc, query_only);
    case 8: return launch_one<8, SMT>(args, smem, st, mc, query_only);
    default: return cudaErrorInvalidValue;
  }
}

template <bool SMT>
static size_t static_smem_t(int NQL) {
  cudaFuncAttributes fa = {};
  cudaError_t e = cudaErrorInvalidValue;
  switch (NQL) {
    case 1: e = cudaFuncGetAttributes(&fa, seq_als_kernel<1, SMT>); break;
    case 2: e = cudaFuncGetAttributes(&fa, seq_als_kernel<2, SMT>); break;
    case 3: e = cudaFuncGetAttributes(&fa, seq_als_kernel<3, SMT>); break;
    case 4: e = cudaFuncGetAttributes(&fa, seq_als_kernel<4, SMT>); break;
    case 5: e = cudaFuncGetAttributes(&fa, seq_als_kernel<5, SMT>); break;
    case 6: e = cudaFuncGetAttributes(&fa, seq_als_kernel<6, SMT>); break;
    case 8: e = cudaFuncGetAttributes(&fa, seq_als_kernel<8, SMT>); break;
    default: break;
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return (size_t)1 << 30;
  }
  return fa.sharedSizeBytes;
}

static size_t static_smem(int NQL, bool smt) {
  return smt ? static_smem_t<true>(NQL) : static_smem_t<false>(NQL);
}

static int nql_for(int TCp) {
  const int nq = TCp / 4;
  int v = (nq + 31) / 32;
  if (v == 7) v = 8;
  return v;
}

struct SeqPlan {
  int NC = 0, CS = 0, TRmax = 0, TCp = 0, NQL = 0;
  bool smt = false;
  size_t smem = 0;
};

// Chooses cluster size, cluster count and tile residency.  Candidates must be
// co-resident (occupancy query).  Shared-memory residency of the whole
// residual wins; among equals the estimated cost per half-step, tile words
// streamed per CTA plus the cross-cluster words each CTA polls, is smallest.
static cudaError_t plan_seq(int m, int n, cudaStream_t st, SeqPlan* out) {
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
  bool best_smt = false;
  for (int CS : cands) {
    if (force_cs > 0 && CS != force_cs) continue;
    if (CS > nchc) continue;
    const int colchunks = (nchc + CS - 1) / CS;
    const int TC = std::min(colchunks * 32, n);
    const int TCp = (TC + 3) & ~3;
    const int NQL = nql_for(TCp);
    if (NQL > 8) continue;
    for (int smt_try = 1; smt_try >= 0; --smt_try) {
      const bool smt = smt_try == 1;
      if (best_smt && !smt) continue;
      int nc = std::min(std::min(m, 64), std::max(1, nsm / CS));
      for (int guard = 0; guard < 16 && nc >= 1; ++guard) {
        const int TRmax = (m + nc - 1) / nc;
        SeqSmem L(TRmax, TCp, nc, NQL, smt);
        const size_t stat = static_smem(NQL, smt);
        if (L.total + stat > (size_t)optin) break;
        SeqArgs probe = {};
        probe.NC = nc;
        probe.CS = CS;
        int maxc = 0;
        cudaError_t qe = smt ? dispatch<true>(NQL, probe, L.total, st, &maxc, true)
                             : dispatch<false>(NQL, probe, L.total, st, &maxc, true);
        if (qe != cudaSuccess) {
          cudaGetLastError();
          break;
        }
        if (maxc >= nc) {
          const double tile_w = (double)TRmax * TCp * (smt ? 1.0 : 4.0);
          const double cost = tile_w + 8.0 * nc * TCp;
          if ((smt && !best_smt) || cost < best_cost) {
            best_cost = cost;
            best_smt = smt;
            best.NC = nc;
            best.CS = CS;
            best.TRmax = TRmax;
            best.TCp = TCp;
            best.NQL = NQL;
            best.smt = smt;
            best.smem = L.total;
          }
          break;
        }
        if (maxc < 1) break;
        nc = std::min(nc - 1, maxc);
      }
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
  cudaError_t e = plan_seq((int)h.m, (int)h.n, st, &pl);
  if (e == cudaErrorNotSupported) return EXTERND_ERR_NO_COOP;
  if (e != cudaSuccess) return EXTERND_ERR_CUDA;
  const int recw = pl.TCp + 16;
  const long long slot_words = (long long)pl.NC * pl.CS * recw;
  const size_t xbytes = sizeof(uint64_t) * 3 * (size_t)slot_words;
  const size_t abort_off = (xbytes + 255) & ~(size_t)255;
  const size_t tile_off = abort_off + 256;
  const size_t tile_bytes =
      pl.smt ? 0 : sizeof(float) * (size_t)pl.NC * pl.CS * (size_t)pl.TRmax * (size_t)pl.TCp;
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
    a.gtile = pl.smt ? nullptr : (float*)((char*)ws + tile_off);
    a.xbuf = (uint64_t*)ws;
    a.abort_word = (int*)((char*)ws + abort_off);
    a.dev_status = status_word_ptr();
    if (!a.dev_status) rc = EXTERND_ERR_CUDA;
    if (rc == EXTERND_OK) {
      int dummy = 0;
      e = pl.smt ? dispatch<true>(pl.NQL, a, pl.smem, st, &dummy, false)
                 : dispatch<false>(pl.NQL, a, pl.smem, st, &dummy, false);
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
  cudaError_t e = plan_seq((int)h.m, (int)h.n, st, &pl);
  if (e == cudaErrorNotSupported) return EXTERND_ERR_NO_COOP;
  if (e != cudaSuccess) return EXTERND_ERR_CUDA;
  if (!pl.smt) return EXTERND_ERR_SCRATCH_LIMIT;
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
  e = dispatch<true>(pl.NQL, a, pl.smem, st, &dummy, false);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return EXTERND_ERR_CUDA;
  }
  return EXTERND_OK;
}

}  // namespace externd
