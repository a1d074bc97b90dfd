// The persistent sequential-deflation ALS kernel (a template instantiated in
// the seq_inst_*.cu units; the host side that plans and launches it is in
// seq_als.cu).
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

#pragma once

#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace externd {

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
  int NSy;       // column segments of the y pass over the shared-memory rows
  int flags;     // EXTERND_TSTAT_MEAN_ABS | EXTERND_VSTEP_NAIVE
  int sweeps;    // refinement sweeps after the greedy pass
  double* sweep_energy;  // [sweeps] energy after each sweep
  float* dpriv;  // [grid][k] each CTA's own copy of the scales it emitted (sweeps)
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
//                   partials, or the row energies in the statistics step);
//                   summed in place into y
//  zred  the z pass's partials per row slot ([RGz][TCp]), the y pass's
//        partials per column segment ([NSy][SRp], then the global rows), and
//        the statistics step's scratch -- lifetimes disjoint
//  rlist the rows of the cluster band with u_i != 0 in ascending order, as i
//        (u_i = +1) or ~i (u_i = -1)
//  zs    per-CTA partial sums pushed to every CTA of the cluster: [0, CS)
//        the threshold statistic of z (sum z_j^2 or sum |z_j|), [CS, 2CS)
//        sum w_j |z_j| and [2CS, 3CS) sum w_j over v_j != 0, [3CS, 4CS) sum w_j
//        over the old component's v_j != 0 (refinement steps)
//  uold, vold  the old component's codes in a refinement step (my cluster's
//        rows, my columns)
//  tile  the first SR rows of this CTA's residual tile, TCp floats per row
//        (TCp a multiple of 32); row i keeps its logical quad q (columns
//        4q .. 4q+3) at physical quad q ^ (i & 7), so that 8 consecutive rows
//        read at one logical quad, or one row read at 8 consecutive quads,
//        touch 8 distinct 16-byte bank groups
struct SeqSmem {
  size_t wp, wpi, misc, rss, xd, xu, erec, abg, uval, gat, rho_p, rmax, zred, wcol, vval, vw,
      zown, nnzu, rlist, zs, uold, vold, wcnt, tile, total;
  int zred_floats;
  __host__ __device__ SeqSmem(int TRmax, int TCp, int NC, int CS, int SR, int NSy) {
    const int TRp = (TRmax + 31) & ~31;
    const int SRp = (SR + 31) & ~31;
    const int RGz = kThreads / (TCp / 4);
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
    xd = take(sizeof(double) * 3 * NC);    // per-cluster fp64 records
    xu = take(sizeof(uint32_t) * 6 * NC);  // per-cluster 32-bit records
    erec = take(sizeof(double) * 4 * CS);  // per-CTA best entry (pushed)
    abg = take(sizeof(int) * CS);          // per-CTA abort flags (pushed)
    uval = take(sizeof(float) * TRp);
    gat = take(sizeof(float) * (size_t)CS * TRp);
    rho_p = take(sizeof(float) * TRp);
    rmax = take(sizeof(float) * TRp);
    long long zf = (long long)RGz * TCp;
    const long long yf = (long long)NSy * SRp + (TRp - SR);
    if (yf > zf) zf = yf;
    if (TRp > zf) zf = TRp;
    if (TCp > zf) zf = TCp;
    zred_floats = (int)zf;
    zred = take(sizeof(float) * (size_t)zf);
    wcol = take(sizeof(float) * TCp);
    vval = take(sizeof(float) * TCp);
    vw = take(sizeof(float) * TCp);
    zown = take(sizeof(float) * TCp);
    nnzu = take(sizeof(int) * NC);
    rlist = take(sizeof(int) * TRp);
    zs = take(sizeof(double) * 4 * CS);
    uold = take(sizeof(float) * TRp);
    vold = take(sizeof(float) * TCp);
    wcnt = take(sizeof(int) * (kWarps + 2));
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
  MS_DOLD,   // the old component's scale in a refinement step
  MS_NUOC,   // rows of my cluster in the old component (refinement)
  MS_VWOQ,   // sum of w_j over my columns of the old v (refinement)
  MS_POT,    // u_o^T R W v_o over all rows (refinement)
  MS_NUOT,   // |u_o|^2 over all rows (refinement)
  MS_PH = 16 // phase timers (long long, CTA 0 thread 0 only)
};

__device__ __forceinline__ float tern(float x, double thr) {
  double a = fabs((double)x);
  return a > thr ? (x > 0.f ? 1.f : -1.f) : 0.f;
}

__device__ __forceinline__ float tern_d(double x, double thr) {
  return fabs(x) > thr ? (x > 0.0 ? 1.f : -1.f) : 0.f;
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

// Same, replacing earlier bits of the entries [g0, g0+len) only (the other
// bits of a shared word belong to the neighbouring bands and are kept).
__device__ __forceinline__ void pack_planes_replace(const float* vals, int len, int g0,
                                                    uint32_t* plane0, int W) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int w0 = g0 >> 5, w1 = (g0 + len + 31) >> 5;
  for (int t = w0 + wid; t < w1; t += kWarps) {
    const int e = t * 32 + lane - g0;
    const bool in = e >= 0 && e < len;
    const float x = in ? vals[e] : 0.f;
    const uint32_t own = __ballot_sync(0xffffffffu, in);
    const uint32_t mk = __ballot_sync(0xffffffffu, x != 0.f);
    const uint32_t sg = __ballot_sync(0xffffffffu, x < 0.f);
    if (lane == 0) {
      atomicAnd(plane0 + t, ~own);
      atomicAnd(plane0 + W + t, ~own);
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

__device__ __forceinline__ float4 lds4(uint32_t a) {
  float4 r;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
               : "r"(a));
  return r;
}
__device__ __forceinline__ void sts4(uint32_t a, float4 x) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(x.x), "f"(x.y), "f"(x.z),
               "f"(x.w)
               : "memory");
}

// Byte offset of logical quad q of shared-memory tile row i (see SeqSmem).
__device__ __forceinline__ uint32_t tile_off(int i, int q, int TCp) {
  return 4u * (uint32_t)(i * TCp + ((q ^ (i & 7)) << 2));
}

// y partials of K groups of 32 shared-memory tile rows over the logical quads
// [q0, q1): lane l of the warp takes row 32 g[t] + l of group t, so a load
// of one logical quad reads 32 rows; rows >= TRs are read from row TRs - 1
// and dropped.  Writes part[row] (one fp32 partial per row), each summed in
// a fixed order.  Quads go in steps of QS, all of a step's loads issued
// before its products.
template <int K, int QS>
__device__ __forceinline__ void y_rows(uint32_t tsb, int TCp, int TRs, const int* g, int q0,
                                       int q1, const float4* vw4, float* part) {
  const int lane = threadIdx.x & 31, sw = lane & 7;  // row & 7 == lane & 7
  uint32_t rb[K];
  int row[K];
#pragma unroll
  for (int t = 0; t < K; ++t) {
    row[t] = g[t] * 32 + lane;
    const int rr = row[t] < TRs ? row[t] : TRs - 1;
    rb[t] = tsb + 4u * (uint32_t)(rr * TCp);
  }
  float a0[K], a1[K];
#pragma unroll
  for (int t = 0; t < K; ++t) a0[t] = a1[t] = 0.f;
  int q = q0;
  for (; q + QS <= q1; q += QS) {
    float4 x[QS][K], v[QS];
#pragma unroll
    for (int u = 0; u < QS; ++u) {
      v[u] = vw4[q + u];
#pragma unroll
      for (int t = 0; t < K; ++t) x[u][t] = lds4(rb[t] + (uint32_t)(((q + u) ^ sw) << 4));
    }
#pragma unroll
    for (int u = 0; u < QS; ++u)
#pragma unroll
      for (int t = 0; t < K; ++t) {
        a0[t] = fmaf(x[u][t].x, v[u].x, a0[t]);
        a1[t] = fmaf(x[u][t].y, v[u].y, a1[t]);
        a0[t] = fmaf(x[u][t].z, v[u].z, a0[t]);
        a1[t] = fmaf(x[u][t].w, v[u].w, a1[t]);
      }
  }
  for (; q < q1; ++q) {
    const float4 vl = vw4[q];
    float4 x[K];
#pragma unroll
    for (int t = 0; t < K; ++t) x[t] = lds4(rb[t] + (uint32_t)((q ^ sw) << 4));
#pragma unroll
    for (int t = 0; t < K; ++t) {
      a0[t] = fmaf(x[t].x, vl.x, a0[t]);
      a1[t] = fmaf(x[t].y, vl.y, a1[t]);
      a0[t] = fmaf(x[t].z, vl.z, a0[t]);
      a1[t] = fmaf(x[t].w, vl.w, a1[t]);
    }
  }
#pragma unroll
  for (int t = 0; t < K; ++t)
    if (row[t] < TRs) part[row[t]] = a0[t] + a1[t];
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

// FULL: the threshold variants and the refinement sweeps are compiled in
// (the plain decomposition runs the FULL == false instantiation, which
// carries none of their state).
template <int NQL, bool HYB, bool FULL>
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
  const int TCp = a.TCp;        // multiple of 32
  const int NQs = TCp >> 2;     // quads per tile row (a multiple of 8)
  const int Wm = (m + 31) >> 5, Wn = (n + 31) >> 5;
  const int SR = a.SR;
  const int TRs = min(TR, SR);  // rows of this tile held in shared memory
  const int SRp = (SR + 31) & ~31;

  const bool weighted = a.w != nullptr;
  const SeqSmem L(a.TRmax, TCp, a.NC, CS, SR, a.NSy);
  double* wp = (double*)(smem + L.wp);
  int* wpi = (int*)(smem + L.wpi);
  double* misc = (double*)(smem + L.misc);
  double* xd = (double*)(smem + L.xd);
  uint32_t* xu = (uint32_t*)(smem + L.xu);
  double* erec = (double*)(smem + L.erec);
  int* abg = (int*)(smem + L.abg);
  float* uval = (float*)(smem + L.uval);
  float* gat = (float*)(smem + L.gat);
  float* rho_p = (float*)(smem + L.rho_p);
  float* rmax = (float*)(smem + L.rmax);
  float* zred = (float*)(smem + L.zred);
  float* part = zred;                     // y partials (lifetime disjoint from zred's)
  float* yfull = (float*)(smem + L.gat);  // summed in place over gat's first row block
  float* wcol = (float*)(smem + L.wcol);
  float* vval = (float*)(smem + L.vval);
  float* vw = (float*)(smem + L.vw);
  float* zown = (float*)(smem + L.zown);
  int* nnzu = (int*)(smem + L.nnzu);
  int* rlist = (int*)(smem + L.rlist);
  double* zs = (double*)(smem + L.zs);
  int* wcnt = (int*)(smem + L.wcnt);
  float* const Ts = (float*)(smem + L.tile);
  const uint32_t tsb = (uint32_t)__cvta_generic_to_shared(Ts);
  float* const Tg = a.gtile + (size_t)blockIdx.x * (size_t)(a.TRmax - SR) * (size_t)TCp;
  // row i of this CTA's tile: shared memory (swizzled quads) for the first SR
  // rows, else the private global region (plain layout).  HYB == false: every
  // row is in shared memory, SR == TRmax.
  auto ld4 = [&](int i, int quad) -> float4 {
    if (!HYB || i < SR) return lds4(tsb + tile_off(i, quad, TCp));
    return ((const float4*)(Tg + (size_t)(i - SR) * TCp))[quad];
  };
  auto st4 = [&](int i, int quad, float4 x) {
    if (!HYB || i < SR)
      sts4(tsb + tile_off(i, quad, TCp), x);
    else
      ((float4*)(Tg + (size_t)(i - SR) * TCp))[quad] = x;
  };
  auto ld1 = [&](int i, int j) -> float {
    if (!HYB || i < SR) return Ts[(tile_off(i, j >> 2, TCp) >> 2) + (j & 3)];
    return Tg[(size_t)(i - SR) * TCp + j];
  };
  auto st1 = [&](int i, int j, float x) {
    if (!HYB || i < SR)
      Ts[(tile_off(i, j >> 2, TCp) >> 2) + (j & 3)] = x;
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

  // ---- setup: A -> tile, weights of my columns, validity ----
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
  for (int j = tid; j < TCp; j += kThreads) {
    float wv = 0.f;
    if (j < TC) {
      wv = weighted ? a.w[c0 + j] : 1.f;
      if (!(wv > 0.f) || !isfinite(wv)) bad = 1;
    }
    wcol[j] = wv;
    vval[j] = 0.f;
    vw[j] = 0.f;
    zown[j] = 0.f;
  }
  for (int i = tid; i < TRp; i += kThreads) {
    uval[i] = 0.f;
    rho_p[i] = 0.f;
    rmax[i] = 0.f;
  }
  {
    double b1[1] = {(double)bad};
    bsum<1>(b1, wp, rph);
    bad = b1[0] > 0.0 ? 1 : 0;
  }

  // ---- deflation of one or two rows with refreshed row statistics ----
  // One warp per row, lanes over logical quads.  Row ia (and ib when
  // ib >= 0) gets R_ij <- fl32(R_ij -+ sd) where v_j = +-1 (sd = u_i d, exact;
  // sd == 0 leaves the row as it is); then rho_p = sum_j w_j R_ij^2 (fp32,
  // fixed order) and rmax = the row's largest score (|R_ij|, or the fp32
  // (R_ij * R_ij) * w_j when weighted).
  auto upd_quad = [&](float4& x, float sd, int quad) {
    const float4 v4 = *(const float4*)(vval + 4 * quad);
    x.x = v4.x > 0.f ? __fsub_rn(x.x, sd) : (v4.x < 0.f ? __fadd_rn(x.x, sd) : x.x);
    x.y = v4.y > 0.f ? __fsub_rn(x.y, sd) : (v4.y < 0.f ? __fadd_rn(x.y, sd) : x.y);
    x.z = v4.z > 0.f ? __fsub_rn(x.z, sd) : (v4.z < 0.f ? __fadd_rn(x.z, sd) : x.z);
    x.w = v4.w > 0.f ? __fsub_rn(x.w, sd) : (v4.w < 0.f ? __fadd_rn(x.w, sd) : x.w);
  };
  auto stat_quad = [&](const float4& x, int quad, float& rh, float& mx) {
    const float4 w4 = *(const float4*)(wcol + 4 * quad);
    const float xs[4] = {x.x, x.y, x.z, x.w};
    const float ws[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float sq = __fmul_rn(xs[e], xs[e]);
      rh = fmaf(ws[e], sq, rh);
      mx = fmaxf(mx, weighted ? __fmul_rn(sq, ws[e]) : fabsf(xs[e]));
    }
  };
  auto rows_update = [&](int ia, float sa, int ib, float sb) {
    float4 xa[NQL], xb[NQL];
#pragma unroll
    for (int k = 0; k < NQL; ++k) {
      const int quad = lane + 32 * k;
      if (quad < NQs) {
        xa[k] = ld4(ia, quad);
        if (ib >= 0) xb[k] = ld4(ib, quad);
      }
    }
    float rha = 0.f, mxa = 0.f, rhb = 0.f, mxb = 0.f;
#pragma unroll
    for (int k = 0; k < NQL; ++k) {
      const int quad = lane + 32 * k;
      if (quad < NQs) {
        if (sa != 0.f) {
          upd_quad(xa[k], sa, quad);
          st4(ia, quad, xa[k]);
        }
        stat_quad(xa[k], quad, rha, mxa);
        if (ib >= 0) {
          if (sb != 0.f) {
            upd_quad(xb[k], sb, quad);
            st4(ib, quad, xb[k]);
          }
          stat_quad(xb[k], quad, rhb, mxb);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      rha += __shfl_xor_sync(0xffffffffu, rha, o);
      mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, o));
      rhb += __shfl_xor_sync(0xffffffffu, rhb, o);
      mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, o));
    }
    if (lane == 0) {
      rho_p[ia] = rha;
      rmax[ia] = mxa;
      if (ib >= 0) {
        rho_p[ib] = rhb;
        rmax[ib] = mxb;
      }
    }
  };

  for (int i = wid; i < TR; i += 2 * kWarps)
    rows_update(i, 0.f, i + kWarps < TR ? i + kWarps : -1, 0.f);
  __syncthreads();

  // ---- the threshold statistic of T_tau: sum x^2 (rms) or sum |x| (mean |x|)
  const bool mean_abs = FULL && (a.flags & EXTERND_TSTAT_MEAN_ABS) != 0;
  const bool naive = FULL && weighted && (a.flags & EXTERND_VSTEP_NAIVE) != 0;
  auto st_acc = [&](double x) -> double { return mean_abs ? fabs(x) : x * x; };
  auto st_thr = [&](double sum, int len) -> double {
    return mean_abs ? tau * (sum / (double)len) : tau * sqrt(sum / (double)len);
  };

  // ---- statistics exchange: row energies, best row, best entry, |R|^2 ----
  // Leaves misc[MS_R2], misc[MS_M], misc[MS_MVAL], misc[MS_MI], misc[MS_MJ],
  // misc[MS_ISTAR], misc[MS_BAD] and, when with_row, the starting v (vval,
  // vw) for this CTA.
  auto stats_exchange = [&](int bad_in, bool with_row) {
    // this CTA's best entry: the row of the largest score (lowest row on
    // ties), then the lowest column of that row holding the score
    double bs = -1.0;
    int bi = 0x7fffffff;
    for (int i = tid; i < TR; i += kThreads) {
      const double s = (double)rmax[i];
      if (s > bs || (s == bs && i < bi)) { bs = s; bi = i; }
    }
    {
      double dummy = 0.0;
      bargmax_sum(bs, bi, dummy, wp, wpi, rph);
    }
    // push row energies to every CTA of the cluster
    for (int e = tid; e < CS * (TRp >> 2); e += kThreads) {
      const int qq = e / (TRp >> 2), i4 = e - qq * (TRp >> 2);
      float4* dst = (float4*)cl.map_shared_rank(gat, qq) + (size_t)q * (TRp >> 2) + i4;
      *dst = ((const float4*)rho_p)[i4];
    }
    if (wid == 0) {
      int jb = 0x7fffffff;
      float val = 0.f;
      if (bi >= 0 && bi < TR) {
        const float target = (float)bs;
        for (int j = lane; j < TC; j += 32) {
          const float x = ld1(bi, j);
          const float sq = __fmul_rn(x, x);
          const float sc = weighted ? __fmul_rn(sq, wcol[j]) : fabsf(x);
          if (sc == target && j < jb) { jb = j; val = x; }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const int oj = __shfl_xor_sync(0xffffffffu, jb, o);
        const float ov = __shfl_xor_sync(0xffffffffu, val, o);
        if (oj < jb) { jb = oj; val = ov; }
      }
      const bool found = bi >= 0 && bi < TR && jb < TC;
      const double flat = found ? (double)((r0 + bi) * n + c0 + jb) : 2147483647.0;
      if (lane < CS) {
        double* dst = cl.map_shared_rank(erec, lane) + 4 * q;
        dst[0] = found ? bs : -1.0;
        dst[1] = flat;
        dst[2] = found ? (double)val : 0.0;
      }
    }
    cl.sync();
    // cluster rows: energies, best row, |R|^2 over the cluster's rows
    double brho = -1.0, r2 = 0.0;
    int bir = 0x7fffffff;
    for (int i = tid; i < TR; i += kThreads) {
      double s = 0.0;
      for (int qq = 0; qq < CS; ++qq) s += (double)gat[(size_t)qq * TRp + i];
      r2 += s;
      if (s > brho) { brho = s; bir = i; }
    }
    bargmax_sum(brho, bir, r2, wp, wpi, rph);
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
    const int ib = (bir >= 0 && bir < TR) ? bir : 0;
    ++ep;
    uint64_t* s = slot(ep);
    uint64_t* mine = rec(s, c, q);
    // my slice of the cluster's best row (pairs of words), then its statistic
    for (int j = 2 * tid; with_row && j < TC; j += 2 * kThreads) {
      const float x0 = ld1(ib, j), x1 = (j + 1 < TC) ? ld1(ib, j + 1) : 0.f;
      xw_store2(mine + j, ep, f2u(x0), f2u(x1));
    }
    if (with_row && wid == 0) {
      double ss = 0.0;
      for (int j = lane; j < TC; j += 32) ss += st_acc((double)ld1(ib, j));
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
    const bool one_round = !with_row || (a.NC <= 16 && TC + a.NC <= kThreads &&
                                         2 * a.NC * CS <= L.zred_floats);
    // the CTAs' slice statistics: fetched by the threads past the record
    // range, each taking every nspare-th one (a few waits at most); only if
    // no thread is spare do the record threads fetch their cluster's
    const int rs0 = TC + a.NC, nspare = kThreads - rs0;
    const bool rsa_spare = nspare > 0;
    const long long cstride = (long long)CS * a.recw;
    const int rbase = (with_row && one_round) ? TC : 0;  // first thread of the record range
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
      if (with_row && one_round && !rsa_spare)
        for (int qq = 0; qq < CS; ++qq) {
          uint32_t p2[2];
          xw_wait_n<2>(rec(s, cc, qq) + TCp, 1, 2, ep, p2, ab, a.budget, a.abort_word);
          rsa[cc * CS + qq] = u2d(p2[0], p2[1]);
        }
    } else if (with_row && one_round && rsa_spare && tid >= rs0) {
      for (int t = tid - rs0; t < a.NC * CS; t += nspare) {
        const int cc = t / CS, qq = t - cc * CS;
        uint32_t p[2];
        xw_wait_n<2>(rec(s, cc, qq) + TCp, 1, 2, ep, p, ab, a.budget, a.abort_word);
        rsa[t] = u2d(p[0], p[1]);
      }
    } else if (with_row && one_round && tid < TC) {
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
    if (!with_row) {
      // no starting row wanted (refinement steps, the end of a pass)
    } else if (one_round) {
      double rs = 0.0;
      for (int qq = 0; qq < CS; ++qq) rs += rsa[win * CS + qq];
      const double thr0 = st_thr(rs, n);
      for (int j = tid; j < TCp; j += kThreads) {
        float x = 0.f;
        if (j < TC) {
#pragma unroll
          for (int t = 0; t < 16; ++t)
            if (t == win) x = u2f(slice[t]);
        }
        const float vv = j < TC ? tern(x, thr0) : 0.f;
        vval[j] = vv;
        vw[j] = vv * wcol[j];
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
      const double thr0 = st_thr(rs, n);
      for (int j = tid; j < TCp; j += kThreads) {
        const float vv = j < TC ? tern(rowbuf[j], thr0) : 0.f;
        vval[j] = vv;
        vw[j] = vv * wcol[j];
      }
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

  stats_exchange(bad, true);
  const double E0 = misc[MS_R2];
  mark(PH_SETUP);

  long long n_fb = 0, n_zero = 0;
  int tpos = 0;
  const int S_tr = 2 * Wn + a.iters * 2 * (Wm + Wn);
  bool stop = false;
  // the y pass's split of the shared-memory rows: column segment sy of NSy,
  // row groups of 32 every gsy-th from gy0
  const int NSy = a.NSy, sy = wid % NSy, gsy = kWarps / NSy;
  const int SQy = (NQs + NSy - 1) / NSy;
  const int qy0 = min(NQs, sy * SQy), qy1 = min(NQs, qy0 + SQy);
  const int NGs = (TRs + 31) >> 5;
  // the global rows (HYB): contiguous blocks per warp
  const int TRg = TR - TRs;
  const int rpwg = (TRg + kWarps - 1) / kWarps;
  const int gr0 = TRs + min(TRg, wid * rpwg), gr1 = TRs + min(TRg, wid * rpwg + rpwg);
  // the z pass's split: thread -> (logical quad, row slot)
  const int RGz = kThreads / NQs;
  const int qz = tid % NQs, rgz = tid / NQs;
  int nlist = 0;  // entries of rlist (rows of the cluster band with u_i != 0)
  float* const uold = (float*)(smem + L.uold);
  float* const vold = (float*)(smem + L.vold);

  // rlist <- the rows of the cluster band whose code in `codes` is nonzero,
  // ascending; returns their number (the same in every thread)
  auto compact = [&](const float* codes) -> int {
    int cnt = 0;
    for (int base = 0; base < TRp; base += kThreads) {
      const int i = base + tid;
      const float uu = i < TR ? codes[i] : 0.f;
      const unsigned bal = __ballot_sync(0xffffffffu, uu != 0.f);
      if (lane == 0) wcnt[wid] = __popc(bal);
      __syncthreads();
      int off = cnt, tot = cnt;
      for (int w2 = 0; w2 < kWarps; ++w2) {
        const int cw = wcnt[w2];
        if (w2 < wid) off += cw;
        tot += cw;
      }
      if (uu != 0.f) rlist[off + __popc(bal & ((1u << lane) - 1u))] = uu > 0.f ? i : ~i;
      cnt = tot;
      __syncthreads();
    }
    return cnt;
  };
  // energy after step tp (a greedy component, or the last step of a sweep)
  auto record_energy = [&](int tp) {
    const double e = E0 > 0.0 ? 1.0 - misc[MS_R2] / E0 : 1.0;
    if (tp < a.k)
      a.energy[tp] = e;
    else if ((tp - a.k) % a.k == a.k - 1)
      a.sweep_energy[(tp - a.k) / a.k] = e;
  };

  // Steps 0 .. k-1 are the greedy components; then each refinement sweep
  // revisits components 0 .. k-1 in order (step k (1 + s) + l is component
  // l in sweep s).
  const int nsteps = FULL ? a.k * (1 + a.sweeps) : a.k;  // < 2^31 (checked on the host)
  for (int t = 0; t < nsteps && !stop; ++t) {
    const bool sweep = FULL && t >= a.k;
    const int comp = t % a.k;
    if (t > 0 && blockIdx.x == 0 && tid == 0) record_energy(t - 1);
    const bool traced = tpos < a.ntrace && a.trace_comp[tpos] == (int64_t)t;
    uint32_t* tb = traced ? a.trace_bits + (size_t)tpos * S_tr : nullptr;
    int nu_total = 0;
    if (sweep) {
      // ---- refinement: the old component l = comp, added back onto R ----
      const uint32_t* pb = a.pB + (size_t)comp * 2 * Wm;
      const uint32_t* pc = a.pC + (size_t)comp * 2 * Wn;
      for (int i = tid; i < TRp; i += kThreads) {
        float u = 0.f;
        if (i < TR) {
          const int r = r0 + i;
          const uint32_t bit = 1u << (r & 31);
          if (pb[r >> 5] & bit) u = (pb[Wm + (r >> 5)] & bit) ? -1.f : 1.f;
        }
        uold[i] = u;
      }
      for (int j = tid; j < TCp; j += kThreads) {
        float v = 0.f;
        if (j < TC) {
          const int cj = c0 + j;
          const uint32_t bit = 1u << (cj & 31);
          if (pc[cj >> 5] & bit) v = (pc[Wn + (cj >> 5)] & bit) ? -1.f : 1.f;
        }
        vold[j] = v;
        vval[j] = v;
        vw[j] = v * wcol[j];
      }
      if (tid == 0) misc[MS_DOLD] = (double)a.dpriv[(size_t)blockIdx.x * a.k + comp];
      __syncthreads();
      const int nuo_c = compact(uold);
      const float d_o = (float)misc[MS_DOLD];
      // R <- R + d_o u_o v_o^T: the deflation routine with the opposite sign
      for (int e = wid; e < nuo_c; e += 2 * kWarps) {
        const int xa = rlist[e];
        int ib = -1;
        float sb = 0.f;
        if (e + kWarps < nuo_c) {
          const int xb = rlist[e + kWarps];
          ib = xb >= 0 ? xb : ~xb;
          sb = xb >= 0 ? -d_o : d_o;
        }
        rows_update(xa >= 0 ? xa : ~xa, xa >= 0 ? -d_o : d_o, ib, sb);
      }
      {
        double vwp[1] = {0.0};
        for (int j = tid; j < TC; j += kThreads)
          if (vold[j] != 0.f) vwp[0] += (double)wcol[j];
        bsum<1>(vwp, wp, rph);  // (also orders the row updates before the exchange)
        if (tid == 0) {
          misc[MS_VWOQ] = vwp[0];
          misc[MS_NUOC] = (double)nuo_c;
        }
      }
      stats_exchange(0, false);
      mark(PH_STATS);
    }
    for (int it = 0; it < a.iters; ++it) {
      // ---- y = R (w o v) over my columns: partial per row ----
      for (int gb = wid / NSy; gb < NGs; gb += 4 * gsy) {
        int g[4];
        int K = 0;
#pragma unroll
        for (int t2 = 0; t2 < 4; ++t2) {
          g[t2] = gb + t2 * gsy;
          if (g[t2] < NGs) K = t2 + 1;
        }
        float* ps = part + (size_t)sy * SRp;
        const float4* vw4 = (const float4*)vw;
        if (K == 4) y_rows<4, 2>(tsb, TCp, TRs, g, qy0, qy1, vw4, ps);
        else if (K == 3) y_rows<3, 3>(tsb, TCp, TRs, g, qy0, qy1, vw4, ps);
        else if (K == 2) y_rows<2, 4>(tsb, TCp, TRs, g, qy0, qy1, vw4, ps);
        else y_rows<1, 12>(tsb, TCp, TRs, g, qy0, qy1, vw4, ps);
      }
      if (HYB && gr0 < gr1) {
        float4 vr[NQL];
#pragma unroll
        for (int k = 0; k < NQL; ++k) {
          const int quad = lane + 32 * k;
          vr[k] = quad < NQs ? *(const float4*)(vw + 4 * quad) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        for (int i = gr0; i < gr1; ++i) {
          float acc = 0.f;
#pragma unroll
          for (int k = 0; k < NQL; ++k) {
            const int quad = lane + 32 * k;
            if (quad < NQs) {
              const float4 r4 = ld4(i, quad);
              acc = fmaf(r4.x, vr[k].x, acc);
              acc = fmaf(r4.y, vr[k].y, acc);
              acc = fmaf(r4.z, vr[k].z, acc);
              acc = fmaf(r4.w, vr[k].w, acc);
            }
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
          if (lane == 0) part[(size_t)NSy * SRp + (i - TRs)] = acc;
        }
      }
      __syncthreads();
      mark(PH_YPASS);
      // sum my row partials and push them (and, once per step, my abort
      // flag) to every CTA of the cluster
      if (pending_wait) {
        cluster_wait();
        pending_wait = false;
      }
      // (the row sums go to uval, free until the u threshold rewrites it,
      // then every push is one load and one store)
      for (int i = tid; i < TRp; i += kThreads) {
        float sacc = 0.f;
        if (i < TRs) {
          for (int ss = 0; ss < NSy; ++ss) sacc += part[(size_t)ss * SRp + i];
        } else if (i < TR) {
          sacc = part[(size_t)NSy * SRp + (i - TRs)];
        }
        uval[i] = sacc;
      }
      __syncthreads();
      for (int e = tid; e < CS * (TRp >> 2); e += kThreads) {
        const int qq = e / (TRp >> 2), i4 = e - qq * (TRp >> 2);
        ((float4*)cl.map_shared_rank(gat, qq))[(size_t)q * (TRp >> 2) + i4] =
            ((const float4*)uval)[i4];
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
        if (!sweep && misc[MS_M] <= 0.0) {
          // the residual vanished: the remaining components are empty
          // (packed_B was zeroed before the launch); no sweep runs
          for (int cc = comp; cc < a.k; ++cc) {
            for (int t2 = (c0 >> 5) + tid; t2 < (c1 + 31) >> 5; t2 += kThreads) {
              a.pC[(size_t)cc * 2 * Wn + t2] = 0u;
              a.pC[(size_t)cc * 2 * Wn + Wn + t2] = 0u;
            }
            if (blockIdx.x == 0 && tid == 0) {
              a.D[cc] = 0.f;
              a.energy[cc] = 1.0;
            }
          }
          if (blockIdx.x == 0 && tid == 0)
            for (int s2 = 0; s2 < a.sweeps; ++s2) a.sweep_energy[s2] = 1.0;
          n_zero = a.k - comp;
          stop = true;
          break;
        }
        if (traced) {
          pack_planes(vval, TC, c0, tb, Wn);
          if (blockIdx.x == 0 && tid == 0)
            a.trace_row[tpos] = sweep ? -1 : (int32_t)misc[MS_ISTAR];
        }
      }
      // y over the cluster's rows (fixed order), its statistic, and in a
      // refinement step's first round u_o^T y (the old pattern's gain)
      const bool first_ref = sweep && it == 0;
      double ys[2] = {0.0, 0.0};
      for (int i = tid; i < TR; i += kThreads) {
        float sy_ = 0.f;
        for (int qq = 0; qq < CS; ++qq) sy_ += gat[(size_t)qq * TRp + i];
        yfull[i] = sy_;  // overwrites gat[i] after its last read, same thread
        ys[0] += st_acc((double)sy_);
        if (first_ref) ys[1] += (double)uold[i] * (double)sy_;
      }
      bsum<2>(ys, wp, rph);
      mark(PH_YGATHER);
      ++ep;
      {
        uint64_t* s = slot(ep);
        if (q == 0 && tid == 0) {
          uint64_t* r = rec(s, c, 0);
          xw_store2(r, ep, dlo(ys[0]), dhi(ys[0]));
          if (FULL) {
            xw_store2(r + 2, ep, dlo(ys[1]), dhi(ys[1]));
            xw_store(r + 4, ep, first_ref ? (uint32_t)misc[MS_NUOC] : 0u);
          }
        }
        double* ysum = xd;
        double* ypo = xd + 2 * a.NC;
        uint32_t* ynu = xu + 5 * a.NC;
        for (int cc = tid; cc < a.NC; cc += kThreads) {
          if (FULL) {
            uint32_t p[5];
            xw_wait_n<5>(rec(s, cc, 0), 1, 5, ep, p, ab, a.budget, a.abort_word);
            ysum[cc] = u2d(p[0], p[1]);
            ypo[cc] = u2d(p[2], p[3]);
            ynu[cc] = p[4];
          } else {
            const uint64_t* r = rec(s, cc, 0);
            uint64_t v0, v1;
            xw_load2(r, v0, v1);
            ysum[cc] = u2d(take(v0, r), take(v1, r + 1));
          }
        }
        ab = __syncthreads_or(ab);
      }
      double sy_all = 0.0;
      for (int cc = 0; cc < a.NC; ++cc) sy_all += xd[cc];
      if (first_ref && tid == 0) {
        double po = 0.0, nuo = 0.0;
        for (int cc = 0; cc < a.NC; ++cc) {
          po += xd[2 * a.NC + cc];
          nuo += (double)xu[5 * a.NC + cc];
        }
        misc[MS_POT] = po;
        misc[MS_NUOT] = nuo;  // (read after later barriers)
      }
      const double thr_u = st_thr(sy_all, m);
      // u over the cluster's rows, and the ordered list of its nonzero rows
      nlist = 0;
      for (int base = 0; base < TRp; base += kThreads) {
        const int i = base + tid;
        const float uu = i < TR ? tern(yfull[i], thr_u) : 0.f;
        if (i < TRp) uval[i] = uu;
        const unsigned bal = __ballot_sync(0xffffffffu, uu != 0.f);
        if (lane == 0) wcnt[wid] = __popc(bal);
        __syncthreads();
        int off = nlist, tot = nlist;
        for (int w2 = 0; w2 < kWarps; ++w2) {
          const int cw = wcnt[w2];
          if (w2 < wid) off += cw;
          tot += cw;
        }
        if (uu != 0.f) rlist[off + __popc(bal & ((1u << lane) - 1u))] = uu > 0.f ? i : ~i;
        nlist = tot;
        __syncthreads();
      }
      const int nnz_c = nlist;
      if (traced && q == 0) pack_planes_or(uval, TR, r0, tb + 2 * Wn + it * 2 * (Wm + Wn), Wm);
      mark(PH_YXCHG);

      // ---- z = R^T u over the cluster's rows, my columns ----
      if (rgz < RGz) {
        float4 za = make_float4(0.f, 0.f, 0.f, 0.f), zb = za;
        int t2 = rgz;
        for (; t2 + 3 * RGz < nnz_c; t2 += 4 * RGz) {
          const int e0 = rlist[t2], e1 = rlist[t2 + RGz], e2 = rlist[t2 + 2 * RGz],
                    e3 = rlist[t2 + 3 * RGz];
          const float4 x0 = ld4(e0 >= 0 ? e0 : ~e0, qz);
          const float4 x1 = ld4(e1 >= 0 ? e1 : ~e1, qz);
          const float4 x2 = ld4(e2 >= 0 ? e2 : ~e2, qz);
          const float4 x3 = ld4(e3 >= 0 ? e3 : ~e3, qz);
          const float s0 = e0 >= 0 ? 1.f : -1.f, s1 = e1 >= 0 ? 1.f : -1.f;
          const float s2 = e2 >= 0 ? 1.f : -1.f, s3 = e3 >= 0 ? 1.f : -1.f;
          za.x = fmaf(s0, x0.x, za.x);
          za.y = fmaf(s0, x0.y, za.y);
          za.z = fmaf(s0, x0.z, za.z);
          za.w = fmaf(s0, x0.w, za.w);
          zb.x = fmaf(s1, x1.x, zb.x);
          zb.y = fmaf(s1, x1.y, zb.y);
          zb.z = fmaf(s1, x1.z, zb.z);
          zb.w = fmaf(s1, x1.w, zb.w);
          za.x = fmaf(s2, x2.x, za.x);
          za.y = fmaf(s2, x2.y, za.y);
          za.z = fmaf(s2, x2.z, za.z);
          za.w = fmaf(s2, x2.w, za.w);
          zb.x = fmaf(s3, x3.x, zb.x);
          zb.y = fmaf(s3, x3.y, zb.y);
          zb.z = fmaf(s3, x3.z, zb.z);
          zb.w = fmaf(s3, x3.w, zb.w);
        }
        for (; t2 + RGz < nnz_c; t2 += 2 * RGz) {
          const int e0 = rlist[t2], e1 = rlist[t2 + RGz];
          const float4 x0 = ld4(e0 >= 0 ? e0 : ~e0, qz);
          const float4 x1 = ld4(e1 >= 0 ? e1 : ~e1, qz);
          const float s0 = e0 >= 0 ? 1.f : -1.f, s1 = e1 >= 0 ? 1.f : -1.f;
          za.x = fmaf(s0, x0.x, za.x);
          za.y = fmaf(s0, x0.y, za.y);
          za.z = fmaf(s0, x0.z, za.z);
          za.w = fmaf(s0, x0.w, za.w);
          zb.x = fmaf(s1, x1.x, zb.x);
          zb.y = fmaf(s1, x1.y, zb.y);
          zb.z = fmaf(s1, x1.z, zb.z);
          zb.w = fmaf(s1, x1.w, zb.w);
        }
        if (t2 < nnz_c) {
          const int e0 = rlist[t2];
          const float4 x0 = ld4(e0 >= 0 ? e0 : ~e0, qz);
          const float s0 = e0 >= 0 ? 1.f : -1.f;
          za.x = fmaf(s0, x0.x, za.x);
          za.y = fmaf(s0, x0.y, za.y);
          za.z = fmaf(s0, x0.z, za.z);
          za.w = fmaf(s0, x0.w, za.w);
        }
        za.x += zb.x;
        za.y += zb.y;
        za.z += zb.z;
        za.w += zb.w;
        *(float4*)(zred + (size_t)rgz * TCp + 4 * qz) = za;
      }
      __syncthreads();
      mark(PH_ZPASS);
      ++ep;
      {
        uint64_t* s = slot(ep);
        uint64_t* mine = rec(s, c, q);
        for (int j = 2 * tid; j < TC; j += 2 * kThreads) {
          float z0 = 0.f, z1 = 0.f;
          for (int g = 0; g < RGz; ++g) {
            z0 += zred[(size_t)g * TCp + j];
            z1 += zred[(size_t)g * TCp + j + 1];
          }
          xw_store2(mine + j, ep, f2u(z0), f2u(j + 1 < TC ? z1 : 0.f));
        }
        if (tid == 0) xw_store(mine + TCp, ep, (uint32_t)nnz_c);
        const long long cstride = (long long)CS * a.recw;
        double zz[1] = {0.0};
        for (int j = tid; j < TC; j += kThreads) {
          float z = 0.f;
          for (int cc0 = 0; cc0 < a.NC; cc0 += 16) {
            uint32_t pl[16];
            const int cnt = min(16, a.NC - cc0);
            xw_wait_n<16>(rec(s, cc0, q) + j, cstride, cnt, ep, pl, ab, a.budget, a.abort_word);
#pragma unroll
            for (int t3 = 0; t3 < 16; ++t3)
              if (t3 < cnt) z += u2f(pl[t3]);
          }
          zown[j] = z;
          zz[0] += st_acc(naive ? (double)wcol[j] * (double)z : (double)z);
        }
        for (int cc = tid; cc < a.NC; cc += kThreads) {
          const uint64_t* r = rec(s, cc, q) + TCp;
          nnzu[cc] = (int)take(xw_load(r), r);
        }
        ab = __syncthreads_or(ab);
        // the statistic over my columns, pushed to every CTA of the cluster
        // (with, in a refinement step's first round, my part of v_o^T W v_o)
        bsum<1>(zz, wp, rph);
        if (tid < CS) {
          double* dst = cl.map_shared_rank(zs, tid);
          dst[q] = zz[0];
          if (first_ref) dst[3 * CS + q] = misc[MS_VWOQ];
        }
      }
      mark(PH_ZXCHG);
      cl.sync();
      {
        double Sz = 0.0;
        for (int qq = 0; qq < CS; ++qq) Sz += zs[qq];
        const double thr_v = st_thr(Sz, n);
        for (int j = tid; j < TCp; j += kThreads) {
          float vv = 0.f;
          if (j < TC)
            vv = naive ? tern_d((double)wcol[j] * (double)zown[j], thr_v) : tern(zown[j], thr_v);
          vval[j] = vv;
          vw[j] = vv * wcol[j];
        }
      }
      nu_total = 0;
      for (int cc = 0; cc < a.NC; ++cc) nu_total += nnzu[cc];
      __syncthreads();
      if (traced) pack_planes(vval, TC, c0, tb + 2 * Wn + it * 2 * (Wm + Wn) + 2 * Wm, Wn);
      mark(PH_ZSYNC);
    }
    if (stop) break;

    // ---- scale, gain, safeguard: sums over the nonzero v_j of the cluster ----
    {
      double pv[2] = {0.0, 0.0};
      for (int j = tid; j < TC; j += kThreads) {
        if (vval[j] != 0.f) {
          const double wv = (double)wcol[j];
          pv[0] += wv * fabs((double)zown[j]);
          pv[1] += wv;
        }
      }
      bsum<2>(pv, wp, rph);
      if (tid < CS) {
        double* dst = cl.map_shared_rank(zs, tid);
        dst[CS + q] = pv[0];
        dst[2 * CS + q] = pv[1];
      }
    }
    cl.sync();
    double P = 0.0, VW = 0.0;
    for (int qq = 0; qq < CS; ++qq) {
      P += zs[CS + qq];
      VW += zs[2 * CS + qq];
    }
    const double den = (double)nu_total * VW;
    const double gain = den > 0.0 ? P * P / den : 0.0;
    // a refinement step's other candidate: the old pattern, its scale
    // re-solved on the current residual
    double g_old = -1.0, d_old = 0.0;
    if (sweep) {
      double vwo = 0.0;
      for (int qq = 0; qq < CS; ++qq) vwo += zs[3 * CS + qq];
      const double deno = misc[MS_NUOT] * vwo, po = misc[MS_POT];
      g_old = deno > 0.0 ? po * po / deno : 0.0;
      d_old = deno > 0.0 ? po / deno : 0.0;
    }
    const double g_best = gain > g_old ? gain : g_old;
    const bool fb = g_best < misc[MS_M];
    const bool keep_old = sweep && !fb && !(gain > g_old);
    float d;
    if (fb) {
      d = (float)misc[MS_MVAL];
      const int ip = (int)misc[MS_MI], jp = (int)misc[MS_MJ];
      for (int i = tid; i < TRp; i += kThreads) uval[i] = (r0 + i == ip && i < TR) ? 1.f : 0.f;
      for (int j = tid; j < TCp; j += kThreads) vval[j] = (c0 + j == jp && j < TC) ? 1.f : 0.f;
      nlist = (ip >= r0 && ip < r1) ? 1 : 0;
      if (tid == 0 && nlist) rlist[0] = ip - r0;
      if (!sweep) ++n_fb;
    } else if (keep_old) {
      d = (float)d_old;
      for (int i = tid; i < TRp; i += kThreads) uval[i] = uold[i];
      for (int j = tid; j < TCp; j += kThreads) vval[j] = vold[j];
    } else {
      d = den > 0.0 ? (float)(P / den) : 0.f;
    }
    __syncthreads();
    if (keep_old) nlist = compact(uval);
    if (traced && blockIdx.x == 0 && tid == 0)
      a.trace_flags[tpos] = (fb ? 1 : 0) | (keep_old ? 2 : 0);
    if (traced) ++tpos;

    // ---- emit (a refinement step replaces component comp) ----
    if (q == 0) {
      if (sweep)
        pack_planes_replace(uval, TR, r0, a.pB + (size_t)comp * 2 * Wm, Wm);
      else
        pack_planes_or(uval, TR, r0, a.pB + (size_t)comp * 2 * Wm, Wm);
    }
    pack_planes(vval, TC, c0, a.pC + (size_t)comp * 2 * Wn, Wn);
    if (blockIdx.x == 0 && tid == 0) a.D[comp] = d;
    if (a.dpriv && tid == 0) a.dpriv[(size_t)blockIdx.x * a.k + comp] = d;
    mark(PH_SCALE);

    // ---- deflate R <- R - d u v^T over the rows with u_i != 0, refresh
    // their statistics ----
    for (int e = wid; e < nlist; e += 2 * kWarps) {
      const int xa = rlist[e];
      const int ia = xa >= 0 ? xa : ~xa;
      const float sa = xa >= 0 ? d : -d;
      int ib = -1;
      float sb = 0.f;
      if (e + kWarps < nlist) {
        const int xb = rlist[e + kWarps];
        ib = xb >= 0 ? xb : ~xb;
        sb = xb >= 0 ? d : -d;
      }
      rows_update(ia, sa, ib, sb);
    }
    __syncthreads();
    mark(PH_DEFLATE);
    // the statistics the next step starts from: a greedy step needs the next
    // start row; the last greedy step and the last step of a sweep need the
    // residual norm for the energy record; other refinement steps need
    // nothing here (the next one refreshes them after its add-back)
    const bool next_greedy = t + 1 < a.k;
    const bool ends_pass = t == a.k - 1 || (sweep && comp == a.k - 1);
    if (next_greedy || ends_pass) stats_exchange(0, next_greedy);
    mark(PH_STATS);
  }

  // final energy entry, counters, status
  __syncthreads();
  if (blockIdx.x == 0 && tid == 0) {
    if (!stop && a.k > 0) record_energy(nsteps - 1);
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



// Explicit instantiations live in seq_inst_*.cu; launching code sees these
// declarations only.
#define EXTERND_SEQ_KERNELS(HYB, FULL, X)                                   \
  X template __global__ void seq_als_kernel<1, HYB, FULL>(const SeqArgs);   \
  X template __global__ void seq_als_kernel<2, HYB, FULL>(const SeqArgs);   \
  X template __global__ void seq_als_kernel<3, HYB, FULL>(const SeqArgs);   \
  X template __global__ void seq_als_kernel<4, HYB, FULL>(const SeqArgs);   \
  X template __global__ void seq_als_kernel<5, HYB, FULL>(const SeqArgs);   \
  X template __global__ void seq_als_kernel<6, HYB, FULL>(const SeqArgs);   \
  X template __global__ void seq_als_kernel<8, HYB, FULL>(const SeqArgs);

}  // namespace externd
