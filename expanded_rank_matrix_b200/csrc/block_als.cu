// Block-ALS for ExTernD (paper Sec. 2.4 with the decorrelated least-squares
// target of Eq. 3, as summarised in the Pith review's referee report; the
// romaanj.github.io review's "Method" calls it the batched block-ALS GPU
// algorithm).  Per block of bb <= 64 components:
//   rows  = the bb largest-energy residual rows (energy desc, index asc)
//   V     = T_col(R[rows, :]^T)
//   repeat iters times:
//     U = T_col(R W V (V^T W V + eps I)^-1)
//     V = T_col(((U^T U + eps I)^-1 U^T R)^T)
//   D = ((U^T U) o (V^T W V) + eps I)^-1 r,  r_l = u_l^T R W v_l   (active set)
//   R <- R - sum_l d_l u_l v_l^T as bb ordered fp32 add/subtracts per entry
// with eps = 1e-6 trace(G) / bb (1 when the trace is 0), T_col thresholding
// each column with its own rms.  Ternary columns are held as 64-bit masks per
// row (bit l = component l): Um/Us over the m rows, Vm/Vs over the n columns.
//
// Every reduction runs in a fixed order (split-K partials are summed in
// split order), so results are bit-reproducible.

#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstdlib>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace externd {
namespace blk {

typedef unsigned long long u64;
constexpr int kMaxB = 64;

__device__ __forceinline__ double warp_sum(double x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Deterministic sum over a block of `nth` threads (multiple of 32).
__device__ double block_sum_d(double x, double* sh) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  x = warp_sum(x);
  __syncthreads();
  if (lane == 0) sh[wid] = x;
  __syncthreads();
  double s = 0.0;
  for (int i = 0; i < nw; ++i) s += sh[i];
  __syncthreads();
  return s;
}

// ---- setup: R = A, row-energy partials per column chunk, validity -----------
// Row energies are kept as partials over column chunks of kChunk columns,
// rhop[chunk][row], summed in chunk order where a full energy is needed.
constexpr int kChunk = 1024;
__global__ void setup_kernel(const float* __restrict__ A, float* __restrict__ R, int m, int n,
                             const float* __restrict__ w, double* __restrict__ rhop,
                             int* __restrict__ bad) {
  const int lane = threadIdx.x & 31;
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int ch = blockIdx.y;
  if (row >= m) return;
  const int j0 = ch * kChunk, j1 = min(n, j0 + kChunk);
  double s = 0.0;
  int b = 0;
  for (int j = j0 + lane; j < j1; j += 32) {
    const float x = A[(size_t)row * n + j];
    R[(size_t)row * n + j] = x;
    if (!isfinite(x)) b = 1;
    const double wj = w ? (double)w[j] : 1.0;
    s += wj * (double)x * (double)x;
  }
  s = warp_sum(s);
  b = __any_sync(0xffffffffu, b);
  if (lane == 0) {
    rhop[(size_t)ch * m + row] = s;
    if (b) atomicExch(bad, 1);
  }
}

__global__ void check_w_kernel(const float* __restrict__ w, int n, int* __restrict__ bad) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j < n) {
    const float x = w[j];
    if (!(x > 0.f) || !isfinite(x)) atomicExch(bad, 1);
  }
}

// ---- top-bb rows: radix select on the fp64 energy bits, then rank ----------
// One CTA of 1024 threads.  Also sums the energies in a fixed order (R2) and,
// on the first block, records it as E0.
__global__ void __launch_bounds__(1024) select_rows_kernel(const double* __restrict__ rhop,
                                                           int nch, double* __restrict__ rho,
                                                           int m, int bb, int* __restrict__ rows,
                                                           double* __restrict__ scal,
                                                           int first) {
  __shared__ unsigned int hist[256];
  __shared__ double sh[32];
  __shared__ unsigned long long s_prefix, s_mask;
  __shared__ int s_remaining;
  __shared__ int cnt_gt[1024], cnt_eq[1024];
  __shared__ int cand[kMaxB];
  const int tid = threadIdx.x;
  double part = 0.0;
  for (int i = tid; i < m; i += 1024) {
    double r = 0.0;
    for (int c = 0; c < nch; ++c) r += rhop[(size_t)c * m + i];
    rho[i] = r;
    part += r;
  }
  const double R2 = block_sum_d(part, sh);
  if (tid == 0) {
    scal[0] = R2;
    if (first) scal[1] = R2;
    s_prefix = 0ull;
    s_mask = 0ull;
    s_remaining = bb;
  }
  __syncthreads();
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int t = tid; t < 256; t += 1024) hist[t] = 0u;
    __syncthreads();
    const u64 pref = s_prefix, msk = s_mask;
    for (int i = tid; i < m; i += 1024) {
      const u64 key = (u64)__double_as_longlong(rho[i]);
      if ((key & msk) == pref) atomicAdd(&hist[(key >> shift) & 0xffu], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      int rem = s_remaining;
      int d = 255;
      for (; d > 0; --d) {
        if ((int)hist[d] >= rem) break;
        rem -= (int)hist[d];
      }
      s_remaining = rem;
      s_prefix = pref | ((u64)d << shift);
      s_mask = msk | (0xffull << shift);
    }
    __syncthreads();
  }
  const u64 kstar = s_prefix;
  const int need_eq = s_remaining;  // rows equal to kstar to take, lowest index first
  // contiguous index ranges per thread keep the scan in index order
  const int per = (m + 1023) / 1024;
  const int i0 = min(m, tid * per), i1 = min(m, i0 + per);
  int g = 0, e = 0;
  for (int i = i0; i < i1; ++i) {
    const u64 key = (u64)__double_as_longlong(rho[i]);
    g += key > kstar;
    e += key == kstar;
  }
  cnt_gt[tid] = g;
  cnt_eq[tid] = e;
  __syncthreads();
  if (tid == 0) {  // exclusive scans (1024 entries, cheap)
    int ag = 0, ae = 0;
    for (int t = 0; t < 1024; ++t) {
      const int tg = cnt_gt[t], te = cnt_eq[t];
      cnt_gt[t] = ag;
      cnt_eq[t] = ae;
      ag += tg;
      ae += te;
    }
  }
  __syncthreads();
  int pg = cnt_gt[tid], pe = cnt_eq[tid];
  const int ngt = bb - need_eq;  // rows strictly above kstar
  for (int i = i0; i < i1; ++i) {
    const u64 key = (u64)__double_as_longlong(rho[i]);
    if (key > kstar) {
      if (pg < kMaxB) cand[pg] = i;
      ++pg;
    } else if (key == kstar) {
      if (pe < need_eq && ngt + pe < kMaxB) cand[ngt + pe] = i;
      ++pe;
    }
  }
  __syncthreads();
  // order the bb candidates by (energy desc, index asc)
  if (tid < bb) {
    const int me = cand[tid];
    const double rm = rho[me];
    int rank = 0;
    for (int t = 0; t < bb; ++t) {
      const int o = cand[t];
      const double ro = rho[o];
      rank += (ro > rm) || (ro == rm && o < me);
    }
    rows[rank] = me;
  }
}

// ---- starting V: column l = T_tau(R[rows[l], :]) ----------------------------
__global__ void vinit_kernel(const float* __restrict__ R, int n, const int* __restrict__ rows,
                             double tau, u64* __restrict__ Vm, u64* __restrict__ Vs) {
  __shared__ double sh[32];
  const int l = blockIdx.x;
  const float* row = R + (size_t)rows[l] * n;
  double s = 0.0;
  for (int j = threadIdx.x; j < n; j += blockDim.x) s += (double)row[j] * (double)row[j];
  s = block_sum_d(s, sh);
  const double thr = tau * sqrt(s / (double)n);
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    const float x = row[j];
    if (fabs((double)x) > thr) {
      atomicOr(Vm + j, 1ull << l);
      if (x < 0.f) atomicOr(Vs + j, 1ull << l);
    }
  }
}

// ---- packed planes [bb][2][W] of per-entry 64-bit masks (warp per word) ------
__global__ void planes_kernel(const u64* __restrict__ Mk, const u64* __restrict__ Sg, int len,
                              int bb, uint32_t* __restrict__ planes, int W) {
  const int lane = threadIdx.x & 31;
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= W) return;
  const int x = t * 32 + lane;
  const u64 mk = x < len ? Mk[x] : 0ull, sg = x < len ? Sg[x] : 0ull;
  uint32_t om[2] = {0u, 0u}, os[2] = {0u, 0u};
  for (int l = 0; l < bb; ++l) {
    const uint32_t bm = __ballot_sync(0xffffffffu, (mk >> l) & 1ull);
    const uint32_t bs = __ballot_sync(0xffffffffu, (sg >> l) & 1ull);
    if (lane == (l & 31)) {
      om[l >> 5] = bm;
      os[l >> 5] = bs;
    }
  }
  for (int h = 0; h < 2; ++h) {
    const int l = lane + 32 * h;
    if (l < bb) {
      planes[(size_t)l * 2 * W + t] = om[h];
      planes[(size_t)l * 2 * W + W + t] = os[h];
    }
  }
}

// ---- Gram matrix from packed planes: G[l][l2] = sum_x w_x s_xl s_xl2 --------
// One warp per pair l <= l2.  Unweighted: exact popcounts.  Weighted: fp64
// over the common support, lanes over words, fixed-order warp tree.
__global__ void gram_kernel(const uint32_t* __restrict__ planes, int W, int bb,
                            const float* __restrict__ w, double* __restrict__ G) {
  const int lane = threadIdx.x & 31;
  const int pr = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int npairs = bb * (bb + 1) / 2;
  if (pr >= npairs) return;
  int l = 0, rem = pr;
  while (rem >= bb - l) {
    rem -= bb - l;
    ++l;
  }
  const int l2 = l + rem;
  const uint32_t* m1 = planes + (size_t)l * 2 * W;
  const uint32_t* m2 = planes + (size_t)l2 * 2 * W;
  double acc = 0.0;
  long long cnt = 0;
  for (int t = lane; t < W; t += 32) {
    const uint32_t mm = m1[t] & m2[t];
    const uint32_t x = m1[W + t] ^ m2[W + t];
    if (!w) {
      cnt += (long long)__popc(mm & ~x) - (long long)__popc(mm & x);
    } else {
      uint32_t bits = mm;
      while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1u;
        const double wj = (double)w[t * 32 + b];
        acc += ((x >> b) & 1u) ? -wj : wj;
      }
    }
  }
  if (!w) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    acc = (double)cnt;
  } else {
    acc = warp_sum(acc);
  }
  if (lane == 0) {
    G[l * bb + l2] = acc;
    G[l2 * bb + l] = acc;
  }
}

// ---- S = (G + eps I)^-1 by Gauss-Jordan on [G + eps I | I] (SPD, no pivots) --
// Dynamic shared memory: bb x 2bb doubles + bb doubles.
__global__ void __launch_bounds__(256) inv_kernel(const double* __restrict__ G, int bb,
                                                  double* __restrict__ S) {
  extern __shared__ double ash[];
  const int w2 = 2 * bb;
  double* Am = ash;
  __shared__ double eps;
  if (threadIdx.x == 0) {
    double tr = 0.0;
    for (int l = 0; l < bb; ++l) tr += G[l * bb + l];
    eps = tr > 0.0 ? 1e-6 * tr / (double)bb : 1.0;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < bb * w2; e += blockDim.x) {
    const int i = e / w2, j = e - i * w2;
    Am[e] = j < bb ? G[i * bb + j] + (i == j ? eps : 0.0) : (j - bb == i ? 1.0 : 0.0);
  }
  __syncthreads();
  // thread (row r = tid / 4, column phase cq = tid % 4) -- blockDim.x == 256
  const int r = threadIdx.x >> 2, cq = threadIdx.x & 3;
  for (int k = 0; k < bb; ++k) {
    const double inv = 1.0 / Am[k * w2 + k];
    const double f = (r < bb && r != k) ? Am[r * w2 + k] : 0.0;
    __syncthreads();
    if (r == k)
      for (int j = cq; j < w2; j += 4) Am[k * w2 + j] *= inv;
    __syncthreads();
    if (r < bb && r != k)
      for (int j = cq; j < w2; j += 4) Am[r * w2 + j] -= f * Am[k * w2 + j];
    __syncthreads();
  }
  for (int e = threadIdx.x; e < bb * bb; e += blockDim.x) {
    const int i = e / bb, j = e - i * bb;
    S[e] = Am[i * w2 + bb + j];
  }
}

// ---- contractions on CUDA cores ---------------------------------------------
// P partials: Pp[split][i][l] = sum_{j in split} R_ij w_j s_jl   (64 x 64 tile)
constexpr int kTile = 64, kKc = 32;
__global__ void __launch_bounds__(256) rv_kernel(const float* __restrict__ R, int m, int n,
                                                 const u64* __restrict__ Vm,
                                                 const u64* __restrict__ Vs,
                                                 const float* __restrict__ w, int bb, int klen,
                                                 float* __restrict__ Pp) {
  __shared__ __align__(16) float As[kKc][kTile + 4];
  __shared__ __align__(16) float Bs[kKc][kTile];
  const int i0 = blockIdx.x * kTile, split = blockIdx.y;
  const int j0 = split * klen, j1 = min(n, j0 + klen);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int jc = j0; jc < j1; jc += kKc) {
    __syncthreads();
    for (int e = threadIdx.x; e < kTile * kKc; e += 256) {
      const int r = e / kKc, kk = e - r * kKc;
      const int i = i0 + r, j = jc + kk;
      As[kk][r] = (i < m && j < j1) ? R[(size_t)i * n + j] : 0.f;
    }
    for (int e = threadIdx.x; e < kKc * kTile; e += 256) {
      const int kk = e / kTile, l = e - kk * kTile;
      const int j = jc + kk;
      float v = 0.f;
      if (j < j1 && l < bb) {
        const u64 mm = Vm[j];
        if ((mm >> l) & 1ull) v = (((Vs[j] >> l) & 1ull) ? -1.f : 1.f) * (w ? w[j] : 1.f);
      }
      Bs[kk][l] = v;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kKc; ++kk) {
      const float4 a = *(const float4*)&As[kk][ty * 4];
      const float4 b = *(const float4*)&Bs[kk][tx * 4];
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(av[r], bv[c], acc[r][c]);
    }
  }
  float* out = Pp + (size_t)split * m * bb;
  for (int r = 0; r < 4; ++r) {
    const int i = i0 + ty * 4 + r;
    if (i >= m) continue;
    for (int c = 0; c < 4; ++c) {
      const int l = tx * 4 + c;
      if (l < bb) out[(size_t)i * bb + l] = acc[r][c];
    }
  }
}

// Q partials: Qp[split][j][l] = sum_{i in split} R_ij s_il   (64 x 64 tile)
__global__ void __launch_bounds__(256) rtu_kernel(const float* __restrict__ R, int m, int n,
                                                  const u64* __restrict__ Um,
                                                  const u64* __restrict__ Us, int bb, int klen,
                                                  float* __restrict__ Qp) {
  __shared__ __align__(16) float As[kKc][kTile];
  __shared__ __align__(16) float Bs[kKc][kTile];
  const int j0c = blockIdx.x * kTile, split = blockIdx.y;
  const int r0 = split * klen, r1 = min(m, r0 + klen);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int ic = r0; ic < r1; ic += kKc) {
    __syncthreads();
    for (int e = threadIdx.x; e < kKc * kTile; e += 256) {
      const int kk = e / kTile, c = e - kk * kTile;
      const int i = ic + kk, j = j0c + c;
      As[kk][c] = (i < r1 && j < n) ? R[(size_t)i * n + j] : 0.f;
    }
    for (int e = threadIdx.x; e < kKc * kTile; e += 256) {
      const int kk = e / kTile, l = e - kk * kTile;
      const int i = ic + kk;
      float v = 0.f;
      if (i < r1 && l < bb) {
        const u64 mm = Um[i];
        if ((mm >> l) & 1ull) v = ((Us[i] >> l) & 1ull) ? -1.f : 1.f;
      }
      Bs[kk][l] = v;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kKc; ++kk) {
      const float4 a = *(const float4*)&As[kk][ty * 4];
      const float4 b = *(const float4*)&Bs[kk][tx * 4];
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(av[r], bv[c], acc[r][c]);
    }
  }
  float* out = Qp + (size_t)split * n * bb;
  for (int r = 0; r < 4; ++r) {
    const int j = j0c + ty * 4 + r;
    if (j >= n) continue;
    for (int c = 0; c < 4; ++c) {
      const int l = tx * 4 + c;
      if (l < bb) out[(size_t)j * bb + l] = acc[r][c];
    }
  }
}

// ---- targets: T[x][l] = sum_l2 (sum_s Xp[s][x][l2]) S[l2][l] (fp64), and
// per-CTA column sums of squares.  16 rows per CTA, 4 per step.
constexpr int kTgtRows = 16;
__global__ void __launch_bounds__(256) target_kernel(const float* __restrict__ Xp, int splits,
                                                     int rows, int bb, const double* __restrict__ S,
                                                     double* __restrict__ T,
                                                     double* __restrict__ colss) {
  __shared__ double Ss[kMaxB * kMaxB];
  __shared__ double xr[4][kMaxB];
  __shared__ double part[4][kMaxB];
  for (int p = threadIdx.x; p < bb * bb; p += 256) Ss[p] = S[p];
  const int l = threadIdx.x & 63, rr = threadIdx.x >> 6;
  double cs = 0.0;
  const int x0 = blockIdx.x * kTgtRows;
  for (int base = x0; base < min(rows, x0 + kTgtRows); base += 4) {
    __syncthreads();
    {
      const int x = base + rr;
      if (l < bb) {
        double s = 0.0;
        if (x < rows)
          for (int sp = 0; sp < splits; ++sp) s += (double)Xp[((size_t)sp * rows + x) * bb + l];
        xr[rr][l] = s;
      }
    }
    __syncthreads();
    const int x = base + rr;
    if (x < rows && l < bb) {
      double t = 0.0;
      for (int l2 = 0; l2 < bb; ++l2) t += xr[rr][l2] * Ss[l2 * bb + l];
      T[(size_t)x * bb + l] = t;
      cs += t * t;
    }
  }
  part[rr][l] = cs;
  __syncthreads();
  if (rr == 0 && l < bb)
    colss[(size_t)blockIdx.x * bb + l] = ((part[0][l] + part[1][l]) + part[2][l]) + part[3][l];
}

// ---- thresholds per column; 64-bit masks per entry and packed planes -------
// One warp per 32 entries (one plane word).
__global__ void tern_kernel(const double* __restrict__ T, int rows, int bb,
                            const double* __restrict__ colss, int nparts, double tau,
                            u64* __restrict__ Mk, u64* __restrict__ Sg,
                            uint32_t* __restrict__ planes, int W) {
  __shared__ double thr[kMaxB];
  if (threadIdx.x < bb) {
    double s = 0.0;
    for (int b = 0; b < nparts; ++b) s += colss[(size_t)b * bb + threadIdx.x];
    thr[threadIdx.x] = tau * sqrt(s / (double)rows);
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= W) return;
  const int x = t * 32 + lane;
  u64 mk = 0ull, sg = 0ull;
  if (x < rows)
    for (int l = 0; l < bb; ++l) {
      const double v = T[(size_t)x * bb + l];
      if (fabs(v) > thr[l]) {
        mk |= 1ull << l;
        if (v < 0.0) sg |= 1ull << l;
      }
    }
  if (x < rows) {
    Mk[x] = mk;
    Sg[x] = sg;
  }
  uint32_t om[2] = {0u, 0u}, os[2] = {0u, 0u};
  for (int l = 0; l < bb; ++l) {
    const uint32_t bm = __ballot_sync(0xffffffffu, (mk >> l) & 1ull);
    const uint32_t bs = __ballot_sync(0xffffffffu, (sg >> l) & 1ull);
    if (lane == (l & 31)) {
      om[l >> 5] = bm;
      os[l >> 5] = bs;
    }
  }
  for (int h = 0; h < 2; ++h) {
    const int l = lane + 32 * h;
    if (l < bb) {
      planes[(size_t)l * 2 * W + t] = om[h];
      planes[(size_t)l * 2 * W + W + t] = os[h];
    }
  }
}

// ---- r_l = u_l^T R W v_l = sum_j (sum_s Qp[s][j][l]) w_j s_jl, per-CTA partials
__global__ void __launch_bounds__(256) rpart_kernel(const float* __restrict__ Qp, int splits, int n,
                                                    int bb, const u64* __restrict__ Vm,
                                                    const u64* __restrict__ Vs,
                                                    const float* __restrict__ w,
                                                    double* __restrict__ rp) {
  __shared__ double part[4][kMaxB];
  const int l = threadIdx.x & 63, rr = threadIdx.x >> 6;
  const int x0 = blockIdx.x * kTgtRows;
  double acc = 0.0;
  if (l < bb)
    for (int j = x0 + rr; j < min(n, x0 + kTgtRows); j += 4) {
      const u64 mm = Vm[j];
      if (!((mm >> l) & 1ull)) continue;
      double q = 0.0;
      for (int sp = 0; sp < splits; ++sp) q += (double)Qp[((size_t)sp * n + j) * bb + l];
      const double wj = w ? (double)w[j] : 1.0;
      acc += (((Vs[j] >> l) & 1ull) ? -q : q) * wj;
    }
  part[rr][l] = acc;
  __syncthreads();
  if (rr == 0 && l < bb)
    rp[(size_t)blockIdx.x * bb + l] = ((part[0][l] + part[1][l]) + part[2][l]) + part[3][l];
}

// ---- joint scales, closed-form energies ---------------------------------------
// r_l = sum_j (sum_s Qp[s][j][l]) w_j s_jl; G = GU o GV; active-set solve.
__global__ void __launch_bounds__(256) dsolve_kernel(const double* __restrict__ GU,
                                                     const double* __restrict__ GV,
                                                     const double* __restrict__ rp, int rparts,
                                                     int bb, const double* __restrict__ scal,
                                                     int c0, float* __restrict__ D,
                                                     double* __restrict__ energy,
                                                     float* __restrict__ dblk) {
  extern __shared__ double dsh[];
  double* G = dsh;                        // bb x bb, (U^T U) o (V^T W V)
  double* Am = dsh + (size_t)bb * bb;      // active system, A x (A+1)
  __shared__ double r[kMaxB], fcol[kMaxB];
  __shared__ float dl[kMaxB];
  __shared__ int act[kMaxB];
  __shared__ int na;
  __shared__ double eps;
  if (threadIdx.x < bb) {
    double s = 0.0;
    for (int b = 0; b < rparts; ++b) s += rp[(size_t)b * bb + threadIdx.x];
    r[threadIdx.x] = s;
    dl[threadIdx.x] = 0.f;
  }
  for (int p = threadIdx.x; p < bb * bb; p += blockDim.x) G[p] = GU[p] * GV[p];
  __syncthreads();
  if (threadIdx.x == 0) {
    double tr = 0.0;
    for (int l = 0; l < bb; ++l) tr += G[l * bb + l];
    eps = tr > 0.0 ? 1e-6 * tr / (double)bb : 1.0;
    int c = 0;
    for (int l = 0; l < bb; ++l)
      if (GU[l * bb + l] > 0.0 && GV[l * bb + l] > 0.0) act[c++] = l;
    na = c;
  }
  __syncthreads();
  const int A = na, w2 = A + 1;
  for (int e = threadIdx.x; e < A * w2; e += blockDim.x) {
    const int a = e / w2, c = e - a * w2;
    Am[e] = c < A ? G[act[a] * bb + act[c]] + (a == c ? eps : 0.0) : r[act[a]];
  }
  __syncthreads();
  {
    const int rr = threadIdx.x >> 2, cq = threadIdx.x & 3;
    for (int k = 0; k < A; ++k) {
      const double inv = 1.0 / Am[k * w2 + k];
      const double f = (rr < A && rr != k) ? Am[rr * w2 + k] : 0.0;
      __syncthreads();
      if (rr == k)
        for (int j = cq; j < w2; j += 4) Am[k * w2 + j] *= inv;
      __syncthreads();
      if (rr < A && rr != k)
        for (int j = cq; j < w2; j += 4) Am[rr * w2 + j] -= f * Am[k * w2 + j];
      __syncthreads();
    }
  }
  for (int a = threadIdx.x; a < A; a += blockDim.x) dl[act[a]] = (float)Am[a * w2 + A];
  __syncthreads();
  // energy after component c0 + l: |R|^2 - 2 sum_{a<=l} d_a r_a + sum_{a,c<=l} d_a d_c G_ac,
  // accumulated over l: inc_l = -2 d_l r_l + d_l^2 G_ll + 2 d_l sum_{a<l} d_a G_al
  if (threadIdx.x < bb) {
    const int l = threadIdx.x;
    double h = 0.0;
    for (int a = 0; a < l; ++a) h += (double)dl[a] * G[a * bb + l];
    const double dd = (double)dl[l];
    fcol[l] = -2.0 * dd * r[l] + dd * dd * G[l * bb + l] + 2.0 * dd * h;
    D[c0 + l] = dl[l];
    dblk[l] = dl[l];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const double R2 = scal[0], E0 = scal[1];
    double e = R2;
    for (int l = 0; l < bb; ++l) {
      e += fcol[l];
      energy[c0 + l] = E0 > 0.0 ? 1.0 - e / E0 : 1.0;
    }
  }
}

// ---- ordered block deflation + next block's row-energy partials ------------
// CTA = 8 warps = 8 rows x one column chunk; V masks of the chunk in shared
// memory; each lane advances 4 entries' ordered add/subtract chains together.
__global__ void __launch_bounds__(256) deflate_kernel(float* __restrict__ R, int m, int n,
                                                      const u64* __restrict__ Um,
                                                      const u64* __restrict__ Us,
                                                      const u64* __restrict__ Vm,
                                                      const u64* __restrict__ Vs,
                                                      const float* __restrict__ dblk,
                                                      const float* __restrict__ w,
                                                      double* __restrict__ rhop) {
  __shared__ u64 vm[kChunk], vs[kChunk];
  __shared__ float d[kMaxB];
  const int ch = blockIdx.y, j0 = ch * kChunk, j1 = min(n, j0 + kChunk);
  for (int j = threadIdx.x; j < j1 - j0; j += blockDim.x) {
    vm[j] = Vm[j0 + j];
    vs[j] = Vs[j0 + j];
  }
  if (threadIdx.x < kMaxB) d[threadIdx.x] = dblk[threadIdx.x];
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int i = blockIdx.x * 8 + wid;
  if (i >= m) return;
  const u64 um = Um[i];
  if (um == 0ull) return;  // untouched row: R and its energy partials stay
  const u64 us = Us[i];
  // signed scales of the row's components, in ascending component order
  // (per-warp lists in shared memory; every lane computes the same list)
  __shared__ int ls_s[8][kMaxB];
  __shared__ float du_s[8][kMaxB];
  int* ls = ls_s[wid];
  float* dus = du_s[wid];
  int nl = 0;
  for (u64 bits = um; bits; bits &= bits - 1ull) {
    const int l = __ffsll((long long)bits) - 1;
    if (lane == 0) {
      ls[nl] = l;
      dus[nl] = ((us >> l) & 1ull) ? -d[l] : d[l];
    }
    ++nl;
  }
  __syncwarp();
  float* row = R + (size_t)i * n;
  double s = 0.0;
  for (int jb = lane; jb < j1 - j0; jb += 128) {
    float x[4];
    u64 m4[4], s4[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = jb + 32 * e;
      const bool ok = j < j1 - j0;
      x[e] = ok ? row[j0 + j] : 0.f;
      m4[e] = ok ? vm[j] : 0ull;
      s4[e] = ok ? vs[j] : 0ull;
    }
    for (int t = 0; t < nl; ++t) {  // same trip count on every lane: no divergence
      const int l = ls[t];
      const float du = dus[t];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float sd = ((s4[e] >> l) & 1ull) ? -du : du;
        const float y = __fsub_rn(x[e], sd);
        x[e] = ((m4[e] >> l) & 1ull) ? y : x[e];
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = jb + 32 * e;
      if (j < j1 - j0) {
        if ((um & m4[e]) != 0ull) row[j0 + j] = x[e];
        const double wj = w ? (double)w[j0 + j] : 1.0;
        s += wj * (double)x[e] * (double)x[e];
      }
    }
  }
  s = warp_sum(s);
  if (lane == 0) rhop[(size_t)ch * m + i] = s;
}

__global__ void set_status_kernel(const int* __restrict__ bad, int* __restrict__ status) {
  if (*bad) atomicCAS(status, 0, EXTERND_ERR_NONFINITE);
}

}  // namespace blk

int block_decompose(const BlockHostArgs& h, cudaStream_t st) {
  using namespace blk;
  const int m = (int)h.m, n = (int)h.n, k = (int)h.k, b = h.block;
  if (b > kMaxB) return EXTERND_ERR_INVALID_ARG;
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  // Contractions run on the tensor cores (tcgen05, 128-row tiles); setting
  // EXTERND_BLOCK_CUDA_CORES=1 selects the CUDA-core kernels (64-row tiles)
  // instead, for comparison.
  const char* cc = getenv("EXTERND_BLOCK_CUDA_CORES");
  const bool tc = !(cc && cc[0] == '1');
  const int tileR = tc ? 128 : kTile, kq = 32;
  // split-K factors so each contraction has about two CTAs per SM
  const int tiles_m = (m + tileR - 1) / tileR, tiles_n = (n + tileR - 1) / tileR;
  int splitP = std::max(1, std::min((2 * nsm + tiles_m - 1) / tiles_m, (n + kq - 1) / kq));
  int splitQ = std::max(1, std::min((2 * nsm + tiles_n - 1) / tiles_n, (m + kq - 1) / kq));
  const int klenP = ((n + splitP - 1) / splitP + kq - 1) / kq * kq;
  const int klenQ = ((m + splitQ - 1) / splitQ + kq - 1) / kq * kq;
  splitP = (n + klenP - 1) / klenP;
  splitQ = (m + klenQ - 1) / klenQ;
  const int tgtU = (m + kTgtRows - 1) / kTgtRows, tgtV = (n + kTgtRows - 1) / kTgtRows;
  const int nch = (n + kChunk - 1) / kChunk;
  const int mx = std::max(m, n);
  const int Wm = (m + 31) / 32, Wn = (n + 31) / 32;
  // workspace carve-up
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t r = off;
    off += (bytes + 255) & ~(size_t)255;
    return r;
  };
  const size_t oR = take(sizeof(float) * (size_t)m * n);
  const size_t oRho = take(sizeof(double) * m);
  const size_t oRhop = take(sizeof(double) * (size_t)nch * m);
  const size_t oRows = take(sizeof(int) * kMaxB);
  const size_t oUm = take(sizeof(u64) * m), oUs = take(sizeof(u64) * m);
  const size_t oVm = take(sizeof(u64) * n), oVs = take(sizeof(u64) * n);
  const size_t oPp = take(sizeof(float) * (size_t)splitP * m * b);
  const size_t oQp = take(sizeof(float) * (size_t)splitQ * n * b);
  const size_t oT = take(sizeof(double) * (size_t)mx * b);
  const size_t oCs = take(sizeof(double) * (size_t)std::max(tgtU, tgtV) * b);
  const size_t oRp = take(sizeof(double) * (size_t)tgtV * b);
  const size_t oSV = take(sizeof(double) * b * b), oSU = take(sizeof(double) * b * b);
  const size_t oGU = take(sizeof(double) * b * b), oGV = take(sizeof(double) * b * b);
  const size_t oScal = take(sizeof(double) * 4);
  const size_t oD = take(sizeof(float) * kMaxB);
  const size_t oBad = take(sizeof(int));
  void* ws = nullptr;
  if (cudaMallocAsync(&ws, off, st) != cudaSuccess) {
    cudaGetLastError();
    return EXTERND_ERR_OOM;
  }
  char* base = (char*)ws;
  float* R = (float*)(base + oR);
  double* rho = (double*)(base + oRho);
  double* rhop = (double*)(base + oRhop);
  int* rows = (int*)(base + oRows);
  u64 *Um = (u64*)(base + oUm), *Us = (u64*)(base + oUs);
  u64 *Vm = (u64*)(base + oVm), *Vs = (u64*)(base + oVs);
  float* Pp = (float*)(base + oPp);
  float* Qp = (float*)(base + oQp);
  double* T = (double*)(base + oT);
  double* Cs = (double*)(base + oCs);
  double* Rp = (double*)(base + oRp);
  double *SV = (double*)(base + oSV), *SU = (double*)(base + oSU);
  double *GU = (double*)(base + oGU), *GV = (double*)(base + oGV);
  double* scal = (double*)(base + oScal);
  float* dblk = (float*)(base + oD);
  int* bad = (int*)(base + oBad);
  const double tau = (double)h.tau;
  int rc = EXTERND_OK;
  auto chk = [&]() {
    if (rc == EXTERND_OK && cudaGetLastError() != cudaSuccess) rc = EXTERND_ERR_CUDA;
  };
  const size_t ism = sizeof(double) * ((size_t)b * 2 * b + b);
  const size_t dsm = sizeof(double) * ((size_t)b * b + (size_t)b * (b + 1));
  if (ism > 48 * 1024) cudaFuncSetAttribute(inv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ism);
  if (dsm > 48 * 1024)
    cudaFuncSetAttribute(dsolve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dsm);
  cudaMemsetAsync(bad, 0, sizeof(int), st);
  cudaMemsetAsync(dblk, 0, sizeof(float) * kMaxB, st);
  setup_kernel<<<dim3((m * 32 + 255) / 256, nch), 256, 0, st>>>(h.A, R, m, n, h.w, rhop, bad);
  if (h.w) check_w_kernel<<<(n + 255) / 256, 256, 0, st>>>(h.w, n, bad);
  chk();
  // trace record of a block: V0, then U_t and V_t per iteration (mask words
  // then sign words); plus the start rows
  const size_t trace_words = 2 * (size_t)n + (size_t)h.iters * 2 * ((size_t)m + n);
  const int gthreads = 256;
  for (int c0 = 0; c0 < k && rc == EXTERND_OK; c0 += b) {
    const int bb = std::min(b, k - c0);
    const int npairs = bb * (bb + 1) / 2;
    const int gblocks = (npairs * 32 + gthreads - 1) / gthreads;
    uint32_t* pB = h.packed_B + (size_t)c0 * 2 * Wm;  // planes of this block's U
    uint32_t* pC = h.packed_C + (size_t)c0 * 2 * Wn;  // planes of this block's V
    int tslot = -1;
    for (int64_t t = 0; t < h.ntrace; ++t)
      if (h.trace_block && h.trace_block[t] == c0 / b) tslot = (int)t;
    u64* tr = tslot >= 0 ? (u64*)h.trace_uv + (size_t)tslot * trace_words : nullptr;
    auto record = [&](u64* dst, const u64* mk, const u64* sg, int len) {
      cudaMemcpyAsync(dst, mk, sizeof(u64) * len, cudaMemcpyDeviceToDevice, st);
      cudaMemcpyAsync(dst + len, sg, sizeof(u64) * len, cudaMemcpyDeviceToDevice, st);
    };
    select_rows_kernel<<<1, 1024, 0, st>>>(rhop, nch, rho, m, bb, rows, scal, c0 == 0);
    cudaMemsetAsync(Vm, 0, sizeof(u64) * n, st);
    cudaMemsetAsync(Vs, 0, sizeof(u64) * n, st);
    vinit_kernel<<<bb, 256, 0, st>>>(R, n, rows, tau, Vm, Vs);
    planes_kernel<<<(Wn * 32 + 255) / 256, 256, 0, st>>>(Vm, Vs, n, bb, pC, Wn);
    if (tr) {
      cudaMemcpyAsync(h.trace_rows + (size_t)tslot * b, rows, sizeof(int) * bb,
                      cudaMemcpyDeviceToDevice, st);
      record(tr, Vm, Vs, n);
    }
    for (int it = 0; it < h.iters; ++it) {
      gram_kernel<<<gblocks, gthreads, 0, st>>>(pC, Wn, bb, h.w, GV);
      inv_kernel<<<1, 256, ism, st>>>(GV, bb, SV);
      if (tc)
        tc_contract_rv(R, m, n, Vm, Vs, h.w, bb, klenP, splitP, Pp, st);
      else
        rv_kernel<<<dim3(tiles_m, splitP), 256, 0, st>>>(R, m, n, Vm, Vs, h.w, bb, klenP, Pp);
      target_kernel<<<tgtU, 256, 0, st>>>(Pp, splitP, m, bb, SV, T, Cs);
      tern_kernel<<<(Wm * 32 + 255) / 256, 256, 0, st>>>(T, m, bb, Cs, tgtU, tau, Um, Us, pB, Wm);
      gram_kernel<<<gblocks, gthreads, 0, st>>>(pB, Wm, bb, nullptr, GU);
      inv_kernel<<<1, 256, ism, st>>>(GU, bb, SU);
      if (tc)
        tc_contract_rtu(R, m, n, Um, Us, bb, klenQ, splitQ, Qp, st);
      else
        rtu_kernel<<<dim3(tiles_n, splitQ), 256, 0, st>>>(R, m, n, Um, Us, bb, klenQ, Qp);
      target_kernel<<<tgtV, 256, 0, st>>>(Qp, splitQ, n, bb, SU, T, Cs);
      tern_kernel<<<(Wn * 32 + 255) / 256, 256, 0, st>>>(T, n, bb, Cs, tgtV, tau, Vm, Vs, pC, Wn);
      if (tr) {
        u64* at = tr + 2 * (size_t)n + (size_t)it * 2 * ((size_t)m + n);
        record(at, Um, Us, m);
        record(at + 2 * (size_t)m, Vm, Vs, n);
      }
    }
    gram_kernel<<<gblocks, gthreads, 0, st>>>(pC, Wn, bb, h.w, GV);
    rpart_kernel<<<tgtV, 256, 0, st>>>(Qp, splitQ, n, bb, Vm, Vs, h.w, Rp);
    dsolve_kernel<<<1, 256, dsm, st>>>(GU, GV, Rp, tgtV, bb, scal, c0, h.D, h.energy, dblk);
    deflate_kernel<<<dim3((m + 7) / 8, nch), 256, 0, st>>>(R, m, n, Um, Us, Vm, Vs, dblk, h.w, rhop);
    chk();
  }
  int* status = status_word_ptr();
  if (status) set_status_kernel<<<1, 1, 0, st>>>(bad, status);
  chk();
  if (cudaFreeAsync(ws, st) != cudaSuccess && rc == EXTERND_OK) rc = EXTERND_ERR_CUDA;
  return rc;
}

}  // namespace externd
