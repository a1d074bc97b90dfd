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
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"
#include "umma_layout.cuh"

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
constexpr int kChunk = 256;
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

// validity of the weights, and their copy zero padded to npad entries
__global__ void check_w_kernel(const float* __restrict__ w, int n, int npad,
                               float* __restrict__ wpad, int* __restrict__ bad) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j < n) {
    const float x = w[j];
    if (!(x > 0.f) || !isfinite(x)) atomicExch(bad, 1);
    wpad[j] = x;
  } else if (j < npad) {
    wpad[j] = 0.f;
  }
}

// ---- top-bb rows: radix select on the fp64 energy bits, then rank ----------
// One CTA of 1024 threads.  Also sums the energies in a fixed order (R2) and,
// on the first block, records it as E0.  With `cached` set the m energy keys
// are kept in dynamic shared memory for the eight radix passes.
__global__ void __launch_bounds__(1024) select_rows_kernel(const double* __restrict__ rhop,
                                                           int nch, double* __restrict__ rho,
                                                           int m, int bb, int* __restrict__ rows,
                                                           double* __restrict__ scal,
                                                           int first, int cached) {
  extern __shared__ unsigned long long keys_sh[];
  __shared__ unsigned int hist[256];
  __shared__ double sh[32];
  __shared__ unsigned long long s_prefix, s_mask;
  __shared__ int s_remaining;
  __shared__ int cnt_gt[64], cnt_eq[64];
  __shared__ int cand[kMaxB];
  const int tid = threadIdx.x;
  double part = 0.0;
  for (int i0 = 0; i0 < m; i0 += 4096) {
    // four rows per thread per round; eight chunks' partial loads in flight
    // together (the sums still run in chunk order)
    double r[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 8
    for (int c = 0; c < nch; ++c) {
      double v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = i0 + tid + 1024 * q;
        v[q] = i < m ? rhop[(size_t)c * m + i] : 0.0;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) r[q] += v[q];
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = i0 + tid + 1024 * q;
      if (i < m) {
        rho[i] = r[q];
        if (cached) keys_sh[i] = (u64)__double_as_longlong(r[q]);
        part += r[q];
      }
    }
  }
  auto key_of = [&](int i) -> u64 {
    return cached ? keys_sh[i] : (u64)__double_as_longlong(rho[i]);
  };
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
      const u64 key = key_of(i);
      if ((key & msk) == pref) atomicAdd(&hist[(key >> shift) & 0xffu], 1u);
    }
    __syncthreads();
    if (tid < 32) {
      // lane L owns digits 255 - 8L down to 248 - 8L; the digit sought is the
      // largest d whose count from the top reaches the rows still needed
      const int rem = s_remaining;
      int cnt[8], tot = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        cnt[q] = (int)hist[255 - 8 * tid - q];
        tot += cnt[q];
      }
      int incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += y;
      }
      const int excl = incl - tot;
      // the owner lane: excl < rem <= incl (the last lane takes digit 0 otherwise)
      const bool own = (excl < rem && rem <= incl) || (tid == 31 && incl < rem);
      if (own) {
        int r = rem - excl, dd = 255 - 8 * tid - 7;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (cnt[q] >= r) {
            dd = 255 - 8 * tid - q;
            break;
          }
          r -= cnt[q];
        }
        s_remaining = r;
        s_prefix = pref | ((u64)dd << shift);
        s_mask = msk | (0xffull << shift);
      }
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
    const u64 key = key_of(i);
    g += key > kstar;
    e += key == kstar;
  }
  // exclusive scans of both counts in thread order: warp scans, then the
  // 32 warp totals scanned by warp 0
  {
    const int lane = tid & 31, wq = tid >> 5;
    int ig = g, ie = e;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int yg = __shfl_up_sync(0xffffffffu, ig, o), ye = __shfl_up_sync(0xffffffffu, ie, o);
      if (lane >= o) {
        ig += yg;
        ie += ye;
      }
    }
    if (lane == 31) {
      cnt_gt[wq] = ig;
      cnt_eq[wq] = ie;
    }
    __syncthreads();
    if (wq == 0) {
      int tg = cnt_gt[lane], te = cnt_eq[lane];
      int sg = tg, se = te;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int yg = __shfl_up_sync(0xffffffffu, sg, o), ye = __shfl_up_sync(0xffffffffu, se, o);
        if (lane >= o) {
          sg += yg;
          se += ye;
        }
      }
      cnt_gt[32 + lane] = sg - tg;
      cnt_eq[32 + lane] = se - te;
    }
    __syncthreads();
    g = cnt_gt[32 + wq] + ig - g;
    e = cnt_eq[32 + wq] + ie - e;
  }
  int pg = g, pe = e;
  const int ngt = bb - need_eq;  // rows strictly above kstar
  for (int i = i0; i < i1; ++i) {
    const u64 key = key_of(i);
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
    const double rm = __longlong_as_double((long long)key_of(me));
    int rank = 0;
    for (int t = 0; t < bb; ++t) {
      const int o = cand[t];
      const double ro = __longlong_as_double((long long)key_of(o));
      rank += (ro > rm) || (ro == rm && o < me);
    }
    rows[rank] = me;
  }
}

// ---- starting V: column l = T_tau(R[rows[l], :]) ----------------------------
// (stat 0: threshold tau * rms of the row; stat 1: tau * mean |x|)
__global__ void vinit_kernel(const float* __restrict__ R, int n, const int* __restrict__ rows,
                             double tau, int stat, u64* __restrict__ Vm, u64* __restrict__ Vs) {
  __shared__ double sh[32];
  const int l = blockIdx.x;
  const float* row = R + (size_t)rows[l] * n;
  double s = 0.0;
  for (int j = threadIdx.x; j < n; j += blockDim.x)
    s += stat ? fabs((double)row[j]) : (double)row[j] * (double)row[j];
  s = block_sum_d(s, sh);
  const double thr = stat ? tau * (s / (double)n) : tau * sqrt(s / (double)n);
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    const float x = row[j];
    if (fabs((double)x) > thr) {
      atomicOr(Vm + j, 1ull << l);
      if (x < 0.f) atomicOr(Vs + j, 1ull << l);
    }
  }
}

// Writes the tensor-core B chunk of plane word t (entries 32t .. 32t+31): lane
// holds the plane words of components lane and lane + 32 (zero beyond bb).
__device__ __forceinline__ void write_bchunk(unsigned char* __restrict__ bop, int t, int lane,
                                             const uint32_t (&om)[2], const uint32_t (&os)[2]) {
  unsigned char* chunk = bop + (size_t)t * umma::kBBytes;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int l = lane + 32 * h;
#pragma unroll
    for (int kg = 0; kg < 4; ++kg)
      *(uint4*)(chunk + umma::kmaj_off(l, kg * 8)) =
          umma::bf16_codes8((om[h] >> (8 * kg)) & 0xffu, (os[h] >> (8 * kg)) & 0xffu);
  }
}

// ---- packed planes [bb][2][W] of per-entry 64-bit masks (warp per word) ------
__global__ void planes_kernel(const u64* __restrict__ Mk, const u64* __restrict__ Sg, int len,
                              int bb, uint32_t* __restrict__ planes, int W,
                              unsigned char* __restrict__ bop) {
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
  if (bop) write_bchunk(bop, t, lane, om, os);
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
  if (!w) {
    // unrolled so the plane loads of several words are in flight together
#pragma unroll 4
    for (int t = lane; t < W; t += 32) {
      const uint32_t mm = m1[t] & m2[t];
      const uint32_t x = m1[W + t] ^ m2[W + t];
      cnt += (long long)__popc(mm & ~x) - (long long)__popc(mm & x);
    }
  } else {
    for (int t = lane; t < W; t += 32) {
      const uint32_t mm = m1[t] & m2[t];
      const uint32_t x = m1[W + t] ^ m2[W + t];
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

// ---- in-place Gauss-Jordan inverse of an SPD matrix (no pivoting) ----------
// The bb x bb matrix (bb <= 64, zero padded to 64 x 64) lives in registers of
// a 256-thread CTA: warp w holds rows 8w .. 8w+7, lane holds columns lane and
// lane + 32.  The pivots are taken in blocks of eight, K = 8w .. 8w+7, which
// are exactly warp w's rows.  Block K: warp w runs the eight in-place pivot
// steps on its own rows alone (for pivot k: n = a_k / a_kk with n_k = 1 / a_kk,
// row k <- n, and a_ij <- a_ij - a_ik n_j (j != k), a_ik <- -a_ik n_k on the
// block's other rows; the factors come by warp shuffles).  Those rows then
// hold [A_KK^-1, A_KK^-1 A_KJ] and are published to shared memory, together
// with every other row's factors a_iK (before the block).  Each other row
// takes the block's eight steps at once, a_ij <- [j not in K] a_ij -
// sum_k a_ik P_kj, which is the same elimination regrouped (the Schur
// complement update).  Two barriers per block; after all blocks the
// registers hold the inverse.  `sm` holds 1024 doubles.
__device__ __forceinline__ void gj_inverse(double (&a)[8][2], int bb, double* sm) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  double* const P = sm;             // [8][64]: the block's transformed rows
  double* const F = sm + 8 * kMaxB;  // [64 rows][8]: each row's factors a_iK
  const int nblk = (bb + 7) >> 3;
  for (int K = 0; K < nblk; ++K) {
    const int kb = 8 * K, nk = min(8, bb - kb);
    const int lk = kb & 31;  // lane holding column kb (columns kb .. kb+7: lanes lk .. lk+7)
    const bool hk = kb >= 32;
    if (wid == K) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        if (kk < nk) {
          const int k = kb + kk;
          const double piv = __shfl_sync(0xffffffffu, hk ? a[kk][1] : a[kk][0], lk + kk);
          const double p = 1.0 / piv;
          const double n0 = lane == k ? p : a[kk][0] * p;
          const double n1 = lane + 32 == k ? p : a[kk][1] * p;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const double f = __shfl_sync(0xffffffffu, hk ? a[q][1] : a[q][0], lk + kk);
            if (q == kk) {
              a[q][0] = n0;
              a[q][1] = n1;
            } else {
              a[q][0] = (lane == k ? 0.0 : a[q][0]) - f * n0;
              a[q][1] = (lane + 32 == k ? 0.0 : a[q][1]) - f * n1;
            }
          }
        }
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        P[q * kMaxB + lane] = a[q][0];
        P[q * kMaxB + lane + 32] = a[q][1];
      }
    } else if (lane >= lk && lane < lk + 8) {
#pragma unroll
      for (int q = 0; q < 8; ++q) F[(wid * 8 + q) * 8 + (lane - lk)] = hk ? a[q][1] : a[q][0];
    }
    __syncthreads();
    if (wid != K) {
      double pv[8][2];
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        pv[kk][0] = P[kk * kMaxB + lane];
        pv[kk][1] = P[kk * kMaxB + lane + 32];
      }
      const bool in0 = lane >= kb && lane < kb + 8, in1 = lane + 32 >= kb && lane + 32 < kb + 8;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const double2* fr = (const double2*)(F + (wid * 8 + q) * 8);
        const double2 f01 = fr[0], f23 = fr[1], f45 = fr[2], f67 = fr[3];
        const double f[8] = {f01.x, f01.y, f23.x, f23.y, f45.x, f45.y, f67.x, f67.y};
        double x0 = in0 ? 0.0 : a[q][0], x1 = in1 ? 0.0 : a[q][1];
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          x0 -= f[kk] * pv[kk][0];
          x1 -= f[kk] * pv[kk][1];
        }
        a[q][0] = x0;
        a[q][1] = x1;
      }
    }
    __syncthreads();  // P and F are rewritten by the next block
  }
  __syncthreads();  // (also when bb == 0)
}

// S = (G + eps I)^-1 with eps = 1e-6 tr(G) / bb (1 when the trace is 0).
__global__ void __launch_bounds__(256, 1) inv_kernel(const double* __restrict__ G, int bb,
                                                  double* __restrict__ S) {
  __shared__ __align__(16) double prow[16 * kMaxB];
  __shared__ double eps;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (wid == 0) {
    double t = (lane < bb ? G[lane * bb + lane] : 0.0) +
               (lane + 32 < bb ? G[(lane + 32) * bb + lane + 32] : 0.0);
    // fixed-order tree over the 64 diagonal entries
    t = warp_sum(t);
    if (lane == 0) eps = t > 0.0 ? 1e-6 * t / (double)bb : 1.0;
  }
  __syncthreads();
  double a[8][2];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int i = wid * 8 + q;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = lane + 32 * h;
      a[q][h] = (i < bb && j < bb) ? G[i * bb + j] + (i == j ? eps : 0.0) : 0.0;
    }
  }
  gj_inverse(a, bb, prow);
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int i = wid * 8 + q;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = lane + 32 * h;
      if (i < bb && j < bb) S[i * bb + j] = a[q][h];
    }
  }
}

// ---- targets: T[x][l] = sum_l2 (sum_s Xp[s][x][l2]) S[l2][l] (fp64) ----------
// The rows are split evenly over at most one CTA per SM: CTA c takes rows
// [c rpc, (c+1) rpc) with rpc <= 80, so no SM holds twice the work of
// another.  The split-K / stream-K partials are summed (in partial order,
// fp64) into a row-major tile Xs[row][l2] in shared memory next to S -- each
// thread loads 4 consecutive columns of 4 rows, float4 per partial, all
// partials in flight (NS >= partials is a compile-time bound).  Thread
// (rg, cg) then forms the 4 x 4 block rows 4rg.., columns 4cg.. of T: 16
// independent fp64 chains per thread.  Each CTA writes its column sums of
// squares (stat 0) or of absolute values (stat 1); the last CTA to finish
// (ticket counter) adds those partials in a fixed order -- thread (q, l)
// takes CTAs q, q + 5, q + 10, ... in CTA order with all its loads in
// flight, then the five sums in q order -- and writes the column thresholds
// thr[l] = tau * rms(T[:, l]) (stat 0) or tau * mean |T[:, l]| (stat 1), then
// rearms the counter.  With Xout set, the partial-summed X (rows x bb, fp64)
// is stored as well.  With wsc set, row x of T is scaled by wsc[x] before it
// is stored and measured (the naive weighted V-step thresholds W times the
// target).
constexpr int kTgtThreads = 320;     // 20 row groups x 16 column groups
constexpr int kTgtMaxRows = 80;      // rows per CTA at most (20 groups x 4)
constexpr int kTgtRedGroups = kTgtThreads / kMaxB;  // 5 summing groups in the last CTA
constexpr int kTgtRedLoads = 32;     // loads in flight per thread in the last CTA
constexpr int kMaxSplits = kMaxSegs;  // partials per output row (split-K or stream-K)
// padded row of the X tile: even (16-byte aligned pairs), and 4 rows apart
// land 16 banks apart, so the two row groups a warp reads never collide
constexpr int kXs = kMaxB + 2;
// rows per CTA for `rows` rows on nsm SMs
inline int target_rpc(int rows, int nsm) {
  const int r = (rows + nsm - 1) / std::max(nsm, 1);
  return std::max(1, std::min(kTgtMaxRows, r));
}
// Partials: split-K layout Xp[split][row][bb] (sk == 0, `splits` of them) or
// stream-K layout Xp[(t Sslots + slot) 128 + row % 128][bb] with the tile's
// segment count from the plan (C, U, G) (sk != 0).
template <int NS>
__global__ void __launch_bounds__(kTgtThreads, 1) target_kernel(
    const float* __restrict__ Xp, int splits, int rows, int rpc, int bb,
    const double* __restrict__ S, double tau, double* __restrict__ T,
    double* __restrict__ colss, unsigned* __restrict__ ticket, double* __restrict__ thr,
    double* __restrict__ Xout, int sk, int C, long long U, int G, int Sslots, int stat,
    const float* __restrict__ wsc) {
  extern __shared__ __align__(16) double tsh[];
  double* Ss = tsh;                                                    // [64][64]: S[l2][l]
  double* Xt = tsh + kMaxB * kMaxB;                                    // [80][kXs]
  double (*part)[kMaxB] = (double (*)[kMaxB])(Xt + kTgtMaxRows * kXs);  // [20][64]
  __shared__ bool last;
  __shared__ int np_s[2];  // partials of the CTA's first and last 128-row tile
  const int tid = threadIdx.x;
  const int x0 = blockIdx.x * rpc, nr = min(rpc, rows - x0);
  if (tid < 2) {
    // the CTA's rows (at most 80) meet at most two tiles; the segment count
    // costs 64-bit divisions, so it is found once per tile, not per row
    const int xt = tid == 0 ? x0 : x0 + nr - 1;
    np_s[tid] = sk ? umma::sk_nseg(xt / umma::kM, C, U, G) : splits;
  }
  {
    constexpr int kSL = (kMaxB * kMaxB + kTgtThreads - 1) / kTgtThreads;
    double sv[kSL];
#pragma unroll
    for (int q = 0; q < kSL; ++q) {
      const int p = tid + kTgtThreads * q, l2 = p >> 6, lc = p & 63;
      sv[q] = (p < kMaxB * kMaxB && l2 < bb && lc < bb) ? __ldg(S + l2 * bb + lc) : 0.0;
    }
#pragma unroll
    for (int q = 0; q < kSL; ++q) {
      const int p = tid + kTgtThreads * q;
      if (p < kMaxB * kMaxB) Ss[p] = sv[q];
    }
  }
  __syncthreads();  // np_s
  {
    // thread: columns lq .. lq+3 (lq = 4 (tid % 16)), rows tid / 16 + 20 h
    const int lq = (tid & 15) * 4, rr = tid >> 4;
    const size_t sstride = sk ? (size_t)umma::kM * bb : (size_t)rows * bb;
    const bool vec = (bb & 3) == 0;
    constexpr int RPR = NS > 8 ? 1 : 2;  // rows per round: at most 64 floats in flight
#pragma unroll 1
    for (int h0 = 0; h0 < 4; h0 += RPR) {
      float4 v[RPR][NS];
      int np[RPR];
#pragma unroll
      for (int h = 0; h < RPR; ++h) {
        const int r = rr + 20 * (h0 + h), x = x0 + r;
        const bool ok = r < nr && lq < bb;
        const int xs = ok ? x : 0;
        np[h] = ok ? np_s[(xs / umma::kM) != (x0 / umma::kM)] : 0;
        const size_t prow = sk ? ((size_t)(xs / umma::kM) * Sslots * umma::kM + xs % umma::kM)
                               : (size_t)xs;
        const float* src = Xp + prow * bb + (ok ? lq : 0);
#pragma unroll
        for (int sp = 0; sp < NS; ++sp) {
          float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
          if (ok && sp < np[h]) {
            const float* q = src + sp * sstride;
            if (vec) {
              t = __ldg((const float4*)q);
            } else {
              t.x = __ldg(q);
              if (lq + 1 < bb) t.y = __ldg(q + 1);
              if (lq + 2 < bb) t.z = __ldg(q + 2);
              if (lq + 3 < bb) t.w = __ldg(q + 3);
            }
          }
          v[h][sp] = t;
        }
      }
#pragma unroll
      for (int h = 0; h < RPR; ++h) {
        double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
#pragma unroll
        for (int sp = 0; sp < NS; ++sp)
          if (sp < np[h]) {
            s0 += (double)v[h][sp].x;
            s1 += (double)v[h][sp].y;
            s2 += (double)v[h][sp].z;
            s3 += (double)v[h][sp].w;
          }
        const int r = rr + 20 * (h0 + h);
        *(double2*)(Xt + r * kXs + lq) = make_double2(s0, s1);
        *(double2*)(Xt + r * kXs + lq + 2) = make_double2(s2, s3);
        const int x = x0 + r;
        if (Xout && r < nr) {
          const double sx[4] = {s0, s1, s2, s3};
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (lq + j < bb) Xout[(size_t)x * bb + lq + j] = sx[j];
        }
      }
    }
  }
  __syncthreads();
  const int rg = tid >> 4, cg = tid & 15;
  double acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
  if (4 * rg < nr) {
    // two l2 per step (X entries past bb and S rows past bb are zero)
    const double* xr = Xt + (4 * rg) * kXs;
#pragma unroll 2
    for (int l2 = 0; l2 < bb; l2 += 2) {
      double2 xp[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) xp[i] = *(const double2*)(xr + i * kXs + l2);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const double2 sa = *(const double2*)(Ss + (l2 + h) * kMaxB + 4 * cg);
        const double2 sb = *(const double2*)(Ss + (l2 + h) * kMaxB + 4 * cg + 2);
        const double svv[4] = {sa.x, sa.y, sb.x, sb.y};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const double xv = h ? xp[i].y : xp[i].x;
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] += xv * svv[j];
        }
      }
    }
  }
  double cs[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = 4 * rg + i, x = x0 + r;
    if (r < nr) {
      if (wsc) {
        const double ws = (double)wsc[x];
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] *= ws;
      }
      if (bb == kMaxB) {
        *(double2*)(T + (size_t)x * bb + 4 * cg) = make_double2(acc[i][0], acc[i][1]);
        *(double2*)(T + (size_t)x * bb + 4 * cg + 2) = make_double2(acc[i][2], acc[i][3]);
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (4 * cg + j < bb) T[(size_t)x * bb + 4 * cg + j] = acc[i][j];
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) cs[j] += stat ? fabs(acc[i][j]) : acc[i][j] * acc[i][j];
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) part[rg][4 * cg + j] = cs[j];
  __syncthreads();
  if (tid < kMaxB) {
    double c = 0.0;
    for (int g = 0; g < kTgtThreads / 16; ++g) c += part[g][tid];
    if (tid < bb) colss[(size_t)blockIdx.x * bb + tid] = c;
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    last = atomicAdd(ticket, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  {
    const int l = tid & 63, q = tid / kMaxB;
    const int nb = (int)gridDim.x;
    double c = 0.0;
    if (l < bb) {
      for (int b0 = q; b0 < nb; b0 += kTgtRedGroups * kTgtRedLoads) {
        double v[kTgtRedLoads];
#pragma unroll
        for (int u = 0; u < kTgtRedLoads; ++u) {
          const int b = b0 + kTgtRedGroups * u;
          v[u] = b < nb ? __ldcg(colss + (size_t)b * bb + l) : 0.0;
        }
#pragma unroll
        for (int u = 0; u < kTgtRedLoads; ++u)
          if (b0 + kTgtRedGroups * u < nb) c += v[u];
      }
    }
    part[q][l] = c;
    __syncthreads();
    if (tid < bb) {
      double t5 = part[0][tid];
#pragma unroll
      for (int g = 1; g < kTgtRedGroups; ++g) t5 += part[g][tid];
      thr[tid] = stat ? tau * (t5 / (double)rows) : tau * sqrt(t5 / (double)rows);
    }
  }
  if (tid == 0) *ticket = 0u;
}
constexpr size_t kTgtSmem =
    sizeof(double) * (kMaxB * kMaxB + kTgtMaxRows * kXs + (kTgtThreads / 16) * kMaxB);
// the target kernel instantiated for a partial-count bound
typedef void (*TargetFn)(const float*, int, int, int, int, const double*, double, double*,
                         double*, unsigned*, double*, double*, int, int, long long, int, int, int,
                         const float*);
inline TargetFn target_for(int splits) {
  if (splits <= 1) return target_kernel<1>;
  if (splits <= 2) return target_kernel<2>;
  if (splits <= 4) return target_kernel<4>;
  if (splits <= 8) return target_kernel<8>;
  return target_kernel<16>;
}

// ---- ternary codes: 64-bit masks per entry and packed planes -----------------
// One CTA of 8 warps per 32 entries (one plane word t).  Warp w thresholds
// entries 4w .. 4w+3: lane l reads T[x][l] and T[x][l + 32] (coalesced), and
// four ballots give entry x's mask and sign words directly.  The 32 entries'
// words meet in shared memory; warp w then transposes components
// 8w .. 8w+7 into plane words (one ballot per component and plane), and every
// thread writes one 16-byte group of the word's bf16 B chunk.
__global__ void __launch_bounds__(256) tern_kernel(const double* __restrict__ T, int rows, int bb,
                                                   const double* __restrict__ thr,
                                                   u64* __restrict__ Mk, u64* __restrict__ Sg,
                                                   uint32_t* __restrict__ planes, int W,
                                                   unsigned char* __restrict__ bop) {
  __shared__ u64 mk_s[32], sg_s[32];
  __shared__ uint32_t om_s[kMaxB], os_s[kMaxB];
  const int t = blockIdx.x, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  double v0[4], v1[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int x = t * 32 + 4 * wid + q;
    v0[q] = (x < rows && lane < bb) ? T[(size_t)x * bb + lane] : 0.0;
    v1[q] = (x < rows && lane + 32 < bb) ? T[(size_t)x * bb + lane + 32] : 0.0;
  }
  const double th0 = lane < bb ? thr[lane] : 0.0, th1 = lane + 32 < bb ? thr[lane + 32] : 0.0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const bool a0 = lane < bb && fabs(v0[q]) > th0, a1 = lane + 32 < bb && fabs(v1[q]) > th1;
    const uint32_t m0 = __ballot_sync(0xffffffffu, a0), m1 = __ballot_sync(0xffffffffu, a1);
    const uint32_t s0 = __ballot_sync(0xffffffffu, a0 && v0[q] < 0.0);
    const uint32_t s1 = __ballot_sync(0xffffffffu, a1 && v1[q] < 0.0);
    if (lane == 0) {
      mk_s[4 * wid + q] = (u64)m0 | ((u64)m1 << 32);
      sg_s[4 * wid + q] = (u64)s0 | ((u64)s1 << 32);
    }
  }
  __syncthreads();
  const u64 mk = mk_s[lane], sg = sg_s[lane];  // entry t * 32 + lane (0 past the end)
  if (wid == 0 && t * 32 + lane < rows) {
    Mk[t * 32 + lane] = mk;
    Sg[t * 32 + lane] = sg;
  }
  uint32_t pm = 0u, ps = 0u;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const int l = 8 * wid + c;
    const uint32_t bm = __ballot_sync(0xffffffffu, (mk >> l) & 1ull);
    const uint32_t bs = __ballot_sync(0xffffffffu, (sg >> l) & 1ull);
    if (lane == c) {
      pm = bm;
      ps = bs;
    }
  }
  if (lane < 8) {
    const int l = 8 * wid + lane;
    om_s[l] = pm;
    os_s[l] = ps;
    if (l < bb) {
      planes[(size_t)l * 2 * W + t] = pm;
      planes[(size_t)l * 2 * W + W + t] = ps;
    }
  }
  if (!bop) return;
  __syncthreads();
  {
    // thread -> component l = tid / 4, 8-entry group kg = tid % 4
    const int l = tid >> 2, kg = tid & 3;
    *(uint4*)(bop + (size_t)t * umma::kBBytes + umma::kmaj_off(l, kg * 8)) =
        umma::bf16_codes8((om_s[l] >> (8 * kg)) & 0xffu, (os_s[l] >> (8 * kg)) & 0xffu);
  }
}

// ---- r_l = u_l^T R W v_l = sum_j Q[j][l] w_j s_jl, per-CTA partials (64 rows)
constexpr int kRpartRows = 64;
// Q = R^T U, split-summed in fp64 by the last V-step target pass.
__global__ void __launch_bounds__(256) rpart_kernel(const double* __restrict__ Q, int n, int bb,
                                                    const u64* __restrict__ Vm,
                                                    const u64* __restrict__ Vs,
                                                    const float* __restrict__ w,
                                                    double* __restrict__ rp) {
  __shared__ double part[4][kMaxB];
  const int l = threadIdx.x & 63, rr = threadIdx.x >> 6;
  const int x0 = blockIdx.x * kRpartRows;
  double acc = 0.0;
  if (l < bb) {
#pragma unroll 4
    for (int t = 0; t < kRpartRows / 4; ++t) {
      const int j = x0 + rr + 4 * t;
      if (j < n) {
        const u64 mm = Vm[j];
        const double q = Q[(size_t)j * bb + l];
        const double wj = w ? (double)w[j] : 1.0;
        if ((mm >> l) & 1ull) acc += (((Vs[j] >> l) & 1ull) ? -q : q) * wj;
      }
    }
  }
  part[rr][l] = acc;
  __syncthreads();
  if (rr == 0 && l < bb)
    rp[(size_t)blockIdx.x * bb + l] = ((part[0][l] + part[1][l]) + part[2][l]) + part[3][l];
}

// ---- joint scales, closed-form energies ---------------------------------------
// r_l = sum_j (sum_s Qp[s][j][l]) w_j s_jl; G = GU o GV; the active set (l
// with u_l != 0 and v_l != 0) solves (G_AA + eps I) d_A = r_A through the
// register Gauss-Jordan inverse; inactive scales are 0.
__global__ void __launch_bounds__(256, 1) dsolve_kernel(const double* __restrict__ GU,
                                                     const double* __restrict__ GV,
                                                     const double* __restrict__ rp, int rparts,
                                                     int bb, const double* __restrict__ scal,
                                                     int c0, float* __restrict__ D,
                                                     double* __restrict__ energy,
                                                     float* __restrict__ dblk) {
  __shared__ double G[kMaxB * kMaxB];
  __shared__ double r[kMaxB], ra[kMaxB], fcol[kMaxB];
  __shared__ __align__(16) double prow[16 * kMaxB];
  __shared__ float dl[kMaxB];
  __shared__ int act[kMaxB];
  __shared__ int na;
  __shared__ double eps;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (threadIdx.x < bb) {
    double s = 0.0;
#pragma unroll 8
    for (int b = 0; b < rparts; ++b) s += rp[(size_t)b * bb + threadIdx.x];
    r[threadIdx.x] = s;
    dl[threadIdx.x] = 0.f;
  }
  for (int p = threadIdx.x; p < bb * bb; p += blockDim.x) G[p] = GU[p] * GV[p];
  __syncthreads();
  if (wid == 0) {
    double t = (lane < bb ? G[lane * bb + lane] : 0.0) +
               (lane + 32 < bb ? G[(lane + 32) * bb + lane + 32] : 0.0);
    t = warp_sum(t);
    const bool a0 = lane < bb && GU[lane * bb + lane] > 0.0 && GV[lane * bb + lane] > 0.0;
    const bool a1 = lane + 32 < bb && GU[(lane + 32) * bb + lane + 32] > 0.0 &&
                    GV[(lane + 32) * bb + lane + 32] > 0.0;
    const unsigned b0 = __ballot_sync(0xffffffffu, a0), b1 = __ballot_sync(0xffffffffu, a1);
    const unsigned below = (1u << lane) - 1u;
    if (a0) act[__popc(b0 & below)] = lane;
    if (a1) act[__popc(b0) + __popc(b1 & below)] = lane + 32;
    if (lane == 0) {
      eps = t > 0.0 ? 1e-6 * t / (double)bb : 1.0;
      na = __popc(b0) + __popc(b1);
    }
  }
  __syncthreads();
  const int A = na;
  if (threadIdx.x < A) ra[threadIdx.x] = r[act[threadIdx.x]];
  double a[8][2];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int i = wid * 8 + q;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = lane + 32 * h;
      a[q][h] = (i < A && j < A) ? G[act[i] * bb + act[j]] + (i == j ? eps : 0.0) : 0.0;
    }
  }
  gj_inverse(a, A, prow);  // ends with a barrier, which also publishes ra
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int i = wid * 8 + q;
    double t = (lane < A ? a[q][0] * ra[lane] : 0.0) + (lane + 32 < A ? a[q][1] * ra[lane + 32] : 0.0);
    t = warp_sum(t);
    if (lane == 0 && i < A) dl[act[i]] = (float)t;
  }
  __syncthreads();
  // energy after component c0 + l: |R|^2 - 2 sum_{a<=l} d_a r_a + sum_{a,c<=l} d_a d_c G_ac,
  // accumulated over l: inc_l = -2 d_l r_l + d_l^2 G_ll + 2 d_l sum_{a<l} d_a G_al
  if (threadIdx.x < bb) {
    const int l = threadIdx.x;
    double h = 0.0;
    for (int q = 0; q < l; ++q) h += (double)dl[q] * G[q * bb + l];
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
// CTA = 8 warps over 64 rows and one chunk of kChunk columns, walked in
// sub-tiles of 128 columns.  Shared memory holds, per component l of the
// block, the negated signed scales of the CTA's rows, nd_il = -(u_il d_l)
// (0 where u_il = 0; stored twice, as a pair), and the sub-tile's V codes
// expanded to fp32, vf_lj = v_jl in {-1, 0, +1}.  Warp w owns rows
// 8w .. 8w+7 and lane t the columns 4t .. 4t+3 of the sub-tile, so a thread
// holds an 8 x 4 block of R.  For l = 0, 1, ..., b-1 in order it takes
// x <- fma(nd_il, vf_lj, x) on column pairs (__ffma2_rn).  The product is
// exact (vf is -1, 0 or +1), so where u_il v_jl != 0 the step is the one fp32
// subtract (or add) of d_l that the ordered deflation makes, rounded once,
// and where u_il v_jl = 0 it adds a zero: x is unchanged (a -0 entry may turn
// into +0, which no later sum, square or threshold can tell apart).  The
// (weighted) row energies of the updated chunk are summed in fp64 on the way
// out: lane partials over the sub-tiles, then across the warp.
constexpr int kDefRows = 64;  // rows per CTA: 8 warps x 8 rows
constexpr int kDefSub = 128;  // columns per sub-tile: 32 lanes x 4
static_assert(kChunk % kDefSub == 0, "sub-tiles tile the chunk");
constexpr size_t kDefSmem = sizeof(float2) * kMaxB * kDefRows + sizeof(float) * kMaxB * kDefSub;

template <bool VEC>
__global__ void __launch_bounds__(256, 3) deflate_kernel(float* __restrict__ R, int m, int n,
                                                         const u64* __restrict__ Um,
                                                         const u64* __restrict__ Us,
                                                         const u64* __restrict__ Vm,
                                                         const u64* __restrict__ Vs,
                                                         const float* __restrict__ dblk, int bb,
                                                         const float* __restrict__ w,
                                                         double* __restrict__ rhop) {
  extern __shared__ __align__(16) unsigned char dsm[];
  float2* nd2 = (float2*)dsm;                                         // [kMaxB][kDefRows]
  float* vf = (float*)(dsm + sizeof(float2) * kMaxB * kDefRows);      // [kMaxB][kDefSub]
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int i0 = blockIdx.x * kDefRows;
  const int ch = blockIdx.y, j0 = ch * kChunk, j1 = min(n, j0 + kChunk);
  {
    const int r = tid & (kDefRows - 1), i = i0 + r;
    const u64 um = i < m ? Um[i] : 0ull, us = i < m ? Us[i] : 0ull;
    for (int l = tid / kDefRows; l < bb; l += 256 / kDefRows) {
      float v = 0.f;
      if ((um >> l) & 1ull) v = ((us >> l) & 1ull) ? dblk[l] : -dblk[l];
      nd2[l * kDefRows + r] = make_float2(v, v);
    }
  }
  const int r0 = 8 * wid;
  double es[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) es[q] = 0.0;
  for (int jt = j0; jt < j1; jt += kDefSub) {
    __syncthreads();  // nd2 written; the previous sub-tile's codes no longer read
    {
      // thread -> column c, components l = tid / 128 + 2 t
      const int c = tid & (kDefSub - 1), j = jt + c;
      const u64 vm = j < j1 ? Vm[j] : 0ull, vs = j < j1 ? Vs[j] : 0ull;
      for (int l = tid / kDefSub; l < bb; l += 256 / kDefSub) {
        const uint32_t on = (uint32_t)(vm >> l) & 1u, neg = (uint32_t)(vs >> l) & 1u;
        vf[l * kDefSub + c] = __uint_as_float(on ? (0x3f800000u | (neg << 31)) : 0u);
      }
    }
    __syncthreads();
    const int jc = jt + 4 * lane;
    float2 x[8][2];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int i = i0 + r0 + q;
      const float* src = R + (size_t)(i < m ? i : 0) * n + jc;
      float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i < m) {
        if (VEC) {
          if (jc < j1) t = *(const float4*)src;
        } else {
          if (jc < j1) t.x = src[0];
          if (jc + 1 < j1) t.y = src[1];
          if (jc + 2 < j1) t.z = src[2];
          if (jc + 3 < j1) t.w = src[3];
        }
      }
      x[q][0] = make_float2(t.x, t.y);
      x[q][1] = make_float2(t.z, t.w);
    }
#pragma unroll 2
    for (int l = 0; l < bb; ++l) {
      const float4 v = *(const float4*)(vf + l * kDefSub + 4 * lane);
      const float2 v01 = make_float2(v.x, v.y), v23 = make_float2(v.z, v.w);
      const float4* np = (const float4*)(nd2 + l * kDefRows + r0);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 a = np[q];  // {nd, nd} of rows r0 + 2q and r0 + 2q + 1
        const float2 a0 = make_float2(a.x, a.y), a1 = make_float2(a.z, a.w);
        x[2 * q][0] = __ffma2_rn(a0, v01, x[2 * q][0]);
        x[2 * q][1] = __ffma2_rn(a0, v23, x[2 * q][1]);
        x[2 * q + 1][0] = __ffma2_rn(a1, v01, x[2 * q + 1][0]);
        x[2 * q + 1][1] = __ffma2_rn(a1, v23, x[2 * q + 1][1]);
      }
    }
    double wj[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) wj[e] = (jc + e < j1) ? (w ? (double)w[jc + e] : 1.0) : 0.0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int i = i0 + r0 + q;
      if (i < m) {
        float* dst = R + (size_t)i * n + jc;
        const float xv[4] = {x[q][0].x, x[q][0].y, x[q][1].x, x[q][1].y};
        if (VEC) {
          if (jc < j1) *(float4*)dst = make_float4(xv[0], xv[1], xv[2], xv[3]);
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (jc + e < j1) dst[e] = xv[e];
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) es[q] += wj[e] * (double)xv[e] * (double)xv[e];
      }
    }
  }
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const double s = warp_sum(es[q]);
    const int i = i0 + r0 + q;
    if (lane == 0 && i < m) rhop[(size_t)ch * m + i] = s;
  }
}

__global__ void set_status_kernel(const int* __restrict__ bad, int* __restrict__ status) {
  if (*bad) atomicCAS(status, 0, EXTERND_ERR_NONFINITE);
}

}  // namespace blk

// Enqueues one whole block-ALS decomposition on st (side stream and events
// for the Gram / inverse overlap supplied by the caller).
static int block_enqueue(const BlockHostArgs& h, cudaStream_t st, cudaStream_t side,
                         cudaEvent_t ev_fork, cudaEvent_t ev_join) {
  using namespace blk;
  const int m = (int)h.m, n = (int)h.n, k = (int)h.k, b = h.block;
  if (b > kMaxB) return EXTERND_ERR_INVALID_ARG;
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  // contractions run on the tensor cores (tcgen05, 128-row tiles)
  const int tileR = 128, kq = 32;
  // threshold variants: the statistic of T_tau, and the weights the naive
  // V-step scales its target by
  const int stat = (h.flags & EXTERND_TSTAT_MEAN_ABS) ? 1 : 0;
  const float* naive_w = (h.flags & EXTERND_VSTEP_NAIVE) ? h.w : nullptr;
  // split-K factors so each contraction has about two CTAs per SM
  const int tiles_m = (m + tileR - 1) / tileR, tiles_n = (n + tileR - 1) / tileR;
  // (at most two CTAs per SM in total, so a contraction runs in one wave)
  int splitP = std::max(1, std::min({2 * nsm / tiles_m, (n + kq - 1) / kq, kMaxSplits}));
  int splitQ = std::max(1, std::min({2 * nsm / tiles_n, (m + kq - 1) / kq, kMaxSplits}));
  const int klenP = ((n + splitP - 1) / splitP + kq - 1) / kq * kq;
  const int klenQ = ((m + splitQ - 1) / splitQ + kq - 1) / kq * kq;
  splitP = (n + klenP - 1) / klenP;
  splitQ = (m + klenQ - 1) / klenQ;
  // the persistent TMA contraction (stream-K partials) whenever R's rows are
  // TMA-addressable; the workspace keeps R at a 256-byte aligned offset
  const bool sk = tc_contract_tma_ok(n);
  TcPlan planP{}, planQ{};
  if (sk) {
    tc_contract_plan(m, n, nsm, &planP);
    tc_contract_plan(n, m, nsm, &planQ);
  }
  const size_t partsP = sk ? (size_t)planP.T * planP.S * 128 : (size_t)splitP * m;
  const size_t partsQ = sk ? (size_t)planQ.T * planQ.S * 128 : (size_t)splitQ * n;
  const int boundP = sk ? planP.S : splitP, boundQ = sk ? planQ.S : splitQ;
  // target CTAs: rows spread evenly over the SMs; rpart keeps 64-row CTAs
  const int rpcU = target_rpc(m, nsm), rpcV = target_rpc(n, nsm);
  const int tgtU = (m + rpcU - 1) / rpcU, tgtV = (n + rpcV - 1) / rpcV;
  const int rpartV = (n + kRpartRows - 1) / kRpartRows;
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
  const size_t oPp = take(sizeof(float) * partsP * b);
  const size_t oQp = take(sizeof(float) * partsQ * b);
  const size_t oT = take(sizeof(double) * (size_t)mx * b);
  const size_t oCs = take(sizeof(double) * (size_t)std::max(tgtU, tgtV) * b);
  const size_t oRp = take(sizeof(double) * (size_t)rpartV * b);
  const size_t oThr = take(sizeof(double) * kMaxB);
  const size_t oTick = take(sizeof(unsigned));
  const size_t oQs = take(sizeof(double) * (size_t)n * b);
  const size_t oBopU = take((size_t)Wm * umma::kBBytes), oBopV = take((size_t)Wn * umma::kBBytes);
  const size_t oWpad = take(sizeof(float) * (size_t)Wn * 32);
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
  double* thr = (double*)(base + oThr);
  unsigned* tick = (unsigned*)(base + oTick);
  double *SV = (double*)(base + oSV), *SU = (double*)(base + oSU);
  double *GU = (double*)(base + oGU), *GV = (double*)(base + oGV);
  double* scal = (double*)(base + oScal);
  float* dblk = (float*)(base + oD);
  int* bad = (int*)(base + oBad);
  double* Qs = (double*)(base + oQs);
  unsigned char* BopU = (unsigned char*)(base + oBopU);
  unsigned char* BopV = (unsigned char*)(base + oBopV);
  float* wpad = (float*)(base + oWpad);
  const double tau = (double)h.tau;
  int rc = EXTERND_OK;
  const TargetFn tgtP = target_for(boundP), tgtQ = target_for(boundQ);
  cudaFuncSetAttribute(deflate_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)kDefSmem);
  cudaFuncSetAttribute(deflate_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)kDefSmem);
  cudaFuncSetAttribute(tgtP, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTgtSmem);
  cudaFuncSetAttribute(tgtQ, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTgtSmem);
  // the row-energy keys of the radix select stay in shared memory when they fit
  const size_t sel_smem = (size_t)m * sizeof(u64) <= 160 * 1024 ? (size_t)m * sizeof(u64) : 0;
  if (sel_smem > 0)
    cudaFuncSetAttribute(select_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sel_smem);
  auto chk = [&]() {
    if (rc == EXTERND_OK && cudaGetLastError() != cudaSuccess) rc = EXTERND_ERR_CUDA;
  };
  cudaMemsetAsync(bad, 0, sizeof(int), st);
  cudaMemsetAsync(tick, 0, sizeof(unsigned), st);
  cudaMemsetAsync(dblk, 0, sizeof(float) * kMaxB, st);
  setup_kernel<<<dim3((m * 32 + 255) / 256, nch), 256, 0, st>>>(h.A, R, m, n, h.w, rhop, bad);
  if (h.w) check_w_kernel<<<(Wn * 32 + 255) / 256, 256, 0, st>>>(h.w, n, Wn * 32, wpad, bad);
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
    select_rows_kernel<<<1, 1024, sel_smem, st>>>(rhop, nch, rho, m, bb, rows, scal, c0 == 0,
                                                  sel_smem > 0);
    cudaMemsetAsync(Vm, 0, sizeof(u64) * n, st);
    cudaMemsetAsync(Vs, 0, sizeof(u64) * n, st);
    vinit_kernel<<<bb, 256, 0, st>>>(R, n, rows, tau, stat, Vm, Vs);
    planes_kernel<<<(Wn * 32 + 255) / 256, 256, 0, st>>>(Vm, Vs, n, bb, pC, Wn, BopV);
    if (tr) {
      cudaMemcpyAsync(h.trace_rows + (size_t)tslot * b, rows, sizeof(int) * bb,
                      cudaMemcpyDeviceToDevice, st);
      record(tr, Vm, Vs, n);
    }
    for (int it = 0; it < h.iters; ++it) {
      // the Gram matrix and its inverse do not feed the contraction: they
      // run on the side stream while it streams R
      cudaEventRecord(ev_fork, st);
      cudaStreamWaitEvent(side, ev_fork, 0);
      gram_kernel<<<gblocks, gthreads, 0, side>>>(pC, Wn, bb, h.w, GV);
      inv_kernel<<<1, 256, 0, side>>>(GV, bb, SV);
      cudaEventRecord(ev_join, side);
      tc_contract_rv(R, m, n, Vm, Vs, BopV, h.w, wpad, bb, sk ? &planP : nullptr, klenP, splitP,
                     Pp, h.wait_budget, st);
      cudaStreamWaitEvent(st, ev_join, 0);
      tgtP<<<tgtU, kTgtThreads, kTgtSmem, st>>>(Pp, splitP, m, rpcU, bb, SV, tau, T, Cs, tick,
                                                 thr, nullptr, sk, planP.C, planP.U, planP.G,
                                                 planP.S, stat, nullptr);
      tern_kernel<<<Wm, 256, 0, st>>>(T, m, bb, thr, Um, Us, pB, Wm, BopU);
      cudaEventRecord(ev_fork, st);
      cudaStreamWaitEvent(side, ev_fork, 0);
      gram_kernel<<<gblocks, gthreads, 0, side>>>(pB, Wm, bb, nullptr, GU);
      inv_kernel<<<1, 256, 0, side>>>(GU, bb, SU);
      cudaEventRecord(ev_join, side);
      tc_contract_rtu(R, m, n, Um, Us, BopU, bb, sk ? &planQ : nullptr, klenQ, splitQ, Qp,
                      h.wait_budget, st);
      cudaStreamWaitEvent(st, ev_join, 0);
      tgtQ<<<tgtV, kTgtThreads, kTgtSmem, st>>>(Qp, splitQ, n, rpcV, bb, SU, tau, T, Cs, tick,
                                                 thr, it == h.iters - 1 ? Qs : nullptr, sk,
                                                 planQ.C, planQ.U, planQ.G, planQ.S, stat,
                                                 naive_w);
      tern_kernel<<<Wn, 256, 0, st>>>(T, n, bb, thr, Vm, Vs, pC, Wn, BopV);
      if (tr) {
        u64* at = tr + 2 * (size_t)n + (size_t)it * 2 * ((size_t)m + n);
        record(at, Um, Us, m);
        record(at + 2 * (size_t)m, Vm, Vs, n);
      }
    }
    gram_kernel<<<gblocks, gthreads, 0, st>>>(pC, Wn, bb, h.w, GV);
    rpart_kernel<<<rpartV, 256, 0, st>>>(Qs, n, bb, Vm, Vs, h.w, Rp);
    dsolve_kernel<<<1, 256, 0, st>>>(GU, GV, Rp, rpartV, bb, scal, c0, h.D, h.energy, dblk);
    if (n % 4 == 0)
      deflate_kernel<true><<<dim3((m + kDefRows - 1) / kDefRows, nch), 256, kDefSmem, st>>>(
          R, m, n, Um, Us, Vm, Vs, dblk, bb, h.w, rhop);
    else
      deflate_kernel<false><<<dim3((m + kDefRows - 1) / kDefRows, nch), 256, kDefSmem, st>>>(
          R, m, n, Um, Us, Vm, Vs, dblk, bb, h.w, rhop);
    chk();
  }
  int* status = status_word_ptr();
  if (status) set_status_kernel<<<1, 1, 0, st>>>(bad, status);
  chk();
  if (cudaFreeAsync(ws, st) != cudaSuccess && rc == EXTERND_OK) rc = EXTERND_ERR_CUDA;
  return rc;
}

// ---- CUDA-graph replay of repeated decompositions -----------------------------
// One decomposition is a fixed sequence of ~40 launches per block.  A call
// identical to an earlier one (same pointers, sizes and knobs, same device)
// is captured once into a CUDA graph on a private stream and replayed from
// then on; the first occurrence runs directly, which also loads every kernel
// before any capture.  Traced calls, and calls on a stream that is itself
// being captured, always run directly.  EXTERND_NO_GRAPH=1 disables replay.
namespace {

struct GraphKey {
  BlockHostArgs h;
  int dev, no_tma;
  bool operator==(const GraphKey& o) const {
    return h.A == o.h.A && h.m == o.h.m && h.n == o.h.n && h.k == o.h.k && h.tau == o.h.tau &&
           h.iters == o.h.iters && h.w == o.h.w && h.block == o.h.block &&
           h.flags == o.h.flags && h.packed_B == o.h.packed_B && h.packed_C == o.h.packed_C &&
           h.D == o.h.D && h.energy == o.h.energy && h.wait_budget == o.h.wait_budget &&
           dev == o.dev && no_tma == o.no_tma;
  }
};

struct GraphSlot {
  GraphKey key;
  cudaGraphExec_t exec = nullptr;
  cudaStream_t cap = nullptr;
  cudaEvent_t ev_in = nullptr, ev_out = nullptr;
};

constexpr size_t kGraphSlots = 8;
std::mutex g_graph_mu;
std::vector<GraphSlot> g_graphs;  // most recently used last
std::vector<GraphKey> g_seen;     // calls seen once, not yet captured

bool env_on(const char* name) {
  const char* v = getenv(name);
  return v && v[0] == '1';
}

void release(GraphSlot& g) {
  if (g.exec) cudaGraphExecDestroy(g.exec);
  if (g.ev_in) cudaEventDestroy(g.ev_in);
  if (g.ev_out) cudaEventDestroy(g.ev_out);
  if (g.cap) cudaStreamDestroy(g.cap);
  g = GraphSlot{};
}

// Runs block_enqueue on st with a freshly made side stream (direct path).
int enqueue_direct(const BlockHostArgs& h, cudaStream_t st) {
  cudaStream_t side = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  if (cudaStreamCreateWithFlags(&side, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&ev_fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&ev_join, cudaEventDisableTiming) != cudaSuccess) {
    cudaGetLastError();
    if (side) cudaStreamDestroy(side);
    if (ev_fork) cudaEventDestroy(ev_fork);
    return EXTERND_ERR_CUDA;
  }
  const int rc = block_enqueue(h, st, side, ev_fork, ev_join);
  // every side-stream launch is joined into st; the handles go once the
  // queued work no longer needs them (destruction is deferred by CUDA)
  cudaEventDestroy(ev_fork);
  cudaEventDestroy(ev_join);
  cudaStreamDestroy(side);
  return rc;
}

// Captures the decomposition on a private stream into g.exec.
int capture(GraphSlot& g, const BlockHostArgs& h) {
  cudaStream_t side = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  cudaGraph_t graph = nullptr;
  int rc = EXTERND_ERR_CUDA;
  if (cudaStreamCreateWithFlags(&g.cap, cudaStreamNonBlocking) == cudaSuccess &&
      cudaStreamCreateWithFlags(&side, cudaStreamNonBlocking) == cudaSuccess &&
      cudaEventCreateWithFlags(&ev_fork, cudaEventDisableTiming) == cudaSuccess &&
      cudaEventCreateWithFlags(&ev_join, cudaEventDisableTiming) == cudaSuccess &&
      cudaEventCreateWithFlags(&g.ev_in, cudaEventDisableTiming) == cudaSuccess &&
      cudaEventCreateWithFlags(&g.ev_out, cudaEventDisableTiming) == cudaSuccess &&
      cudaStreamBeginCapture(g.cap, cudaStreamCaptureModeThreadLocal) == cudaSuccess) {
    const int erc = block_enqueue(h, g.cap, side, ev_fork, ev_join);
    const cudaError_t ce = cudaStreamEndCapture(g.cap, &graph);
    if (erc == EXTERND_OK && ce == cudaSuccess && graph &&
        cudaGraphInstantiate(&g.exec, graph, 0) == cudaSuccess)
      rc = EXTERND_OK;
  }
  if (graph) cudaGraphDestroy(graph);
  if (ev_fork) cudaEventDestroy(ev_fork);
  if (ev_join) cudaEventDestroy(ev_join);
  if (side) cudaStreamDestroy(side);
  if (rc != EXTERND_OK) {
    cudaGetLastError();
    release(g);
  }
  return rc;
}

// Replays g on st: the private stream waits for st, runs the graph, and st
// waits for it in turn.
int replay(GraphSlot& g, cudaStream_t st) {
  if (cudaEventRecord(g.ev_in, st) != cudaSuccess ||
      cudaStreamWaitEvent(g.cap, g.ev_in, 0) != cudaSuccess ||
      cudaGraphLaunch(g.exec, g.cap) != cudaSuccess ||
      cudaEventRecord(g.ev_out, g.cap) != cudaSuccess ||
      cudaStreamWaitEvent(st, g.ev_out, 0) != cudaSuccess) {
    cudaGetLastError();
    return EXTERND_ERR_CUDA;
  }
  return EXTERND_OK;
}

}  // namespace

int block_decompose(const BlockHostArgs& h, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (h.ntrace > 0 || env_on("EXTERND_NO_GRAPH") ||
      cudaStreamIsCapturing(st, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) {
    cudaGetLastError();
    return enqueue_direct(h, st);
  }
  GraphKey key{h, 0, getenv("EXTERND_CONTRACT_NO_TMA") ? 1 : 0};
  cudaGetDevice(&key.dev);
  std::lock_guard<std::mutex> lock(g_graph_mu);
  for (size_t i = 0; i < g_graphs.size(); ++i)
    if (g_graphs[i].key == key) {
      std::rotate(g_graphs.begin() + i, g_graphs.begin() + i + 1, g_graphs.end());
      return replay(g_graphs.back(), st);
    }
  bool seen = false;
  for (const GraphKey& k2 : g_seen) seen = seen || k2 == key;
  if (!seen) {
    if (g_seen.size() >= kGraphSlots) g_seen.erase(g_seen.begin());
    g_seen.push_back(key);
    return enqueue_direct(h, st);
  }
  GraphSlot g;
  g.key = key;
  if (capture(g, h) != EXTERND_OK) return enqueue_direct(h, st);
  if (g_graphs.size() >= kGraphSlots) {
    const int edev = g_graphs.front().key.dev;
    release(g_graphs.front());
    g_graphs.erase(g_graphs.begin());
    // the evicted graph's workspace goes back to the device once it is idle
    int cur = 0;
    if (cudaGetDevice(&cur) == cudaSuccess && cur == edev) cudaDeviceGraphMemTrim(edev);
    cudaGetLastError();
  }
  g_graphs.push_back(g);
  return replay(g_graphs.back(), st);
}

int block_release_graphs() {
  std::lock_guard<std::mutex> lock(g_graph_mu);
  bool devs[64] = {};
  for (GraphSlot& g : g_graphs) {
    if (g.key.dev >= 0 && g.key.dev < 64) devs[g.key.dev] = true;
    release(g);
  }
  g_graphs.clear();
  g_seen.clear();
  int rc = EXTERND_OK;
  for (int d = 0; d < 64; ++d)
    if (devs[d] && cudaDeviceGraphMemTrim(d) != cudaSuccess) {
      cudaGetLastError();
      rc = EXTERND_ERR_CUDA;
    }
  return rc;
}

}  // namespace externd
