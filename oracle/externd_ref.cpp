// ExTernD CPU oracle -- TEST INFRASTRUCTURE ONLY.
//
// A plain, slow, single-threaded statement of the expanded-rank ternary
// decomposition, used only by the tests, by the package's smoke check and by
// the benchmark's CPU-baseline leg to check and time the CUDA path.  The CUDA
// library never links, loads or calls this file, and this file shares no code
// with it.
//
// Sources (web pages on arXiv:2607.13511, "ExTernD: Expanded-Rank Ternary
// Decomposition"):
//   [REV]  "Paper Review: ExTernD ..." (romaanj.github.io), sections "Method"
//          and "Key idea".
//   [PITH] "Pith review of ExTernD ..." (pith.science), "What carries the
//          argument", the referee report (paper Sec. 2.3 greedy ALS,
//          Sec. 2.4 block-ALS with Eq. 3, Sec. 2.5 importance weighting,
//          Appendix A Prop. 1 and Prop. 2) and "Assumptions & free
//          parameters" (Eq. 2 threshold, Eq. 5 packing).
//   [ABS]  the paper's abstract as reprinted on arxivlens.com.
//
// Readings taken where the pages leave a step open (each is listed in the
// design notes with its reason):
//   * T_tau(x)_j = sign(x_j) if |x_j| > tau * s(x) else 0, strict, with the
//     statistic s computed in fp64 over the whole vector: s = rms(x) by
//     default; s = mean |x| in the threshold variant ([REV] "Method" quotes
//     zero shares, tau = 0.7 -> ~41% and tau = 2.0 -> ~87%, that a mean-|x|
//     statistic reproduces on Gaussian data and rms does not).
//   * Naive weighted V-step (the ablation [REV] "Validation" names):
//     v = T_tau(W R^T u); the default (corrected) V-step thresholds R^T u.
//   * Refinement sweeps (backfitting, [REV] "Results"): component l is added
//     back onto the residual and refit by ALS from its own v; the refit
//     replaces it only if it removes more than the old pattern with its
//     scale re-solved on that residual, so no sweep step raises the residual;
//     the single-entry step applies as in the greedy pass.
//   * The residual R is kept in the input's precision (fp32).  A deflation
//     R_ij <- R_ij - u_i v_j d is one IEEE fp32 add or subtract of the fp32
//     scale d (u_i v_j is +-1 or 0), never fused with anything else.
//   * Every other reduction (matrix-vector products, norms, scales) is fp64.
//   * Ties in every argmax go to the lowest (row-major) index.
//   * Weighted mode: the u-step thresholds y = R (w o v); the v-step
//     thresholds z = R^T u unweighted (per-column weights do not move the
//     column-wise least-squares minimiser); d = u^T R W v / (|u|^2 v^T W v).
//   * The single-entry safeguard scores entries by w_j R_ij^2; in weighted
//     mode that score is formed in fp32 as (R_ij * R_ij) * w_j so that the
//     argmax is decided in the same precision as the kernel's.
//   * Block mode: eps = 1e-6 * trace(G) / b for each b x b Gram system G
//     (1.0 when the trace is zero); U-step target R W V (V^T W V + eps I)^-1;
//     V-step target ((U^T U + eps I)^-1 U^T R)^T (Eq. 3); joint scales
//     D = (G + eps I)^-1 r with G = (U^T U) o (V^T W V), r_l = u_l^T R W v_l;
//     b ordered rank-1 deflations; no safeguard.
//
// Build: g++ -O2 -ffp-contract=off -fno-fast-math -shared -fPIC (see build.py).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

inline double wt(const float* w, int64_t j) { return w ? (double)w[j] : 1.0; }

// Cholesky factorisation and solve of a small symmetric positive definite
// system, fp64, in place.  Returns false if a pivot is not positive.
bool chol_solve(std::vector<double>& G, int64_t b, std::vector<double>& rhs, int64_t nrhs) {
  // G is b x b row-major; rhs is b x nrhs row-major.
  for (int64_t i = 0; i < b; ++i) {
    for (int64_t j = 0; j <= i; ++j) {
      double s = G[i * b + j];
      for (int64_t p = 0; p < j; ++p) s -= G[i * b + p] * G[j * b + p];
      if (i == j) {
        if (!(s > 0.0)) return false;
        G[i * b + i] = std::sqrt(s);
      } else {
        G[i * b + j] = s / G[j * b + j];
      }
    }
  }
  for (int64_t c = 0; c < nrhs; ++c) {
    for (int64_t i = 0; i < b; ++i) {  // L y = r
      double s = rhs[i * nrhs + c];
      for (int64_t p = 0; p < i; ++p) s -= G[i * b + p] * rhs[p * nrhs + c];
      rhs[i * nrhs + c] = s / G[i * b + i];
    }
    for (int64_t i = b - 1; i >= 0; --i) {  // L^T x = y
      double s = rhs[i * nrhs + c];
      for (int64_t p = i + 1; p < b; ++p) s -= G[p * b + i] * rhs[p * nrhs + c];
      rhs[i * nrhs + c] = s / G[i * b + i];
    }
  }
  return true;
}

double ridge_eps(const std::vector<double>& G, int64_t b) {
  double tr = 0.0;
  for (int64_t i = 0; i < b; ++i) tr += G[i * b + i];
  return tr > 0.0 ? 1e-6 * tr / (double)b : 1.0;
}

}  // namespace

extern "C" {

// T_tau, the adaptive ternarisation operator ([PITH] Eq. 2 via "Assumptions &
// free parameters"; [REV] "Method": tau sets the share of zeros).  Writes the
// ternary codes and returns the threshold tau * s(x), s = rms (stat 0) or
// mean |x| (stat 1).
double orc_ternarize2(const double* x, int64_t len, double tau, int stat, int8_t* out) {
  double s = 0.0;
  for (int64_t j = 0; j < len; ++j) s += stat == 1 ? std::fabs(x[j]) : x[j] * x[j];
  double thr = 0.0;
  if (len > 0) thr = stat == 1 ? tau * (s / (double)len) : tau * std::sqrt(s / (double)len);
  for (int64_t j = 0; j < len; ++j) {
    double a = std::fabs(x[j]);
    out[j] = (a > thr) ? (x[j] > 0.0 ? 1 : -1) : 0;
  }
  return thr;
}

double orc_ternarize(const double* x, int64_t len, double tau, int8_t* out) {
  return orc_ternarize2(x, len, tau, 0, out);
}

// ALS u half-step ([PITH] referee summary, Sec. 2.3: ternarise against the
// current residual): y = R (w o v), u = T_tau(y).  Returns the threshold.
double orc_u_step2(const float* R, int64_t m, int64_t n, const int8_t* v, const float* w,
                   double tau, int stat, double* y, int8_t* u) {
  for (int64_t i = 0; i < m; ++i) {
    double s = 0.0;
    const float* row = R + i * n;
    for (int64_t j = 0; j < n; ++j)
      if (v[j]) s += (double)row[j] * ((double)v[j] * wt(w, j));
    y[i] = s;
  }
  return orc_ternarize2(y, m, tau, stat, u);
}

double orc_u_step(const float* R, int64_t m, int64_t n, const int8_t* v, const float* w,
                  double tau, double* y, int8_t* u) {
  return orc_u_step2(R, m, n, v, w, tau, 0, y, u);
}

// ALS v half-step: z = R^T u, v = T_tau(z) -- or, for the naive weighted
// V-step, v = T_tau(w o z).  z is returned unweighted either way.  Returns
// the threshold.
double orc_v_step2(const float* R, int64_t m, int64_t n, const int8_t* u, const float* w,
                   double tau, int stat, int naive, double* z, int8_t* v) {
  for (int64_t j = 0; j < n; ++j) z[j] = 0.0;
  for (int64_t i = 0; i < m; ++i) {
    if (!u[i]) continue;
    const float* row = R + i * n;
    for (int64_t j = 0; j < n; ++j) z[j] += (double)u[i] * (double)row[j];
  }
  if (!naive || !w) return orc_ternarize2(z, n, tau, stat, v);
  std::vector<double> wz(n);
  for (int64_t j = 0; j < n; ++j) wz[j] = (double)w[j] * z[j];
  return orc_ternarize2(wz.data(), n, tau, stat, v);
}

double orc_v_step(const float* R, int64_t m, int64_t n, const int8_t* u, double tau,
                  double* z, int8_t* v) {
  return orc_v_step2(R, m, n, u, nullptr, tau, 0, 0, z, v);
}

// Row energies rho_i = sum_j w_j R_ij^2; returns the index of the largest
// (lowest index on ties).  The component's starting row.
int64_t orc_row_norms(const float* R, int64_t m, int64_t n, const float* w, double* rho) {
  int64_t best = 0;
  for (int64_t i = 0; i < m; ++i) {
    double s = 0.0;
    const float* row = R + i * n;
    for (int64_t j = 0; j < n; ++j) s += wt(w, j) * (double)row[j] * (double)row[j];
    rho[i] = s;
    if (s > rho[best]) best = i;
  }
  return best;
}

// Weighted squared Frobenius norm sum_ij w_j R_ij^2 (energy, [PITH]
// "Load-bearing premise": E = 1 - |A - Ahat|^2 / |A|^2).
double orc_sumsq(const float* R, int64_t m, int64_t n, const float* w) {
  double s = 0.0;
  for (int64_t i = 0; i < m; ++i)
    for (int64_t j = 0; j < n; ++j) s += wt(w, j) * (double)R[i * n + j] * (double)R[i * n + j];
  return s;
}

// Best single entry for the safeguard ([PITH] referee major comment 1,
// Appendix A Prop. 2): argmax of w_j R_ij^2, lowest row-major index on ties.
// Writes the score M (as fp64) and returns the flat index.
int64_t orc_entry_max(const float* R, int64_t m, int64_t n, const float* w, double* M) {
  int64_t best = 0;
  if (w) {
    float bs = -1.0f;
    for (int64_t i = 0; i < m; ++i)
      for (int64_t j = 0; j < n; ++j) {
        float r = R[i * n + j];
        float sq = r * r;
        float s = sq * w[j];
        if (s > bs) { bs = s; best = i * n + j; }
      }
    *M = (double)bs;
  } else {
    float ba = -1.0f;
    for (int64_t i = 0; i < m; ++i)
      for (int64_t j = 0; j < n; ++j) {
        float a = std::fabs(R[i * n + j]);
        if (a > ba) { ba = a; best = i * n + j; }
      }
    *M = (double)ba * (double)ba;
  }
  return best;
}

// Closed-form scale and gain ([PITH] "What carries the argument": d = u^T R v /
// (|u|^2 |v|^2); Prop. 1: the residual falls by (u^T R v)^2 / (|u|^2 |v|^2)).
// z must be R^T u for the given u; then u^T R W v = sum_j w_j v_j z_j.
// out[0]=p=u^T R W v, out[1]=n_u, out[2]=n_v, out[3]=|u|^2 v^T W v,
// out[4]=d (exact fp64), out[5]=gain.
void orc_scale(const double* z, const int8_t* u, const int8_t* v, int64_t m, int64_t n,
               const float* w, double* out) {
  double p = 0.0, vw = 0.0;
  int64_t nu = 0, nv = 0;
  for (int64_t i = 0; i < m; ++i) nu += u[i] != 0;
  for (int64_t j = 0; j < n; ++j)
    if (v[j]) {
      ++nv;
      p += wt(w, j) * (double)v[j] * z[j];
      vw += wt(w, j);
    }
  double den = (double)nu * vw;
  out[0] = p;
  out[1] = (double)nu;
  out[2] = (double)nv;
  out[3] = den;
  out[4] = den > 0.0 ? p / den : 0.0;
  out[5] = den > 0.0 ? p * p / den : 0.0;
}

// Rank-1 deflation R <- R - d u v^T ([REV] "Method": deflate the residual
// before the next component), one fp32 add or subtract per touched entry.
void orc_deflate(float* R, int64_t m, int64_t n, const int8_t* u, const int8_t* v, float d) {
  for (int64_t i = 0; i < m; ++i) {
    if (!u[i]) continue;
    float* row = R + i * n;
    for (int64_t j = 0; j < n; ++j) {
      int s = (int)u[i] * (int)v[j];
      if (s > 0) row[j] = row[j] - d;
      else if (s < 0) row[j] = row[j] + d;
    }
  }
}

// Greedy sequential-deflation ALS (paper Sec. 2.3 per [PITH]; [REV] "Method"
// and "Key idea"), with the best-single-entry safeguard of Prop. 2.
// flags: bit 0 = mean-|x| threshold statistic, bit 1 = naive weighted V-step.
// Outputs: U k x m and V k x n ternary codes (row c = component c), D[k],
// energy[k] = 1 - |R_{c+1}|_W^2 / |A|_W^2, init_row[k] (row whose ternarised
// copy started the component), fallback[k] (1 when the safeguard fired).
// After the greedy pass, `sweeps` refinement sweeps (orc_refine_sweep) run
// over the k components; sweep_energy[s] (may be NULL when sweeps == 0) is the
// energy after sweep s and sweep_flags[s*k + l] the step's flags.  energy[]
// keeps the greedy pass's trace.  Returns the number of safeguard
// activations of the greedy pass.
int64_t orc_refine_sweep(float* R, int64_t m, int64_t n, int64_t k, double tau, int iters,
                         const float* w, int flags, int8_t* U, int8_t* V, float* D,
                         uint8_t* step_flags);

int64_t orc_decompose_seq2(const float* A, int64_t m, int64_t n, int64_t k, double tau, int iters,
                           const float* w, int flags, int sweeps, int8_t* U, int8_t* V, float* D,
                           double* energy, int64_t* init_row, uint8_t* fallback,
                           double* sweep_energy, uint8_t* sweep_flags) {
  const int stat = flags & 1, naive = (flags >> 1) & 1;
  std::vector<float> R(A, A + m * n);
  std::vector<double> rho(m), y(m), z(n), rowd(n);
  std::vector<int8_t> u(m), v(n);
  const double E0 = orc_sumsq(A, m, n, w);
  int64_t nfb = 0;
  bool zero = false;
  for (int64_t c = 0; c < k; ++c) {
    int8_t* Uc = U + c * m;
    int8_t* Vc = V + c * n;
    if (!zero) {
      double M = 0.0;
      int64_t flat = orc_entry_max(R.data(), m, n, w, &M);
      if (M == 0.0) zero = true;
      if (!zero) {
        int64_t istar = orc_row_norms(R.data(), m, n, w, rho.data());
        init_row[c] = istar;
        for (int64_t j = 0; j < n; ++j) rowd[j] = (double)R[istar * n + j];
        orc_ternarize2(rowd.data(), n, tau, stat, v.data());
        for (int t = 0; t < iters; ++t) {
          orc_u_step2(R.data(), m, n, v.data(), w, tau, stat, y.data(), u.data());
          orc_v_step2(R.data(), m, n, u.data(), w, tau, stat, naive, z.data(), v.data());
        }
        double sc[6];
        orc_scale(z.data(), u.data(), v.data(), m, n, w, sc);
        float d;
        if (sc[5] < M) {  // safeguard: single best entry removal
          std::fill(u.begin(), u.end(), 0);
          std::fill(v.begin(), v.end(), 0);
          int64_t ip = flat / n, jp = flat % n;
          u[ip] = 1;
          v[jp] = 1;
          d = R[flat];
          fallback[c] = 1;
          ++nfb;
        } else {
          d = (float)sc[4];
          fallback[c] = 0;
        }
        orc_deflate(R.data(), m, n, u.data(), v.data(), d);
        std::memcpy(Uc, u.data(), m);
        std::memcpy(Vc, v.data(), n);
        D[c] = d;
        energy[c] = E0 > 0.0 ? 1.0 - orc_sumsq(R.data(), m, n, w) / E0 : 1.0;
        continue;
      }
    }
    // R is identically zero: the remaining components are empty.
    std::memset(Uc, 0, m);
    std::memset(Vc, 0, n);
    D[c] = 0.0f;
    energy[c] = 1.0;
    init_row[c] = -1;
    fallback[c] = 0;
  }
  for (int sw = 0; sw < sweeps; ++sw) {
    orc_refine_sweep(R.data(), m, n, k, tau, iters, w, flags, U, V, D, sweep_flags + sw * k);
    sweep_energy[sw] = E0 > 0.0 ? 1.0 - orc_sumsq(R.data(), m, n, w) / E0 : 1.0;
  }
  return nfb;
}

int64_t orc_decompose_seq(const float* A, int64_t m, int64_t n, int64_t k, double tau, int iters,
                          const float* w, int8_t* U, int8_t* V, float* D, double* energy,
                          int64_t* init_row, uint8_t* fallback) {
  return orc_decompose_seq2(A, m, n, k, tau, iters, w, 0, 0, U, V, D, energy, init_row, fallback,
                            nullptr, nullptr);
}

// One refinement sweep over the k components on the residual R (backfitting;
// [REV] "Results": sweeps add ~0.4 energy points and cut the rank a target
// needs by 4-8%).  For l = 0 .. k-1:
//   1. add component l back: R <- R + d_l u_l v_l^T (one fp32 add or
//      subtract per touched entry);
//   2. the old pattern, rescaled on this residual: p_o = u_l^T R W v_l,
//      gain g_o = p_o^2 / (|u_l|^2 v_l^T W v_l), scale p_o / (|u_l|^2 v_l^T W v_l);
//   3. the refit: `iters` ALS rounds from v = v_l, gain g_n and scale as in
//      the greedy pass;
//   4. the refit replaces the old pattern only if g_n > g_o; if the larger
//      gain is below the best single entry's w_j R_ij^2, that entry is taken
//      instead (Prop. 2);
//   5. deflate with the choice and store it as component l.
// Since the old pattern with its re-solved scale removes at least what d_l
// did, no step raises |R|_W^2 (up to fp32 rounding of the updates).
// step_flags[l]: bit 0 = single entry, bit 1 = old pattern kept.  Returns the
// number of single-entry steps.
int64_t orc_refine_sweep(float* R, int64_t m, int64_t n, int64_t k, double tau, int iters,
                         const float* w, int flags, int8_t* U, int8_t* V, float* D,
                         uint8_t* step_flags) {
  const int stat = flags & 1, naive = (flags >> 1) & 1;
  std::vector<double> y(m), z(n);
  std::vector<int8_t> u(m), v(n);
  int64_t nsingle = 0;
  for (int64_t l = 0; l < k; ++l) {
    int8_t* Ul = U + l * m;
    int8_t* Vl = V + l * n;
    orc_deflate(R, m, n, Ul, Vl, -D[l]);  // add back
    double p_old = 0.0, vw_old = 0.0;
    int64_t nu_old = 0;
    for (int64_t i = 0; i < m; ++i) {
      if (!Ul[i]) continue;
      ++nu_old;
      for (int64_t j = 0; j < n; ++j)
        if (Vl[j]) p_old += (double)Ul[i] * (double)R[i * n + j] * wt(w, j) * (double)Vl[j];
    }
    for (int64_t j = 0; j < n; ++j)
      if (Vl[j]) vw_old += wt(w, j);
    const double den_old = (double)nu_old * vw_old;
    const double g_old = den_old > 0.0 ? p_old * p_old / den_old : 0.0;
    std::memcpy(v.data(), Vl, n);
    for (int t = 0; t < iters; ++t) {
      orc_u_step2(R, m, n, v.data(), w, tau, stat, y.data(), u.data());
      orc_v_step2(R, m, n, u.data(), w, tau, stat, naive, z.data(), v.data());
    }
    double sc[6];
    orc_scale(z.data(), u.data(), v.data(), m, n, w, sc);
    double M = 0.0;
    const int64_t flat = orc_entry_max(R, m, n, w, &M);
    uint8_t fl = 0;
    float d;
    const double g_best = sc[5] > g_old ? sc[5] : g_old;
    if (g_best < M) {  // the best single entry beats both patterns
      for (int64_t i = 0; i < m; ++i) u[i] = 0;
      for (int64_t j = 0; j < n; ++j) v[j] = 0;
      u[flat / n] = 1;
      v[flat % n] = 1;
      d = R[flat];
      fl = 1;
      ++nsingle;
    } else if (sc[5] > g_old) {
      d = (float)sc[4];
    } else {
      std::memcpy(u.data(), Ul, m);
      std::memcpy(v.data(), Vl, n);
      d = den_old > 0.0 ? (float)(p_old / den_old) : 0.0f;
      fl = 2;
    }
    orc_deflate(R, m, n, u.data(), v.data(), d);
    std::memcpy(Ul, u.data(), m);
    std::memcpy(Vl, v.data(), n);
    D[l] = d;
    step_flags[l] = fl;
  }
  return nsingle;
}

// Replays components [0, upto) onto A with the same fp32 deflation; the
// residual R_upto it yields is the one component `upto` started from.
void orc_replay(const float* A, int64_t m, int64_t n, const int8_t* U, const int8_t* V,
                const float* D, int64_t upto, float* R) {
  std::memcpy(R, A, sizeof(float) * m * n);
  for (int64_t c = 0; c < upto; ++c) orc_deflate(R, m, n, U + c * m, V + c * n, D[c]);
}

// In-place replay of components [from, to) onto R (R must hold R_from).
void orc_replay_range(float* R, int64_t m, int64_t n, const int8_t* U, const int8_t* V,
                      const float* D, int64_t from, int64_t to) {
  for (int64_t c = from; c < to; ++c) orc_deflate(R, m, n, U + c * m, V + c * n, D[c]);
}

// Ahat = B diag(D) C in fp64 ([ABS]: A ~ B diag(D) C).
void orc_reconstruct(const int8_t* U, const int8_t* V, const float* D, int64_t m, int64_t n,
                     int64_t k, double* Ahat) {
  std::memset(Ahat, 0, sizeof(double) * m * n);
  for (int64_t c = 0; c < k; ++c) {
    const int8_t* u = U + c * m;
    const int8_t* v = V + c * n;
    double d = D[c];
    for (int64_t i = 0; i < m; ++i) {
      if (!u[i]) continue;
      for (int64_t j = 0; j < n; ++j)
        if (v[j]) Ahat[i * n + j] += d * (double)(u[i] * v[j]);
    }
  }
}

// Per-matrix rank allocation to an energy target ([REV] "Results": mu is set
// per matrix so that its energy matches a reference quantiser's, 1.97 .. 3.43
// per [PITH] "Assumptions & free parameters").  Greedy deflation fixes
// components in order, so a run at rank k contains every shorter run as its
// prefix; the smallest rank reaching the target is the first c with
// energy[c] >= target, plus one.  Returns 0 when no prefix reaches it.
int64_t orc_rank_for_energy(const double* energy, int64_t k, double target) {
  for (int64_t c = 0; c < k; ++c)
    if (energy[c] >= target) return c + 1;
  return 0;
}

// Indices of the b largest row energies, distinct, descending, lowest index
// first on ties (block-ALS initialisation).
void orc_top_rows(const double* rho, int64_t m, int64_t b, int64_t* rows) {
  std::vector<int64_t> idx(m);
  for (int64_t i = 0; i < m; ++i) idx[i] = i;
  std::stable_sort(idx.begin(), idx.end(),
                   [&](int64_t a, int64_t c) { return rho[a] > rho[c]; });
  for (int64_t l = 0; l < b; ++l) rows[l] = idx[l];
}

// Block-ALS U half-step (paper Sec. 2.4 per [PITH]; the U-step target is the
// reading R W V (V^T W V + eps I)^-1): U = T_col of that target, each column
// thresholded with its own rms over the m rows.  V and U are column-major
// per component: V[l*n + j], U[l*m + i].  targets (m x bb, row-major, may be
// NULL) receives the target, thr (bb, may be NULL) the thresholds.
void orc_block_u_step2(const float* R, int64_t m, int64_t n, int64_t bb, const int8_t* V,
                       const float* w, double tau, int stat, int8_t* U, double* targets,
                       double* thr) {
  std::vector<double> G(bb * bb);
  for (int64_t l = 0; l < bb; ++l)
    for (int64_t l2 = 0; l2 < bb; ++l2) {
      double s = 0.0;
      for (int64_t j = 0; j < n; ++j) s += wt(w, j) * V[l * n + j] * V[l2 * n + j];
      G[l * bb + l2] = s;
    }
  const double eps = ridge_eps(G, bb);
  for (int64_t l = 0; l < bb; ++l) G[l * bb + l] += eps;
  // P = R W V (m x bb); targets are the rows of P solved against G: G t_i = p_i
  std::vector<double> Pt(bb * m);
  for (int64_t i = 0; i < m; ++i)
    for (int64_t l = 0; l < bb; ++l) {
      double s = 0.0;
      for (int64_t j = 0; j < n; ++j)
        if (V[l * n + j]) s += (double)R[i * n + j] * wt(w, j) * V[l * n + j];
      Pt[l * m + i] = s;
    }
  chol_solve(G, bb, Pt, m);
  for (int64_t l = 0; l < bb; ++l) {
    const double t = orc_ternarize2(&Pt[l * m], m, tau, stat, U + l * m);
    if (thr) thr[l] = t;
    if (targets)
      for (int64_t i = 0; i < m; ++i) targets[i * bb + l] = Pt[l * m + i];
  }
}

void orc_block_u_step(const float* R, int64_t m, int64_t n, int64_t bb, const int8_t* V,
                      const float* w, double tau, int8_t* U, double* targets, double* thr) {
  orc_block_u_step2(R, m, n, bb, V, w, tau, 0, U, targets, thr);
}

// Block-ALS V half-step (Eq. 3): V = T_col(((U^T U + eps I)^-1 U^T R)^T); the
// naive weighted V-step thresholds each column of W times that target.
// targets (n x bb) receives the thresholded values (weighted when naive).
void orc_block_v_step2(const float* R, int64_t m, int64_t n, int64_t bb, const int8_t* U,
                       const float* w, double tau, int stat, int naive, int8_t* V,
                       double* targets, double* thr) {
  std::vector<double> G(bb * bb);
  for (int64_t l = 0; l < bb; ++l)
    for (int64_t l2 = 0; l2 < bb; ++l2) {
      double s = 0.0;
      for (int64_t i = 0; i < m; ++i) s += (double)(U[l * m + i] * U[l2 * m + i]);
      G[l * bb + l2] = s;
    }
  const double eps = ridge_eps(G, bb);
  for (int64_t l = 0; l < bb; ++l) G[l * bb + l] += eps;
  std::vector<double> Q(bb * n, 0.0);  // U^T R
  for (int64_t l = 0; l < bb; ++l)
    for (int64_t i = 0; i < m; ++i) {
      const int8_t ui = U[l * m + i];
      if (!ui) continue;
      for (int64_t j = 0; j < n; ++j) Q[l * n + j] += (double)ui * (double)R[i * n + j];
    }
  chol_solve(G, bb, Q, n);
  if (naive && w)
    for (int64_t l = 0; l < bb; ++l)
      for (int64_t j = 0; j < n; ++j) Q[l * n + j] *= (double)w[j];
  for (int64_t l = 0; l < bb; ++l) {
    const double t = orc_ternarize2(&Q[l * n], n, tau, stat, V + l * n);
    if (thr) thr[l] = t;
    if (targets)
      for (int64_t j = 0; j < n; ++j) targets[j * bb + l] = Q[l * n + j];
  }
}

void orc_block_v_step(const float* R, int64_t m, int64_t n, int64_t bb, const int8_t* U,
                      double tau, int8_t* V, double* targets, double* thr) {
  orc_block_v_step2(R, m, n, bb, U, nullptr, tau, 0, 0, V, targets, thr);
}

// Joint block scales: (G + eps I) D = r with G = (U^T U) o (V^T W V) and
// r_l = u_l^T R W v_l, over the components whose u and v are both nonzero
// (the others take d = 0).  Also returns G (raw, bb x bb) and r.
void orc_block_scales(const float* R, int64_t m, int64_t n, int64_t bb, const int8_t* U,
                      const int8_t* V, const float* w, double* D, double* Graw, double* r) {
  std::vector<double> GU(bb * bb), GV(bb * bb), G(bb * bb);
  for (int64_t l = 0; l < bb; ++l)
    for (int64_t l2 = 0; l2 < bb; ++l2) {
      double su = 0.0, sv = 0.0;
      for (int64_t i = 0; i < m; ++i) su += (double)(U[l * m + i] * U[l2 * m + i]);
      for (int64_t j = 0; j < n; ++j) sv += wt(w, j) * V[l * n + j] * V[l2 * n + j];
      GU[l * bb + l2] = su;
      GV[l * bb + l2] = sv;
    }
  for (int64_t l = 0; l < bb; ++l) {
    double s = 0.0;
    for (int64_t i = 0; i < m; ++i) {
      const int8_t ui = U[l * m + i];
      if (!ui) continue;
      for (int64_t j = 0; j < n; ++j)
        if (V[l * n + j]) s += (double)ui * (double)R[i * n + j] * wt(w, j) * V[l * n + j];
    }
    r[l] = s;
  }
  for (int64_t l = 0; l < bb * bb; ++l) G[l] = GU[l] * GV[l];
  for (int64_t l = 0; l < bb * bb; ++l) Graw[l] = G[l];
  const double eps = ridge_eps(G, bb);
  std::vector<int64_t> act;
  for (int64_t l = 0; l < bb; ++l)
    if (GU[l * bb + l] > 0.0 && GV[l * bb + l] > 0.0) act.push_back(l);
  for (int64_t l = 0; l < bb; ++l) D[l] = 0.0;
  if (!act.empty()) {
    const int64_t na = (int64_t)act.size();
    std::vector<double> Ga(na * na), ra(na);
    for (int64_t a = 0; a < na; ++a) {
      ra[a] = r[act[a]];
      for (int64_t c = 0; c < na; ++c) Ga[a * na + c] = G[act[a] * bb + act[c]];
      Ga[a * na + a] += eps;
    }
    chol_solve(Ga, na, ra, 1);
    for (int64_t a = 0; a < na; ++a) D[act[a]] = ra[a];
  }
}

// Starting V of a block: column l = T_tau(R[rows[l], :]) (each row's own
// statistic).
void orc_block_init2(const float* R, int64_t m, int64_t n, int64_t bb, const int64_t* rows,
                     double tau, int stat, int8_t* V) {
  std::vector<double> row(n);
  for (int64_t l = 0; l < bb; ++l) {
    for (int64_t j = 0; j < n; ++j) row[j] = (double)R[rows[l] * n + j];
    orc_ternarize2(row.data(), n, tau, stat, V + l * n);
  }
}

void orc_block_init(const float* R, int64_t m, int64_t n, int64_t bb, const int64_t* rows,
                    double tau, int8_t* V) {
  orc_block_init2(R, m, n, bb, rows, tau, 0, V);
}

// Block-ALS with decorrelated least-squares targets (paper Sec. 2.4, Eq. 3 per
// [PITH]; [REV] "Method": batched block-ALS).  Fits bb = min(b, k - c0)
// components per sweep: start from the bb largest-energy rows, `iters`
// rounds of the U and V half-steps above, joint scales, then bb ordered
// rank-1 deflations.  Energy per component from the closed form
// |R|^2 - 2 sum d_l r_l + sum d_l d_l' G_ll' over the block prefix.
void orc_decompose_block2(const float* A, int64_t m, int64_t n, int64_t k, double tau,
                          int iters, const float* w, int flags, int64_t b, int8_t* U, int8_t* V,
                          float* D, double* energy, int64_t* init_row) {
  const int stat = flags & 1, naive = (flags >> 1) & 1;
  std::vector<float> R(A, A + m * n);
  const double E0 = orc_sumsq(A, m, n, w);
  std::vector<double> rho(m);
  for (int64_t c0 = 0; c0 < k; c0 += b) {
    const int64_t bb = std::min(b, k - c0);
    orc_row_norms(R.data(), m, n, w, rho.data());
    std::vector<int64_t> rows(bb);
    orc_top_rows(rho.data(), m, bb, rows.data());
    for (int64_t l = 0; l < bb; ++l) init_row[c0 + l] = rows[l];
    std::vector<int8_t> Ub(bb * m, 0), Vb(bb * n, 0);
    orc_block_init2(R.data(), m, n, bb, rows.data(), tau, stat, Vb.data());
    for (int t = 0; t < iters; ++t) {
      orc_block_u_step2(R.data(), m, n, bb, Vb.data(), w, tau, stat, Ub.data(), nullptr, nullptr);
      orc_block_v_step2(R.data(), m, n, bb, Ub.data(), w, tau, stat, naive, Vb.data(), nullptr,
                        nullptr);
    }
    std::vector<double> dsol(bb), Graw(bb * bb), r(bb);
    orc_block_scales(R.data(), m, n, bb, Ub.data(), Vb.data(), w, dsol.data(), Graw.data(),
                     r.data());
    std::vector<float> dl(bb);
    for (int64_t l = 0; l < bb; ++l) dl[l] = (float)dsol[l];
    const double base = orc_sumsq(R.data(), m, n, w);
    for (int64_t l = 0; l < bb; ++l) {
      orc_deflate(R.data(), m, n, &Ub[l * m], &Vb[l * n], dl[l]);
      std::memcpy(U + (c0 + l) * m, &Ub[l * m], m);
      std::memcpy(V + (c0 + l) * n, &Vb[l * n], n);
      D[c0 + l] = dl[l];
      double e = base;
      for (int64_t a = 0; a <= l; ++a) {
        e -= 2.0 * (double)dl[a] * r[a];
        for (int64_t c = 0; c <= l; ++c) e += (double)dl[a] * (double)dl[c] * Graw[a * bb + c];
      }
      energy[c0 + l] = E0 > 0.0 ? 1.0 - e / E0 : 1.0;
    }
  }
}

void orc_decompose_block(const float* A, int64_t m, int64_t n, int64_t k, double tau, int iters,
                         const float* w, int64_t b, int8_t* U, int8_t* V, float* D,
                         double* energy, int64_t* init_row) {
  orc_decompose_block2(A, m, n, k, tau, iters, w, 0, b, U, V, D, energy, init_row);
}

// Inference with the factors ([REV] "Significance": inference stays
// multiplication-free -- ternary adds and subtracts plus one scale per
// component; "Limitations" / "Future work": a fused inference kernel is the
// missing piece): for each of the nb input vectors x (rows of X, nb x n),
// t_c = sum_j C_cj x_j, then y_i = sum_c B_ic D_c t_c, in fp64.  U is k x m
// (row c = column c of B), V is k x n (row c of C); Y is nb x m.
void orc_ternary_apply(const int8_t* U, const int8_t* V, const float* D, int64_t m, int64_t n,
                       int64_t k, const float* X, int64_t nb, double* Y) {
  std::vector<double> t(k);
  for (int64_t b = 0; b < nb; ++b) {
    const float* x = X + b * n;
    for (int64_t c = 0; c < k; ++c) {
      double s = 0.0;
      for (int64_t j = 0; j < n; ++j)
        if (V[c * n + j]) s += (double)V[c * n + j] * (double)x[j];
      t[c] = s;
    }
    double* y = Y + b * m;
    for (int64_t i = 0; i < m; ++i) y[i] = 0.0;
    for (int64_t c = 0; c < k; ++c) {
      const double sc = (double)D[c] * t[c];
      for (int64_t i = 0; i < m; ++i)
        if (U[c * m + i]) y[i] += (double)U[c * m + i] * sc;
    }
  }
}

}  // extern "C"
