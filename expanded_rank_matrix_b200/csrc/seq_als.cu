// Greedy sequential-deflation ALS for ExTernD: the host side (planning and launch) of the persistent kernel in seq_kernel.cuh.
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
#include "seq_kernel.cuh"

namespace externd {

__device__ int g_status = 0;  // per-device sticky status (first error wins)

int* status_word_ptr() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
  return (int*)p;
}

EXTERND_SEQ_KERNELS(false, false, extern)
EXTERND_SEQ_KERNELS(true, false, extern)
EXTERND_SEQ_KERNELS(false, true, extern)
EXTERND_SEQ_KERNELS(true, true, extern)

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

template <int NQL, bool HYB, bool FULL>
static cudaError_t launch_one(const SeqArgs& args, size_t smem, cudaStream_t st,
                              int* max_clusters_out, bool query_only) {
  auto kern = seq_als_kernel<NQL, HYB, FULL>;
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

template <bool HYB, bool FULL>
static cudaError_t dispatch_t(int NQL, const SeqArgs& args, size_t smem, cudaStream_t st, int* mc,
                              bool query_only) {
  switch (NQL) {
    case 1: return launch_one<1, HYB, FULL>(args, smem, st, mc, query_only);
    case 2: return launch_one<2, HYB, FULL>(args, smem, st, mc, query_only);
    case 3: return launch_one<3, HYB, FULL>(args, smem, st, mc, query_only);
    case 4: return launch_one<4, HYB, FULL>(args, smem, st, mc, query_only);
    case 5: return launch_one<5, HYB, FULL>(args, smem, st, mc, query_only);
    case 6: return launch_one<6, HYB, FULL>(args, smem, st, mc, query_only);
    case 8: return launch_one<8, HYB, FULL>(args, smem, st, mc, query_only);
    default: return cudaErrorInvalidValue;
  }
}

// HYB is chosen from the arguments (rows outside shared memory need the
// hybrid kernel), FULL from the variant flags and the sweep count.
static cudaError_t dispatch(int NQL, const SeqArgs& args, size_t smem, cudaStream_t st, int* mc,
                            bool query_only) {
  const bool full = args.flags != 0 || args.sweeps != 0;
  if (args.SR < args.TRmax)
    return full ? dispatch_t<true, true>(NQL, args, smem, st, mc, query_only)
                : dispatch_t<true, false>(NQL, args, smem, st, mc, query_only);
  return full ? dispatch_t<false, true>(NQL, args, smem, st, mc, query_only)
              : dispatch_t<false, false>(NQL, args, smem, st, mc, query_only);
}

template <bool HYB, bool FULL>
static size_t static_smem_t(int NQL) {
  cudaFuncAttributes fa = {};
  cudaError_t e = cudaErrorInvalidValue;
  switch (NQL) {
    case 1: e = cudaFuncGetAttributes(&fa, seq_als_kernel<1, HYB, FULL>); break;
    case 2: e = cudaFuncGetAttributes(&fa, seq_als_kernel<2, HYB, FULL>); break;
    case 3: e = cudaFuncGetAttributes(&fa, seq_als_kernel<3, HYB, FULL>); break;
    case 4: e = cudaFuncGetAttributes(&fa, seq_als_kernel<4, HYB, FULL>); break;
    case 5: e = cudaFuncGetAttributes(&fa, seq_als_kernel<5, HYB, FULL>); break;
    case 6: e = cudaFuncGetAttributes(&fa, seq_als_kernel<6, HYB, FULL>); break;
    case 8: e = cudaFuncGetAttributes(&fa, seq_als_kernel<8, HYB, FULL>); break;
    default: break;
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return (size_t)1 << 30;
  }
  return fa.sharedSizeBytes;
}

static size_t static_smem(int NQL) {
  return std::max(std::max(static_smem_t<true, false>(NQL), static_smem_t<false, false>(NQL)),
                  std::max(static_smem_t<true, true>(NQL), static_smem_t<false, true>(NQL)));
}

// Column segments of the y pass: each warp takes one segment of the tile's
// quads and every (16/NSy)-th group of 32 shared-memory rows; the count that
// gives the smallest per-warp share is taken (the fewest on ties).
static int choose_nsy(int rows, int NQs) {
  const int NG = (rows + 31) / 32;
  int best = 1;
  long long best_w = -1;
  for (int ns = 1; ns <= kWarps && ns <= NQs; ns *= 2) {
    const int gs = kWarps / ns;
    const long long w = (long long)((NG + gs - 1) / gs) * ((NQs + ns - 1) / ns);
    if (best_w < 0 || w < best_w) {
      best_w = w;
      best = ns;
    }
  }
  return best;
}

static int nql_for(int TCp) {
  const int nq = TCp / 4;
  int v = (nq + 31) / 32;
  if (v == 7) v = 8;
  return v;
}

struct SeqPlan {
  int NC = 0, CS = 0, TRmax = 0, TCp = 0, NQL = 0, SR = 0, NSy = 1;
  size_t smem = 0;
};

// Bytes of caller-provided scratch a plan needs when nothing is allocated:
// the three exchange rings, then the abort word on its own 256-byte line.
static size_t fixed_scratch_bytes(int NC, int CS, int TCp) {
  const size_t xbytes = sizeof(uint64_t) * 3 * (size_t)NC * CS * (TCp + 16);
  return ((xbytes + 255) & ~(size_t)255) + 256;
}

// Chooses cluster size, cluster count and how many rows of each CTA's tile
// stay in shared memory (the rest stream from global memory).  Candidates
// must be co-resident (occupancy query).  The estimated cost per half-step
// -- tile words read per CTA, global rows weighted 4x, plus the cross-cluster
// words each CTA polls -- is minimised.  With scratch_limit > 0 only plans
// that keep the whole residual in shared memory and whose exchange rings fit
// in scratch_limit bytes are candidates; the best of all plans is among them
// whenever it qualifies, so such a call takes the same plan as an
// unrestricted one in that case.
static cudaError_t plan_seq(int m, int n, bool weighted, cudaStream_t st, SeqPlan* out,
                            size_t scratch_limit = 0) {
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
    const int TCp = (TC + 31) & ~31;
    const int NQL = nql_for(TCp);
    if (NQL > 8) continue;
    const size_t stat = static_smem(NQL);
    int nc = std::min(std::min(m, 64), std::max(1, nsm / CS));
    for (int guard = 0; guard < 16 && nc >= 1; ++guard) {
      const int TRmax = (m + nc - 1) / nc;
      const SeqSmem L0(TRmax, TCp, nc, CS, 0, 1);
      if (L0.total + stat > (size_t)optin) break;
      const size_t room = (size_t)optin - stat - L0.total;
      int SR = (int)std::min((size_t)TRmax, room / (sizeof(float) * (size_t)TCp));
      int NSy = choose_nsy(SR, TCp / 4);
      SeqSmem L(TRmax, TCp, nc, CS, SR, NSy);
      while (SR > 0 && L.total + stat > (size_t)optin) {
        SR = std::max(0, SR - 8);
        NSy = choose_nsy(SR, TCp / 4);
        L = SeqSmem(TRmax, TCp, nc, CS, SR, NSy);
      }
      if (L.total + stat > (size_t)optin) break;
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
        if (scratch_limit > 0 &&
            (SR < TRmax || fixed_scratch_bytes(nc, CS, TCp) > scratch_limit))
          break;  // fewer clusters only lengthen the tile rows
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
          best.NSy = NSy;
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
  a.NSy = pl.NSy;
  a.recw = recw;
  a.slot_words = slot_words;
  a.flags = (int)h.flags;
  a.sweeps = h.sweeps;
  a.sweep_energy = h.sweep_energy;
  a.dpriv = nullptr;
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
  // refinement sweeps: every CTA keeps its own copy of the emitted scales
  const size_t dpriv_off = (tile_off + tile_bytes + 255) & ~(size_t)255;
  const size_t dpriv_bytes =
      h.sweeps > 0 ? sizeof(float) * (size_t)pl.NC * pl.CS * (size_t)h.k : 0;
  void* ws = nullptr;
  e = cudaMallocAsync(&ws, dpriv_off + dpriv_bytes, st);
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
    a.dpriv = dpriv_bytes ? (float*)((char*)ws + dpriv_off) : nullptr;
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
  if (h.sweeps != 0) return EXTERND_ERR_INVALID_ARG;
  if (scratch_bytes < 256) return EXTERND_ERR_SCRATCH_LIMIT;
  SeqPlan pl;
  cudaError_t e = plan_seq((int)h.m, (int)h.n, h.w != nullptr, st, &pl, scratch_bytes);
  if (e == cudaErrorNotSupported) return EXTERND_ERR_SCRATCH_LIMIT;
  if (e != cudaSuccess) return EXTERND_ERR_CUDA;
  const int recw = pl.TCp + 16;
  const long long slot_words = (long long)pl.NC * pl.CS * recw;
  const size_t need = fixed_scratch_bytes(pl.NC, pl.CS, pl.TCp);
  const size_t abort_off = need - 256;
  if (pl.SR < pl.TRmax || need > scratch_bytes) return EXTERND_ERR_SCRATCH_LIMIT;
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
