/*
 * externd.h -- C ABI of libexternd.so, the B200 (sm_100a) ExTernD library.
 *
 * ExTernD ("Expanded-Rank Ternary Decomposition", arXiv:2607.13511) factors
 * an fp32 matrix A (m x n) as A ~ B diag(D) C with ternary B in
 * {-1,0,+1}^{m x k}, ternary C in {-1,0,+1}^{k x n}, real D in R^k and an
 * inner rank k = floor(mu * min(m, n)) that may exceed min(m, n)
 * (the paper's abstract; "Method" in the romaanj.github.io review).
 *
 * Conventions shared by every entry point:
 *  - Every array pointer is a caller-owned DEVICE pointer on the current CUDA
 *    device, at least 4-byte aligned.  The library never frees or keeps them.
 *  - Matrices are row-major (C order); A[i*n + j] is row i, column j.
 *  - Packed ternary vectors ("bitplanes", mask+sign as in the paper's Eq. 5
 *    bit accounting): a vector of length L is 2 planes of W = ceil(L/32)
 *    uint32 words.  Bit b of word t stands for entry 32*t + b.  Plane 0 is the
 *    mask (1 = nonzero), plane 1 the sign (1 = -1).  The sign bit is 0
 *    wherever the mask bit is 0, and bits past L are 0, so packed outputs can
 *    be compared bit for bit.
 *      packed_B: k x 2 x ceil(m/32) words -- component c's column of B.
 *      packed_C: k x 2 x ceil(n/32) words -- component c's row of C.
 *  - Calls are ordered on `stream`.  The return value reports errors found on
 *    the host (arguments, allocation, launch).  Errors found on the device
 *    (a wait that ran out, non-finite input) go to a per-device status word
 *    that externd_sync_status() returns.
 *  - Scratch memory is taken with cudaMallocAsync on `stream` and released on
 *    `stream` before the call returns.
 */
#ifndef EXTERND_H
#define EXTERND_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define EXTERND_OK 0
#define EXTERND_ERR_INVALID_ARG (-1) /* bad size, pointer, alignment or knob   */
#define EXTERND_ERR_CUDA (-2)        /* a CUDA runtime call failed              */
#define EXTERND_ERR_OOM (-3)         /* scratch allocation failed               */
#define EXTERND_ERR_NO_COOP (-4)     /* the persistent grid cannot be resident  */
#define EXTERND_ERR_TIMEOUT (-5)     /* a bounded device-side wait ran out      */
#define EXTERND_ERR_NONFINITE (-6)   /* NaN/Inf in A, or w not finite and > 0   */
#define EXTERND_ERR_SCRATCH_LIMIT (-7) /* problem too large for the fixed scratch  */

typedef struct CUstream_st* externd_stream_t; /* same object as cudaStream_t */

/*
 * Variant flags of externd_decompose_ex (the threshold and V-step options the
 * romaanj.github.io review names in "Method" and "Validation").
 *
 * EXTERND_TSTAT_MEAN_ABS: T_tau(x)_j = sign(x_j) if |x_j| > tau * mean_j |x_j|
 *   (instead of tau * rms(x)).  The review's zero shares (tau = 0.7 -> ~41%,
 *   tau = 2.0 -> ~87%) are those of this statistic on Gaussian data.
 * EXTERND_VSTEP_NAIVE: with weights, the V-step thresholds W R^T u (the
 *   "naive" importance-weighted V-step of the review's ablation) instead of
 *   R^T u (the corrected one, the default).  No effect without weights.
 */
#define EXTERND_TSTAT_MEAN_ABS 1u
#define EXTERND_VSTEP_NAIVE 2u
#define EXTERND_MAX_SWEEPS 64

/*
 * externd_rank -- the inner rank k = floor(mu * min(m, n)) (the paper's
 * abstract: k = mu min(m, n)).  Returns 0 when an argument is out of range.
 */
int64_t externd_rank(int64_t m, int64_t n, float mu);

/*
 * externd_decompose -- the whole ExTernD decomposition of one matrix.
 *
 * block == 1: greedy sequential-deflation ALS (paper Sec. 2.3, per the Pith
 *   review's referee summary and the review's "Method"/"Key idea"): for each
 *   component c = 0..k-1 on the residual R (R = A at the start):
 *     i*  = argmax_i sum_j w_j R_ij^2;  v = T_tau(R[i*, :])
 *     repeat iters times: u = T_tau(R W v); v = T_tau(R^T u)
 *     d = u^T R W v / (|u|^2 v^T W v), gain g = (u^T R W v)^2 / (|u|^2 v^T W v)
 *     if g < max_ij w_j R_ij^2: u = e_i', v = e_j', d = R_i'j' (single-entry
 *       safeguard of Appendix A, Prop. 2)
 *     R <- R - d u v^T  (one fp32 add or subtract per touched entry)
 *   where T_tau(x)_j = sign(x_j) if |x_j| > tau * rms(x) else 0 (Eq. 2) and
 *   W = diag(w) (W = I when w is NULL; the importance weighting of Sec. 2.5).
 * block > 1: block-ALS (Sec. 2.4, Eq. 3): b = block components per sweep
 *   against decorrelated least-squares targets, joint scales, b ordered
 *   rank-1 deflations.
 *
 * Arguments:
 *   A            [m*n] fp32, read only.
 *   m, n         1 <= m, n and m*n < 2^31.
 *   mu           rank multiplier, > 0; k = externd_rank(m, n, mu) >= 1.
 *   tau          threshold factor, finite and >= 0.
 *   iters        ALS iterations per component (or per block), >= 1.
 *   w            [n] fp32 per-input-column importance weights, finite and
 *                > 0, or NULL for the unweighted objective.
 *   block        1 (sequential) or 2..min(k, m, n, 64) (block-ALS).
 *   packed_B     [k][2][ceil(m/32)] uint32 out.
 *   packed_C     [k][2][ceil(n/32)] uint32 out.
 *   D            [k] fp32 out.
 *   energy_trace [k] fp64 out: 1 - |R_{c+1}|_W^2 / |A|_W^2 after component c
 *                (|X|_W^2 = sum_ij w_j X_ij^2; 1 when A == 0).
 *   stream       CUDA stream (NULL = legacy default stream).
 * Returns EXTERND_OK or a negative status.  On a device-detected error the
 * outputs are undefined and externd_sync_status() returns the error.
 *
 * Scratch: the call allocates its workspace stream-ordered on `stream`
 * (cudaMallocAsync) and frees it before the work it queued completes.
 * Block mode replays repeated calls: a call whose pointers, sizes and knobs
 * equal an earlier call's on the same device (the second such call) is
 * captured once into a CUDA graph on a library-owned stream and replayed
 * from then on, joined to `stream` by events; the library keeps up to 8
 * such graphs (least recently used first out), whose workspace lives in the
 * device's graph memory pool.  The replay reads A and w at launch time, so
 * new contents under the same pointers are honoured.  Calls on a stream that
 * is being captured run directly (they become part of the caller's graph);
 * setting the environment variable EXTERND_NO_GRAPH=1 disables replay, and
 * externd_release_cache() drops the cached graphs with their memory.
 */
int externd_decompose(const float* A, int64_t m, int64_t n, float mu, float tau, int iters,
                      const float* w, int block, uint32_t* packed_B, uint32_t* packed_C,
                      float* D, double* energy_trace, externd_stream_t stream);

/*
 * externd_decompose_ex -- externd_decompose with the threshold variants and
 * refinement sweeps.
 *
 *   flags        EXTERND_TSTAT_MEAN_ABS | EXTERND_VSTEP_NAIVE, or 0 (the
 *                externd_decompose behaviour).  Both modes.
 *   sweeps       refinement sweeps after the greedy pass, 0 .. EXTERND_MAX_SWEEPS;
 *                block == 1 only.  A sweep backfits every component in order
 *                (the review's "Results": sweeps add about 0.4 energy points):
 *                component l is added back onto the residual, refit by
 *                `iters` ALS rounds from its own v, and replaced by the refit
 *                only if the refit removes more than the old pattern with its
 *                scale re-solved on that residual (otherwise the old pattern
 *                stays, rescaled); the single-entry safeguard applies as in
 *                the greedy pass.  No step raises the residual beyond fp32
 *                rounding.  The outputs then hold the refined factors;
 *                energy_trace keeps the greedy pass's trace.
 *   sweep_energy [sweeps] fp64 out: the energy after each sweep (NULL when
 *                sweeps == 0).
 * Other arguments, scratch and errors as for externd_decompose (sweeps add
 * 4 * k bytes per CTA of the persistent grid to the stream-ordered scratch).
 */
int externd_decompose_ex(const float* A, int64_t m, int64_t n, float mu, float tau, int iters,
                         const float* w, int block, unsigned flags, int sweeps,
                         uint32_t* packed_B, uint32_t* packed_C, float* D, double* energy_trace,
                         double* sweep_energy, externd_stream_t stream);

/*
 * externd_decompose_traced -- externd_decompose_ex plus a record of the ALS
 * trajectory of selected steps (used to compare the device path with a
 * reference half-step by half-step).  Tracing is sequential-mode
 * (block == 1) only.  Step t < k is greedy component t; step k (1 + s) + l
 * is component l's refit in sweep s.
 *
 *   trace_comp   [ntrace] int64, strictly increasing step indices below
 *                k (1 + sweeps), or NULL when ntrace == 0.
 *   trace_bits   [ntrace][S] uint32 out, S = 2*Wn + iters*2*(Wm + Wn),
 *                Wm = ceil(m/32), Wn = ceil(n/32): for each traced component
 *                the packed starting v (a refit's: the old component's v),
 *                then for t = 1..iters the packed u_t and the packed v_t.
 *                May be NULL when ntrace == 0.
 *   trace_row    [ntrace] int32 out: the starting row i* (-1 for a refit).
 *   trace_flags  [ntrace] uint8 out: bit 0 = the safeguard replaced the ALS
 *                pair of this step, bit 1 = a refit kept the old pattern.
 *   stats        [16] int64 out or NULL: [0] safeguard activations over all
 *                components, [1] components emitted as zero because the
 *                residual vanished, [2] launch clusters, [3] CTAs per cluster,
 *                [4] rows of each CTA's residual tile kept in shared memory,
 *                [5] rows of each CTA's tile (the rest stream from global memory),
 *                [6..15] SM cycles CTA 0 spent per phase (setup, R W v pass,
 *                cluster gather of y, y exchange, R^T u pass, z exchange,
 *                z cluster step, scale and emit, deflation, statistics).
 *   wait_budget  upper bound, in SM clock cycles, on every device-side wait
 *                for another CTA's data; 0 selects the default (about 1 s).
 *                A wait that runs out sets EXTERND_ERR_TIMEOUT and the kernel
 *                winds down without further waits.
 */
int externd_decompose_traced(const float* A, int64_t m, int64_t n, float mu, float tau, int iters,
                             const float* w, int block, unsigned flags, int sweeps,
                             uint32_t* packed_B, uint32_t* packed_C, float* D,
                             double* energy_trace, double* sweep_energy, int64_t ntrace,
                             const int64_t* trace_comp, uint32_t* trace_bits, int32_t* trace_row,
                             uint8_t* trace_flags, int64_t* stats, int64_t wait_budget,
                             externd_stream_t stream);

/*
 * externd_decompose_block_traced -- externd_decompose_ex with block >= 2
 * (flags as there, no sweeps) plus a
 * record of the block-ALS trajectory of selected blocks (used to compare the
 * device path with a reference half-step by half-step).  Block t covers
 * components t*block .. min(k, (t+1)*block) - 1; bit l of a mask word stands
 * for the block's component l.
 *
 *   trace_block  [ntrace] int64 HOST array of block indices (may be NULL when
 *                ntrace == 0).
 *   trace_uv     [ntrace][2n + iters*2(m+n)] uint64 (device) out: per traced
 *                block the n mask words then the n sign words of the starting
 *                V, then for t = 1..iters the m mask and m sign words of U_t
 *                and the n mask and n sign words of V_t.
 *   trace_rows   [ntrace][block] int32 (device) out: the block's start rows in
 *                order (energy descending, index ascending).
 *   wait_budget  upper bound, in SM clock cycles, on the tensor-core
 *                contractions' waits for their pipeline stages; 0 selects the
 *                default (about 1 s).  A wait that runs out sets
 *                EXTERND_ERR_TIMEOUT; the CTA then drains its own copies and
 *                MMAs (with the default bound), frees its tensor memory and
 *                returns, so the call completes with undefined outputs.
 */
int externd_decompose_block_traced(const float* A, int64_t m, int64_t n, float mu, float tau,
                                   int iters, const float* w, int block, unsigned flags,
                                   uint32_t* packed_B,
                                   uint32_t* packed_C, float* D, double* energy_trace,
                                   int64_t ntrace, const int64_t* trace_block, uint64_t* trace_uv,
                                   int32_t* trace_rows, int64_t wait_budget,
                                   externd_stream_t stream);

/*
 * externd_reconstruct -- A_hat = B diag(D) C from the packed factors (the
 * factor form of the paper's abstract), accumulated in fp64 in component
 * order and rounded once to fp32.
 *   packed_B [k][2][ceil(m/32)], packed_C [k][2][ceil(n/32)], D [k] in;
 *   A_hat [m*n] fp32 out.  1 <= m, n, k; m*n < 2^31.
 */
int externd_reconstruct(const uint32_t* packed_B, const uint32_t* packed_C, const float* D,
                        int64_t m, int64_t n, int64_t k, float* A_hat, externd_stream_t stream);

/*
 * externd_ternary_apply -- inference with the factors: Y = X (B diag(D) C)^T
 * from the packed bitplanes, without forming the dense matrix.  For each
 * input vector x (a row of X): t_c = sum_j C_cj x_j, then
 * y_i = sum_c B_ic D_c t_c -- ternary additions and subtractions plus one
 * scale per component (the romaanj.github.io review, "Significance":
 * inference stays multiplication-free; "Limitations": no fused inference
 * kernel exists yet).  Sums are fp32 in a fixed order (reproducible run to
 * run).
 *
 *   packed_B [k][2][ceil(m/32)], packed_C [k][2][ceil(n/32)], D [k]: the
 *            factors as externd_decompose writes them (device, in).
 *   m, n, k  1 <= m <= EXTERND_APPLY_MAX_ROWS, 1 <= n, m*n < 2^31, k >= 1.
 *   X        [nb][n] fp32 (device, in): nb input vectors, row-major.
 *   nb       1 .. 65536 vectors (processed two at a time).
 *   Y        [nb][m] fp32 (device, out).
 * Scratch: SMs * m * 2 floats, stream-ordered on `stream` from a memory pool
 * the library owns on each device, which keeps that memory mapped between
 * calls (until the process exits).  One cooperative launch per two vectors (every CTA
 * resident; its two grid barriers are bounded waits that raise
 * EXTERND_ERR_TIMEOUT in the status word if they ever run out).  Returns
 * EXTERND_OK, EXTERND_ERR_INVALID_ARG, EXTERND_ERR_OOM, EXTERND_ERR_NO_COOP
 * or EXTERND_ERR_CUDA.
 */
#define EXTERND_APPLY_MAX_ROWS 16384
int externd_ternary_apply(const uint32_t* packed_B, const uint32_t* packed_C, const float* D,
                          int64_t m, int64_t n, int64_t k, const float* X, int64_t nb, float* Y,
                          externd_stream_t stream);

/*
 * externd_decompose_noalloc -- externd_decompose (block == 1 only) without
 * any memory allocation.  The paper has no counterpart; this is a service of
 * this library.
 *
 * Some callers cannot let a library allocate device memory: programs whose
 * memory manager has already reserved the device's memory (a framework's
 * caching allocator, a serving process that sizes its pools at start-up), in
 * which a library's own allocation can fail or fragment what they hold; and
 * latency-bound request paths that forbid allocation after start-up because
 * allocation calls can stall or synchronise the device.  This entry point
 * takes all of its scratch (the cross-CTA exchange ring and the abort word)
 * from one fixed array compiled into the library, EXTERND_NOALLOC_SCRATCH_BYTES
 * bytes per device, which every device that loads the library holds until the
 * process exits.  It calls no cudaMalloc, cudaMallocAsync, cudaFree or other
 * allocating routine.  The caller still owns and passes every input and
 * output, with the same meaning as for externd_decompose.
 *
 * Limits: the launch plan is the cheapest one (of those externd_decompose
 * chooses among) that keeps the whole residual in the persistent grid's
 * shared memory (about 26 MB of fp32 on a B200, e.g. 2560 x 2560) and whose
 * exchange ring fits in the fixed array; when no plan qualifies the call
 * returns EXTERND_ERR_SCRATCH_LIMIT without launching anything.  Where
 * externd_decompose's own plan qualifies (2560 x 2560 and smaller square
 * problems do) both entry points run the same plan and give identical
 * factors.
 * The first call on a device looks up the device address of the fixed array
 * (a one-time set-up per device, done with that device current); make that
 * first call before any stream capture.
 * Every call on a device shares the one array and clears the part it uses at
 * the start of the call.  Calls that overlap on the GPU (issued on different
 * streams without ordering between them) race on it and give undefined
 * results; order them on one stream or with events.
 */
#define EXTERND_NOALLOC_SCRATCH_BYTES (4u << 20)
int externd_decompose_noalloc(const float* A, int64_t m, int64_t n, float mu, float tau,
                              int iters, const float* w, uint32_t* packed_B, uint32_t* packed_C,
                              float* D, double* energy_trace, externd_stream_t stream);

/*
 * externd_rank_for_energy -- per-matrix rank allocation to an energy target
 * (the romaanj.github.io review, "Results": the rank multiplier is chosen per
 * matrix to reach a reference quantiser's per-matrix energy; the Pith
 * review's "Assumptions & free parameters": mu from 1.97 to 3.43 per matrix).
 * Greedy sequential deflation (block == 1) makes a rank-k decomposition hold
 * every shorter one as its prefix, bit for bit, so the smallest rank whose
 * energy reaches `target` is read off one run's energy trace: the first c
 * with energy_trace[c] >= target, plus one.  The first r components of
 * packed_B, packed_C and D are then exactly the rank-r decomposition.  (In
 * block mode a prefix is a shorter run only where it ends on a block
 * boundary.)
 *
 *   energy_trace [k] fp64 (device) in, as written by externd_decompose.
 *   k            >= 1 entries.
 *   target       finite energy target (e.g. 0.994).
 *   rank         [1] int64 (device) out: that rank in 1..k, or 0 when no
 *                prefix reaches the target.
 * Stream-ordered on `stream`; returns EXTERND_OK, EXTERND_ERR_INVALID_ARG
 * (NULL or misaligned pointer, k < 1, target not finite) or EXTERND_ERR_CUDA.
 */
int externd_rank_for_energy(const double* energy_trace, int64_t k, double target, int64_t* rank,
                            externd_stream_t stream);

/*
 * externd_probe_read_bandwidth -- a read-bandwidth probe for the on-chip
 * rooflines (measurement, not part of the method).  kind
 * EXTERND_PROBE_SMEM: one CTA per SM streams its own shared memory (about
 * 220 KB) `reps` times with 128-bit loads; buf and bytes are ignored.
 * EXTERND_PROBE_L2: every SM streams the device buffer `buf` (`bytes` long,
 * 16-byte aligned; size it well below the L2 so it stays resident) `reps`
 * times with 128-bit L2 loads.  *bytes_read (host) receives the bytes the
 * launch reads; time it with events on `stream`.  Returns EXTERND_OK,
 * EXTERND_ERR_INVALID_ARG, EXTERND_ERR_OOM or EXTERND_ERR_CUDA.
 */
#define EXTERND_PROBE_SMEM 0
#define EXTERND_PROBE_L2 1
int externd_probe_read_bandwidth(int kind, const void* buf, int64_t bytes, int reps,
                                 int64_t* bytes_read, externd_stream_t stream);

/*
 * externd_release_cache -- gives back the device memory the library keeps
 * between calls: destroys every CUDA graph that block-mode replay has
 * captured (each holds its own workspace, including a copy of the residual,
 * in its device's graph memory pool), returns that graph memory to the
 * devices (cudaDeviceGraphMemTrim), and trims the inference scratch pools
 * to zero (cudaMemPoolTrimTo).  Work already queued keeps what it uses:
 * destruction and trimming leave alone memory that queued work still needs.
 * Later calls capture and allocate again as usual.  Not stream-ordered;
 * safe to call from any thread.  Returns EXTERND_OK, or EXTERND_ERR_CUDA if a trim failed (the caches are
 * emptied regardless).
 */
int externd_release_cache(void);

/*
 * externd_sync_status -- synchronises `stream`, then returns and clears the
 * current device's status word: EXTERND_OK, or the first device-side error
 * (EXTERND_ERR_TIMEOUT, EXTERND_ERR_NONFINITE) raised by any call on this
 * device since the last read; EXTERND_ERR_CUDA if the synchronisation
 * itself failed.
 */
int externd_sync_status(externd_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* EXTERND_H */
