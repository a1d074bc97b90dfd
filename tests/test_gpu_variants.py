"""Parity of the T_tau variants (mean-|x| statistic, naive weighted V-step)
and of the refinement sweeps with the CPU oracle, through the C ABI
(externd_decompose_ex / externd_decompose_traced).  Every traced half-step
is re-run by the oracle from the device's own iterates (teacher forced);
refinement steps are checked on the residual the oracle rebuilds from the
device's greedy factors.  Needs a B200."""
import numpy as np
import pytest
import torch

from expanded_rank_matrix_b200 import externd as X
from expanded_rank_matrix_b200 import workloads as W
from tests.parity import BlockReport, RefitReport, Report, check_block, check_component, check_refit

pytestmark = pytest.mark.gpu

FREE_ENERGY_ATOL = 1e-4


def _dev(a):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _seq_teacher_forced(oracle, A, mu, tau, iters, flags, w=None, comps=None):
    m, n = A.shape
    k = X.rank(m, n, mu)
    comps = list(range(k)) if comps is None else sorted(set(comps))
    f, tr, status = X.decompose_traced(_dev(A), mu, tau, iters, comps, w=_dev(w), flags=flags)
    assert status == X.OK
    U, V, D, E = X.to_codes(f)
    rows, fl = tr.row.cpu().numpy(), tr.flags.cpu().numpy()
    E0 = oracle.sumsq(A, w)
    rep = Report()
    R = np.array(A, dtype=np.float32, copy=True)
    at = 0
    stat, naive = flags & 1, bool(flags & 2)
    for ti, c in enumerate(tr.comps.tolist()):
        oracle.replay_range(R, U, V, D, at, c)
        v0, us, vs = X.trace_vectors(tr, ti, m, n)
        R = check_component(oracle, rep, c, R, E0, tau, iters, w, rows[ti], v0, us, vs, fl[ti],
                            U[c], V[c], D[c], E[c], stat=stat, naive=naive)
        at = c + 1
    return rep, f


@pytest.mark.parametrize("flags,weighted", [(X.TSTAT_MEAN_ABS, False), (X.TSTAT_MEAN_ABS, True),
                                            (X.VSTEP_NAIVE, True),
                                            (X.TSTAT_MEAN_ABS | X.VSTEP_NAIVE, True)])
def test_variant_teacher_forced_every_component(oracle, flags, weighted):
    A = W.llm_like(192, 160, 93, n_outliers=4)
    w = W.lognormal_weights(160, 93) if weighted else None
    rep, f = _seq_teacher_forced(oracle, A, 2.0, 0.7, 4, flags, w=w)
    print(f"flags {flags} weighted {weighted}: band {rep.band_total} (mismatch "
          f"{rep.band_mismatch}), fallbacks {rep.fallbacks}")
    assert rep.ok, rep.bad
    ref = oracle.decompose(A, f.k, 0.7, 4, w=w, flags=flags)
    assert abs(float(f.energy[-1]) - ref.energy[-1]) <= FREE_ENERGY_ATOL


def test_mean_abs_llm1024_sampled_and_sparsity(oracle):
    """mean-|x| on the 1024 x 1024 LLM-like matrix at tau = 0.7 and 2.0: sampled
    components teacher-forced; the zero shares of B and C are reported (the
    review's ~41% and ~87% are Gaussian-data figures)."""
    wl = W.config_llm1024(0.5)
    for tau in (0.7, 2.0):
        rep, f = _seq_teacher_forced(oracle, wl.a, 0.25, tau, wl.iters, X.TSTAT_MEAN_ABS,
                                     comps=[0, 1, 2, 50, 255])
        assert rep.ok, rep.bad
        U, V, _, _ = X.to_codes(f)
        print(f"llm1024 mean-|x| tau={tau}: zero share B {np.mean(U == 0):.3f} "
              f"C {np.mean(V == 0):.3f}")


def test_unit_weights_naive_equals_corrected():
    A = _dev(W.llm_like(160, 128, 31, n_outliers=2))
    f0 = X.decompose(A, 1.0, 0.5, 3, flags=X.TSTAT_MEAN_ABS)
    f1 = X.decompose(A, 1.0, 0.5, 3, w=torch.ones(128, device="cuda"),
                     flags=X.TSTAT_MEAN_ABS | X.VSTEP_NAIVE)
    assert torch.equal(f0.packed_B, f1.packed_B) and torch.equal(f0.packed_C, f1.packed_C)
    assert torch.equal(f0.D, f1.D)


@pytest.mark.parametrize("flags,weighted", [(X.TSTAT_MEAN_ABS, False),
                                            (X.TSTAT_MEAN_ABS | X.VSTEP_NAIVE, True)])
def test_block_variant_teacher_forced(oracle, flags, weighted):
    A = W.llm_like(192, 160, 95, n_outliers=4)
    w = W.lognormal_weights(160, 95) if weighted else None
    m, n = A.shape
    mu, tau, iters, b = 2.0, 0.7, 3, 16
    k = X.rank(m, n, mu)
    nb = (k + b - 1) // b
    f, tr = X.decompose_block_traced(_dev(A), mu, tau, iters, b, list(range(nb)), w=_dev(w),
                                     flags=flags)
    U, V, D, E = X.to_codes(f)
    E0 = oracle.sumsq(A, w)
    rep = BlockReport()
    R = np.array(A, dtype=np.float32, copy=True)
    for ti, blk in enumerate(tr.blocks.tolist()):
        c0 = blk * b
        bb = min(b, k - c0)
        rows, V0, us, vs = X.block_trace_vectors(tr, ti, m, n, bb)
        R = check_block(oracle, rep, c0, R, E0, tau, iters, w, rows, V0, us, vs,
                        U[c0:c0 + bb], V[c0:c0 + bb], D[c0:c0 + bb], E[c0:c0 + bb],
                        stat=flags & 1, naive=bool(flags & 2))
    print(f"block flags {flags}: band {rep.band_total} mismatch {rep.band_mismatch}")
    assert rep.ok, rep.bad
    ref = oracle.decompose(A, k, tau, iters, w=w, block=b, flags=flags)
    assert abs(float(f.energy[-1]) - ref.energy[-1]) <= FREE_ENERGY_ATOL


# --- refinement sweeps -----------------------------------------------------

def _sweep_teacher_forced(oracle, A, mu, tau, iters, w=None, flags=0, steps=None):
    """One sweep, every (or the listed) refinement step traced and checked."""
    m, n = A.shape
    k = X.rank(m, n, mu)
    g = X.decompose(_dev(A), mu, tau, iters, w=_dev(w), flags=flags)
    U0, V0, D0, E0g = X.to_codes(g)
    steps = list(range(k)) if steps is None else sorted(set(steps))
    f, tr, status = X.decompose_traced(_dev(A), mu, tau, iters, [k + l for l in steps],
                                       w=_dev(w), flags=flags, sweeps=1)
    assert status == X.OK
    U, V, D, E = X.to_codes(f)
    assert np.array_equal(E, E0g)  # the greedy pass under the sweep is the plain run
    fl = tr.flags.cpu().numpy()
    rows = tr.row.cpu().numpy()
    assert np.all(rows == -1)
    R = oracle.replay(A, U0, V0, D0, k)
    rep = RefitReport()
    traced = {l: i for i, l in enumerate(steps)}
    for l in range(k):
        R = oracle.deflate(R, U0[l], V0[l], -D0[l])  # add back the old component
        if l in traced:
            v0, us, vs = X.trace_vectors(tr, traced[l], m, n)
            R = check_refit(oracle, rep, l, R, tau, iters, w, v0, us, vs, fl[traced[l]], U0[l],
                            V0[l], U[l], V[l], D[l], stat=flags & 1, naive=bool(flags & 2))
        else:
            R = oracle.deflate(R, U[l], V[l], D[l])
    Ew = oracle.sumsq(A, w)
    se = float(f.sweep_energy[0])
    res_o = oracle.sumsq(R, w)
    assert abs((1.0 - se) * Ew - res_o) <= 1e-5 * res_o + 1e-12 * Ew
    return rep, f, E


@pytest.mark.parametrize("weighted", [False, True])
def test_sweep_teacher_forced_every_step(oracle, weighted):
    A = W.llm_like(192, 160, 97, n_outliers=4)
    w = W.lognormal_weights(160, 97) if weighted else None
    rep, f, E = _sweep_teacher_forced(oracle, A, 2.0, 0.5, 4, w=w)
    print(f"sweep weighted={weighted}: refit {rep.refit} kept {rep.kept} single {rep.fallbacks} "
          f"choice ties {rep.choice_ties}; band {rep.band_total} mismatch {rep.band_mismatch}")
    assert rep.ok, rep.bad
    se = float(f.sweep_energy[0])
    assert se >= E[-1] - 8 * 2.0 ** -24
    ref = oracle.decompose(A, f.k, 0.5, 4, w=w, sweeps=1)
    assert abs(se - ref.sweep_energy[0]) <= FREE_ENERGY_ATOL


def test_sweeps_iid256_free_running(oracle):
    """Config-1 shape (256 x 256 i.i.d., mu = 2, I = 4): two sweeps, sampled
    refinement steps of the first teacher-forced, sweep energies against the
    oracle's free-running ones."""
    wl = W.config_small()
    rep, f, E = _sweep_teacher_forced(oracle, wl.a, wl.mu, wl.tau, wl.iters,
                                      steps=[0, 1, 100, 255, 256, 511])
    assert rep.ok, rep.bad
    f2 = X.decompose(_dev(wl.a), wl.mu, wl.tau, wl.iters, sweeps=2)
    se = f2.sweep_energy.cpu().numpy()
    ref = oracle.decompose(wl.a, wl.k, wl.tau, wl.iters, sweeps=2)
    print(f"iid256: greedy {E[-1]:.6f}, sweeps {se.tolist()} (oracle {ref.sweep_energy.tolist()})")
    assert np.all(np.abs(se - ref.sweep_energy) <= FREE_ENERGY_ATOL)
    assert se[0] >= E[-1] - 8 * 2.0 ** -24 and se[1] >= se[0] - 8 * 2.0 ** -24
    # the stored factors are the refined ones: reconstruction gives the sweep energy
    Ahat = X.reconstruct(f2).cpu().numpy().astype(np.float64)
    A64 = wl.a.astype(np.float64)
    assert 1.0 - ((A64 - Ahat) ** 2).sum() / (A64 ** 2).sum() == pytest.approx(se[-1], abs=1e-5)
