"""Teacher-forced comparison of the CUDA path with the CPU oracle.

The oracle rebuilds the device's residual R_c exactly by replaying the
device's emitted (u, v, d) components onto A with the same fp32 deflation,
then re-runs each traced half-step from the device's own input iterate:
  v0  = T_tau(R_c[i*, :])          from the device's starting row i*
  u_t = T_tau(R_c W v_{t-1})       from the device's v_{t-1}
  v_t = T_tau(R_c^T u_t)           from the device's u_t
and checks every ternary code bit for bit, except codes whose |x_j| lies
within BAND (relative) of the threshold tau * rms(x); those are counted and
reported, not hidden.  Scales agree to D_RTOL relative, residual norms to
NORM_RTOL relative.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

BAND = 1e-5
D_RTOL = 1e-5
NORM_RTOL = 1e-5


@dataclass
class Report:
    comps: int = 0
    codes: int = 0
    band_total: int = 0
    band_mismatch: int = 0
    bad: list = field(default_factory=list)
    fallbacks: int = 0
    init_ties: int = 0

    def fail(self, msg):
        if len(self.bad) < 20:
            self.bad.append(msg)

    @property
    def ok(self) -> bool:
        return not self.bad


def _cmp(rep: Report, tag: str, gpu: np.ndarray, ora: np.ndarray, x: np.ndarray, thr: float):
    band = np.abs(np.abs(x) - thr) <= BAND * max(thr, 1e-300)
    mism = gpu != ora
    rep.codes += gpu.size
    rep.band_total += int(band.sum())
    rep.band_mismatch += int((mism & band).sum())
    hard = mism & ~band
    if hard.any():
        idx = np.flatnonzero(hard)[:5]
        rep.fail(f"{tag}: {int(hard.sum())} codes differ outside the band, e.g. at {idx.tolist()} "
                 f"x={x[idx].tolist()} thr={thr}")


def _half_steps(oracle, rep, tag, R, tau, iters, w, v0, us, vs, stat, naive):
    """Re-runs the traced ALS rounds from the device's own iterates; returns
    the last z (R^T u, unweighted)."""
    vprev = v0
    z = None
    for t in range(iters):
        uo, y, thr = oracle.u_step(R, vprev, tau, w, stat=stat)
        _cmp(rep, f"{tag} u{t + 1}", us[t], uo, y, thr)
        vo, z, thr2 = oracle.v_step(R, us[t], tau, w=w, stat=stat, naive=naive)
        x = z * w.astype(np.float64) if (naive and w is not None) else z
        _cmp(rep, f"{tag} v{t + 1}", vs[t], vo, x, thr2)
        vprev = vs[t]
    return z


def check_component(oracle, rep: Report, c: int, R: np.ndarray, E0: float, tau: float, iters: int,
                    w, trace_row: int, v0: np.ndarray, us, vs, flag: int, U_c: np.ndarray,
                    V_c: np.ndarray, D_c: float, energy_c: float, stat: int = 0,
                    naive: bool = False) -> np.ndarray:
    """Checks component c given R = R_c; returns R_{c+1} (replayed with the
    device's emitted component).  stat / naive select the threshold
    variants (mean-|x| statistic, naive weighted V-step)."""
    rep.comps += 1
    rho, best = oracle.row_norms(R, w)
    i0 = int(trace_row)
    if not (0 <= i0 < R.shape[0]) or rho[i0] < rho.max() * (1 - 1e-5):
        rep.fail(f"comp {c}: start row {i0} is not a largest-energy row (best {best})")
        return oracle.deflate(R, U_c, V_c, D_c)
    if i0 != best:
        rep.init_ties += 1
    row = R[i0].astype(np.float64)
    v0o, thr0 = oracle.ternarize(row, tau, stat=stat)
    _cmp(rep, f"comp {c} v0", v0, v0o, row, thr0)
    z = _half_steps(oracle, rep, f"comp {c}", R, tau, iters, w, v0, us, vs, stat, naive)
    s = oracle.scale(z, us[-1], vs[-1], w)
    flat, M = oracle.entry_max(R, w)
    fb_o = s.gain < M
    close = abs(s.gain - M) <= 1e-5 * max(M, 1e-300)
    if bool(flag) != fb_o and not close:
        rep.fail(f"comp {c}: safeguard decision differs (gain {s.gain}, M {M}, device {flag})")
    if flag:
        rep.fallbacks += 1
        i = int(np.flatnonzero(U_c)[0]) if U_c.any() else -1
        j = int(np.flatnonzero(V_c)[0]) if V_c.any() else -1
        if i < 0 or j < 0 or np.count_nonzero(U_c) != 1 or np.count_nonzero(V_c) != 1:
            rep.fail(f"comp {c}: safeguard component is not a single entry")
        else:
            wj = 1.0 if w is None else float(w[j])
            sc = float(np.float32(np.float32(R[i, j] * R[i, j]) * np.float32(wj))) if w is not None \
                else float(R[i, j]) ** 2
            if sc < M * (1 - 1e-6):
                rep.fail(f"comp {c}: safeguard entry ({i},{j}) is not a largest entry")
            if np.float32(D_c) != R[i, j]:
                rep.fail(f"comp {c}: safeguard scale {D_c} != R_ij {R[i, j]}")
    else:
        if not (np.array_equal(U_c, us[-1]) and np.array_equal(V_c, vs[-1])):
            rep.fail(f"comp {c}: emitted factors differ from the last iterates")
        if abs(float(D_c) - s.d) > D_RTOL * abs(s.d) + 1e-30:
            rep.fail(f"comp {c}: scale {D_c} vs oracle {s.d}")
    Rn = oracle.deflate(R, U_c, V_c, D_c)
    res_o = oracle.sumsq(Rn, w)
    res_g = (1.0 - float(energy_c)) * E0
    if abs(res_g - res_o) > NORM_RTOL * res_o + 1e-12 * E0:
        rep.fail(f"comp {c}: residual |R|^2 {res_g} vs oracle {res_o}")
    return Rn


@dataclass
class RefitReport(Report):
    kept: int = 0
    refit: int = 0
    choice_ties: int = 0


def check_refit(oracle, rep: RefitReport, l: int, R: np.ndarray, tau: float, iters: int, w,
                v0, us, vs, flag: int, U_old, V_old, U_l, V_l, D_l, stat: int = 0,
                naive: bool = False) -> np.ndarray:
    """Checks one refinement step of component l given R = the residual with
    the old component added back (replayed from the device's own factors);
    returns the residual after the device's emitted component."""
    rep.comps += 1
    if not np.array_equal(v0, V_old):
        rep.fail(f"refit {l}: the refit did not start from the old v")
    z = _half_steps(oracle, rep, f"refit {l}", R, tau, iters, w, v0, us, vs, stat, naive)
    s = oracle.scale(z, us[-1], vs[-1], w)
    wv = np.ones(R.shape[1]) if w is None else w.astype(np.float64)
    R64 = R.astype(np.float64)
    p_o = float(U_old.astype(np.float64) @ R64 @ (wv * V_old))
    den_o = float(np.count_nonzero(U_old)) * float(wv[V_old != 0].sum())
    g_o = p_o * p_o / den_o if den_o > 0 else 0.0
    d_o = p_o / den_o if den_o > 0 else 0.0
    _, M = oracle.entry_max(R, w)
    g_best = max(s.gain, g_o)
    fb_o = g_best < M
    same = np.array_equal(us[-1], U_old) and np.array_equal(vs[-1], V_old)
    keep_o = (not fb_o) and not (s.gain > g_o)
    fb_d, keep_d = bool(flag & 1), bool(flag & 2)
    near_m = abs(g_best - M) <= 1e-5 * max(M, 1e-300)
    near_g = same or abs(s.gain - g_o) <= 1e-5 * max(g_o, s.gain, 1e-300)
    if fb_d != fb_o and not near_m:
        rep.fail(f"refit {l}: single-entry decision differs (gain {g_best}, M {M}, flag {flag})")
    if not fb_d and not fb_o and keep_d != keep_o:
        if near_g:
            rep.choice_ties += 1
        else:
            rep.fail(f"refit {l}: keep/replace differs (new {s.gain}, old {g_o}, flag {flag})")
    if fb_d:
        rep.fallbacks += 1
        if np.count_nonzero(U_l) != 1 or np.count_nonzero(V_l) != 1:
            rep.fail(f"refit {l}: single-entry component is not a single entry")
    elif keep_d:
        rep.kept += 1
        if not (np.array_equal(U_l, U_old) and np.array_equal(V_l, V_old)):
            rep.fail(f"refit {l}: kept component differs from the old pattern")
        if abs(float(D_l) - d_o) > D_RTOL * abs(d_o) + 1e-30:
            rep.fail(f"refit {l}: kept scale {D_l} vs re-solved {d_o}")
    else:
        rep.refit += 1
        if not (np.array_equal(U_l, us[-1]) and np.array_equal(V_l, vs[-1])):
            rep.fail(f"refit {l}: emitted factors differ from the last iterates")
        if abs(float(D_l) - s.d) > D_RTOL * abs(s.d) + 1e-30:
            rep.fail(f"refit {l}: scale {D_l} vs oracle {s.d}")
    return oracle.deflate(R, U_l, V_l, D_l)


D_RTOL_BLOCK = 1e-5  # joint block scales (same bound as the sequential scales)


@dataclass
class BlockReport(Report):
    blocks: int = 0
    d_rel_max: float = 0.0


def check_block(oracle, rep: "BlockReport", c0: int, R: np.ndarray, E0: float, tau: float,
                iters: int, w, rows, V0, us, vs, U_emit, V_emit, D_gpu, E_gpu, stat: int = 0,
                naive: bool = False) -> np.ndarray:
    """Teacher-forced check of one block (components c0 .. c0+bb-1) given R = R_c0;
    returns the residual after replaying the device's block."""
    bb = len(D_gpu)
    rep.blocks += 1
    rep.comps += bb
    rho, _ = oracle.row_norms(R, w)
    top = oracle.top_rows(rho, bb)
    if not np.array_equal(np.sort(rows), np.sort(top)):
        # allowed only where energies tie to rounding
        if not np.allclose(np.sort(rho[rows])[::-1], rho[top], rtol=1e-12, atol=0):
            rep.fail(f"block {c0}: start rows are not the {bb} largest-energy rows")
        rep.init_ties += 1
    if np.any(np.diff(rho[rows]) > 1e-12 * rho[rows][:-1]):
        rep.fail(f"block {c0}: start rows not in descending energy order")
    V0o = oracle.block_init(R, rows, tau, stat=stat)
    for l in range(bb):
        x = R[rows[l]].astype(np.float64)
        thr = tau * (np.mean(np.abs(x)) if stat else np.sqrt(np.mean(x * x)))
        _cmp(rep, f"block {c0} v0[{l}]", V0[l], V0o[l], x, thr)
    Vprev = V0
    for t in range(iters):
        Uo, T, thr = oracle.block_u_step(R, Vprev, tau, w, stat=stat)
        for l in range(bb):
            _cmp(rep, f"block {c0} u{t + 1}[{l}]", us[t][l], Uo[l], T[:, l], thr[l])
        Vo, T, thr = oracle.block_v_step(R, us[t], tau, w, stat=stat, naive=naive)
        for l in range(bb):
            _cmp(rep, f"block {c0} v{t + 1}[{l}]", vs[t][l], Vo[l], T[:, l], thr[l])
        Vprev = vs[t]
    if not (np.array_equal(U_emit, us[-1]) and np.array_equal(V_emit, vs[-1])):
        rep.fail(f"block {c0}: emitted factors differ from the last iterates")
    Do, G, r = oracle.block_scales(R, us[-1], vs[-1], w)
    for l in range(bb):
        err = abs(float(D_gpu[l]) - Do[l])
        if Do[l] != 0.0:
            rep.d_rel_max = max(rep.d_rel_max, err / abs(Do[l]))
        if err > D_RTOL_BLOCK * abs(Do[l]) + 1e-30:
            rep.fail(f"block {c0}: scale {l} {D_gpu[l]} vs oracle {Do[l]}")
    Rn = R
    for l in range(bb):
        Rn = oracle.deflate(Rn, U_emit[l], V_emit[l], D_gpu[l])
    res_o = oracle.sumsq(Rn, w)
    res_g = (1.0 - float(E_gpu[-1])) * E0
    if abs(res_g - res_o) > NORM_RTOL * res_o + 1e-12 * E0:
        rep.fail(f"block {c0}: residual |R|^2 {res_g} vs replay {res_o}")
    return Rn
