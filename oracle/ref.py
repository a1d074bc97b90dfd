"""Python view of the ExTernD CPU oracle -- TEST INFRASTRUCTURE ONLY.

Thin numpy/ctypes marshalling over ``externd_ref.cpp``.  Only the tests, the
package's smoke check and the benchmark's CPU-baseline leg import this
module; the CUDA library never does.  Codes are int8 in {-1, 0, +1}; U is
k x m and V is k x n (row c holds component c), so B = U^T and C = V.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Optional

import numpy as np

from . import build as _build

_lib = None

_F = ctypes.POINTER(ctypes.c_float)
_D = ctypes.POINTER(ctypes.c_double)
_I8 = ctypes.POINTER(ctypes.c_int8)
_U8 = ctypes.POINTER(ctypes.c_uint8)
_I64 = ctypes.POINTER(ctypes.c_int64)
_i64 = ctypes.c_int64


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(_build.build())
        L.orc_ternarize.argtypes = [_D, _i64, ctypes.c_double, _I8]
        L.orc_ternarize.restype = ctypes.c_double
        L.orc_ternarize2.argtypes = [_D, _i64, ctypes.c_double, ctypes.c_int, _I8]
        L.orc_ternarize2.restype = ctypes.c_double
        L.orc_u_step2.argtypes = [_F, _i64, _i64, _I8, _F, ctypes.c_double, ctypes.c_int, _D, _I8]
        L.orc_u_step2.restype = ctypes.c_double
        L.orc_v_step2.argtypes = [_F, _i64, _i64, _I8, _F, ctypes.c_double, ctypes.c_int,
                                  ctypes.c_int, _D, _I8]
        L.orc_v_step2.restype = ctypes.c_double
        L.orc_decompose_seq2.argtypes = [_F, _i64, _i64, _i64, ctypes.c_double, ctypes.c_int, _F,
                                         ctypes.c_int, ctypes.c_int, _I8, _I8, _F, _D, _I64, _U8,
                                         _D, _U8]
        L.orc_decompose_seq2.restype = _i64
        L.orc_refine_sweep.argtypes = [_F, _i64, _i64, _i64, ctypes.c_double, ctypes.c_int, _F,
                                       ctypes.c_int, _I8, _I8, _F, _U8]
        L.orc_refine_sweep.restype = _i64
        L.orc_block_u_step2.argtypes = [_F, _i64, _i64, _i64, _I8, _F, ctypes.c_double,
                                        ctypes.c_int, _I8, _D, _D]
        L.orc_block_u_step2.restype = None
        L.orc_block_v_step2.argtypes = [_F, _i64, _i64, _i64, _I8, _F, ctypes.c_double,
                                        ctypes.c_int, ctypes.c_int, _I8, _D, _D]
        L.orc_block_v_step2.restype = None
        L.orc_block_init2.argtypes = [_F, _i64, _i64, _i64, _I64, ctypes.c_double, ctypes.c_int, _I8]
        L.orc_block_init2.restype = None
        L.orc_decompose_block2.argtypes = [_F, _i64, _i64, _i64, ctypes.c_double, ctypes.c_int, _F,
                                           ctypes.c_int, _i64, _I8, _I8, _F, _D, _I64]
        L.orc_decompose_block2.restype = None
        L.orc_u_step.argtypes = [_F, _i64, _i64, _I8, _F, ctypes.c_double, _D, _I8]
        L.orc_u_step.restype = ctypes.c_double
        L.orc_v_step.argtypes = [_F, _i64, _i64, _I8, ctypes.c_double, _D, _I8]
        L.orc_v_step.restype = ctypes.c_double
        L.orc_row_norms.argtypes = [_F, _i64, _i64, _F, _D]
        L.orc_row_norms.restype = _i64
        L.orc_sumsq.argtypes = [_F, _i64, _i64, _F]
        L.orc_sumsq.restype = ctypes.c_double
        L.orc_entry_max.argtypes = [_F, _i64, _i64, _F, _D]
        L.orc_entry_max.restype = _i64
        L.orc_scale.argtypes = [_D, _I8, _I8, _i64, _i64, _F, _D]
        L.orc_scale.restype = None
        L.orc_deflate.argtypes = [_F, _i64, _i64, _I8, _I8, ctypes.c_float]
        L.orc_deflate.restype = None
        L.orc_decompose_seq.argtypes = [_F, _i64, _i64, _i64, ctypes.c_double, ctypes.c_int, _F,
                                        _I8, _I8, _F, _D, _I64, _U8]
        L.orc_decompose_seq.restype = _i64
        L.orc_replay.argtypes = [_F, _i64, _i64, _I8, _I8, _F, _i64, _F]
        L.orc_replay.restype = None
        L.orc_replay_range.argtypes = [_F, _i64, _i64, _I8, _I8, _F, _i64, _i64]
        L.orc_replay_range.restype = None
        L.orc_reconstruct.argtypes = [_I8, _I8, _F, _i64, _i64, _i64, _D]
        L.orc_reconstruct.restype = None
        L.orc_rank_for_energy.argtypes = [_D, _i64, ctypes.c_double]
        L.orc_rank_for_energy.restype = _i64
        L.orc_ternary_apply.argtypes = [_I8, _I8, _F, _i64, _i64, _i64, _F, _i64, _D]
        L.orc_ternary_apply.restype = None
        L.orc_top_rows.argtypes = [_D, _i64, _i64, _I64]
        L.orc_top_rows.restype = None
        L.orc_block_u_step.argtypes = [_F, _i64, _i64, _i64, _I8, _F, ctypes.c_double, _I8, _D, _D]
        L.orc_block_u_step.restype = None
        L.orc_block_v_step.argtypes = [_F, _i64, _i64, _i64, _I8, ctypes.c_double, _I8, _D, _D]
        L.orc_block_v_step.restype = None
        L.orc_block_scales.argtypes = [_F, _i64, _i64, _i64, _I8, _I8, _F, _D, _D, _D]
        L.orc_block_scales.restype = None
        L.orc_block_init.argtypes = [_F, _i64, _i64, _i64, _I64, ctypes.c_double, _I8]
        L.orc_block_init.restype = None
        L.orc_decompose_block.argtypes = [_F, _i64, _i64, _i64, ctypes.c_double, ctypes.c_int, _F,
                                          _i64, _I8, _I8, _F, _D, _I64]
        L.orc_decompose_block.restype = None
        _lib = L
    return _lib


def _p(a: Optional[np.ndarray], t):
    if a is None:
        return ctypes.cast(None, t)
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(t)


def _f32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float32)


# variant flags (same bits as the library's): threshold statistic mean |x|,
# naive weighted V-step
MEAN_ABS = 1
NAIVE_VSTEP = 2


def ternarize(x: np.ndarray, tau: float, stat: int = 0):
    """T_tau with the rms (stat 0) or mean-|x| (stat 1) statistic."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape[0], np.int8)
    if stat == 0:
        thr = lib().orc_ternarize(_p(x, _D), x.shape[0], tau, _p(out, _I8))
    else:
        thr = lib().orc_ternarize2(_p(x, _D), x.shape[0], tau, stat, _p(out, _I8))
    return out, thr


def u_step(R: np.ndarray, v: np.ndarray, tau: float, w=None, stat: int = 0):
    R = _f32(R); w = _f32(w)
    m, n = R.shape
    v = np.ascontiguousarray(v, np.int8)
    y = np.empty(m); u = np.empty(m, np.int8)
    if stat == 0:
        thr = lib().orc_u_step(_p(R, _F), m, n, _p(v, _I8), _p(w, _F), tau, _p(y, _D), _p(u, _I8))
    else:
        thr = lib().orc_u_step2(_p(R, _F), m, n, _p(v, _I8), _p(w, _F), tau, stat, _p(y, _D),
                                _p(u, _I8))
    return u, y, thr


def v_step(R: np.ndarray, u: np.ndarray, tau: float, w=None, stat: int = 0, naive: bool = False):
    """v = T_tau(R^T u), or T_tau(w o R^T u) for the naive weighted V-step;
    returns (v, z = R^T u unweighted, threshold)."""
    R = _f32(R)
    m, n = R.shape
    u = np.ascontiguousarray(u, np.int8)
    z = np.empty(n); v = np.empty(n, np.int8)
    if stat == 0 and not naive:
        thr = lib().orc_v_step(_p(R, _F), m, n, _p(u, _I8), tau, _p(z, _D), _p(v, _I8))
    else:
        w = _f32(w)
        thr = lib().orc_v_step2(_p(R, _F), m, n, _p(u, _I8), _p(w, _F), tau, stat, int(naive),
                                _p(z, _D), _p(v, _I8))
    return v, z, thr


def row_norms(R, w=None):
    R = _f32(R); w = _f32(w)
    m, n = R.shape
    rho = np.empty(m)
    best = lib().orc_row_norms(_p(R, _F), m, n, _p(w, _F), _p(rho, _D))
    return rho, int(best)


def sumsq(R, w=None):
    R = _f32(R); w = _f32(w)
    return float(lib().orc_sumsq(_p(R, _F), R.shape[0], R.shape[1], _p(w, _F)))


def entry_max(R, w=None):
    R = _f32(R); w = _f32(w)
    M = ctypes.c_double()
    flat = lib().orc_entry_max(_p(R, _F), R.shape[0], R.shape[1], _p(w, _F), ctypes.byref(M))
    return int(flat), float(M.value)


@dataclass
class Scale:
    p: float
    n_u: int
    n_v: int
    den: float
    d: float
    gain: float


def scale(z, u, v, w=None) -> Scale:
    z = np.ascontiguousarray(z, np.float64)
    u = np.ascontiguousarray(u, np.int8); v = np.ascontiguousarray(v, np.int8)
    w = _f32(w)
    out = np.empty(6)
    lib().orc_scale(_p(z, _D), _p(u, _I8), _p(v, _I8), u.shape[0], v.shape[0], _p(w, _F),
                    _p(out, _D))
    return Scale(out[0], int(out[1]), int(out[2]), out[3], out[4], out[5])


def deflate(R: np.ndarray, u, v, d: float) -> np.ndarray:
    """Returns a deflated copy of R."""
    R = np.array(R, dtype=np.float32, order="C", copy=True)
    u = np.ascontiguousarray(u, np.int8); v = np.ascontiguousarray(v, np.int8)
    lib().orc_deflate(_p(R, _F), R.shape[0], R.shape[1], _p(u, _I8), _p(v, _I8),
                      ctypes.c_float(np.float32(d)))
    return R


@dataclass
class Decomposition:
    U: np.ndarray         # k x m int8 (B^T)
    V: np.ndarray         # k x n int8 (C)
    D: np.ndarray         # k fp32
    energy: np.ndarray    # k fp64 (the greedy pass)
    init_row: np.ndarray  # k int64
    fallback: np.ndarray  # k uint8 (sequential mode only)
    n_fallback: int
    sweep_energy: np.ndarray = None  # [sweeps] fp64: energy after each refinement sweep
    sweep_flags: np.ndarray = None   # [sweeps, k] uint8: bit 0 single entry, bit 1 old kept


def decompose(A, k: int, tau: float, iters: int, w=None, block: int = 1,
              block_path: bool = False, flags: int = 0, sweeps: int = 0) -> Decomposition:
    """Free-running decomposition; block > 1 (or block_path) runs block-ALS.
    flags: MEAN_ABS | NAIVE_VSTEP; sweeps: refinement sweeps (sequential)."""
    A = _f32(A); w = _f32(w)
    m, n = A.shape
    U = np.zeros((k, m), np.int8); V = np.zeros((k, n), np.int8)
    D = np.zeros(k, np.float32); E = np.zeros(k); rows = np.zeros(k, np.int64)
    fb = np.zeros(k, np.uint8)
    se = np.zeros(max(sweeps, 1)); sf = np.zeros((max(sweeps, 1), k), np.uint8)
    if block <= 1 and not block_path:
        if flags == 0 and sweeps == 0:
            nfb = lib().orc_decompose_seq(_p(A, _F), m, n, k, tau, iters, _p(w, _F), _p(U, _I8),
                                          _p(V, _I8), _p(D, _F), _p(E, _D), _p(rows, _I64),
                                          _p(fb, _U8))
        else:
            nfb = lib().orc_decompose_seq2(_p(A, _F), m, n, k, tau, iters, _p(w, _F), flags,
                                           sweeps, _p(U, _I8), _p(V, _I8), _p(D, _F), _p(E, _D),
                                           _p(rows, _I64), _p(fb, _U8), _p(se, _D), _p(sf, _U8))
    else:
        if flags == 0:
            lib().orc_decompose_block(_p(A, _F), m, n, k, tau, iters, _p(w, _F), block,
                                      _p(U, _I8), _p(V, _I8), _p(D, _F), _p(E, _D),
                                      _p(rows, _I64))
        else:
            lib().orc_decompose_block2(_p(A, _F), m, n, k, tau, iters, _p(w, _F), flags, block,
                                       _p(U, _I8), _p(V, _I8), _p(D, _F), _p(E, _D),
                                       _p(rows, _I64))
        nfb = 0
    return Decomposition(U, V, D, E, rows, fb, int(nfb), se[:sweeps], sf[:sweeps])


def refine_sweep(R, U, V, D, tau: float, iters: int, w=None, flags: int = 0):
    """One refinement sweep on copies: returns (R, U, V, D, step_flags)."""
    R = np.array(R, dtype=np.float32, order="C", copy=True)
    U = np.array(U, dtype=np.int8, order="C", copy=True)
    V = np.array(V, dtype=np.int8, order="C", copy=True)
    D = np.array(D, dtype=np.float32, order="C", copy=True)
    w = _f32(w)
    m, n = R.shape
    k = D.shape[0]
    fl = np.zeros(k, np.uint8)
    lib().orc_refine_sweep(_p(R, _F), m, n, k, tau, iters, _p(w, _F), flags, _p(U, _I8),
                           _p(V, _I8), _p(D, _F), _p(fl, _U8))
    return R, U, V, D, fl


def replay(A, U, V, D, upto: int) -> np.ndarray:
    A = _f32(A)
    m, n = A.shape
    R = np.empty_like(A)
    U = np.ascontiguousarray(U, np.int8); V = np.ascontiguousarray(V, np.int8)
    D = _f32(D)
    lib().orc_replay(_p(A, _F), m, n, _p(U, _I8), _p(V, _I8), _p(D, _F), upto, _p(R, _F))
    return R


def replay_range(R: np.ndarray, U, V, D, start: int, stop: int) -> None:
    """Deflates R in place by components [start, stop)."""
    assert R.dtype == np.float32 and R.flags["C_CONTIGUOUS"]
    U = np.ascontiguousarray(U, np.int8); V = np.ascontiguousarray(V, np.int8)
    D = _f32(D)
    lib().orc_replay_range(_p(R, _F), R.shape[0], R.shape[1], _p(U, _I8), _p(V, _I8), _p(D, _F),
                           start, stop)


def reconstruct(U, V, D, m: int, n: int) -> np.ndarray:
    U = np.ascontiguousarray(U, np.int8); V = np.ascontiguousarray(V, np.int8)
    D = _f32(D)
    out = np.empty((m, n))
    lib().orc_reconstruct(_p(U, _I8), _p(V, _I8), _p(D, _F), m, n, D.shape[0], _p(out, _D))
    return out


def rank_for_energy(energy, target: float) -> int:
    """Smallest rank r whose prefix reaches the energy target (0: none)."""
    e = np.ascontiguousarray(energy, np.float64)
    return int(lib().orc_rank_for_energy(_p(e, _D), e.shape[0], target))


def ternary_apply(U, V, D, X) -> np.ndarray:
    """Y = X (B diag(D) C)^T for the nb x n inputs X (fp64 result, nb x m)."""
    U = np.ascontiguousarray(U, np.int8); V = np.ascontiguousarray(V, np.int8)
    D = _f32(D)
    X = np.ascontiguousarray(np.atleast_2d(X), np.float32)
    k, m = U.shape
    n = V.shape[1]
    nb = X.shape[0]
    Y = np.empty((nb, m))
    lib().orc_ternary_apply(_p(U, _I8), _p(V, _I8), _p(D, _F), m, n, k, _p(X, _F), nb, _p(Y, _D))
    return Y


def top_rows(rho, b: int):
    rho = np.ascontiguousarray(rho, np.float64)
    rows = np.empty(b, np.int64)
    lib().orc_top_rows(_p(rho, _D), rho.shape[0], b, _p(rows, _I64))
    return rows


# --- block-ALS half-steps (component-major codes: U[l, i], V[l, j]) ---------

def block_init(R, rows, tau, stat: int = 0):
    R = _f32(R)
    m, n = R.shape
    rows = np.ascontiguousarray(rows, np.int64)
    V = np.zeros((rows.shape[0], n), np.int8)
    lib().orc_block_init2(_p(R, _F), m, n, rows.shape[0], _p(rows, _I64), tau, stat, _p(V, _I8))
    return V


def block_u_step(R, V, tau, w=None, stat: int = 0):
    R = _f32(R); w = _f32(w)
    m, n = R.shape
    V = np.ascontiguousarray(V, np.int8)
    bb = V.shape[0]
    U = np.zeros((bb, m), np.int8)
    T = np.zeros((m, bb)); thr = np.zeros(bb)
    lib().orc_block_u_step2(_p(R, _F), m, n, bb, _p(V, _I8), _p(w, _F), tau, stat, _p(U, _I8),
                            _p(T, _D), _p(thr, _D))
    return U, T, thr


def block_v_step(R, U, tau, w=None, stat: int = 0, naive: bool = False):
    """V half-step; T is the thresholded target (times w when naive)."""
    R = _f32(R); w = _f32(w)
    m, n = R.shape
    U = np.ascontiguousarray(U, np.int8)
    bb = U.shape[0]
    V = np.zeros((bb, n), np.int8)
    T = np.zeros((n, bb)); thr = np.zeros(bb)
    lib().orc_block_v_step2(_p(R, _F), m, n, bb, _p(U, _I8), _p(w, _F), tau, stat, int(naive),
                            _p(V, _I8), _p(T, _D), _p(thr, _D))
    return V, T, thr


def block_scales(R, U, V, w=None):
    R = _f32(R); w = _f32(w)
    m, n = R.shape
    U = np.ascontiguousarray(U, np.int8); V = np.ascontiguousarray(V, np.int8)
    bb = U.shape[0]
    D = np.zeros(bb); G = np.zeros((bb, bb)); r = np.zeros(bb)
    lib().orc_block_scales(_p(R, _F), m, n, bb, _p(U, _I8), _p(V, _I8), _p(w, _F), _p(D, _D),
                           _p(G, _D), _p(r, _D))
    return D, G, r
