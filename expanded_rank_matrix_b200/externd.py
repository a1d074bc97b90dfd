"""ctypes binding to libexternd.so (the C ABI in include/externd.h).

Argument marshalling only: every step of the decomposition runs in the CUDA
library.  PyTorch supplies device memory and streams.  There is no fallback:
if the library is missing or no CUDA device is present the calls raise.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libexternd.so")

OK = 0
ERR_INVALID_ARG = -1
ERR_CUDA = -2
ERR_OOM = -3
ERR_NO_COOP = -4
ERR_TIMEOUT = -5
ERR_NONFINITE = -6
ERR_SCRATCH_LIMIT = -7

# variant flags of externd_decompose_ex
TSTAT_MEAN_ABS = 1
VSTEP_NAIVE = 2
MAX_SWEEPS = 64

# every symbol include/externd.h declares
EXPORTS = ("externd_rank", "externd_decompose", "externd_decompose_ex", "externd_decompose_traced",
           "externd_reconstruct", "externd_sync_status", "externd_decompose_noalloc",
           "externd_decompose_block_traced", "externd_rank_for_energy",
           "externd_ternary_apply", "externd_probe_read_bandwidth", "externd_release_cache")

_lib = None
_vp = ctypes.c_void_p
_i64 = ctypes.c_int64


class ExterndError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what} failed with status {code}")
        self.code = code


def load(path: str = LIB_PATH):
    """Loads the library (no GPU needed) and declares the signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libexternd.so is not built ({path}); run __graft_entry__.build()")
    L = ctypes.CDLL(path)
    L.externd_rank.argtypes = [_i64, _i64, ctypes.c_float]
    L.externd_rank.restype = _i64
    L.externd_decompose.argtypes = [_vp, _i64, _i64, ctypes.c_float, ctypes.c_float, ctypes.c_int,
                                    _vp, ctypes.c_int, _vp, _vp, _vp, _vp, _vp]
    L.externd_decompose.restype = ctypes.c_int
    L.externd_decompose_ex.argtypes = [_vp, _i64, _i64, ctypes.c_float, ctypes.c_float,
                                       ctypes.c_int, _vp, ctypes.c_int, ctypes.c_uint, ctypes.c_int,
                                       _vp, _vp, _vp, _vp, _vp, _vp]
    L.externd_decompose_ex.restype = ctypes.c_int
    L.externd_decompose_traced.argtypes = [_vp, _i64, _i64, ctypes.c_float, ctypes.c_float,
                                           ctypes.c_int, _vp, ctypes.c_int, ctypes.c_uint,
                                           ctypes.c_int, _vp, _vp, _vp, _vp, _vp,
                                           _i64, _vp, _vp, _vp, _vp, _vp, _i64, _vp]
    L.externd_decompose_traced.restype = ctypes.c_int
    L.externd_reconstruct.argtypes = [_vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp]
    L.externd_reconstruct.restype = ctypes.c_int
    L.externd_decompose_noalloc.argtypes = [_vp, _i64, _i64, ctypes.c_float, ctypes.c_float,
                                            ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp]
    L.externd_decompose_noalloc.restype = ctypes.c_int
    L.externd_decompose_block_traced.argtypes = [_vp, _i64, _i64, ctypes.c_float, ctypes.c_float,
                                                 ctypes.c_int, _vp, ctypes.c_int, ctypes.c_uint,
                                                 _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _i64, _vp]
    L.externd_decompose_block_traced.restype = ctypes.c_int
    L.externd_rank_for_energy.argtypes = [_vp, _i64, ctypes.c_double, _vp, _vp]
    L.externd_rank_for_energy.restype = ctypes.c_int
    L.externd_ternary_apply.argtypes = [_vp, _vp, _vp, _i64, _i64, _i64, _vp, _i64, _vp, _vp]
    L.externd_ternary_apply.restype = ctypes.c_int
    L.externd_probe_read_bandwidth.argtypes = [ctypes.c_int, _vp, _i64, ctypes.c_int,
                                               ctypes.POINTER(ctypes.c_int64), _vp]
    L.externd_probe_read_bandwidth.restype = ctypes.c_int
    L.externd_sync_status.argtypes = [_vp]
    L.externd_sync_status.restype = ctypes.c_int
    L.externd_release_cache.argtypes = []
    L.externd_release_cache.restype = ctypes.c_int
    _lib = L
    return L


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def rank(m: int, n: int, mu: float) -> int:
    return int(load().externd_rank(m, n, mu))


def words(length: int) -> int:
    return (length + 31) // 32


@dataclass
class Factors:
    """Device-resident result of one decomposition."""
    packed_B: torch.Tensor  # int32 view of uint32 [k, 2, ceil(m/32)]
    packed_C: torch.Tensor  # [k, 2, ceil(n/32)]
    D: torch.Tensor         # fp32 [k]
    energy: torch.Tensor    # fp64 [k] (the greedy pass)
    m: int
    n: int
    sweep_energy: Optional[torch.Tensor] = None  # fp64 [sweeps]: after each refinement sweep

    @property
    def k(self) -> int:
        return int(self.D.shape[0])


def alloc_factors(m: int, n: int, k: int, device) -> Factors:
    return Factors(torch.empty((k, 2, words(m)), dtype=torch.int32, device=device),
                   torch.empty((k, 2, words(n)), dtype=torch.int32, device=device),
                   torch.empty(k, dtype=torch.float32, device=device),
                   torch.empty(k, dtype=torch.float64, device=device), m, n)


def decompose_into(out: Factors, A: torch.Tensor, mu: float, tau: float, iters: int,
                   w: Optional[torch.Tensor] = None, block: int = 1,
                   stream: Optional[torch.cuda.Stream] = None, flags: int = 0,
                   sweeps: int = 0) -> None:
    """Runs externd_decompose (externd_decompose_ex with variant flags or
    refinement sweeps) into preallocated outputs (stream ordered)."""
    m, n = A.shape
    if flags == 0 and sweeps == 0:
        rc = load().externd_decompose(_ptr(A), m, n, mu, tau, iters, _ptr(w), block,
                                      _ptr(out.packed_B), _ptr(out.packed_C), _ptr(out.D),
                                      _ptr(out.energy), _stream(stream))
    else:
        if sweeps > 0 and (out.sweep_energy is None or out.sweep_energy.numel() < sweeps):
            out.sweep_energy = torch.empty(sweeps, dtype=torch.float64, device=out.D.device)
        rc = load().externd_decompose_ex(_ptr(A), m, n, mu, tau, iters, _ptr(w), block, flags,
                                         sweeps, _ptr(out.packed_B), _ptr(out.packed_C),
                                         _ptr(out.D), _ptr(out.energy),
                                         _ptr(out.sweep_energy) if sweeps > 0 else None,
                                         _stream(stream))
    if rc != OK:
        raise ExterndError(rc, "externd_decompose")


def decompose(A: torch.Tensor, mu: float, tau: float, iters: int,
              w: Optional[torch.Tensor] = None, block: int = 1,
              stream: Optional[torch.cuda.Stream] = None, check: bool = True, flags: int = 0,
              sweeps: int = 0) -> Factors:
    if A.dtype != torch.float32 or A.dim() != 2:
        raise ValueError("A must be a 2-D fp32 CUDA tensor")
    m, n = A.shape
    k = rank(m, n, mu)
    if k < 1:
        raise ExterndError(ERR_INVALID_ARG, "externd_rank")
    out = alloc_factors(m, n, k, A.device)
    decompose_into(out, A, mu, tau, iters, w, block, stream, flags, sweeps)
    if check:
        st = sync_status(stream)
        if st != OK:
            raise ExterndError(st, "externd_decompose (device)")
    return out


def decompose_noalloc_into(out: Factors, A: torch.Tensor, mu: float, tau: float, iters: int,
                           w: Optional[torch.Tensor] = None,
                           stream: Optional[torch.cuda.Stream] = None) -> int:
    """externd_decompose_noalloc into preallocated outputs; returns the C
    status (the entry point allocates nothing itself)."""
    m, n = A.shape
    return int(load().externd_decompose_noalloc(_ptr(A), m, n, mu, tau, iters, _ptr(w),
                                                _ptr(out.packed_B), _ptr(out.packed_C),
                                                _ptr(out.D), _ptr(out.energy), _stream(stream)))


@dataclass
class Trace:
    comps: np.ndarray   # traced component indices
    bits: torch.Tensor  # [ntrace, S] int32
    row: torch.Tensor   # [ntrace] int32
    flags: torch.Tensor  # [ntrace] uint8
    stats: torch.Tensor  # [16] int64 (see externd_decompose_traced)
    iters: int


def decompose_traced(A: torch.Tensor, mu: float, tau: float, iters: int,
                     trace_comps: Sequence[int], w: Optional[torch.Tensor] = None,
                     wait_budget: int = 0, stream: Optional[torch.cuda.Stream] = None,
                     check: bool = True, flags: int = 0, sweeps: int = 0):
    """Traced sequential run.  trace_comps are step indices: component c of
    the greedy pass is step c, component l's refit in sweep s is step
    k (1 + s) + l."""
    m, n = A.shape
    k = rank(m, n, mu)
    out = alloc_factors(m, n, k, A.device)
    if sweeps > 0:
        out.sweep_energy = torch.empty(sweeps, dtype=torch.float64, device=A.device)
    nsteps = k * (1 + sweeps)
    comps = np.array(sorted(set(int(c) for c in trace_comps if 0 <= c < nsteps)), dtype=np.int64)
    nt = int(comps.size)
    S = 2 * words(n) + iters * 2 * (words(m) + words(n))
    dev = A.device
    tc = torch.from_numpy(comps).to(dev) if nt else None
    tb = torch.zeros((max(nt, 1), S), dtype=torch.int32, device=dev)
    tr = torch.zeros(max(nt, 1), dtype=torch.int32, device=dev)
    tf = torch.zeros(max(nt, 1), dtype=torch.uint8, device=dev)
    stats = torch.zeros(16, dtype=torch.int64, device=dev)
    rc = load().externd_decompose_traced(
        _ptr(A), m, n, mu, tau, iters, _ptr(w), 1, flags, sweeps, _ptr(out.packed_B),
        _ptr(out.packed_C), _ptr(out.D), _ptr(out.energy),
        _ptr(out.sweep_energy) if sweeps > 0 else None, nt, _ptr(tc), _ptr(tb) if nt else None,
        _ptr(tr) if nt else None, _ptr(tf) if nt else None, _ptr(stats), wait_budget,
        _stream(stream))
    if rc != OK:
        raise ExterndError(rc, "externd_decompose_traced")
    status = sync_status(stream)
    if check and status != OK:
        raise ExterndError(status, "externd_decompose_traced (device)")
    return out, Trace(comps, tb[:nt], tr[:nt], tf[:nt], stats, iters), status


def reconstruct(f: Factors, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    out = torch.empty((f.m, f.n), dtype=torch.float32, device=f.D.device)
    rc = load().externd_reconstruct(_ptr(f.packed_B), _ptr(f.packed_C), _ptr(f.D), f.m, f.n, f.k,
                                    _ptr(out), _stream(stream))
    if rc != OK:
        raise ExterndError(rc, "externd_reconstruct")
    return out


def rank_for_energy(energy: torch.Tensor, target: float,
                    stream: Optional[torch.cuda.Stream] = None) -> int:
    """Smallest rank whose prefix of a sequential decomposition reaches the
    energy target (0: none does), found by externd_rank_for_energy."""
    if energy.dtype != torch.float64 or energy.dim() != 1:
        raise ValueError("energy must be a 1-D fp64 CUDA tensor")
    out = torch.empty(1, dtype=torch.int64, device=energy.device)
    rc = load().externd_rank_for_energy(_ptr(energy), energy.shape[0], float(target), _ptr(out),
                                        _stream(stream))
    if rc != OK:
        raise ExterndError(rc, "externd_rank_for_energy")
    return int(out.item())


def truncate(f: Factors, r: int) -> Factors:
    """The first r components (views): the rank-r decomposition of a
    sequential run, since greedy deflation is prefix-consistent."""
    return Factors(f.packed_B[:r], f.packed_C[:r], f.D[:r], f.energy[:r], f.m, f.n)


def allocate_rank(A: torch.Tensor, target: float, mu_max: float, tau: float, iters: int,
                  w: Optional[torch.Tensor] = None,
                  stream: Optional[torch.cuda.Stream] = None):
    """Per-matrix rank allocation: decomposes A sequentially at mu_max and
    returns (rank, mu, factors) for the smallest rank reaching `target`
    (rank 0 and the full factors when even mu_max falls short)."""
    f = decompose(A, mu_max, tau, iters, w=w, block=1, stream=stream)
    r = rank_for_energy(f.energy, target, stream)
    if r == 0:
        return 0, mu_max, f
    return r, r / min(f.m, f.n), truncate(f, r)


def apply_into(f: Factors, X: torch.Tensor, Y: torch.Tensor,
               stream: Optional[torch.cuda.Stream] = None) -> None:
    """Y = X (B diag(D) C)^T from the packed factors (externd_ternary_apply);
    X is [nb, n] fp32, Y [nb, m] fp32, both on the device."""
    nb = X.shape[0]
    rc = load().externd_ternary_apply(_ptr(f.packed_B), _ptr(f.packed_C), _ptr(f.D), f.m, f.n, f.k,
                                      _ptr(X), nb, _ptr(Y), _stream(stream))
    if rc != OK:
        raise ExterndError(rc, "externd_ternary_apply")


def apply(f: Factors, X: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    X2 = X.reshape(-1, f.n).contiguous()
    Y = torch.empty((X2.shape[0], f.m), dtype=torch.float32, device=X.device)
    apply_into(f, X2, Y, stream)
    return Y.reshape(*X.shape[:-1], f.m)


PROBE_SMEM = 0
PROBE_L2 = 1


def probe_read_bandwidth(kind: int, reps: int, buf: Optional[torch.Tensor] = None,
                         stream: Optional[torch.cuda.Stream] = None) -> float:
    """Measured read bandwidth (bytes/s) of shared memory (PROBE_SMEM, every
    SM) or of an L2-resident buffer (PROBE_L2), timed with CUDA events."""
    out = ctypes.c_int64(0)
    s = stream if stream is not None else torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    nbytes = 0 if buf is None else buf.numel() * buf.element_size()
    ev0.record(s)
    rc = load().externd_probe_read_bandwidth(kind, _ptr(buf) if buf is not None else None, nbytes,
                                             reps, ctypes.byref(out), _stream(s))
    ev1.record(s)
    if rc != OK:
        raise ExterndError(rc, "externd_probe_read_bandwidth")
    ev1.synchronize()
    return out.value / (ev0.elapsed_time(ev1) / 1000.0)


def sync_status(stream: Optional[torch.cuda.Stream] = None) -> int:
    return int(load().externd_sync_status(_stream(stream)))


def release_cache() -> int:
    """externd_release_cache: drops the block path's cached graphs (with
    their workspaces) and trims the inference scratch pools; returns the C
    status."""
    return int(load().externd_release_cache())


# --- decoding of packed outputs (host side, for inspection and tests) -------

def unpack_planes(packed: np.ndarray, length: int) -> np.ndarray:
    """[..., 2, W] uint32 bitplanes -> [..., length] int8 codes in {-1,0,1}."""
    p = np.ascontiguousarray(packed).view(np.uint32)
    bits = ((p[..., :, :, None] >> np.arange(32, dtype=np.uint32)) & 1).astype(np.int8)
    bits = bits.reshape(*p.shape[:-1], -1)[..., :length]
    mask, sign = bits[..., 0, :], bits[..., 1, :]
    return (mask * (1 - 2 * sign)).astype(np.int8)


def to_codes(f: Factors):
    """(U k x m, V k x n, D, energy) on the host."""
    U = unpack_planes(f.packed_B.cpu().numpy(), f.m)
    V = unpack_planes(f.packed_C.cpu().numpy(), f.n)
    return U, V, f.D.cpu().numpy(), f.energy.cpu().numpy()


def trace_vectors(tr: Trace, t_idx: int, m: int, n: int):
    """Decodes traced component t_idx into (v0, [u_1..u_I], [v_1..v_I])."""
    Wm, Wn = words(m), words(n)
    b = tr.bits[t_idx].cpu().numpy().view(np.uint32)
    v0 = unpack_planes(b[:2 * Wn].reshape(2, Wn), n)
    us, vs = [], []
    off = 2 * Wn
    for _ in range(tr.iters):
        us.append(unpack_planes(b[off:off + 2 * Wm].reshape(2, Wm), m))
        off += 2 * Wm
        vs.append(unpack_planes(b[off:off + 2 * Wn].reshape(2, Wn), n))
        off += 2 * Wn
    return v0, us, vs


@dataclass
class BlockTrace:
    blocks: np.ndarray     # traced block indices
    uv: torch.Tensor       # [ntrace, 2n + iters*2(m+n)] int64 masks
    rows: torch.Tensor     # [ntrace, block] int32
    iters: int
    block: int


def decompose_block_traced(A: torch.Tensor, mu: float, tau: float, iters: int, block: int,
                           trace_blocks: Sequence[int], w: Optional[torch.Tensor] = None,
                           stream: Optional[torch.cuda.Stream] = None, check: bool = True,
                           flags: int = 0, wait_budget: int = 0):
    m, n = A.shape
    k = rank(m, n, mu)
    out = alloc_factors(m, n, k, A.device)
    nblocks = (k + block - 1) // block
    blocks = np.array(sorted(set(int(b) for b in trace_blocks if 0 <= b < nblocks)), np.int64)
    nt = int(blocks.size)
    words_ = 2 * n + iters * 2 * (m + n)
    uv = torch.zeros((max(nt, 1), words_), dtype=torch.int64, device=A.device)
    rows = torch.zeros((max(nt, 1), block), dtype=torch.int32, device=A.device)
    rc = load().externd_decompose_block_traced(
        _ptr(A), m, n, mu, tau, iters, _ptr(w), block, flags, _ptr(out.packed_B),
        _ptr(out.packed_C),
        _ptr(out.D), _ptr(out.energy), nt,
        blocks.ctypes.data_as(ctypes.c_void_p) if nt else None, _ptr(uv) if nt else None,
        _ptr(rows) if nt else None, wait_budget, _stream(stream))
    if rc != OK:
        raise ExterndError(rc, "externd_decompose_block_traced")
    status = sync_status(stream)
    if check and status != OK:
        raise ExterndError(status, "externd_decompose_block_traced (device)")
    tr = BlockTrace(blocks, uv[:nt], rows[:nt], iters, block)
    tr.status = status
    return out, tr


def _mask_codes(mask: np.ndarray, sign: np.ndarray, bb: int) -> np.ndarray:
    """[len] uint64 masks -> [bb, len] int8 codes."""
    mk = mask.view(np.uint64)[None, :] >> np.arange(bb, dtype=np.uint64)[:, None]
    sg = sign.view(np.uint64)[None, :] >> np.arange(bb, dtype=np.uint64)[:, None]
    mk = (mk & np.uint64(1)).astype(np.int8)
    sg = (sg & np.uint64(1)).astype(np.int8)
    return (mk * (1 - 2 * sg)).astype(np.int8)


def block_trace_vectors(tr: BlockTrace, t_idx: int, m: int, n: int, bb: int):
    """Traced block t_idx -> (rows[bb], V0 [bb, n], [U_t [bb, m]], [V_t [bb, n]])."""
    a = tr.uv[t_idx].cpu().numpy()
    rows = tr.rows[t_idx].cpu().numpy()[:bb].astype(np.int64)
    V0 = _mask_codes(a[:n], a[n:2 * n], bb)
    us, vs = [], []
    off = 2 * n
    for _ in range(tr.iters):
        us.append(_mask_codes(a[off:off + m], a[off + m:off + 2 * m], bb))
        off += 2 * m
        vs.append(_mask_codes(a[off:off + n], a[off + n:off + 2 * n], bb))
        off += 2 * n
    return rows, V0, us, vs
