"""externd_decompose_noalloc: the sequential decomposition for callers that
cannot let a library allocate device memory (programs whose memory manager
has reserved the device's memory up front, and latency-bound request paths
that forbid allocation after start-up).  Its scratch is a fixed array inside
the library, so it must give the same factors as the allocating entry point,
call after call, without touching the device memory pool.

Collected last on purpose (file name), so a stop-at-first-failure run has run
every other test before this one.  Needs a B200."""
import numpy as np
import pytest
import torch

from expanded_rank_matrix_b200 import externd as X
from expanded_rank_matrix_b200 import workloads as W

pytestmark = pytest.mark.gpu

D_RTOL = 1e-5       # scale tolerance of the parity tests
NORM_RTOL = 1e-5    # residual-norm tolerance of the parity tests


def _pool_used_high():
    """High-water mark of the current device's default memory pool (the pool
    cudaMallocAsync draws from), or None when the bindings are missing."""
    try:
        from cuda.bindings import runtime as rt
    except ImportError:
        return None
    err, pool = rt.cudaDeviceGetDefaultMemPool(torch.cuda.current_device())
    if err != rt.cudaError_t.cudaSuccess:
        return None
    err, val = rt.cudaMemPoolGetAttribute(pool, rt.cudaMemPoolAttr.cudaMemPoolAttrUsedMemHigh)
    return None if err != rt.cudaError_t.cudaSuccess else int(val)


def _reset_pool_high():
    try:
        from cuda.bindings import driver as dr
        from cuda.bindings import runtime as rt
    except ImportError:
        return
    err, pool = rt.cudaDeviceGetDefaultMemPool(torch.cuda.current_device())
    if err == rt.cudaError_t.cudaSuccess:
        # the high-water mark can only be reset to zero
        rt.cudaMemPoolSetAttribute(pool, rt.cudaMemPoolAttr.cudaMemPoolAttrUsedMemHigh,
                                   dr.cuuint64_t(0))


def test_noalloc_matches_allocating_entry_point_on_two_calls():
    wl = W.config_llm1024(0.5)
    A = torch.from_numpy(wl.a).cuda()
    ref = X.decompose(A, wl.mu, wl.tau, wl.iters)  # the allocating entry point
    torch.cuda.synchronize()
    for call in range(2):
        out = X.alloc_factors(wl.m, wl.n, wl.k, A.device)
        torch.cuda.synchronize()
        _reset_pool_high()
        before = _pool_used_high()
        rc = X.decompose_noalloc_into(out, A, wl.mu, wl.tau, wl.iters)
        assert rc == X.OK, rc
        assert X.sync_status() == X.OK
        after = _pool_used_high()
        if before is not None and after is not None:
            assert after == before == 0, (before, after)
        # ternary factors: bit for bit; scales and residual norms within the
        # parity tolerances
        assert torch.equal(out.packed_B, ref.packed_B), call
        assert torch.equal(out.packed_C, ref.packed_C), call
        D, Dr = out.D.cpu().numpy(), ref.D.cpu().numpy()
        assert np.all(np.abs(D - Dr) <= D_RTOL * np.abs(Dr)), call
        E, Er = out.energy.cpu().numpy(), ref.energy.cpu().numpy()
        assert np.all(np.abs((1 - E) - (1 - Er)) <= NORM_RTOL * np.abs(1 - Er) + 1e-12), call


def test_noalloc_rejects_problems_beyond_its_scratch():
    A = torch.zeros((4096, 4096), device="cuda")
    out = X.alloc_factors(4096, 4096, 4096, A.device)
    assert X.decompose_noalloc_into(out, A, 1.0, 0.5, 2) == X.ERR_SCRATCH_LIMIT
