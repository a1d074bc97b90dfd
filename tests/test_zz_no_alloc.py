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


def _bindings():
    """The CUDA runtime bindings the allocation checks read the device's
    memory pool through.  They ship with the image; without them the checks
    cannot run, and the test fails rather than pass unchecked."""
    try:
        from cuda.bindings import driver as dr
        from cuda.bindings import runtime as rt
    except ImportError as exc:  # pragma: no cover - the image has them
        pytest.fail(f"cuda.bindings is required for the no-allocation checks: {exc}")
    return rt, dr


def _default_pool():
    rt, _ = _bindings()
    err, pool = rt.cudaDeviceGetDefaultMemPool(torch.cuda.current_device())
    assert err == rt.cudaError_t.cudaSuccess, err
    return pool


def _pool_used_high():
    """High-water mark of the current device's default memory pool (the pool
    cudaMallocAsync draws from)."""
    rt, _ = _bindings()
    err, val = rt.cudaMemPoolGetAttribute(_default_pool(),
                                          rt.cudaMemPoolAttr.cudaMemPoolAttrUsedMemHigh)
    assert err == rt.cudaError_t.cudaSuccess, err
    return int(val)


def _reset_pool_high():
    rt, dr = _bindings()
    # the high-water mark can only be reset to zero
    (err,) = rt.cudaMemPoolSetAttribute(_default_pool(),
                                        rt.cudaMemPoolAttr.cudaMemPoolAttrUsedMemHigh,
                                        dr.cuuint64_t(0))
    assert err == rt.cudaError_t.cudaSuccess, err


def _case(name):
    if name == "llm1024":
        wl = W.config_llm1024(0.5)
        return wl, None
    if name == "llm1024_weighted":
        wl = W.config_llm1024(0.5)
        return wl, torch.from_numpy(W.lognormal_weights(wl.n, 7)).cuda()
    if name == "attn2560":
        return W.config_attn2560(), None
    raise ValueError(name)


@pytest.mark.parametrize("name", ["llm1024", "llm1024_weighted", "attn2560"])
def test_noalloc_matches_allocating_entry_point_on_two_calls(name):
    wl, w = _case(name)
    A = torch.from_numpy(wl.a).cuda()
    ref = X.decompose(A, wl.mu, wl.tau, wl.iters, w=w)  # the allocating entry point
    torch.cuda.synchronize()
    for call in range(2):
        out = X.alloc_factors(wl.m, wl.n, wl.k, A.device)
        torch.cuda.synchronize()
        _reset_pool_high()
        free0 = torch.cuda.mem_get_info()[0]  # cudaMemGetInfo: the whole device
        rc = X.decompose_noalloc_into(out, A, wl.mu, wl.tau, wl.iters, w=w)
        assert rc == X.OK, rc
        assert X.sync_status() == X.OK
        free1 = torch.cuda.mem_get_info()[0]
        # nothing drawn from the stream-ordered pool, on any call
        assert _pool_used_high() == 0, call
        if call == 1:
            # and nothing from cudaMalloc or any other allocator once the
            # first call has loaded the kernels and looked up the fixed array
            assert free1 == free0, (call, free0, free1)
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
