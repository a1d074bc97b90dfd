"""The C ABI library loads and exports every entry point that
include/externd.h declares; host-side argument checks answer without a GPU.
CPU only: no call here reaches a kernel."""
import ctypes
import os
import re

import pytest

from expanded_rank_matrix_b200 import externd as X

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    hdrs = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
            if f.endswith(".h")]
    names = set()
    for h in hdrs:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(externd_\w+)\s*\(", text))
    return names


@pytest.fixture(scope="module")
def lib():
    from expanded_rank_matrix_b200 import build
    build.build()
    return X.load()


def test_every_declared_symbol_is_exported(lib):
    declared = _declared()
    assert declared >= set(X.EXPORTS)
    for name in declared:
        assert hasattr(lib, name), name


def test_rank():
    assert X.rank(2560, 2560, 3.0) == 7680
    assert X.rank(256, 256, 2.0) == 512
    assert X.rank(1024, 1024, 1.5) == 1536
    assert X.rank(9728, 2560, 2.0) == 5120
    assert X.rank(1024, 2560, 3.0) == 3072
    assert X.rank(10, 3, 1.0) == 3
    assert X.rank(0, 5, 1.0) == 0
    assert X.rank(5, 5, 0.0) == 0
    assert X.rank(5, 5, float("nan")) == 0
    assert X.rank(5, 5, 0.1) == 0


def test_host_argument_checks(lib):
    L = lib
    nul = None
    # null pointers and bad knobs are rejected before any CUDA call
    assert L.externd_decompose(nul, 8, 8, 1.0, 0.5, 2, nul, 1, nul, nul, nul, nul, nul) == X.ERR_INVALID_ARG
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: rejected on the knobs first
    for args in ((8, 8, 1.0, -0.5, 2, 1), (8, 8, 1.0, 0.5, 0, 1), (8, 8, 0.0, 0.5, 2, 1),
                 (0, 8, 1.0, 0.5, 2, 1), (8, 8, 1.0, 0.5, 2, 0), (8, 8, 1.0, 0.5, 2, 9),
                 (1 << 16, 1 << 16, 1.0, 0.5, 2, 1)):
        m, n, mu, tau, it, blk = args
        assert L.externd_decompose(fake, m, n, mu, tau, it, nul, blk, fake, fake, fake, fake,
                                   nul) == X.ERR_INVALID_ARG, args
    mis = ctypes.c_void_p((1 << 20) + 2)
    assert L.externd_decompose(mis, 8, 8, 1.0, 0.5, 2, nul, 1, fake, fake, fake, fake,
                               nul) == X.ERR_INVALID_ARG
    assert L.externd_reconstruct(nul, fake, fake, 4, 4, 4, fake, nul) == X.ERR_INVALID_ARG
    assert L.externd_reconstruct(fake, fake, fake, 4, 4, 0, fake, nul) == X.ERR_INVALID_ARG
    # tracing is a sequential-mode feature and needs its buffers
    assert L.externd_decompose_traced(fake, 8, 8, 1.0, 0.5, 2, nul, 1, 0, 0, fake, fake, fake, fake,
                                      nul, 2, nul, nul, nul, nul, nul, 0, nul) == X.ERR_INVALID_ARG
    assert L.externd_decompose_traced(fake, 8, 8, 1.0, 0.5, 2, nul, 1, 0, 0, fake, fake, fake, fake,
                                      nul, 0, nul, nul, nul, nul, nul, -1, nul) == X.ERR_INVALID_ARG


def test_variant_and_sweep_argument_checks(lib):
    L = lib
    nul = None
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: rejected before any CUDA call
    ok_flags = X.TSTAT_MEAN_ABS | X.VSTEP_NAIVE
    # unknown flag bits
    assert L.externd_decompose_ex(fake, 64, 64, 1.0, 0.5, 2, nul, 1, 4, 0, fake, fake, fake, fake,
                                  nul, nul) == X.ERR_INVALID_ARG
    # sweeps: sequential mode only, bounded, and they need their energy output
    assert L.externd_decompose_ex(fake, 64, 64, 1.0, 0.5, 2, nul, 16, ok_flags, 1, fake, fake,
                                  fake, fake, fake, nul) == X.ERR_INVALID_ARG
    assert L.externd_decompose_ex(fake, 64, 64, 1.0, 0.5, 2, nul, 1, 0, -1, fake, fake, fake,
                                  fake, fake, nul) == X.ERR_INVALID_ARG
    assert L.externd_decompose_ex(fake, 64, 64, 1.0, 0.5, 2, nul, 1, 0, X.MAX_SWEEPS + 1, fake,
                                  fake, fake, fake, fake, nul) == X.ERR_INVALID_ARG
    assert L.externd_decompose_ex(fake, 64, 64, 1.0, 0.5, 2, nul, 1, 0, 2, fake, fake, fake, fake,
                                  nul, nul) == X.ERR_INVALID_ARG
    assert L.externd_decompose_block_traced(fake, 64, 64, 1.0, 0.5, 2, nul, 16, 8, fake, fake,
                                            fake, fake, 0, nul, nul, nul, 0, nul) == X.ERR_INVALID_ARG


def test_block_argument_checks(lib):
    L = lib
    nul = None
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: rejected before any CUDA call
    # block-ALS: at most 64 components per block, and no more than k or min(m, n)
    assert L.externd_decompose(fake, 4096, 4096, 1.0, 0.5, 2, nul, 65, fake, fake, fake, fake,
                               nul) == X.ERR_INVALID_ARG
    assert L.externd_decompose(fake, 40, 30, 1.0, 0.5, 2, nul, 31, fake, fake, fake, fake,
                               nul) == X.ERR_INVALID_ARG
    # the block-traced entry is block-mode only and needs its trace buffers
    assert L.externd_decompose_block_traced(fake, 64, 64, 1.0, 0.5, 2, nul, 1, 0, fake, fake, fake,
                                            fake, 0, nul, nul, nul, 0, nul) == X.ERR_INVALID_ARG
    assert L.externd_decompose_block_traced(fake, 64, 64, 1.0, 0.5, 2, nul, 16, 0, fake, fake,
                                            fake, fake, 2, nul, nul, nul, 0, nul) == X.ERR_INVALID_ARG
    assert L.externd_decompose_block_traced(fake, 64, 64, 1.0, 0.5, 2, nul, 16, 0, fake, fake,
                                            fake, fake, -1, nul, nul, nul, 0, nul) == X.ERR_INVALID_ARG
    assert L.externd_decompose_block_traced(fake, 64, 64, 1.0, 0.5, 2, nul, 65, 0, fake, fake,
                                            fake, fake, 0, nul, nul, nul, 0, nul) == X.ERR_INVALID_ARG


def test_unpack_planes_layout():
    import numpy as np
    # entries: +1 at 0, -1 at 1, 0 at 2, +1 at 33 (second word)
    packed = np.zeros((2, 2), np.uint32)
    packed[0, 0] = 0b011
    packed[1, 0] = 0b010
    packed[0, 1] = 0b10
    packed[1, 1] = 0
    codes = X.unpack_planes(packed, 40)
    expect = np.zeros(40, np.int8)
    expect[0], expect[1], expect[33] = 1, -1, 1
    assert np.array_equal(codes, expect)


def test_rank_for_energy_argument_checks(lib):
    L = lib
    nul = None
    fake = ctypes.c_void_p(1 << 20)
    assert L.externd_rank_for_energy(nul, 4, 0.5, fake, nul) == X.ERR_INVALID_ARG
    assert L.externd_rank_for_energy(fake, 4, 0.5, nul, nul) == X.ERR_INVALID_ARG
    assert L.externd_rank_for_energy(fake, 0, 0.5, fake, nul) == X.ERR_INVALID_ARG
    assert L.externd_rank_for_energy(fake, 4, float("nan"), fake, nul) == X.ERR_INVALID_ARG
    mis = ctypes.c_void_p((1 << 20) + 4)  # fp64 / int64 need 8-byte alignment
    assert L.externd_rank_for_energy(mis, 4, 0.5, fake, nul) == X.ERR_INVALID_ARG


def test_ternary_apply_argument_checks(lib):
    L = lib
    nul = None
    fake = ctypes.c_void_p(1 << 20)
    assert L.externd_ternary_apply(nul, fake, fake, 8, 8, 4, fake, 1, fake, nul) == X.ERR_INVALID_ARG
    assert L.externd_ternary_apply(fake, fake, fake, 8, 8, 0, fake, 1, fake, nul) == X.ERR_INVALID_ARG
    assert L.externd_ternary_apply(fake, fake, fake, 8, 8, 4, fake, 0, fake, nul) == X.ERR_INVALID_ARG
    assert L.externd_ternary_apply(fake, fake, fake, 16385, 8, 4, fake, 1, fake,
                                   nul) == X.ERR_INVALID_ARG  # more rows than one launch covers
    mis = ctypes.c_void_p((1 << 20) + 2)
    assert L.externd_ternary_apply(fake, fake, fake, 8, 8, 4, mis, 1, fake, nul) == X.ERR_INVALID_ARG


def test_probe_argument_checks(lib):
    L = lib
    out = ctypes.c_int64(0)
    fake = ctypes.c_void_p(1 << 20)
    assert L.externd_probe_read_bandwidth(7, None, 0, 1, ctypes.byref(out), None) == X.ERR_INVALID_ARG
    assert L.externd_probe_read_bandwidth(X.PROBE_SMEM, None, 0, 0, ctypes.byref(out),
                                          None) == X.ERR_INVALID_ARG
    assert L.externd_probe_read_bandwidth(X.PROBE_L2, None, 1 << 20, 1, ctypes.byref(out),
                                          None) == X.ERR_INVALID_ARG
    mis = ctypes.c_void_p((1 << 20) + 8)
    assert L.externd_probe_read_bandwidth(X.PROBE_L2, mis, 1 << 20, 1, ctypes.byref(out),
                                          None) == X.ERR_INVALID_ARG


def test_block_wait_budget_must_not_be_negative(lib):
    fake = ctypes.c_void_p(1 << 20)
    assert lib.externd_decompose_block_traced(fake, 64, 64, 1.0, 0.5, 2, None, 16, 0, fake, fake,
                                              fake, fake, 0, None, None, None, -1,
                                              None) == X.ERR_INVALID_ARG


def test_release_cache_with_nothing_cached(lib):
    # no graph captured and no pool created in this process: nothing to do
    assert lib.externd_release_cache() == X.OK
