"""Parity of the CUDA block-ALS path (block >= 2) with the CPU oracle through
the C ABI: every traced block is checked half-step by half-step from the
device's own iterates (teacher forced).  Needs a B200."""
import json
import os

import numpy as np
import pytest
import torch

from expanded_rank_matrix_b200 import externd as X
from expanded_rank_matrix_b200 import workloads as W
from tests.parity import BlockReport, check_block

pytestmark = pytest.mark.gpu

FREE_ENERGY_ATOL = 1e-4
# Long block-ALS runs (80 blocks of 64 on 9728 x 2560): the free-running
# trajectory is chaotic at the 1e-4 level -- one threshold-band code decided
# differently (allowed by the teacher-forced bar; the first block alone holds
# ~60 band entries) changes a whole block's joint fit, and relative
# perturbations of 1e-7 in tau move the device's final energy by 4e-5 .. 2e-4.
# The teacher-forced check of the first blocks is the parity bar there; the
# final energy is held to 1e-3.
FREE_ENERGY_ATOL_LONG_BLOCK = 1e-3


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def block_teacher_forced(oracle, A, mu, tau, iters, b, blocks=None, w=None):
    m, n = A.shape
    k = X.rank(m, n, mu)
    nb = (k + b - 1) // b
    blocks = list(range(nb)) if blocks is None else sorted(set(blocks))
    f, tr = X.decompose_block_traced(_dev(A), mu, tau, iters, b, blocks,
                                     w=None if w is None else _dev(w))
    U, V, D, E = X.to_codes(f)
    E0 = oracle.sumsq(A, w)
    rep = BlockReport()
    R = np.array(A, dtype=np.float32, copy=True)
    at = 0
    for ti, blk in enumerate(tr.blocks.tolist()):
        c0 = blk * b
        bb = min(b, k - c0)
        oracle.replay_range(R, U, V, D, at, c0)
        rows, V0, us, vs = X.block_trace_vectors(tr, ti, m, n, bb)
        R = check_block(oracle, rep, c0, R, E0, tau, iters, w, rows, V0, us, vs,
                        U[c0:c0 + bb], V[c0:c0 + bb], D[c0:c0 + bb], E[c0:c0 + bb])
        at = c0 + bb
    return rep, f


@pytest.mark.parametrize("weighted", [False, True])
def test_small_every_block(oracle, weighted):
    A = W.llm_like(192, 160, 91, n_outliers=4)
    w = W.lognormal_weights(160, 91) if weighted else None
    rep, f = block_teacher_forced(oracle, A, 2.0, 0.5, 3, 16, w=w)
    print(f"192x160 b=16 weighted={weighted}: {rep.blocks} blocks, band {rep.band_total} "
          f"(mismatch {rep.band_mismatch}), max D rel err {rep.d_rel_max:.2e}")
    assert rep.ok, rep.bad
    ref = oracle.decompose(A, f.k, 0.5, 3, w=w, block=16)
    assert abs(float(f.energy[-1]) - ref.energy[-1]) <= FREE_ENERGY_ATOL


def test_ragged_last_block_and_max_block(oracle):
    A = W.iid_gaussian(100, 90, 5)
    rep, f = block_teacher_forced(oracle, A, 1.0, 0.5, 2, 16)   # k = 90: last block 10
    assert rep.ok, rep.bad
    A2 = W.llm_like(130, 128, 6, n_outliers=2)
    rep2, f2 = block_teacher_forced(oracle, A2, 1.0, 0.5, 2, 64, blocks=[0, 1])
    assert rep2.ok, rep2.bad


def test_llm1024_sampled_blocks_and_free_running(oracle):
    wl = W.config_llm1024(0.5)
    rep, f = block_teacher_forced(oracle, wl.a, wl.mu, wl.tau, wl.iters, 64,
                                  blocks=[0, 1, 12, 23])
    print(f"llm1024 b=64: band {rep.band_total} mismatch {rep.band_mismatch} "
          f"max D rel {rep.d_rel_max:.2e} ties {rep.init_ties}")
    assert rep.ok, rep.bad
    ref = oracle.decompose(wl.a, wl.k, wl.tau, wl.iters, block=64)
    E = f.energy.cpu().numpy()
    print(f"  final energy device {E[-1]:.8f} oracle {ref.energy[-1]:.8f}")
    assert abs(E[-1] - ref.energy[-1]) <= FREE_ENERGY_ATOL


def test_mlp9728_blocks_across_the_run(oracle):
    """Config 4 (9728 x 2560, mu = 2, I = 4, b = 64): blocks spread over the whole
    80-block run are teacher-forced -- the oracle replays the device's emitted
    components up to each one, so late blocks are checked on the residual the
    ordered deflations and stream-K partials have built up; the energy after
    block 0 is held to 1e-4 against the stored oracle value."""
    wl = W.config_mlp9728(64)
    rep, f = block_teacher_forced(oracle, wl.a, wl.mu, wl.tau, wl.iters, 64,
                                  blocks=[0, 1, 20, 40, 79])
    print(f"mlp9728 b=64: blocks {rep.blocks}, band {rep.band_total} mismatch "
          f"{rep.band_mismatch}, max D rel {rep.d_rel_max:.2e}")
    assert rep.ok, rep.bad
    p = os.path.join(os.path.dirname(__file__), "golden", "oracle_energy.json")
    g = json.load(open(p))["mlp9728_b64"]
    assert g["k"] == wl.k and g["block"] == 64
    E = f.energy.cpu().numpy()
    print(f"  energy after block 0: device {E[63]:.8f} oracle {g['energy_at']['63']:.8f}; "
          f"final: device {E[-1]:.8f} oracle {g['final_energy']:.8f}")
    assert abs(E[63] - g["energy_at"]["63"]) <= FREE_ENERGY_ATOL
    assert abs(E[-1] - g["final_energy"]) <= FREE_ENERGY_ATOL_LONG_BLOCK


def test_block_zero_matrix():
    A = torch.zeros((96, 80), device="cuda")
    f = X.decompose(A, 1.0, 0.5, 2, block=16)
    assert not f.packed_B.any() and not f.packed_C.any() and not f.D.any()
    assert torch.all(f.energy == 1.0)


def test_block_deterministic():
    A = _dev(W.llm_like(300, 256, 12, n_outliers=3))
    f1 = X.decompose(A, 1.5, 0.5, 3, block=32)
    f2 = X.decompose(A, 1.5, 0.5, 3, block=32)
    for a, b in ((f1.packed_B, f2.packed_B), (f1.packed_C, f2.packed_C), (f1.D, f2.D),
                 (f1.energy, f2.energy)):
        assert torch.equal(a, b)


def test_transformer_block_weighted(oracle):
    """The seven importance-weighted matrices of one transformer block (mu = 3,
    b = 64): the first block of q teacher-forced, every matrix free-running
    against the oracle's stored final energy."""
    wls = W.config_block_matrices(64)
    q = wls[0]
    rep, f = block_teacher_forced(oracle, q.a, q.mu, q.tau, q.iters, 64, blocks=[0], w=q.w)
    print(f"block_q b=64 weighted: band {rep.band_total} mismatch {rep.band_mismatch} "
          f"max D rel {rep.d_rel_max:.2e}")
    assert rep.ok, rep.bad
    p = os.path.join(os.path.dirname(__file__), "golden", "oracle_energy.json")
    g = json.load(open(p))
    for wl in wls:
        ref = g[wl.name]
        assert ref["k"] == wl.k and ref["block"] == 64
        fw = X.decompose(_dev(wl.a), wl.mu, wl.tau, wl.iters, block=64, w=_dev(wl.w))
        e = float(fw.energy[-1])
        print(f"  {wl.name} {wl.m}x{wl.n}: device {e:.8f} oracle {ref['final_energy']:.8f}")
        assert abs(e - ref["final_energy"]) <= FREE_ENERGY_ATOL


def test_graph_replay_matches_direct(monkeypatch):
    """Repeated identical calls are replayed from a captured CUDA graph (the
    first runs directly, the second captures); the replayed results equal a
    direct run bit for bit, also when A's contents change between calls."""
    A = _dev(W.llm_like(640, 512, 21, n_outliers=2))
    A0 = A.clone()
    k = X.rank(640, 512, 0.5)
    f = X.alloc_factors(640, 512, k, A.device)
    outs = []
    for _ in range(3):  # direct, capture + replay, replay
        X.decompose_into(f, A, 0.5, 0.5, 3, block=32)
        outs.append([t.clone() for t in (f.packed_B, f.packed_C, f.D, f.energy)])
    A.mul_(1.5)  # new contents under the same pointer: the replay must see them
    X.decompose_into(f, A, 0.5, 0.5, 3, block=32)
    scaled = [t.clone() for t in (f.packed_B, f.packed_C, f.D, f.energy)]
    assert X.sync_status() == X.OK
    monkeypatch.setenv("EXTERND_NO_GRAPH", "1")
    g = X.alloc_factors(640, 512, k, A.device)
    X.decompose_into(g, A, 0.5, 0.5, 3, block=32)
    direct_scaled = [t.clone() for t in (g.packed_B, g.packed_C, g.D, g.energy)]
    A.copy_(A0)
    X.decompose_into(g, A, 0.5, 0.5, 3, block=32)
    direct = [g.packed_B, g.packed_C, g.D, g.energy]
    for run in outs:
        for a, b in zip(run, direct):
            assert torch.equal(a, b)
    for a, b in zip(scaled, direct_scaled):
        assert torch.equal(a, b)


def test_contraction_wait_budget_runs_out_cleanly():
    """A one-cycle budget on the tensor-core contractions' pipeline waits: the
    first stage a converter waits for has not landed yet, so the call ends
    with EXTERND_ERR_TIMEOUT; the CTAs drain their own copies and MMAs and free
    their tensor memory, and the next call on the same context is exact."""
    A = _dev(W.llm_like(640, 512, 21, n_outliers=2))
    f, tr = X.decompose_block_traced(A, 0.25, 0.5, 2, 32, [], check=False, wait_budget=1)
    assert tr.status == X.ERR_TIMEOUT
    g = X.decompose(A, 0.25, 0.5, 2, block=32)
    assert X.sync_status() == X.OK
    ref = X.decompose(A, 0.25, 0.5, 2, block=32)
    assert torch.equal(g.D, ref.D) and float(g.energy[-1]) > 0.3


def test_direct_contraction_many_ctas(oracle):
    """Rows of R not 16-byte aligned (n % 4 != 0) take the direct contraction,
    which keeps several CTAs on an SM: 2000 x 1998 launches far more CTAs than
    SMs.  The first two 64-wide blocks are teacher-forced."""
    A = W.llm_like(2000, 1998, 33, n_outliers=3)
    rep, f = block_teacher_forced(oracle, A, 0.5, 0.5, 2, 64, blocks=[0, 1])
    print(f"2000x1998 b=64 (direct path): band {rep.band_total} mismatch {rep.band_mismatch} "
          f"max D rel {rep.d_rel_max:.2e}")
    assert rep.ok, rep.bad


def test_release_cache_drops_graphs():
    """externd_release_cache destroys the captured graphs and trims their
    memory; calls after it run directly, capture again and replay, with the
    same results as before."""
    A = _dev(W.llm_like(640, 512, 22, n_outliers=2))
    k = X.rank(640, 512, 0.5)
    f = X.alloc_factors(640, 512, k, A.device)
    for _ in range(3):  # direct, capture + replay, replay
        X.decompose_into(f, A, 0.5, 0.5, 3, block=32)
    before = [t.clone() for t in (f.packed_B, f.packed_C, f.D, f.energy)]
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    assert X.release_cache() == X.OK
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] >= free0
    assert X.release_cache() == X.OK  # nothing left to release
    for _ in range(3):
        X.decompose_into(f, A, 0.5, 0.5, 3, block=32)
        for a, b in zip(before, (f.packed_B, f.packed_C, f.D, f.energy)):
            assert torch.equal(a, b)
    assert X.sync_status() == X.OK
