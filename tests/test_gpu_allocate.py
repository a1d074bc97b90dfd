"""Per-matrix rank allocation to an energy target (externd_rank_for_energy)
on the device, against the oracle's first-index search, and the prefix
property it rests on: a mu = 3 sequential run cut at the chosen rank equals a
run of exactly that rank, bit for bit.  Needs a B200."""
import numpy as np
import pytest
import torch

from expanded_rank_matrix_b200 import externd as X
from expanded_rank_matrix_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_rank_for_energy_matches_oracle_search(oracle):
    rng = np.random.default_rng(3)
    for k in (1, 7, 255, 256, 257, 5000):
        e = np.sort(rng.uniform(0.0, 1.0, k))
        e[rng.integers(0, k, size=min(k, 5))] -= 1e-9  # small non-monotone dips
        dev = torch.from_numpy(e).cuda()
        for target in (-1.0, 0.0, 0.3, float(e[k // 2]), float(e[-1]), 0.999999, 2.0):
            assert X.rank_for_energy(dev, target) == oracle.rank_for_energy(e, target), (k, target)
    assert X.sync_status() == X.OK


def test_cut_run_equals_run_of_that_rank():
    wl = W.config_llm1024(0.5)
    A = torch.from_numpy(wl.a).cuda()
    target = 0.994
    r, mu, f = X.allocate_rank(A, target, 3.0, wl.tau, wl.iters)
    assert 1 <= r <= X.rank(wl.m, wl.n, 3.0)
    E = f.energy.cpu().numpy()
    assert E[-1] >= target and (r == 1 or E[-2] < target)
    # a decomposition asked for exactly r components reproduces the prefix
    g = X.decompose(A, (r + 0.5) / min(wl.m, wl.n), wl.tau, wl.iters)
    assert g.k == r
    for a, b in ((f.packed_B, g.packed_B), (f.packed_C, g.packed_C), (f.D, g.D),
                 (f.energy, g.energy)):
        assert torch.equal(a, b)
    print(f"llm1024: energy {target} needs rank {r} (mu {mu:.3f})")
