"""Inference with the packed factors (externd_ternary_apply) against the CPU
oracle's fp64 y = B diag(D) C x, element by element, within a bound derived
from the kernel's fp32 arithmetic.  Needs a B200."""
import numpy as np
import pytest
import torch

from expanded_rank_matrix_b200 import externd as X
from expanded_rank_matrix_b200 import workloads as W

pytestmark = pytest.mark.gpu

U32 = 2.0 ** -24  # unit roundoff of fp32


def _bound(oracle, U, V, D, Xh):
    """First-order bound on |y_fp32 - y_exact| for the kernel's order of
    operations: t_c sums at most n terms (error <= n u sum_j |C_cj x_j|),
    s_c = fl(D_c t_c) adds u |D_c t_c|, and y_i sums at most k terms in
    per-stream, per-CTA and CTA-order partials (at most k + 1024 additions on
    any path): (k + 1026) u sum_c |B_ic s_c| + n u sum_c |B_ic D_c| sum_j |C_cj x_j|.
    Doubled for second-order terms."""
    Ua = np.abs(U).astype(np.float64)
    Va = np.abs(V).astype(np.float64)
    Da = np.abs(D.astype(np.float64))
    Xa = np.abs(Xh.astype(np.float64))
    n, k = V.shape[1], U.shape[0]
    absx = Va @ Xa.T                      # [k, nb]: sum_j |C_cj x_j|
    s_abs = Da[:, None] * np.abs(V.astype(np.float64) @ Xh.T.astype(np.float64))
    term1 = (k + 1026) * U32 * (Ua.T @ s_abs)
    term2 = n * U32 * (Ua.T @ (Da[:, None] * absx))
    return 2.0 * (term1 + term2).T       # [nb, m]


def _check(oracle, f, Xh):
    U, V, D, _ = X.to_codes(f)
    Y = X.apply(f, torch.from_numpy(Xh).cuda()).cpu().numpy().astype(np.float64)
    assert X.sync_status() == X.OK
    ref = oracle.ternary_apply(U, V, D, Xh)
    bound = _bound(oracle, U, V, D, Xh)
    err = np.abs(Y - ref)
    assert np.all(err <= bound), (float((err / np.maximum(bound, 1e-300)).max()))
    return float((err / np.maximum(np.abs(ref), 1e-30)).max())


@pytest.mark.parametrize("nb", [1, 2, 3])
def test_apply_llm_factors(oracle, nb):
    A = W.llm_like(200, 168, 111, n_outliers=3)
    f = X.decompose(torch.from_numpy(A).cuda(), 2.0, 0.5, 3)
    Xh = np.random.default_rng(nb).standard_normal((nb, 168)).astype(np.float32)
    _check(oracle, f, Xh)


@pytest.mark.parametrize("shape", [(1, 1), (5, 33), (33, 5), (97, 130), (1000, 70)])
def test_apply_ragged_shapes(oracle, shape):
    m, n = shape
    A = W.iid_gaussian(m, n, 7 + m + n)
    f = X.decompose(torch.from_numpy(A).cuda(), 1.5 if min(m, n) > 1 else 2.0, 0.5, 2)
    Xh = np.random.default_rng(m).standard_normal((2, n)).astype(np.float32)
    _check(oracle, f, Xh)


def test_apply_attn2560_full_size(oracle):
    """The benchmark matrix's factors (mu = 3, k = 7680): one vector checked
    element by element; the dense reconstruction agrees."""
    wl = W.config_attn2560()
    f = X.decompose(torch.from_numpy(wl.a).cuda(), wl.mu, wl.tau, wl.iters)
    Xh = np.random.default_rng(5).standard_normal((1, wl.n)).astype(np.float32)
    rel = _check(oracle, f, Xh)
    print(f"attn2560 apply: max relative error {rel:.2e}")
    Ahat = X.reconstruct(f)
    yd = (torch.from_numpy(Xh).cuda().double() @ Ahat.double().T).cpu().numpy()
    Y = X.apply(f, torch.from_numpy(Xh).cuda()).cpu().numpy()
    assert np.allclose(Y, yd, rtol=1e-4, atol=1e-4 * np.abs(yd).max())


def test_apply_reproducible_and_linear():
    A = W.llm_like(300, 256, 12, n_outliers=3)
    f = X.decompose(torch.from_numpy(A).cuda(), 1.5, 0.5, 3)
    x = torch.randn(4, 256, device="cuda")
    y1 = X.apply(f, x)
    y2 = X.apply(f, x)
    assert torch.equal(y1, y2)
    # vectors are independent: a batch equals its rows applied one by one
    for b in range(4):
        assert torch.equal(X.apply(f, x[b:b + 1])[0], y1[b])
