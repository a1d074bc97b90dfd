"""Seeded synthetic input matrices for the ExTernD decomposition.

This module only draws random inputs.  It holds none of the decomposition's
arithmetic and is the one piece of code that both the CUDA path's tests and
the CPU oracle's tests use, so that both sides read the same bytes.

The real model tensors that the ExTernD pages measure on (Gemma-4-E2B and
Qwen3.5-4B projections) are not available; these matrices stand in for their
shapes and statistics:

* ``iid``      -- entries i.i.d. N(0, 1).
* ``llm_like`` -- A0 = U diag(s) V^T with Haar-random orthonormal U (m x r) and
  V (n x r), r = min(m, n), singular values s_i proportional to i^-alpha and
  scaled so that the entry rms of A0 is 0.02; plus Student-t(nu=4) noise
  multiplied by 0.002; then a set of outlier columns (or rows) multiplied
  by 10 after the noise.

All draws are fp64 from numpy's PCG64 and the matrix is stored as fp32
(row-major, C order).  The draw order is fixed: U's Gaussian, V's Gaussian,
the t noise, then the outlier indices.  Importance weights come from a
second PCG64 stream seeded with (seed, 1) so that they do not perturb the
matrix draws.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np


def _haar_columns(rng: np.random.Generator, rows: int, cols: int) -> np.ndarray:
    """Orthonormal columns from the QR of a Gaussian matrix, with the sign of
    R's diagonal folded into Q so the result is Haar distributed
    (Mezzadri's correction)."""
    g = rng.standard_normal((rows, cols))
    q, r = np.linalg.qr(g, mode="reduced")
    d = np.sign(np.diag(r))
    d[d == 0] = 1.0
    return q * d[None, :]


def iid_gaussian(m: int, n: int, seed: int) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.standard_normal((m, n)).astype(np.float32)


def llm_like(m: int, n: int, seed: int, alpha: float = 0.5, n_outliers: int = 8,
             outlier_axis: str = "col", entry_rms: float = 0.02,
             noise_scale: float = 0.002, outlier_gain: float = 10.0) -> np.ndarray:
    """Power-law spectrum matrix with heavy-tailed noise and outlier lines."""
    rng = np.random.Generator(np.random.PCG64(seed))
    r = min(m, n)
    u = _haar_columns(rng, m, r)
    v = _haar_columns(rng, n, r)
    s = np.arange(1, r + 1, dtype=np.float64) ** (-alpha)
    # entry rms of U diag(s) V^T is ||s||_2 / sqrt(m n) because U, V have
    # orthonormal columns
    s *= entry_rms * np.sqrt(m * n) / np.linalg.norm(s)
    a = (u * s[None, :]) @ v.T
    a += noise_scale * rng.standard_t(4.0, size=(m, n))
    if outlier_axis == "col":
        idx = rng.choice(n, size=n_outliers, replace=False)
        a[:, idx] *= outlier_gain
    elif outlier_axis == "row":
        idx = rng.choice(m, size=n_outliers, replace=False)
        a[idx, :] *= outlier_gain
    else:
        raise ValueError(outlier_axis)
    return np.ascontiguousarray(a.astype(np.float32))


def lognormal_weights(n: int, seed: int, sigma: float = 1.0) -> np.ndarray:
    """Per-input-column importance weights w_j = exp(N(0, sigma^2)),
    normalised to mean 1 (stand-in for imatrix second moments)."""
    rng = np.random.Generator(np.random.PCG64([seed, 1]))
    w = np.exp(sigma * rng.standard_normal(n))
    w /= w.mean()
    return w.astype(np.float32)


@dataclass
class Workload:
    """One decomposition problem: a matrix plus the method's knobs."""
    name: str
    a: np.ndarray
    mu: float
    tau: float
    iters: int
    block: int = 1
    w: Optional[np.ndarray] = None
    meta: dict = field(default_factory=dict)

    @property
    def m(self) -> int:
        return int(self.a.shape[0])

    @property
    def n(self) -> int:
        return int(self.a.shape[1])

    @property
    def k(self) -> int:
        return int(np.floor(self.mu * min(self.m, self.n) + 1e-9))


def config_small(tau: float = 0.5) -> Workload:
    """256 x 256 i.i.d. N(0,1), mu=2 (k=512), tau=0.5, 4 ALS iterations."""
    return Workload("iid256", iid_gaussian(256, 256, 101), mu=2.0, tau=tau, iters=4,
                    meta={"seed": 101})


def config_llm1024(tau: float = 0.5) -> Workload:
    """1024 x 1024 LLM-like matrix, mu=1.5, tau in {0.3, 0.5, 0.7}, 4 iterations."""
    return Workload(f"llm1024_tau{tau}", llm_like(1024, 1024, 102), mu=1.5, tau=tau,
                    iters=4, meta={"seed": 102})


def config_attn2560() -> Workload:
    """2560 x 2560 attention-projection-shaped matrix with 16 outlier columns,
    mu=3 (k=7680), tau=0.5, 6 iterations."""
    return Workload("attn2560", llm_like(2560, 2560, 103, n_outliers=16), mu=3.0, tau=0.5,
                    iters=6, meta={"seed": 103})


def config_mlp9728(block: int = 64) -> Workload:
    """9728 x 2560 MLP-up-shaped matrix, spectrum exponent 0.4, 32 outlier rows,
    mu=2, tau=0.5, 4 iterations, block-ALS with b components per sweep."""
    a = llm_like(9728, 2560, 104, alpha=0.4, n_outliers=32, outlier_axis="row")
    return Workload(f"mlp9728_b{block}", a, mu=2.0, tau=0.5, iters=4, block=block,
                    meta={"seed": 104})


# one synthetic transformer block: hidden 2560, intermediate 9728,
# 32 query heads / 8 key-value heads of dimension 128
BLOCK_MATRICES = (
    ("q", 4096, 2560),
    ("k", 1024, 2560),
    ("v", 1024, 2560),
    ("o", 2560, 4096),
    ("gate", 9728, 2560),
    ("up", 9728, 2560),
    ("down", 2560, 9728),
)


def config_block_matrices(block: int = 64):
    """The seven matrices of one transformer block, importance weighted,
    mu=3, tau=0.5, 4 iterations, b=64.  Matrix i uses seed 105+i."""
    out = []
    for i, (nm, m, n) in enumerate(BLOCK_MATRICES):
        seed = 105 + i
        a = llm_like(m, n, seed)
        w = lognormal_weights(n, seed)
        out.append(Workload(f"blk_{nm}", a, mu=3.0, tau=0.5, iters=4, block=block, w=w,
                            meta={"seed": seed}))
    return out
