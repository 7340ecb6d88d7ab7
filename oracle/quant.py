"""Quantiser helpers of the oracle (fp64, numpy): greedy +-1 decomposition and
least-squares refit of the scales.

TEST INFRASTRUCTURE (see oracle/__init__.py).  Nothing here is on the GEMV
path; these helpers are pinned by the worked example on the BiLoCo page and
are the building blocks of the offline BCQ quantiser.

Sources, by page title and section:
  * "BiLoCo: Binary Low-Rank Corrections for Post-Training Quantization",
    section "二值向量怎么找": rank-one +-1 components are found one at a time by
    alternating u = sign(R v), v = sign(R^T u); the error-minimising scale of a
    +-1 component is u^T R v divided by the number of entries; the component is
    subtracted from the residual; after all components are found, all scales
    are refit jointly because the components overlap.
  * "AnyBCQ ..." (Paper-Notes page), "关键设计 / 渐进式精度扩展": greedy BCQ
    initialisation, least squares for the scales.

sign(0) is read as +1 (the pages do not say).
"""
from __future__ import annotations

import numpy as np


def sign_pm1(a: np.ndarray) -> np.ndarray:
    """Elementwise sign with sign(0) = +1, as float64 in {-1, +1}."""
    return np.where(np.asarray(a, dtype=np.float64) >= 0.0, 1.0, -1.0)


def greedy_rank1_pm1(W, n_components: int, iters: int = 5, v0=None, rng=None):
    """Greedy rank-one +-1 decomposition W ~ sum_r alpha_r u_r v_r^T.

    For each component: start from v0 (or a random +-1 vector), alternate
    u = sign(R v), v = sign(R^T u) ``iters`` times, take
    alpha = u^T R v / numel(R), subtract alpha u v^T from the residual R.

    Returns (us [r][rows], vs [r][cols], alphas [r], residual R).
    """
    R = np.array(W, dtype=np.float64, copy=True)
    rows, cols = R.shape
    rng = np.random.default_rng(0) if rng is None else rng
    us, vs, alphas = [], [], []
    for r in range(n_components):
        if v0 is not None:
            v = sign_pm1(v0[r] if np.ndim(v0) == 2 else v0)
        else:
            v = sign_pm1(rng.standard_normal(cols))
        u = sign_pm1(R @ v)
        for _ in range(iters):
            u = sign_pm1(R @ v)
            v = sign_pm1(R.T @ u)
        alpha = float(u @ R @ v) / R.size
        R = R - alpha * np.outer(u, v)
        us.append(u)
        vs.append(v)
        alphas.append(alpha)
    return np.array(us), np.array(vs), np.array(alphas), R


def lsq_scales(W, mats) -> np.ndarray:
    """Least-squares scales: argmin_a || W - sum_i a_i M_i ||_F^2.

    Solves the normal equations Gram a = rhs with Gram_ij = <M_i, M_j> and
    rhs_i = <M_i, W> (np.linalg.lstsq on the Gram system, which also covers a
    singular Gram).
    """
    W = np.asarray(W, dtype=np.float64)
    Ms = [np.asarray(m, dtype=np.float64) for m in mats]
    r = len(Ms)
    gram = np.empty((r, r))
    rhs = np.empty(r)
    for i in range(r):
        rhs[i] = np.sum(Ms[i] * W)
        for j in range(r):
            gram[i, j] = np.sum(Ms[i] * Ms[j])
    sol, *_ = np.linalg.lstsq(gram, rhs, rcond=None)
    return sol


def sse(W, mats, scales) -> float:
    """Squared Frobenius norm of W - sum_i scales_i M_i."""
    W = np.asarray(W, dtype=np.float64)
    approx = np.zeros_like(W)
    for a, m in zip(scales, mats):
        approx += a * np.asarray(m, dtype=np.float64)
    return float(np.sum((W - approx) ** 2))


def greedy_bcq(w, p: int):
    """Greedy BCQ of a vector: for i = 1..p, B_i = sign(r), alpha_i = mean|r|
    (the error-minimising scale u^T r / numel for u = sign(r)), r -= alpha_i B_i.

    Returns (B [p][n] in {-1,+1}, alpha [p], residual r).
    """
    r = np.array(w, dtype=np.float64, copy=True).ravel()
    Bs, alphas = [], []
    for _ in range(p):
        b = sign_pm1(r)
        a = float(b @ r) / r.size
        r = r - a * b
        Bs.append(b)
        alphas.append(a)
    return np.array(Bs), np.array(alphas), r
