"""Seeded synthetic inputs for the multi-precision BCQ matmul.

This module holds no arithmetic of the method: it only draws random bit-planes,
scales, offsets, activations and per-row precisions with numpy, in a fixed
order, so that the CUDA path and the CPU oracle see identical inputs.

Recipe (one numpy PCG64 generator, ``np.random.default_rng(seed)``; draws in
this order):
  1. planes   uint32 [p_H][N][K/32], every bit Bernoulli(0.5)
               (uniform 32-bit words), bit j of word w <-> column 32w + j,
               bit 1 = +1, bit 0 = -1;
  2. alpha^(q) for q in ``precisions`` (ascending): fp16 [N][G][q],
               alpha_i = 0.02 * 2^-(i-1) * U(0.8, 1.2), i = 1..q;
  3. z        fp16 [N][G] ~ N(0, 0.005^2) (0.005 is the standard deviation);
  4. x        fp16 [M][K] ~ N(0, 1);
  5. outlier channels (only when ``outliers``): max(1, round(0.001 K))
               columns of x, without replacement, multiplied by 20 before the
               fp16 rounding;
  6. p_row    (only when ``mixed``): int32 [M], uniform in {2, 3, 4}.
Values are rounded to fp16 before anyone sees them.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

GROUP = 128


@dataclass
class Problem:
    x: np.ndarray            # fp16 [M][K]
    planes: np.ndarray       # uint32 [p_H][N][K/32]
    alphas: dict             # {q: fp16 [N][G][q]}
    z: np.ndarray            # fp16 [N][G]
    p_row: np.ndarray | None = None   # int32 [M] or None
    meta: dict = field(default_factory=dict)

    @property
    def M(self) -> int:
        return self.x.shape[0]

    @property
    def K(self) -> int:
        return self.x.shape[1]

    @property
    def N(self) -> int:
        return self.planes.shape[1]

    @property
    def p_H(self) -> int:
        return self.planes.shape[0]


def make_problem(N: int, K: int, M: int = 1, *, seed: int = 0, p_H: int = 4,
                 precisions=(2, 3, 4), outliers: bool = False,
                 mixed: bool = False, group: int = GROUP) -> Problem:
    if K % group or K % 32:
        raise ValueError("K must be a multiple of the group size and of 32")
    rng = np.random.default_rng(seed)
    G = K // group
    planes = rng.integers(0, 2**32, size=(p_H, N, K // 32), dtype=np.uint32)
    alphas = {}
    for q in sorted(precisions):
        u = rng.uniform(0.8, 1.2, size=(N, G, q))
        scale = 0.02 * np.exp2(-np.arange(q, dtype=np.float64))
        alphas[q] = (u * scale).astype(np.float16)
    z = rng.normal(0.0, 0.005, size=(N, G)).astype(np.float16)
    x = rng.normal(0.0, 1.0, size=(M, K))
    chans = None
    if outliers:
        n_out = max(1, int(round(0.001 * K)))
        chans = rng.choice(K, size=n_out, replace=False)
        x[:, chans] *= 20.0
    x = x.astype(np.float16)
    p_row = rng.integers(2, 5, size=M).astype(np.int32) if mixed else None
    meta = dict(N=N, K=K, M=M, seed=seed, p_H=p_H, outliers=outliers,
                mixed=mixed, outlier_channels=None if chans is None else
                sorted(int(c) for c in chans))
    return Problem(x=x, planes=planes, alphas=alphas, z=z, p_row=p_row,
                   meta=meta)


def make_x(M: int, K: int, *, seed: int) -> np.ndarray:
    """Extra activations ~ N(0,1), fp16, from their own seeded generator."""
    rng = np.random.default_rng(seed)
    return rng.normal(0.0, 1.0, size=(M, K)).astype(np.float16)


def make_weights(N: int, K: int, *, seed: int, outliers: bool = True) -> np.ndarray:
    """fp16 weights [N][K] for the offline quantiser, shaped like a trained
    projection matrix.  Recipe (``np.random.default_rng(seed)``, draws in this
    order): row scales s_n = 0.02 * U(0.5, 1.5); w = s_n * N(0, 1); when
    ``outliers``, round(0.001 N K) entries (positions without replacement)
    multiplied by 8; then rounded to fp16."""
    rng = np.random.default_rng(seed)
    s = 0.02 * rng.uniform(0.5, 1.5, size=(N, 1))
    w = s * rng.normal(0.0, 1.0, size=(N, K))
    if outliers and N * K > 0:
        n_out = int(round(0.001 * N * K))
        if n_out:
            idx = rng.choice(N * K, size=n_out, replace=False)
            w.reshape(-1)[idx] *= 8.0
    return w.astype(np.float16)
