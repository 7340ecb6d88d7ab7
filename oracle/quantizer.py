"""Oracle of the offline multi-precision BCQ quantiser (fp64, numpy).

TEST INFRASTRUCTURE (see oracle/__init__.py): only tests/, the package's
smoke check and bench.py's CPU baseline may use it.  It shares no code with
the CUDA library.  Parity status: pinned (tests/test_quantizer_oracle.py:
closed forms, brute-force code search and least squares on tiny groups,
exactly representable groups, the monotone-error invariants, the BiLoCo
worked example for the least-squares step).

What it computes, by page title and section:
  * "AnyBCQ ..." (Paper-Notes page), "关键设计 / 渐进式精度扩展": at the base
    precision p_L the codes are initialised greedily and refined by
    alternating a least-squares solve for the scales with a search for the
    best code of every weight; each expansion p -> p + 1 freezes B_1..B_p,
    adds B_{p+1} = sign(R_p) (the sign of the residual at precision p) and
    refits all p + 1 scales alpha^(p+1) by least squares only.
  * same page, "训练策略": asymmetric BCQ, groups of 128 columns, 20 rounds
    of alternating refinement at initialisation.
  * "BiLoCo ..." page, "二值向量怎么找": the greedy scale of a +-1 component is
    its inner product with the residual over the number of entries, and the
    component is then subtracted from the residual.

Readings (the pages leave them open):
  * one offset z per (row, group), shared by every precision (the format
    the GEMV reads): z is a least-squares variable -- the scale of an
    all-ones plane -- during the base precision's refinement, started at the
    group mean, and is frozen afterwards, so that, like the codes, it is
    shared and the error can only fall as planes are added;
  * greedy initialisation: b_i = sign(r), alpha_i = <b_i, r> / n, r -= alpha_i b_i,
    starting from r = w - mean(w);
  * "BS" (the code update) is read as its result: every weight takes the
    code in {-1,+1}^p whose value z + sum_i alpha_i b_i is nearest to the
    weight; ties go to the candidate enumerated first (candidate c has
    b_i = +1 where bit i of c is set).  A binary search over the sorted
    candidate values finds the same nearest value;
  * one refinement round = least squares, then code update; after the last
    round the scales are refit once more, so they are the least-squares
    optimum for the final codes;
  * a least-squares system whose columns are linearly dependent (a plane
    equal to another, to its negation or to the all-ones plane, or any
    other exact dependence) is solved on the columns that are independent
    of the columns before them, in column order (the all-ones column of z
    first, then planes 1..p); the others get scale 0.  A constant group is
    thus all offset (z = its value, alpha = 0).  The Gram matrix of +-1 and all-ones columns is integer-valued, so the
    dependence is decided exactly (rational elimination);
  * candidate values and residuals are formed in fp64 as
    z + (((alpha_1 b_1) + alpha_2 b_2) + ...), left to right;
  * sign(0) = +1; inputs are fp16 weights widened to fp64; scales and offsets
    are rounded to fp16 (nearest even) only when stored.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

from .quant import sign_pm1


def independent_columns(gram) -> list:
    """Columns of an integer Gram matrix that are linearly independent of
    the columns before them, decided in exact rational arithmetic.

    Column j is kept when the Gram matrix of the kept columns plus j is
    non-singular, i.e. when Gaussian elimination (over the rationals) of
    that matrix finds a non-zero pivot in every column."""
    G = [[Fraction(int(round(v))) for v in row] for row in np.asarray(gram)]
    kept = []
    for j in range(len(G)):
        trial = kept + [j]
        A = [[G[r][c] for c in trial] for r in trial]
        n = len(trial)
        full = True
        for col in range(n):
            piv = next((r for r in range(col, n) if A[r][col] != 0), None)
            if piv is None:
                full = False
                break
            A[col], A[piv] = A[piv], A[col]
            for r in range(col + 1, n):
                f = A[r][col] / A[col][col]
                if f:
                    A[r] = [a - f * b for a, b in zip(A[r], A[col])]
        if full:
            kept.append(j)
    return kept


def lsq(W, B, z=None):
    """Least squares per problem.  W [P][n]; B [P][p][n] in {-1,+1}.
    With z None the unknowns are (z, alpha_1..alpha_p) (an all-ones column
    first); otherwise z [P] is fixed and only alpha is solved.
    Returns (alpha [P][p], z [P])."""
    W = np.asarray(W, dtype=np.float64)
    P, p, n = B.shape
    if z is None:
        A = np.concatenate([np.ones((P, 1, n)), B], axis=1)
        target = W
    else:
        A = B
        target = W - z[:, None]
    gram = np.einsum("qin,qjn->qij", A, A)        # integers, exact in fp64
    rhs = np.einsum("qin,qn->qi", A, target)
    sol = np.zeros_like(rhs)
    for q in range(P):
        kept = independent_columns(gram[q])
        sol[q, kept] = np.linalg.solve(gram[q][np.ix_(kept, kept)], rhs[q, kept])
    if z is None:
        return sol[:, 1:], sol[:, 0]
    return sol, np.array(z, dtype=np.float64, copy=True)


def candidates(p: int) -> np.ndarray:
    """The 2^p codes in enumeration order: row c, column i = +1 if bit i of c."""
    c = np.arange(2 ** p)[:, None]
    return np.where((c >> np.arange(p)[None, :]) & 1, 1.0, -1.0)


def code_values(alpha, z, codes):
    """z + (((alpha_1 b_1) + alpha_2 b_2) + ...) in fp64, left to right.
    alpha [P][p], z [P], codes [P][p][...] -> [P][...]."""
    p = alpha.shape[1]
    extra = (1,) * (codes.ndim - 2)
    acc = alpha[:, 0].reshape((-1,) + extra) * codes[:, 0]
    for i in range(1, p):
        acc = acc + alpha[:, i].reshape((-1,) + extra) * codes[:, i]
    return z.reshape((-1,) + extra) + acc


def best_codes(W, alpha, z):
    """Code update: for every weight the code whose value is nearest.
    W [P][n], alpha [P][p], z [P] -> B [P][p][n]."""
    W = np.asarray(W, dtype=np.float64)
    P, n = W.shape
    p = alpha.shape[1]
    C = candidates(p)                                            # [2^p][p]
    vals = code_values(alpha, z, np.broadcast_to(C.T[None], (P, p, 2 ** p)))
    err = np.abs(W[:, :, None] - vals[:, None, :])               # [P][n][2^p]
    idx = np.argmin(err, axis=2)                                 # first minimum
    return np.transpose(C[idx], (0, 2, 1))                       # [P][p][n]


def residual(W, B, alpha, z):
    """R = w - (z + sum_i alpha_i b_i) per weight, [P][n]."""
    return np.asarray(W, dtype=np.float64) - code_values(alpha, z, B)


def group_sse(W, B, alpha, z):
    """Squared error of every problem, [P]."""
    return np.sum(residual(W, B, alpha, z) ** 2, axis=1)


def quantize_groups(W, p_L: int = 2, p_H: int = 4, rounds: int = 20, trace=None):
    """Quantise P independent groups W [P][n] (fp64).

    Returns (B [P][p_H][n] in {-1,+1}, {p: alpha^(p) [P][p]} for p = p_L..p_H,
    z [P]).  trace, if a list, receives (stage, sse [P]) after every step."""
    W = np.asarray(W, dtype=np.float64)
    P, n = W.shape
    if not 1 <= p_L <= p_H:
        raise ValueError("need 1 <= p_L <= p_H")

    def record(stage, B, alpha, z):
        if trace is not None:
            trace.append((stage, group_sse(W, B, alpha, z)))

    # base precision, greedy: peel sign(r) off the residual of the group mean
    z = W.mean(axis=1)
    r = W - z[:, None]
    Bs, alphas = [], []
    for _ in range(p_L):
        b = sign_pm1(r)
        a = np.sum(b * r, axis=1) / n
        r = r - a[:, None] * b
        Bs.append(b)
        alphas.append(a)
    B = np.stack(Bs, axis=1)
    alpha = np.stack(alphas, axis=1)
    record("greedy", B, alpha, z)
    # alternating refinement: least squares for (alpha, z), then nearest codes
    for _ in range(rounds):
        alpha, z = lsq(W, B)
        record("lsq", B, alpha, z)
        B = best_codes(W, alpha, z)
        record("codes", B, alpha, z)
    alpha, z = lsq(W, B)
    out_alpha = {p_L: alpha}
    record(f"p{p_L}", B, alpha, z)
    # progressive expansion: codes and z frozen, the residual's sign appended
    for p in range(p_L, p_H):
        B = np.concatenate([B, sign_pm1(residual(W, B, alpha, z))[:, None, :]], axis=1)
        alpha, _ = lsq(W, B, z)
        out_alpha[p + 1] = alpha
        record(f"p{p + 1}", B, alpha, z)
    return B, out_alpha, z


def quantize(W, group: int = 128, p_L: int = 2, p_H: int = 4, rounds: int = 20):
    """Quantise a weight W [N][K] (K a multiple of the group size and of 32)
    into the canonical format the GEMV reads.

    Returns (planes uint32 [p_H][N][K/32], bit j of word w = column 32w + j,
    bit 1 = +1; {p: alpha^(p) fp64 [N][K/group][p]} for p = p_L..p_H;
    z fp64 [N][K/group])."""
    W = np.asarray(W, dtype=np.float64)
    N, K = W.shape
    if K % group or K % 32:
        raise ValueError("K must be a multiple of the group size and of 32")
    G = K // group
    B, alphas, z = quantize_groups(W.reshape(N * G, group), p_L, p_H, rounds)
    bits = (B > 0).reshape(N, G, p_H, group).transpose(2, 0, 1, 3).reshape(p_H, N, K)
    words = bits.reshape(p_H, N, K // 32, 32).astype(np.uint64)
    planes = np.sum(words << np.arange(32, dtype=np.uint64), axis=3).astype(np.uint32)
    out = {p: a.reshape(N, G, p) for p, a in alphas.items()}
    return planes, out, z.reshape(N, G)
