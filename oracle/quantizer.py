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
    starting from r = w - mean(w); <b_i, r> is evaluated as
    sum(b_i w) - z sum(b_i) - sum_j alpha_j <b_i, b_j> (exact sums and
    integers, left to right);
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
    thus all offset (z = its value, alpha = 0).  The Gram matrix of +-1 and
    all-ones columns is integer-valued, so the dependence is decided exactly
    (integer determinants), and the normal equations are solved by Cramer's
    rule with the exact integer adjugate and determinant;
  * candidate values and residuals are formed in fp64 as
    z + (((alpha_1 b_1) + alpha_2 b_2) + ...), left to right;
  * sign(0) = +1; inputs are fp16 weights widened to fp64; scales and offsets
    are rounded to fp16 (nearest even) only when stored;
  * variant with offsets per precision (offsets="per_precision", for the
    format in which every precision keeps its own z^(p) as it keeps its own
    scales): each expansion refits z jointly with all p + 1 scales (the
    all-ones column first, as at the base precision); the residual of
    precision p uses z^(p).
"""
from __future__ import annotations

import numpy as np

from .quant import sign_pm1


def det_int(M) -> int:
    """Exact determinant of a small integer matrix (Python integers, Laplace
    expansion along the first row)."""
    M = [[int(v) for v in row] for row in M]
    if not M:
        return 1
    if len(M) == 2:
        return M[0][0] * M[1][1] - M[0][1] * M[1][0]
    if len(M) == 1:
        return M[0][0]
    return sum((-1) ** j * M[0][j] * det_int([r[:j] + r[j + 1:] for r in M[1:]])
               for j in range(len(M)))


def adjugate_int(M) -> list:
    """Exact adjugate: adj[i][j] = (-1)^(i+j) det(M without row j and column i)."""
    M = [[int(v) for v in row] for row in M]
    n = len(M)
    return [[(-1) ** (i + j) * det_int([r[:i] + r[i + 1:] for k, r in enumerate(M) if k != j])
             for j in range(n)] for i in range(n)]


def independent_columns(gram) -> list:
    """Columns of an integer Gram matrix that are linearly independent of
    the kept columns before them: column j is kept when the Gram matrix of
    the kept columns plus j has a non-zero determinant (exact integers)."""
    G = [[int(round(float(v))) for v in row] for row in gram]
    kept = []
    for j in range(len(G)):
        trial = kept + [j]
        if det_int([[G[a][b] for b in trial] for a in trial]) != 0:
            kept.append(j)
    return kept


def solve_normal_equations(gram, rhs):
    """x with gram x = rhs on the kept columns (0 elsewhere), by Cramer's rule
    with the exact integer adjugate and determinant of the kept columns' Gram
    matrix: x_a = (adj[a][0] r_0 + adj[a][1] r_1 + ...) / det, the products
    and sums in fp64 from left to right."""
    kept = independent_columns(gram)
    G = [[int(round(float(v))) for v in row] for row in gram]
    Gk = [[G[a][b] for b in kept] for a in kept]
    r = [float(v) for v in rhs]
    adj = adjugate_int(Gk)
    det = float(det_int(Gk))
    x = np.zeros(len(r))
    for a, ka in enumerate(kept):
        acc = float(adj[a][0]) * r[kept[0]]
        for b in range(1, len(kept)):
            acc = acc + float(adj[a][b]) * r[kept[b]]
        x[ka] = acc / det
    return x


def lsq(W, B, z=None):
    """Least squares per problem.  W [P][n]; B [P][p][n] in {-1,+1}.
    With z None the unknowns are (z, alpha_1..alpha_p) (an all-ones column
    first); otherwise z [P] is fixed and only alpha is solved.
    Returns (alpha [P][p], z [P]).

    Right-hand sides: with z free, sum(w) and sum(b_i w); with z fixed,
    sum(b_i (w - z)) evaluated as sum(b_i w) - z sum(b_i).  For fp16 weights
    sum(b_i w) is exact in fp64 in any order (every partial sum is a multiple
    of 2^-24 below 2^23) and sum(b_i) is an integer, so every right-hand
    side is exact or one rounding from exact."""
    W = np.asarray(W, dtype=np.float64)
    P, p, n = B.shape
    if z is None:
        A = np.concatenate([np.ones((P, 1, n)), B], axis=1)
        rhs = np.einsum("qin,qn->qi", A, W)
    else:
        A = B
        rhs = np.einsum("qin,qn->qi", B, W) - z[:, None] * B.sum(axis=2)
    gram = np.einsum("qin,qjn->qij", A, A)        # integers, exact in fp64
    sol = np.stack([solve_normal_equations(gram[q], rhs[q]) for q in range(P)])
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


def quantize_groups(W, p_L: int = 2, p_H: int = 4, rounds: int = 20, trace=None,
                    offsets: str = "shared"):
    """Quantise P independent groups W [P][n] (fp64).

    Returns (B [P][p_H][n] in {-1,+1}, {p: alpha^(p) [P][p]} for p = p_L..p_H,
    z [P]; with offsets="per_precision", z is {p: z^(p) [P]}).  trace, if a
    list, receives (stage, sse [P]) after every step."""
    W = np.asarray(W, dtype=np.float64)
    P, n = W.shape
    if not 1 <= p_L <= p_H:
        raise ValueError("need 1 <= p_L <= p_H")
    if offsets not in ("shared", "per_precision"):
        raise ValueError("offsets must be 'shared' or 'per_precision'")

    def record(stage, B, alpha, z):
        if trace is not None:
            trace.append((stage, group_sse(W, B, alpha, z)))

    # base precision, greedy: peel sign(r) off the residual of the group mean
    z = W.mean(axis=1)
    r = W - z[:, None]
    Bs, alphas = [], []
    for _ in range(p_L):
        b = sign_pm1(r)
        # <b, r> = sum(b w) - z sum(b) - sum_j alpha_j <b, b_j>, left to right
        t = np.sum(b * W, axis=1) - z * np.sum(b, axis=1)
        for bj, aj in zip(Bs, alphas):
            t = t - aj * np.sum(b * bj, axis=1)
        a = t / n
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
    out_alpha, out_z = {p_L: alpha}, {p_L: z}
    record(f"p{p_L}", B, alpha, z)
    # progressive expansion: codes (and shared z) frozen, the residual's sign appended
    for p in range(p_L, p_H):
        B = np.concatenate([B, sign_pm1(residual(W, B, alpha, z))[:, None, :]], axis=1)
        if offsets == "shared":
            alpha, _ = lsq(W, B, z)
        else:
            alpha, z = lsq(W, B)
        out_alpha[p + 1] = alpha
        out_z[p + 1] = z
        record(f"p{p + 1}", B, alpha, z)
    return B, out_alpha, (z if offsets == "shared" else out_z)


def quantize(W, group: int = 128, p_L: int = 2, p_H: int = 4, rounds: int = 20, trace=None,
             offsets: str = "shared"):
    """Quantise a weight W [N][K] (K a multiple of the group size and of 32)
    into the canonical format the GEMV reads.

    Returns (planes uint32 [p_H][N][K/32], bit j of word w = column 32w + j,
    bit 1 = +1; {p: alpha^(p) fp64 [N][K/group][p]} for p = p_L..p_H;
    z fp64 [N][K/group], or {p: z^(p)} with offsets="per_precision").  trace:
    as for quantize_groups (groups row-major)."""
    W = np.asarray(W, dtype=np.float64)
    N, K = W.shape
    if K % group or K % 32:
        raise ValueError("K must be a multiple of the group size and of 32")
    G = K // group
    B, alphas, z = quantize_groups(W.reshape(N * G, group), p_L, p_H, rounds, trace, offsets)
    bits = (B > 0).reshape(N, G, p_H, group).transpose(2, 0, 1, 3).reshape(p_H, N, K)
    words = bits.reshape(p_H, N, K // 32, 32).astype(np.uint64)
    planes = np.sum(words << np.arange(32, dtype=np.uint64), axis=3).astype(np.uint32)
    out = {p: a.reshape(N, G, p) for p, a in alphas.items()}
    if isinstance(z, dict):
        return planes, out, {p: zp.reshape(N, G) for p, zp in z.items()}
    return planes, out, z.reshape(N, G)
