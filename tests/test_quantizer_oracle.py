"""Pins of the quantiser oracle (oracle/quantizer.py), CPU only.

Each test fixes the oracle to something other than itself: the BiLoCo worked
example (tests/golden/biloco_greedy_3x2.txt), closed forms, brute force on
tiny groups, exactly representable groups and the monotone-error guarantee
of progressive expansion (AnyBCQ page, "关键设计 / 渐进式精度扩展": adding a
plane and refitting every scale can only lower the error, because the old
scales with a zero for the new plane are one of the candidates).

BCQ_QUANTIZER_ORACLE, if set, names another copy of quantizer.py to test
(tests/test_quantizer_mutants.py plants mistakes in copies and expects these
pins to fail).
"""
import importlib.util
import itertools
import os

import numpy as np
import pytest

import oracle
from oracle import quant

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load_quantizer():
    path = os.environ.get("BCQ_QUANTIZER_ORACLE")
    if not path:
        from oracle import quantizer
        return quantizer
    spec = importlib.util.spec_from_file_location("oracle._quantizer_under_test", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


Q = _load_quantizer()


def _read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split(":", 1)
            rows = [np.array([float(t) for t in r.split()]) for r in val.split(";")]
            v = np.stack(rows) if len(rows) > 1 else rows[0]
            out[key.strip()] = float(v[0]) if v.size == 1 else v
    return out


def _pm1(bits):
    return np.where(np.asarray(bits) != 0, 1.0, -1.0)


def _weights(shape, seed, kind="normal"):
    rng = np.random.default_rng(seed)
    if kind == "normal":
        w = rng.standard_normal(shape) * 0.02
    elif kind == "laplace":
        w = rng.laplace(size=shape) * 0.02
    else:
        w = rng.standard_t(3, size=shape) * 0.02
    return w.astype(np.float16).astype(np.float64)


# ------------------------------------------------------------ exact dependence

def _rank_incremental(G):
    kept = []
    for j in range(G.shape[0]):
        t = kept + [j]
        if np.linalg.matrix_rank(G[np.ix_(t, t)]) == len(t):
            kept.append(j)
    return kept


def test_independent_columns_planted_dependencies():
    rng = np.random.default_rng(0)
    b1 = _pm1(rng.integers(0, 2, 128))
    b2 = _pm1(rng.integers(0, 2, 128))
    ones = np.ones(128)
    # b1 + b2 = b3 + 1 wherever (b1, b2) != (-1, -1): b3 is +1 only at (+,+)
    keep = ~((b1 < 0) & (b2 < 0))
    c1, c2 = b1[keep], b2[keep]
    c3 = np.where((c1 > 0) & (c2 > 0), 1.0, -1.0)
    cases = [
        (np.stack([ones, b1, b2]), [0, 1, 2]),
        (np.stack([ones, b1, b1]), [0, 1]),
        (np.stack([ones, b1, -b1, b2]), [0, 1, 3]),
        (np.stack([ones, ones, b2]), [0, 2]),
        (np.stack([ones, ones, ones]), [0]),
        (np.stack([b1, b2, b1 * 0 + 1]), [0, 1, 2]),
        (np.stack([np.ones(c1.size), c1, c2, c3]), [0, 1, 2]),
        (np.stack([c1, c2, c3, np.ones(c1.size)]), [0, 1, 2]),
    ]
    for A, want in cases:
        G = A @ A.T
        assert Q.independent_columns(G) == want
        assert _rank_incremental(G) == want


def test_independent_columns_random_against_rank():
    rng = np.random.default_rng(1)
    for _ in range(60):
        n = int(rng.integers(3, 9))
        k = int(rng.integers(1, 6))
        A = _pm1(rng.integers(0, 2, (k, n)))
        G = A @ A.T
        assert Q.independent_columns(G) == _rank_incremental(G)


# --------------------------------------------------------------- least squares

def test_adjugate_and_determinant_identities():
    # M adj(M) = adj(M) M = det(M) I on random integer matrices (not symmetric),
    # and det against numpy's floating-point determinant
    rng = np.random.default_rng(4)
    for k in range(1, 6):
        for _ in range(20):
            M = rng.integers(-9, 10, (k, k))
            adj = np.array(Q.adjugate_int(M), dtype=np.int64)
            d = Q.det_int(M)
            assert np.array_equal(M @ adj, d * np.eye(k, dtype=np.int64))
            assert np.array_equal(adj @ M, d * np.eye(k, dtype=np.int64))
            assert abs(d - np.linalg.det(M)) < 1e-6 * max(1.0, abs(d))
    assert Q.det_int(np.zeros((0, 0))) == 1


def test_solve_normal_equations_closed_forms():
    # 1x1: x = r / g; 2x2 [[2, 1], [1, 2]] x = (3, 3) -> (1, 1); a dependent
    # middle column gets 0 and the others solve the reduced system
    assert np.array_equal(Q.solve_normal_equations(np.array([[128.0]]), np.array([64.0])), [0.5])
    assert np.array_equal(Q.solve_normal_equations(np.array([[2.0, 1], [1, 2]]), np.array([3.0, 3])),
                          [1.0, 1.0])
    G = np.array([[4.0, 4, 0], [4, 4, 0], [0, 0, 4]])
    assert np.array_equal(Q.solve_normal_equations(G, np.array([8.0, 8, 2])), [2.0, 0.0, 0.5])

def test_lsq_reproduces_biloco_joint_refit():
    g = _read_golden("biloco_greedy_3x2.txt")
    W = g["W"].reshape(1, -1)                                   # 3x2 flattened
    c1 = np.outer(g["c1_u"], g["c1_v"]).reshape(-1)
    c2 = np.outer(g["c2_u"], g["c2_v"]).reshape(-1)
    alpha, z = Q.lsq(W, np.stack([c1, c2])[None], np.zeros(1))
    assert np.allclose(alpha[0], g["joint_alpha"], atol=1e-12)
    assert abs(Q.group_sse(W, np.stack([c1, c2])[None], alpha, z)[0] -
               float(g["joint_sse"])) < 1e-12
    # the greedy scale of the first component is the BiLoCo rule <u v^T, R>/numel
    assert abs(float(c1 @ W[0]) / W.size - float(g["c1_alpha"])) < 1e-12


@pytest.mark.parametrize("p", [1, 2, 3, 4])
@pytest.mark.parametrize("fixed_z", [False, True])
def test_lsq_is_the_least_squares_minimum(p, fixed_z):
    rng = np.random.default_rng(10 + p)
    P, n = 40, 128
    W = _weights((P, n), 3 + p)
    B = _pm1(rng.integers(0, 2, (P, p, n)))
    z0 = rng.normal(size=P) * 0.01 if fixed_z else None
    alpha, z = Q.lsq(W, B, z0)
    for q in range(P):
        if fixed_z:
            A, t = B[q].T, W[q] - z0[q]
        else:
            A, t = np.concatenate([np.ones((n, 1)), B[q].T], axis=1), W[q]
        best = np.linalg.lstsq(A, t, rcond=None)[0]
        sse_best = float(np.sum((t - A @ best) ** 2))
        sse = float(np.sum((W[q] - z[q] - alpha[q] @ B[q]) ** 2))
        assert abs(sse - sse_best) <= 1e-12 * max(1.0, float(t @ t))
        # normal equations: the residual is orthogonal to every column
        res = W[q] - z[q] - alpha[q] @ B[q]
        assert np.max(np.abs(A.T @ res)) < 1e-12
    if fixed_z:
        assert np.array_equal(z, z0)


def test_lsq_dependent_columns_get_zero_scale():
    rng = np.random.default_rng(5)
    n = 128
    b1 = _pm1(rng.integers(0, 2, n))
    w = 0.3 + 0.7 * b1 + rng.normal(size=n) * 0.01
    # planes (b1, -b1): the second is dependent and gets 0
    alpha, z = Q.lsq(w[None], np.stack([b1, -b1])[None])
    assert alpha[0, 1] == 0.0
    assert abs(z[0] - np.mean(w - alpha[0, 0] * b1)) < 1e-12
    # planes (+1, b1): the first equals the offset column and gets 0
    alpha, z = Q.lsq(w[None], np.stack([np.ones(n), b1])[None])
    assert alpha[0, 0] == 0.0
    a_ls = np.linalg.lstsq(np.stack([np.ones(n), b1], axis=1), w, rcond=None)[0]
    assert np.allclose([z[0], alpha[0, 1]], a_ls, atol=1e-12)


# ------------------------------------------------------------------ code update

def test_best_codes_brute_force():
    rng = np.random.default_rng(6)
    for p in (1, 2, 3):
        P, n = 5, 24
        W = rng.normal(size=(P, n))
        alpha = np.abs(rng.normal(size=(P, p))) + 0.1
        z = rng.normal(size=P) * 0.1
        B = Q.best_codes(W, alpha, z)
        for q in range(P):
            for k in range(n):
                errs = []
                for c in range(2 ** p):
                    v = 0.0
                    for i in range(p):
                        v += alpha[q, i] * (1.0 if (c >> i) & 1 else -1.0)
                    errs.append(abs(W[q, k] - (z[q] + v)))
                best = int(np.argmin(errs))
                assert errs[best] < min(e for j, e in enumerate(errs) if j != best)
                want = [1.0 if (best >> i) & 1 else -1.0 for i in range(p)]
                assert list(B[q, :, k]) == want


def test_best_codes_ties_go_to_the_first_candidate():
    # alpha_2 = 0: codes differing only in plane 2 tie; the first (b_2 = -1) wins
    W = np.array([[0.9, -0.4, 0.0, 2.0]])
    B = Q.best_codes(W, np.array([[0.5, 0.0]]), np.array([0.0]))
    assert np.array_equal(B[0, 1], -np.ones(4))
    assert np.array_equal(B[0, 0], [1.0, -1.0, -1.0, 1.0])  # w = 0 ties -0.5/+0.5: code 0 first
    # alpha_1 = alpha_2: (+,-) and (-,+) both give z; the first enumerated,
    # candidate 1 = (+,-), wins
    B = Q.best_codes(np.array([[0.1, -0.1]]), np.array([[0.5, 0.5]]), np.array([0.0]))
    assert np.array_equal(B[0, :, 0], [1.0, -1.0]) and np.array_equal(B[0, :, 1], [1.0, -1.0])
    # all candidates equal: code 0 (every plane -1)
    B = Q.best_codes(W, np.array([[0.0, 0.0]]), np.array([0.3]))
    assert np.array_equal(B[0], -np.ones((2, 4)))


# --------------------------------------------------------------- whole quantiser

def test_greedy_stage_closed_form():
    w = _weights((3, 128), 7)
    tr = []
    Q.quantize_groups(w, p_L=1, p_H=1, rounds=0, trace=tr)
    r = w - w.mean(axis=1, keepdims=True)
    a = np.mean(np.abs(r), axis=1, keepdims=True)
    assert tr[0][0] == "greedy"
    assert np.allclose(tr[0][1], np.sum((np.abs(r) - a) ** 2, axis=1), rtol=1e-12, atol=0)
    # p_L = 2: the second scale is the mean |residual| of the first step
    tr = []
    Q.quantize_groups(w, p_L=2, p_H=2, rounds=0, trace=tr)
    r2 = np.abs(r) - a
    a2 = np.mean(np.abs(r2), axis=1, keepdims=True)
    assert np.allclose(tr[0][1], np.sum((np.abs(r2) - a2) ** 2, axis=1), rtol=1e-12, atol=0)


def test_one_round_worked_example():
    # n = 8, p_L = p_H = 1, one round, worked by hand.  mean = 0.29375, so the
    # greedy code puts 0.35 with the ones.  The joint least squares for
    # (z, alpha) on clusters {0 x5} and {0.35, 1, 1} gives z = alpha = 47/120,
    # a threshold of 0.39167 that moves 0.35 to the lower code.  The final
    # refit on {0 x5, 0.35} and {1, 1}: lower level 0.35/6, upper level 1.
    w = np.array([[0, 0, 0, 0, 0, 0.35, 1, 1]], dtype=np.float64)
    tr = []
    B, al, z = Q.quantize_groups(w, p_L=1, p_H=1, rounds=1, trace=tr)
    assert np.array_equal(B[0, 0], [-1, -1, -1, -1, -1, -1, 1, 1])
    lo, hi = 0.35 / 6, 1.0
    assert abs(z[0] - (lo + hi) / 2) < 1e-15 and abs(al[1][0, 0] - (hi - lo) / 2) < 1e-15
    assert abs(tr[1][1][0] - ((0.35 - 47 / 60) ** 2 + 2 * (1 - 47 / 60) ** 2)) < 1e-15
    assert abs(tr[-1][1][0] - (5 * lo ** 2 + (0.35 - lo) ** 2)) < 1e-15


def test_two_level_group_is_exact_after_one_round():
    rng = np.random.default_rng(8)
    lo, hi = -0.013, 0.021
    w = np.where(rng.random((4, 128)) < 0.3, hi, lo)
    B, al, z = Q.quantize_groups(w, p_L=1, p_H=1, rounds=1)
    assert np.allclose(z, (lo + hi) / 2, atol=1e-15)
    assert np.allclose(al[1][:, 0], (hi - lo) / 2, atol=1e-15)
    assert np.array_equal(B[:, 0], np.where(w == hi, 1.0, -1.0))


def test_representable_group_is_recovered():
    rng = np.random.default_rng(9)
    for balanced in (True, False):
        if balanced:
            c = rng.permutation(np.repeat(np.arange(4), 32))
        else:
            c = rng.integers(0, 4, 128)
        b1, b2 = _pm1(c & 1), _pm1(c & 2)
        w = 0.004 + 0.02 * b1 + 0.007 * b2
        tr = []
        B, al, z = Q.quantize_groups(w[None], p_L=2, p_H=4, trace=tr)
        assert abs(z[0] - 0.004) < 1e-14
        assert np.allclose(al[2][0], [0.02, 0.007], atol=1e-14)
        assert np.array_equal(B[0, 0], b1) and np.array_equal(B[0, 1], b2)
        assert tr[-3][1][0] < 1e-28
        if balanced:                                    # greedy already exact
            assert tr[0][1][0] < 1e-28


def test_constant_and_zero_groups_are_all_offset():
    w = np.stack([np.full(128, 0.25), np.zeros(128), np.full(128, -3.0)])
    B, al, z = Q.quantize_groups(w, p_L=2, p_H=4)
    assert np.array_equal(z, [0.25, 0.0, -3.0])
    for p in (2, 3, 4):
        assert np.array_equal(al[p], np.zeros((3, p)))


@pytest.mark.parametrize("kind", ["normal", "laplace", "t3"])
def test_error_never_rises(kind):
    w = _weights((48, 128), 11, kind)
    tr = []
    B, al, z = Q.quantize_groups(w, p_L=2, p_H=4, trace=tr)
    names = [s for s, _ in tr]
    assert names == ["greedy"] + ["lsq", "codes"] * 20 + ["p2", "p3", "p4"]
    scale = np.sum(w ** 2, axis=1)
    for (_, e1), (_, e2) in zip(tr, tr[1:]):
        assert np.all(e2 <= e1 + 1e-12 * scale)
    # each added plane lowers the error substantially on continuous weights
    e2, e3, e4 = tr[-3][1], tr[-2][1], tr[-1][1]
    assert np.all(e3 < e2) and np.all(e4 < e3)
    assert np.mean(e4 / scale) < 0.1 and np.mean(e2 / scale) < 0.3


def test_expansion_freezes_codes_and_appends_residual_sign():
    w = _weights((16, 128), 12)
    B4, al4, z4 = Q.quantize_groups(w, p_L=2, p_H=4)
    B3, al3, z3 = Q.quantize_groups(w, p_L=2, p_H=3)
    assert np.array_equal(B4[:, :3], B3) and np.array_equal(z4, z3)
    for p in (2, 3):
        assert np.array_equal(al4[p], al3[p])
    for p in (2, 3):
        res = w - z4[:, None] - np.einsum("qi,qin->qn", al4[p], B4[:, :p])
        assert np.array_equal(B4[:, p], np.where(res >= 0, 1.0, -1.0))


def test_expansion_refits_every_scale():
    w = _weights((16, 128), 13)
    B, al, z = Q.quantize_groups(w, p_L=2, p_H=4)
    for p in (3, 4):
        res = w - z[:, None] - np.einsum("qi,qin->qn", al[p], B[:, :p])
        grad = np.einsum("qin,qn->qi", B[:, :p], res)
        assert np.max(np.abs(grad)) < 1e-12
        # the new scales differ from the old ones: all of them were refit
        assert np.max(np.abs(al[p][:, :p - 1] - al[p - 1])) > 1e-6
    # base precision: z and alpha are jointly least squares for the final codes
    res = w - z[:, None] - np.einsum("qi,qin->qn", al[2], B[:, :2])
    assert np.max(np.abs(res.sum(axis=1))) < 1e-12
    assert np.max(np.abs(np.einsum("qin,qn->qi", B[:, :2], res))) < 1e-12


def test_codes_are_nearest_after_refinement():
    # the last refinement step leaves every weight at its nearest code for
    # the scales it was chosen with, so one more code update changes nothing
    w = _weights((8, 128), 14)
    tr = []
    B, al, z = Q.quantize_groups(w, p_L=2, p_H=2, rounds=20, trace=tr)
    Bn = Q.best_codes(w, al[2], z)
    assert np.mean(Bn == B[:, :2]) > 0.97


def test_quantize_canonical_packing_and_reconstruction():
    N, K = 3, 256
    w = _weights((N, K), 15)
    planes, alphas, z = Q.quantize(w)
    assert planes.shape == (4, N, K // 32) and planes.dtype == np.uint32
    B, al, zg = Q.quantize_groups(w.reshape(N * 2, 128))
    for i, n, k in itertools.product(range(4), range(N), range(0, K, 7)):
        bit = (int(planes[i, n, k // 32]) >> (k % 32)) & 1
        assert (1.0 if bit else -1.0) == B[n * 2 + k // 128, i, k % 128]
    for p in (2, 3, 4):
        assert alphas[p].shape == (N, 2, p)
        assert np.array_equal(alphas[p].reshape(-1, p), al[p])
    # the canonical outputs, rounded to fp16, feed the GEMV oracle: its result
    # equals x . W_hat^T with W_hat rebuilt densely from the same values
    a16 = {p: alphas[p].astype(np.float16) for p in (2, 3, 4)}
    z16 = z.astype(np.float16)
    x = _weights((2, K), 16) * 50
    for p in (2, 3, 4):
        y = oracle.gemm(x.astype(np.float16), planes, a16, z16, p=p)
        What = np.zeros((N, K))
        for n, k in itertools.product(range(N), range(K)):
            g = k // 128
            v = float(z16[n, g])
            for i in range(p):
                bit = (int(planes[i, n, k // 32]) >> (k % 32)) & 1
                v += float(a16[p][n, g, i]) * (1.0 if bit else -1.0)
            What[n, k] = v
        ref = x.astype(np.float16).astype(np.float64) @ What.T
        assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_quantize_rejects_ragged_k():
    with pytest.raises(ValueError):
        Q.quantize(np.zeros((2, 200)))
    with pytest.raises(ValueError):
        Q.quantize_groups(np.zeros((2, 128)), p_L=3, p_H=2)


# ------------------------------------------------- variant: offsets per precision

def test_per_precision_offsets_variant():
    w = _weights((24, 128), 17)
    tr_s, tr_v = [], []
    Bs, als, zs = Q.quantize_groups(w, 2, 4, trace=tr_s)
    Bv, alv, zv = Q.quantize_groups(w, 2, 4, trace=tr_v, offsets="per_precision")
    # the base precision is the same; z^(p_L) is the shared z
    assert np.array_equal(Bv[:, :3], Bs[:, :3]) and np.array_equal(alv[2], als[2])
    assert np.array_equal(zv[2], zs)
    # every precision: (z^(p), alpha^(p)) jointly least squares for its codes
    for p in (2, 3, 4):
        res = w - zv[p][:, None] - np.einsum("qi,qin->qn", alv[p], Bv[:, :p])
        assert np.max(np.abs(res.sum(axis=1))) < 1e-12
        assert np.max(np.abs(np.einsum("qin,qn->qi", Bv[:, :p], res))) < 1e-12
    # B_{p+1} = sign of the residual with z^(p); the error falls with p and is
    # never above the shared-offset variant's (a larger least-squares space)
    for p in (2, 3):
        res = w - zv[p][:, None] - np.einsum("qi,qin->qn", alv[p], Bv[:, :p])
        assert np.array_equal(Bv[:, p], np.where(res >= 0, 1.0, -1.0))
    e = [t for s, t in tr_v if s in ("p2", "p3", "p4")]
    assert np.all(e[1] <= e[0] * (1 + 1e-12)) and np.all(e[2] <= e[1] * (1 + 1e-12))
    es = [t for s, t in tr_s if s == "p3"][0]
    assert np.all(e[1] <= es * (1 + 1e-12))
    with pytest.raises(ValueError):
        Q.quantize_groups(w, 2, 4, offsets="bogus")
