"""Pins for the fp64 oracle: each test checks it against something other than
itself -- a value printed on the pages, a closed form, an invariant, or a
brute-force computation by an independent route (numpy bit unpacking + dense
matmul).  CPU only.

Sources, by page title and section:
  * BiLoCo page, "核心思路：修正项只用 +1 和 −1" -- the hand example 3.4.
  * BiLoCo page, "二值向量怎么找" -- the 3x2 greedy + joint-refit example.
  * AnyBCQ (Paper-Notes page), "切入角度", "训练策略", "直接bit-plane运算的CUDA内核"
    -- W_hat = sum_i alpha_i B_i (+ z per group of 128); p-bit uses planes 1..p.
"""
import os

import numpy as np
import pytest

import oracle
from oracle import quant
from bit_gemv_bcq_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split(":", 1)
            rows = [r.split() for r in val.split(";")]
            arr = [[float(t) for t in r] for r in rows]
            val = np.array(arr if len(arr) > 1 else arr[0])
            out[key.strip()] = float(val[0]) if val.size == 1 else val
    return out


def _pack_bits(b01):
    """Pack a 0/1 array along its last axis LSB-first into uint32 words
    (numpy packbits, an independent route from the oracle's bit reader)."""
    b01 = np.asarray(b01, dtype=np.uint8)
    K = b01.shape[-1]
    assert K % 32 == 0
    by = np.packbits(b01, axis=-1, bitorder="little")
    return np.ascontiguousarray(by).view("<u4").reshape(*b01.shape[:-1], K // 32)


def _unpack_pm1(planes):
    """uint32 words -> +-1 float64 array, LSB first (numpy unpackbits)."""
    by = np.ascontiguousarray(planes).view(np.uint8)
    bits = np.unpackbits(by, axis=-1, bitorder="little")
    return bits.astype(np.float64) * 2.0 - 1.0


# ---------------------------------------------------------------- fp16 decode

def test_half_decoder_all_codes_match_numpy():
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.halves_to_double(codes)
    ref = codes.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # signed zeros keep their sign
    assert np.signbit(got[0x8000]) and not np.signbit(got[0])


# -------------------------------------------------------- signed sum (3.4)

def test_signed_sum_hand_example():
    g = _read_golden("biloco_signed_sum.txt")
    x, v, vx = g["x"], g["v"], float(g["vx"])
    bits = (v > 0).astype(np.uint8)
    word = int(sum(int(b) << j for j, b in enumerate(bits)))
    assert word == 0b0101  # LSB-first: column 0 is bit 0
    got = oracle.signed_sum(x, np.array([word], dtype=np.uint32))
    assert abs(got - vx) < 1e-12


def test_gemm_reproduces_hand_example():
    """The same example through the full GEMM: K = 128 (one group), p = 1,
    alpha = 1, z = 0, x = the printed vector padded with zeros."""
    g = _read_golden("biloco_signed_sum.txt")
    K = 128
    x = np.zeros((1, K), dtype=np.float16)
    x[0, :4] = g["x"]
    bits = np.zeros((1, 1, K), dtype=np.uint8)
    bits[0, 0, :4] = (g["v"] > 0)
    planes = _pack_bits(bits)
    alphas = {1: np.ones((1, 1, 1), dtype=np.float16)}
    y = oracle.gemm(x, planes, alphas, None, p=1)
    # the padded zeros contribute +-0; the only error is the fp16 rounding of x
    bound = float(np.sum(np.abs(x[0, :4].astype(np.float64) - g["x"])))
    assert abs(y[0, 0] - float(g["vx"])) <= bound + 1e-12
    assert bound < 1e-3


# ------------------------------------------------------------------ the LUT

def test_lut_closed_forms():
    rng = np.random.default_rng(7)
    x = rng.normal(size=(2, 64)).astype(np.float16)
    T = oracle.lut(x)
    xd = x.astype(np.float64)
    assert T.shape == (2, 8, 256)
    for m in range(2):
        for c in range(8):
            xc = xd[m, 8 * c:8 * c + 8]
            tot = xc.sum()
            t = T[m, c]
            assert abs(t[0xFF] - tot) < 1e-12          # all +1
            assert abs(t[0x00] + tot) < 1e-12          # all -1
            for j in range(8):                         # one +1 at column j
                assert abs(t[1 << j] - (2 * xc[j] - tot)) < 1e-12
            b = np.arange(256)
            assert np.allclose(t[b] + t[255 - b], 0.0, atol=1e-12)  # T[~b] = -T[b]
            for j in range(8):                         # flipping bit j moves by 2 x_j
                hi = b[(b >> j) & 1 == 1]
                assert np.allclose(t[hi] - t[hi ^ (1 << j)], 2 * xc[j], atol=1e-12)


def test_lut_all_bytes_brute_force():
    rng = np.random.default_rng(3)
    x = rng.normal(size=(1, 8)).astype(np.float16)
    T = oracle.lut(x)[0, 0]
    b = np.arange(256, dtype=np.uint8)
    signs = np.unpackbits(b[:, None], axis=1, bitorder="little").astype(np.float64) * 2 - 1
    assert np.allclose(T, signs @ x[0].astype(np.float64), atol=1e-12)


def test_group_sums():
    rng = np.random.default_rng(5)
    x = rng.normal(size=(3, 512)).astype(np.float16)
    S = oracle.group_sums(x)
    ref = x.astype(np.float64).reshape(3, 4, 128).sum(axis=2)
    assert np.allclose(S, ref, atol=1e-12)
    T = oracle.lut(x)                                  # = sum of T[0xFF] over chunks
    assert np.allclose(S, T[:, :, 0xFF].reshape(3, 4, 16).sum(axis=2), atol=1e-12)


# ------------------------------------------------------------------- GEMM

def _dense_reference(prob, p=None, p_row=None):
    """Independent route: unpack with numpy, build W_hat densely, matmul."""
    N, K, G = prob.N, prob.K, prob.K // 128
    signs = _unpack_pm1(prob.planes)                       # [p_H][N][K]
    z = prob.z.astype(np.float64).repeat(128, axis=1)      # [N][K]
    xs = prob.x.astype(np.float64)
    y = np.empty((prob.M, N))
    for m in range(prob.M):
        q = p if p is not None else int(p_row[m])
        a = prob.alphas[q].astype(np.float64)              # [N][G][q]
        W = z.copy()
        for i in range(q):
            W += a[:, :, i].repeat(128, axis=1) * signs[i]
        y[m] = W @ xs[m]
    return y


@pytest.mark.parametrize("N,K,M", [(8, 128, 1), (5, 256, 2), (3, 384, 3)])
@pytest.mark.parametrize("p", [1, 2, 3, 4])
def test_gemm_brute_force_tiny(N, K, M, p):
    prob = synth.make_problem(N, K, M, seed=N * 1000 + K + p, precisions=(1, 2, 3, 4))
    y = oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p=p)
    ref = _dense_reference(prob, p=p)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_gemm_closed_form_all_ones_planes():
    prob = synth.make_problem(6, 384, 2, seed=11)
    prob.planes[:] = 0xFFFFFFFF
    S = oracle.group_sums(prob.x)                          # [M][G]
    for p in (2, 3, 4):
        y = oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p=p)
        coef = prob.alphas[p].astype(np.float64).sum(axis=2) + prob.z.astype(np.float64)
        assert np.allclose(y, S @ coef.T, rtol=1e-12, atol=1e-12)


def test_gemm_closed_form_zero_alpha_is_offset_only():
    prob = synth.make_problem(7, 256, 2, seed=12)
    zero = {q: np.zeros_like(a) for q, a in prob.alphas.items()}
    y = oracle.gemm(prob.x, prob.planes, zero, prob.z, p=3)
    S = oracle.group_sums(prob.x)
    assert np.allclose(y, S @ prob.z.astype(np.float64).T, rtol=1e-12, atol=1e-12)
    y0 = oracle.gemm(prob.x, prob.planes, zero, None, p=3)
    assert np.all(y0 == 0.0)


def test_gemm_pm1_gemv_matches_signed_sums():
    """p = 1, alpha = 1, z = 0: each output is the signed sum of x."""
    prob = synth.make_problem(4, 256, 1, seed=13, precisions=(1,))
    one = {1: np.ones_like(prob.alphas[1])}
    y = oracle.gemm(prob.x, prob.planes, one, None, p=1)
    xd = prob.x[0].astype(np.float64)
    for n in range(4):
        assert abs(y[0, n] - oracle.signed_sum(xd, prob.planes[0, n])) < 1e-12


def test_gemm_p_prefix_ignores_higher_planes():
    prob = synth.make_problem(9, 512, 2, seed=14)
    rng = np.random.default_rng(99)
    for p in (2, 3):
        y = oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p=p)
        poisoned = prob.planes.copy()
        poisoned[p:] = rng.integers(0, 2**32, size=poisoned[p:].shape, dtype=np.uint32)
        y2 = oracle.gemm(prob.x, poisoned, prob.alphas, prob.z, p=p)
        assert np.array_equal(y, y2)
        changed = prob.planes.copy()
        changed[p - 1] ^= 0x1                               # a used plane does matter
        y3 = oracle.gemm(prob.x, changed, prob.alphas, prob.z, p=p)
        assert not np.array_equal(y, y3)


def test_gemm_sign_symmetry():
    prob = synth.make_problem(5, 256, 2, seed=15)
    y = oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p=4)
    for i in range(4):
        flipped = prob.planes.copy()
        flipped[i] = ~flipped[i]
        a = {q: v.copy() for q, v in prob.alphas.items()}
        a[4][:, :, i] = -a[4][:, :, i]
        y2 = oracle.gemm(prob.x, flipped, a, prob.z, p=4)
        assert np.allclose(y, y2, rtol=1e-12, atol=1e-12)


def test_gemm_linear_in_x():
    prob = synth.make_problem(6, 256, 1, seed=16)
    rng = np.random.default_rng(1)
    x1 = rng.integers(-8, 9, size=(1, 256)).astype(np.float16)   # exact sums
    x2 = rng.integers(-8, 9, size=(1, 256)).astype(np.float16)
    f = lambda x: oracle.gemm(x, prob.planes, prob.alphas, prob.z, p=3)
    assert np.allclose(f(x1 + x2), f(x1) + f(x2), rtol=1e-12, atol=1e-12)
    assert np.allclose(f(-x1), -f(x1), rtol=0, atol=0)


def test_gemm_per_row_precision_equals_uniform_rows():
    prob = synth.make_problem(10, 384, 6, seed=17, mixed=True)
    prob.p_row[:] = [4, 2, 3, 3, 2, 4]
    y = oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p_row=prob.p_row)
    for m, q in enumerate(prob.p_row):
        yq = oracle.gemm(prob.x[m:m + 1], prob.planes, prob.alphas, prob.z, p=int(q))
        assert np.array_equal(y[m], yq[0])
    assert np.allclose(y, _dense_reference(prob, p_row=prob.p_row), rtol=1e-12, atol=1e-12)


def test_gemm_row_selection():
    prob = synth.make_problem(12, 256, 2, seed=18)
    full = oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p=2)
    rows = np.array([11, 0, 5, 5], dtype=np.int32)
    part = oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p=2, rows=rows)
    assert np.array_equal(part, full[:, rows])


def test_gemm_rejects_bad_arguments():
    prob = synth.make_problem(4, 256, 1, seed=19)
    with pytest.raises(ValueError):
        oracle.gemm(prob.x, prob.planes, {2: prob.alphas[2]}, prob.z, p=3)  # no alpha^(3)
    with pytest.raises(ValueError):
        oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p=5)
    with pytest.raises(ValueError):
        oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, group=96)     # K % group


# ---------------------------------------------- quantiser helpers (BiLoCo 3x2)

def test_greedy_and_joint_refit_example():
    g = _read_golden("biloco_greedy_3x2.txt")
    W = g["W"]
    us, vs, alphas, R = quant.greedy_rank1_pm1(W, 2, iters=5, v0=g["v0"])
    assert np.array_equal(vs[0], g["c1_v"])
    assert np.array_equal(W @ vs[0], g["c1_Rv"])
    assert np.array_equal(us[0], g["c1_u"])
    assert np.array_equal(W.T @ us[0], g["c1_RTu"])
    assert abs(alphas[0] - float(g["c1_alpha"])) < 1e-12
    R1 = W - alphas[0] * np.outer(us[0], vs[0])
    assert np.allclose(R1, g["residual1"], atol=1e-12)
    assert np.array_equal(us[1], g["c2_u"])
    assert np.array_equal(vs[1], g["c2_v"])
    assert abs(alphas[1] - float(g["c2_alpha"])) < 1e-12
    assert abs(float(np.sum(R ** 2)) - float(g["greedy_sse"])) < 1e-12
    assert us[0] @ us[1] == float(g["u1_dot_u2"])
    mats = [np.outer(us[r], vs[r]) for r in range(2)]
    a = quant.lsq_scales(W, mats)
    assert np.allclose(a, g["joint_alpha"], atol=1e-12)
    assert abs(quant.sse(W, mats, a) - float(g["joint_sse"])) < 1e-12


def test_lsq_scales_never_worse_than_greedy():
    rng = np.random.default_rng(2)
    for _ in range(20):
        W = rng.normal(size=(6, 5))
        us, vs, al, R = quant.greedy_rank1_pm1(W, 3, rng=rng)
        mats = [np.outer(us[r], vs[r]) for r in range(3)]
        a = quant.lsq_scales(W, mats)
        assert quant.sse(W, mats, a) <= float(np.sum(R ** 2)) + 1e-9


def test_greedy_bcq_scale_is_mean_abs_and_error_monotone():
    rng = np.random.default_rng(4)
    w = rng.normal(size=128)
    B, a, r = quant.greedy_bcq(w, 4)
    assert abs(a[0] - np.mean(np.abs(w))) < 1e-12
    errs = [float(np.sum((w - (a[:q, None] * B[:q]).sum(axis=0)) ** 2)) for q in range(1, 5)]
    assert all(e2 <= e1 + 1e-12 for e1, e2 in zip(errs, errs[1:]))


def test_gemm_per_precision_offsets_closed_forms():
    # alpha = 0: y[m][n] = sum_g z^(p_m)[n][g] * (sum of x[m] over group g),
    # the group sums taken directly with numpy; one shared array in every
    # slot of the dict is the single-offset call
    prob = synth.make_problem(48, 384, 5, seed=23)
    rng = np.random.default_rng(24)
    zq = {q: rng.normal(0.0, 0.01, size=(48, 3)).astype(np.float16) for q in (2, 3, 4)}
    zero = {q: np.zeros_like(a) for q, a in prob.alphas.items()}
    p_row = np.array([2, 4, 3, 3, 2], dtype=np.int32)
    y = oracle.gemm(prob.x, prob.planes, zero, zq, p_row=p_row)
    xs = prob.x.astype(np.float64).reshape(5, 3, 128).sum(axis=2)
    for m in range(5):
        ref = zq[int(p_row[m])].astype(np.float64) @ xs[m]
        assert np.allclose(y[m], ref, rtol=1e-12, atol=1e-12)
    same = {q: prob.z for q in (2, 3, 4)}
    assert np.array_equal(oracle.gemm(prob.x, prob.planes, prob.alphas, same, p_row=p_row),
                          oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p_row=p_row))
