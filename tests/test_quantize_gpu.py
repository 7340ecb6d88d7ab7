"""GPU parity of the offline quantiser (bcq_quantize, through the C ABI)
against the fp64 oracle (oracle/quantizer.py).

Both sides take the same fp64 steps: right-hand sides that are exact sums of
+-fp16 weights (or one rounding from them), integer Gram matrices, Cramer's
rule with the exact integer adjugate, products and sums in one fixed order,
and round-to-nearest-even to fp16.  So every output must be bit-identical:
planes, the fp16 scales of every precision and the offsets, in every group,
including groups whose residual is exactly zero at some weight (there sign(R)
depends on the rounding, identical on both sides).  The per-group squared
error is a sum in a different order on each side and agrees to 1e-9
relative.
"""
import numpy as np
import pytest
import torch

from bit_gemv_bcq_b200 import api, synth
from oracle import quantizer as Q

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    api.lib()
    yield
    assert api.device_error() == api.BCQ_OK


def _gpu(w16, p_L=2, p_H=4, rounds=20):
    w = torch.from_numpy(w16.view(np.int16)).view(torch.float16).cuda()
    planes, alphas, z, sse = api.quantize(w, p_L, p_H, rounds, with_sse=True)
    torch.cuda.synchronize()
    return (planes.cpu().numpy().view(np.uint32), {p: a.cpu().numpy() for p, a in alphas.items()},
            z.cpu().numpy(), sse.cpu().numpy())


def _oracle(w16, p_L=2, p_H=4, rounds=20):
    w = w16.astype(np.float64)
    N, K = w.shape
    tr = []
    planes, alphas, z = Q.quantize(w, 128, p_L, p_H, rounds, trace=tr)
    sse = np.stack([e for s, e in tr if s.startswith("p")]).reshape(p_H - p_L + 1, N, K // 128)
    return planes, alphas, z, sse


def _compare(gpu, ref, p_L, p_H):
    gp, ga, gz, gs = gpu
    rp, ra, rz, rs = ref
    assert np.array_equal(gp, rp), f"planes differ in {np.sum(gp != rp)} words"
    for p in range(p_L, p_H + 1):
        g16, r16 = ga[p].view(np.uint16), ra[p].astype(np.float16).view(np.uint16)
        assert np.array_equal(g16, r16), f"alpha^({p}) differs in {np.sum(g16 != r16)} values"
    assert np.array_equal(gz.view(np.uint16), rz.astype(np.float16).view(np.uint16)), "z differs"
    assert np.allclose(gs, rs, rtol=1e-9, atol=1e-30)


@pytest.mark.parametrize("N,K,seed", [(40, 384, 1), (7, 128, 2), (300, 1024, 3)])
def test_parity_generic_weights(N, K, seed):
    w16 = synth.make_weights(N, K, seed=seed)
    _compare(_gpu(w16), _oracle(w16), 2, 4)


@pytest.mark.parametrize("p_L,p_H,rounds", [(1, 4, 20), (3, 4, 20), (2, 2, 20), (1, 1, 5),
                                             (4, 4, 3), (2, 3, 0), (2, 4, 1), (1, 2, 40)])
def test_parity_precision_ranges_and_rounds(p_L, p_H, rounds):
    w16 = synth.make_weights(33, 256, seed=10 + 4 * p_L + p_H, outliers=True)
    _compare(_gpu(w16, p_L, p_H, rounds), _oracle(w16, p_L, p_H, rounds), p_L, p_H)


def _structured(seed):
    rng = np.random.default_rng(seed)
    rows = []
    rows.append(np.full(256, 0.0))                        # all zero
    rows.append(np.full(256, 0.0311))                     # constant
    two = np.where(rng.random(256) < 0.3, 0.021, -0.013)  # two values
    rows.append(two)
    c = rng.integers(0, 4, 256)                            # exactly 2-bit representable
    rows.append(0.004 + 0.02 * np.where(c & 1, 1, -1) + 0.007 * np.where(c & 2, 1, -1))
    sym = rng.choice([-0.5, 0.5], 256) * 0.01              # symmetric two-level, mean ~ 0
    rows.append(sym)
    return np.stack(rows).astype(np.float16)


def _rebuild(planes, alphas, z, p):
    N, G = z.shape
    bits = ((planes[:p, :, :, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(p, N, G, 128)
    a = alphas[p].astype(np.float64)
    return (z.astype(np.float64)[None, :, :, None] +
            np.einsum("ngi,ingk->ngk", a, np.where(bits, 1.0, -1.0))[None]).reshape(N, G * 128)


def test_structured_groups():
    # constant, zero, two-valued and exactly representable groups: dependent
    # least-squares columns, exactly zero residuals and exact ties in the code
    # update are decided identically on both sides
    w16 = _structured(5)
    for p_L, p_H in [(2, 4), (1, 4), (3, 4), (1, 1), (4, 4)]:
        _compare(_gpu(w16, p_L, p_H), _oracle(w16, p_L, p_H), p_L, p_H)
    gp, ga, gz, gs = _gpu(w16)
    assert np.array_equal(gz[0], np.zeros(2, np.float16))
    assert np.array_equal(gz[1], np.full(2, np.float16(0.0311)))
    for p in (2, 3, 4):
        assert not np.any(ga[p][:2].astype(np.float64))
    # every structured group is exact from two bits on
    w64 = w16.astype(np.float64)
    for p in (2, 3, 4):
        assert np.allclose(_rebuild(gp, ga, gz, p), w64, rtol=0, atol=1e-4)


def test_full_size_sampled_groups():
    N, K = 14336, 4096
    w16 = synth.make_weights(N, K, seed=21)
    gp, ga, gz, gs = _gpu(w16)
    rng = np.random.default_rng(22)
    G = K // 128
    picks = rng.choice(N * G, size=192, replace=False)
    picks = np.concatenate([picks, [0, N * G - 1]])
    rows, groups = picks // G, picks % G
    sub = np.stack([w16[n, g * 128:(g + 1) * 128] for n, g in zip(rows, groups)])
    ref = _oracle(sub)
    # the sampled groups as an [S][1]-group matrix on both sides
    S = len(picks)
    mine = (np.stack([gp[:, n, 4 * g:4 * g + 4] for n, g in zip(rows, groups)], axis=1),
            {p: ga[p][rows, groups].reshape(S, 1, p) for p in (2, 3, 4)},
            gz[rows, groups].reshape(S, 1), gs[:, rows, groups].reshape(3, S, 1))
    _compare(mine, ref, 2, 4)
    # every group: the error falls as planes are added
    assert np.all(gs[1] <= gs[0] * (1 + 1e-12)) and np.all(gs[2] <= gs[1] * (1 + 1e-12))


def test_quantised_weights_feed_the_gemm():
    import oracle
    N, K = 96, 512
    w16 = synth.make_weights(N, K, seed=31)
    w = torch.from_numpy(w16.view(np.int16)).view(torch.float16).cuda()
    planes, alphas, z, _ = api.quantize(w)
    bw = api.BcqWeights.from_canonical(planes, alphas, z)
    x16 = synth.make_x(3, K, seed=32)
    x = torch.from_numpy(x16.view(np.int16)).view(torch.float16).cuda()
    pl = planes.cpu().numpy().view(np.uint32)
    al = {p: a.cpu().numpy() for p, a in alphas.items()}
    zz = z.cpu().numpy()
    for p in (2, 3, 4):
        y = bw.gemm(x, p=p).float().cpu().numpy().astype(np.float64)
        ref = oracle.gemm(x16, pl, al, zz, p=p)
        assert np.all(np.abs(y - ref) <= 1e-2 + 2e-3 * np.abs(ref))
    # quantisation error of the product falls with p
    dense = x16.astype(np.float64) @ w16.astype(np.float64).T
    errs = [np.linalg.norm(oracle.gemm(x16, pl, al, zz, p=p) - dense) for p in (2, 3, 4)]
    assert errs[0] > errs[1] > errs[2]


def test_empty_and_bad_arguments():
    w = torch.zeros((4, 256), dtype=torch.float16, device="cuda")
    pl, al, z, _ = api.quantize(w[:0])                     # N = 0: nothing to do
    assert pl.numel() == 0
    for p_L, p_H in [(0, 4), (3, 2), (1, 5)]:
        with pytest.raises(api.BcqError) as e:
            api.quantize(w, p_L, p_H)
        assert e.value.status == api.BCQ_ERR_PRECISION
    with pytest.raises(api.BcqError) as e:
        api.quantize(w, rounds=-1)
    assert e.value.status == api.BCQ_ERR_SHAPE
    with pytest.raises(api.BcqError) as e:
        api.quantize(torch.zeros((4, 200), dtype=torch.float16, device="cuda"))
    assert e.value.status == api.BCQ_ERR_SHAPE


# ------------------------------------------------- variant: offsets per precision

def _gpu_zp(w16, p_L=2, p_H=4, rounds=20):
    w = torch.from_numpy(w16.view(np.int16)).view(torch.float16).cuda()
    planes, alphas, z, sse = api.quantize(w, p_L, p_H, rounds, with_sse=True,
                                          offsets="per_precision")
    torch.cuda.synchronize()
    return (planes.cpu().numpy().view(np.uint32), {p: a.cpu().numpy() for p, a in alphas.items()},
            {p: v.cpu().numpy() for p, v in z.items()}, sse.cpu().numpy())


@pytest.mark.parametrize("p_L,p_H", [(2, 4), (1, 4), (3, 4), (1, 2)])
def test_parity_per_precision_offsets(p_L, p_H):
    structured = np.tile(_structured(6), (1, 2))[:, :384]   # 5 rows of special groups
    w16 = np.concatenate([synth.make_weights(37, 384, seed=40 + p_L), structured])
    gp, ga, gz, gs = _gpu_zp(w16, p_L, p_H)
    tr = []
    rp, ra, rz = Q.quantize(w16.astype(np.float64), 128, p_L, p_H, 20, trace=tr,
                            offsets="per_precision")
    rs = np.stack([e for s, e in tr if s.startswith("p")]).reshape(p_H - p_L + 1, 42, 3)
    assert np.array_equal(gp, rp)
    for p in range(p_L, p_H + 1):
        assert np.array_equal(ga[p].view(np.uint16), ra[p].astype(np.float16).view(np.uint16))
        assert np.array_equal(gz[p].view(np.uint16), rz[p].astype(np.float16).view(np.uint16))
    assert np.allclose(gs, rs, rtol=1e-9, atol=1e-30)
    # the base precision equals the shared-offset quantiser's
    sp, sa, sz, _ = _gpu(w16, p_L, p_H)
    assert np.array_equal(gz[p_L].view(np.uint16), sz.view(np.uint16))
    assert np.array_equal(ga[p_L].view(np.uint16), sa[p_L].view(np.uint16))


def test_per_precision_weights_feed_gemm_zp():
    import oracle
    N, K = 128, 512
    w16 = synth.make_weights(N, K, seed=51)
    w = torch.from_numpy(w16.view(np.int16)).view(torch.float16).cuda()
    bw = api.BcqWeights.quantize(w, offsets="per_precision")
    planes, alphas, z, _ = api.quantize(w, offsets="per_precision")
    pl = planes.cpu().numpy().view(np.uint32)
    al = {p: a.cpu().numpy() for p, a in alphas.items()}
    zq = {p: v.cpu().numpy() for p, v in z.items()}
    x16 = synth.make_x(5, K, seed=52)
    x = torch.from_numpy(x16.view(np.int16)).view(torch.float16).cuda()
    p_row = np.array([2, 4, 3, 2, 4], dtype=np.int32)
    y = bw.gemm(x, p_row=p_row).float().cpu().numpy().astype(np.float64)
    ref = oracle.gemm(x16, pl, al, zq, p_row=p_row)
    assert np.all(np.abs(y - ref) <= 1e-2 + 2e-3 * np.abs(ref))
