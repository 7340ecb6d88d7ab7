"""GPU parity of bcq_gemm_zp (offsets per precision) against the fp64 oracle.

Each precision q keeps its own offsets z^(q); row m of x uses z^(p_m) with
alpha^(p_m).  Covered: every kernel (lookup launches of one and two rows,
two rows of different precisions in one lookup launch, mma.sync and
tcgen05 batches, 64-row tcgen05 launches), mixed batches, a precision
without offsets, and bitwise agreement with bcq_gemm when every precision
has the same offsets.  Bar: |y - ref| <= 1e-2 + 2e-3 |ref|.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_gemv_bcq_b200 import api, synth

pytestmark = pytest.mark.gpu

ATOL, RTOL = 1e-2, 2e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    api.lib()
    yield
    assert api.device_error() == api.BCQ_OK


@pytest.fixture(params=["sync", "tcgen05"])
def kind(request, monkeypatch):
    if request.param == "tcgen05":
        monkeypatch.setenv("BCQ_MMA_KIND", "tcgen05")
    else:
        monkeypatch.delenv("BCQ_MMA_KIND", raising=False)
    return request.param


def _offsets(N, G, seed, missing=None):
    rng = np.random.default_rng(seed)
    zq = {q: rng.normal(0.0, 0.01, size=(N, G)).astype(np.float16) for q in (1, 2, 3, 4)}
    if missing is not None:
        zq[missing] = None
    return zq


def _check(y, ref):
    y = y.float().cpu().numpy().astype(np.float64)
    err = np.abs(y - ref)
    assert np.all(err <= ATOL + RTOL * np.abs(ref)), f"max err {err.max():.3e}"


def _x(prob, M=None):
    x = prob.x if M is None else synth.make_x(M, prob.K, seed=91)
    return x, torch.from_numpy(x.view(np.int16)).view(torch.float16).cuda()


@pytest.mark.parametrize("N,K", [(300, 768), (4096, 4096)])
@pytest.mark.parametrize("M", [1, 2, 4, 16, 33, 64])
def test_uniform_precision(N, K, M, kind):
    prob = synth.make_problem(N, K, 1, seed=N + K, precisions=(1, 2, 3, 4))
    zq = _offsets(N, K // 128, seed=M)
    w = api.BcqWeights.from_canonical(prob.planes, prob.alphas, zq)
    x16, x = _x(prob, M)
    for p in (1, 2, 3, 4):
        ref = oracle.gemm(x16, prob.planes, prob.alphas, zq, p=p)
        _check(w.gemm(x, p=p), ref)


@pytest.mark.parametrize("M", [2, 3, 7, 16, 40, 64])
def test_mixed_rows(M, kind):
    # M = 2: one lookup launch with two precisions (row 1's offsets read apart)
    N, K = 1000, 1024
    prob = synth.make_problem(N, K, 1, seed=M, precisions=(2, 3, 4))
    zq = _offsets(N, K // 128, seed=100 + M, missing=3)
    zq.pop(1)
    w = api.BcqWeights.from_canonical(prob.planes, prob.alphas, zq)
    x16, x = _x(prob, M)
    rng = np.random.default_rng(M)
    p_row = rng.integers(2, 5, size=M).astype(np.int32)
    if M == 2:
        p_row[:] = (2, 4)
    ref = oracle.gemm(x16, prob.planes, prob.alphas, {q: v for q, v in zq.items()}, p_row=p_row)
    _check(w.gemm(x, p_row=p_row), ref)


def test_same_offsets_match_bcq_gemm_bitwise():
    N, K = 2048, 2048
    prob = synth.make_problem(N, K, 8, seed=5)
    x = torch.from_numpy(prob.x.view(np.int16)).view(torch.float16).cuda()
    w1 = api.BcqWeights.from_canonical(prob.planes, prob.alphas, prob.z)
    wq = api.BcqWeights.from_canonical(prob.planes, prob.alphas, {q: prob.z for q in (2, 3, 4)})
    for M, p_row in [(1, [3]), (2, [2, 4]), (8, [2, 3, 4, 4, 2, 3, 4, 2])]:
        a = w1.gemm(x[:M], p_row=p_row)
        b = wq.gemm(x[:M], p_row=p_row)
        torch.cuda.synchronize()
        assert torch.equal(a, b)


def test_rejects_and_guards():
    prob = synth.make_problem(64, 256, 1, seed=6)
    zq = _offsets(64, 2, seed=7)
    w = api.BcqWeights.from_canonical(prob.planes, prob.alphas, zq)
    x = torch.zeros((1, 256), dtype=torch.float16, device="cuda")
    with pytest.raises(ValueError):
        api.gemm_noalloc(x, w, p=2)
    # a misaligned offset array of a used precision is refused
    arr = api._alpha_array(w.alphas)
    zbad = api._alpha_array({q: z for q, z in w.zq.items()}, "z")
    zbad[1] = zbad[1] + 2
    y = torch.empty((1, 64), dtype=torch.float16, device="cuda")
    st = api.lib().bcq_gemm_zp(api._ptr(x), api._ptr(w.packed), api.ctypes.cast(arr, api.ctypes.c_void_p),
                               api.ctypes.cast(zbad, api.ctypes.c_void_p), 2, None, 1, 64, 256, 4,
                               128, api._ptr(y), None, 0, api._stream())
    assert st == api.BCQ_ERR_ALIGN
