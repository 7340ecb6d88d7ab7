"""Matrices with the same input (an MLP's gate and up projections) stacked
along N into one weight: one launch shares the lookup table, the activation
tiles and the split-K reduction.  Each row's sum does not depend on which
CTA computes it, so with row offsets that are multiples of 32 the stacked
call equals the separate calls bit for bit; ragged parts are checked against
the oracle."""
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


@pytest.fixture(params=["lut", "sync", "tcgen05"])
def path(request, monkeypatch):
    monkeypatch.setenv("BCQ_MMA_MIN_ROWS", "1000" if request.param == "lut" else "1")
    if request.param != "lut":
        monkeypatch.setenv("BCQ_MMA_KIND", request.param)
    return request.param


def _parts(Ns, K, M, seed):
    probs = [synth.make_problem(N, K, M, seed=seed + i) for i, N in enumerate(Ns)]
    return probs, [(p.planes, p.alphas, p.z) for p in probs]


@pytest.mark.parametrize("Ns,K,M", [((4096, 4096), 4096, 1), ((14336, 14336), 4096, 2),
                                    ((1024, 2048, 512), 1536, 4), ((2048, 2048), 256, 16)])
def test_stacked_equals_separate_bitwise(Ns, K, M, path):
    probs, parts = _parts(Ns, K, M, seed=40)
    x = torch.from_numpy(probs[0].x.view(np.int16)).view(torch.float16).cuda()
    ws = api.BcqWeights.stack(parts)
    assert ws.N == sum(Ns) and ws.row_splits == tuple(Ns)
    for p in (2, 4):
        y = ws.gemm(x, p=p)
        for (pl, al, z), y_part in zip(parts, ws.split_rows(y)):
            w = api.BcqWeights.from_canonical(pl, al, z)
            ref = w.gemm(x, p=p)
            torch.cuda.synchronize()
            assert torch.equal(y_part, ref), f"Ns={Ns} M={M} p={p}"


def test_stacked_ragged_parts_match_the_oracle(path):
    Ns, K, M = (1000, 300, 77), 640, 3
    probs, parts = _parts(Ns, K, M, seed=50)
    x = probs[0].x
    ws = api.BcqWeights.stack(parts)
    y = ws.gemm(torch.from_numpy(x.view(np.int16)).view(torch.float16).cuda(), p=3)
    torch.cuda.synchronize()
    for (pl, al, z), y_part in zip(parts, ws.split_rows(y)):
        ref = oracle.gemm(x, pl, al, z, p=3)
        got = y_part.float().cpu().numpy().astype(np.float64)
        assert (np.abs(got - ref) <= ATOL + RTOL * np.abs(ref)).all()


def test_stack_rejects_mismatched_parts():
    a = synth.make_problem(64, 256, 1, seed=1)
    b = synth.make_problem(64, 256, 1, seed=2, precisions=(2, 3))
    with pytest.raises(ValueError):
        api.BcqWeights.stack([(a.planes, a.alphas, a.z), (b.planes, b.alphas, b.z)])
    with pytest.raises(ValueError):
        api.BcqWeights.stack([(a.planes, a.alphas, a.z), (a.planes, a.alphas, None)])
