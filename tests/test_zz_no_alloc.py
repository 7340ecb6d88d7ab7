"""bcq_gemm_noalloc: the matmul for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc (code inside an allocator or memory pool,
a plug-in whose host framework owns every device allocation, a loop that must
not block on the driver's allocator), yet bcq_gemm needs split-K scratch from
its caller.  bcq_gemm_noalloc takes that scratch from a static array built
into the library.  These tests call it through the C ABI on two calls in a
row and check each result against the fp64 oracle (within the tolerance of
the other parity tests) and bit for bit against bcq_gemm with a caller
workspace: both run the same kernels in the same order, only the scratch
differs.  The file is named to be collected last.
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


def _check_oracle(y, y_ref, what):
    a = y.float().cpu().numpy().astype(np.float64)
    bad = np.abs(a - y_ref) > ATOL + RTOL * np.abs(y_ref)
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outputs outside tolerance"


@pytest.mark.parametrize("N,K,M", [(4096, 4096, 1), (4096, 4096, 2), (1000, 2048, 5),
                                   (4096, 4096, 16), (300, 256, 3), (14336, 4096, 16)])
def test_noalloc_matches_gemm_twice_in_a_row(N, K, M):
    prob = synth.make_problem(N, K, M, seed=7 * N + K + M)
    w = api.BcqWeights.from_canonical(prob.planes, prob.alphas, prob.z)
    x = torch.from_numpy(prob.x.view(np.int16)).view(torch.float16).cuda()
    assert api.workspace_bytes(M, N, K) <= api.NOALLOC_SCRATCH_BYTES
    for p in (2, 4):
        y_ref = oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p=p)
        ref = w.gemm(x, p=p)
        y1 = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        y2 = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        api.gemm_noalloc(x, w, p=p, out=y1)
        api.gemm_noalloc(x, w, p=p, out=y2)   # second call reuses the same scratch
        torch.cuda.synchronize()
        assert api.device_error() == api.BCQ_OK
        for y, which in ((y1, "first"), (y2, "second")):
            _check_oracle(y, y_ref, f"{which} call N={N} K={K} M={M} p={p}")
            assert torch.equal(y, ref), f"{which} call N={N} K={K} M={M} p={p}: not bcq_gemm's bits"


def test_noalloc_mixed_precision_rows():
    N, K, M = 2048, 4096, 4
    prob = synth.make_problem(N, K, M, seed=11)
    w = api.BcqWeights.from_canonical(prob.planes, prob.alphas, prob.z)
    x = torch.from_numpy(prob.x.view(np.int16)).view(torch.float16).cuda()
    p_row = np.array([2, 4, 3, 2], dtype=np.int32)
    y_ref = oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p_row=p_row)
    ref = w.gemm(x, p_row=p_row)
    for _ in range(2):
        y = api.gemm_noalloc(x, w, p_row=p_row)
        torch.cuda.synchronize()
        _check_oracle(y, y_ref, "mixed precisions")
        assert torch.equal(y, ref)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # 16 rows of a 65536 x 8192 weight need ~128 MiB of partial sums: more
    # than the built-in array.  Only the shape matters; nothing is launched.
    N, K, M = 65536, 8192, 16
    assert api.workspace_bytes(M, N, K) > api.NOALLOC_SCRATCH_BYTES
    dummy = torch.zeros(1024, dtype=torch.int32, device="cuda")
    scales = torch.zeros(1024, dtype=torch.float16, device="cuda")
    w = api.BcqWeights(packed=dummy, alphas={2: scales}, z=None, N=N, K=K, p_H=2)
    x = torch.zeros((M, K), dtype=torch.float16, device="cuda")
    y = torch.zeros((M, 8), dtype=torch.float16, device="cuda")
    # the binding refuses the undersized output itself ...
    with pytest.raises(ValueError):
        api.gemm_noalloc(x, w, p=2, out=y)
    # ... and the library, given the same pointers, refuses the shape
    alpha = api._alpha_array(w.alphas)
    st = api.lib().bcq_gemm_noalloc(api._ptr(x), api._ptr(dummy),
                                    api.ctypes.cast(alpha, api.ctypes.c_void_p), None, 2, None,
                                    M, N, K, 2, 128, api._ptr(y), api._stream())
    assert st == api.BCQ_ERR_SCRATCH
    torch.cuda.synchronize()
    assert torch.count_nonzero(y).item() == 0
