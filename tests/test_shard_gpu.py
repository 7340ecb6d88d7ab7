"""The N-sharded layer through the CUDA kernels on one GPU: every rank's
rows packed and computed with bcq_gemm (here the ranks run one after the
other on the same GPU), the slices put together as the all-gather of
gather_rows lays them out, and the result checked against the fp64 oracle
on every output.  world = 1 runs the whole path (no collective)."""
import numpy as np
import pytest
import torch

import oracle
from bit_gemv_bcq_b200 import api, shard, synth

pytestmark = pytest.mark.gpu

ATOL, RTOL = 1e-2, 2e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    api.lib()
    yield
    assert api.device_error() == api.BCQ_OK


@pytest.mark.parametrize("N,K,world", [(14336, 4096, 2), (4096, 14336, 4), (1000, 2048, 3),
                                       (4096, 4096, 8), (700, 1024, 1)])
def test_sharded_rows_match_the_oracle(N, K, world):
    prob = synth.make_problem(N, K, 4, seed=N + world, mixed=True)
    x = torch.from_numpy(prob.x.view(np.int16)).view(torch.float16).cuda()
    width = shard.shard_width(N, world)
    parts = torch.zeros((world, 4, width), dtype=torch.float16, device="cuda")
    for r in range(world):
        w = shard.ShardedBcqWeights.from_canonical(prob.planes, prob.alphas, prob.z, world, r)
        if w.local is not None:
            parts[r, :, :w.r1 - w.r0] = w.local.gemm(x, p_row=prob.p_row)
    y = shard.assemble(parts, N, world) if world > 1 else \
        shard.ShardedBcqWeights.from_canonical(prob.planes, prob.alphas, prob.z, 1, 0).gemm(
            x, p_row=prob.p_row)
    torch.cuda.synchronize()
    ref = oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p_row=prob.p_row)
    err = np.abs(y.float().cpu().numpy().astype(np.float64) - ref)
    assert (err <= ATOL + RTOL * np.abs(ref)).all(), f"{N}x{K} over {world}: {err.max()}"
