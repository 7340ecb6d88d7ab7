"""The N-sharded (column-parallel) layer on CPU: two gloo ranks.

Each rank takes its rows of the weight (shard_rows), computes its slice of y
-- here with the fp64 oracle, the CUDA kernels being for the GPU tests --
and the slices are all-gathered (gather_rows, the one collective of the
sharded path).  Every rank must end with the full oracle output.  Also the
partition itself: contiguous, whole 32-row blocks, every row exactly once.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from bit_gemv_bcq_b200 import shard, synth


@pytest.mark.parametrize("N", [1, 31, 32, 100, 1000, 4096, 14336])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_shard_rows_partition(N, world):
    spans = [shard.shard_rows(N, world, r) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == N
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 == b0                      # contiguous, no overlap, no gap
    for r0, r1 in spans:
        assert (r0 % 32 == 0 or r0 == N) and (r1 % 32 == 0 or r1 == N) and r1 >= r0
    sizes = [-(-(r1 - r0) // 32) for r0, r1 in spans]
    assert max(sizes) - min(sizes) <= 1
    assert shard.shard_width(N, world) == max(r1 - r0 for r0, r1 in spans)


def test_assemble_puts_slices_in_row_order():
    N, world, M = 100, 3, 2
    width = shard.shard_width(N, world)
    parts = torch.full((world, M, width), -1.0)
    for r in range(world):
        r0, r1 = shard.shard_rows(N, world, r)
        parts[r, :, :r1 - r0] = torch.arange(r0, r1, dtype=torch.float32)
    y = shard.assemble(parts, N, world)
    assert torch.equal(y, torch.arange(N, dtype=torch.float32).expand(M, N))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        prob = synth.make_problem(300, 512, 2, seed=41, mixed=True)
        r0, r1 = shard.shard_rows(300, world, rank)
        pl, al, z = shard.slice_canonical(prob.planes, prob.alphas, prob.z, r0, r1)
        y_local = torch.from_numpy(oracle.gemm(prob.x, np.ascontiguousarray(pl),
                                               {q: np.ascontiguousarray(a) for q, a in al.items()},
                                               np.ascontiguousarray(z), p_row=prob.p_row))
        y = shard.gather_rows(y_local, 300, world)
        out[rank] = y.numpy()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_layer_gathers_the_full_output(world):
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
        out = dict(out)
    prob = synth.make_problem(300, 512, 2, seed=41, mixed=True)
    ref = oracle.gemm(prob.x, prob.planes, prob.alphas, prob.z, p_row=prob.p_row)
    for r in range(world):
        assert np.array_equal(out[r], ref)
