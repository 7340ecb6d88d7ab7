"""Column-parallel (N-sharded) BCQ layers over several GPUs.

Output rows n are independent (y[m][n] needs row n of the weight only), so a
layer splits over `world` ranks by rows: rank r holds rows [r0, r1) of the
planes, scales and offsets, packs them with bcq_pack_planes /
bcq_pack_scales like any weight, runs bcq_gemm on them with its own copy of
x, and the output slices are put together with one all-gather of y
(M x ceil(N / world) fp16 per rank) -- the only collective, over NCCL
between GPUs (NVLink / NVSwitch), gloo on CPU tensors.  No kernel here reads
another GPU's memory.

One process per GPU, torch.distributed for the plumbing; every step of the
matmul runs in libbcq's kernels on each rank.
"""
from __future__ import annotations

import numpy as np
import torch

from . import api

ROW_ALIGN = 32  # rows of a row-block: shard boundaries fall on them


def shard_rows(N: int, world: int, rank: int) -> tuple:
    """Rows [r0, r1) of rank `rank` of `world`: contiguous, whole 32-row
    blocks except at the end, sizes differing by at most one block.  A rank
    may get no rows when N is small (r0 == r1)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank / world")
    blocks = -(-N // ROW_ALIGN)
    q, r = divmod(blocks, world)
    b0 = rank * q + min(rank, r)
    b1 = b0 + q + (1 if rank < r else 0)
    return min(N, b0 * ROW_ALIGN), min(N, b1 * ROW_ALIGN)


def shard_width(N: int, world: int) -> int:
    """Rows per rank in the all-gather buffer (the largest shard)."""
    return max(shard_rows(N, world, r)[1] - shard_rows(N, world, r)[0] for r in range(world))


def slice_canonical(planes, alphas: dict, z, r0: int, r1: int):
    """Rows [r0, r1) of canonical planes [p_H][N][K/32], scales {q: [N][G][q]}
    and offsets [N][G] (or {q: [N][G]}, or None)."""
    pl = planes[:, r0:r1]
    al = {q: a[r0:r1] for q, a in alphas.items()}
    if isinstance(z, dict):
        zz = {q: v[r0:r1] for q, v in z.items()}
    else:
        zz = None if z is None else z[r0:r1]
    return pl, al, zz


def assemble(parts, N: int, world: int) -> torch.Tensor:
    """y [M][N] from the all-gathered buffer parts [world][M][width]: rank r's
    first (r1 - r0) columns go to rows [r0, r1)."""
    cols = []
    for r in range(world):
        r0, r1 = shard_rows(N, world, r)
        cols.append(parts[r, :, :r1 - r0])
    return torch.cat(cols, dim=1)


def gather_rows(y_local: torch.Tensor, N: int, world: int, group=None) -> torch.Tensor:
    """All-gather the ranks' output slices y_local [M][r1 - r0] into y [M][N]
    (every rank gets all of it).  One all_gather_into_tensor of
    [M][shard_width] per rank; world == 1 returns y_local."""
    if world == 1:
        return y_local
    import torch.distributed as dist
    M = y_local.shape[0]
    width = shard_width(N, world)
    send = torch.zeros((M, width), dtype=y_local.dtype, device=y_local.device)
    send[:, :y_local.shape[1]] = y_local
    recv = torch.empty((world * M, width), dtype=y_local.dtype, device=y_local.device)
    dist.all_gather_into_tensor(recv, send, group=group)
    return assemble(recv.view(world, M, width), N, world)


class ShardedBcqWeights:
    """This rank's rows of a BCQ weight: a BcqWeights of rows [r0, r1)."""

    def __init__(self, local, N: int, r0: int, r1: int, world: int, rank: int):
        self.local, self.N, self.r0, self.r1 = local, N, r0, r1
        self.world, self.rank = world, rank

    @classmethod
    def from_canonical(cls, planes, alphas: dict, z, world: int, rank: int, device="cuda"):
        """Take rows shard_rows(N, world, rank) of the canonical arrays
        (numpy or tensors, all ranks holding the same full arrays) and pack
        them on `device`."""
        N = planes.shape[1]
        r0, r1 = shard_rows(N, world, rank)
        pl, al, zz = slice_canonical(planes, alphas, z, r0, r1)
        if r1 == r0:
            return cls(None, N, r0, r1, world, rank)
        if isinstance(pl, np.ndarray):
            pl = np.ascontiguousarray(pl)
            al = {q: np.ascontiguousarray(a) for q, a in al.items()}
            if isinstance(zz, dict):
                zz = {q: np.ascontiguousarray(v) for q, v in zz.items()}
            elif zz is not None:
                zz = np.ascontiguousarray(zz)
        local = api.BcqWeights.from_canonical(pl, al, zz, device=device)
        return cls(local, N, r0, r1, world, rank)

    def gemm(self, x: torch.Tensor, p=None, p_row=None, group=None, stream=None) -> torch.Tensor:
        """y = x . W_hat^T [M][N] on every rank: this rank's rows through
        bcq_gemm, then the all-gather of the slices."""
        M = x.shape[0]
        if self.local is None:
            y_local = torch.empty((M, 0), dtype=torch.float16, device=x.device)
        else:
            y_local = self.local.gemm(x, p=p, p_row=p_row, stream=stream)
        return gather_rows(y_local, self.N, self.world, group)
