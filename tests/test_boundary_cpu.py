"""The C-ABI library without a GPU: it loads, exports every function that
include/bcq.h declares, and rejects invalid arguments on the host before any
CUDA call (so these checks never touch a device)."""
import ctypes
import os
import re

import pytest

from bit_gemv_bcq_b200 import api
from bit_gemv_bcq_b200 import build as libbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bcq.h")


@pytest.fixture(scope="module")
def L():
    libbuild.build()
    return api.lib()


def _declared_functions():
    text = open(HEADER, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bcq_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    names = _declared_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(L, n), n
    assert sorted(api.EXPORTED) == names


def test_version_and_status_strings(L):
    assert api.lib().bcq_version() == 200
    for s in range(8):
        assert api.status_string(s).startswith("BCQ_")
    assert api.status_string(99) == "BCQ_ERR_UNKNOWN"


def test_packed_bytes_formula(L):
    # 8 KiB per (plane, 256 rows, 256 columns), rows and columns padded
    assert api.packed_planes_bytes(4, 14336, 4096) == 16 * 56 * 4 * 8192
    assert api.packed_planes_bytes(4, 14336, 4096) == 14336 * 4096 * 4 // 8
    assert api.packed_planes_bytes(2, 33, 384) == 2 * 1 * 2 * 8192     # padded
    for bad in [(0, 32, 256), (5, 32, 256), (4, 0, 256), (4, 32, 100), (4, 32, 0)]:
        assert api.packed_planes_bytes(*bad) == 0
    # K-blocks x row-blocks x 32 lanes x 2 groups x q halves
    assert api.packed_scales_bytes(3, 14336, 4096) == 16 * 448 * 32 * 2 * 3 * 2
    assert api.packed_scales_bytes(3, 14336, 4096) == 14336 * 32 * 3 * 2
    assert api.packed_scales_bytes(1, 33, 384) == 2 * 2 * 32 * 2 * 1 * 2
    assert api.packed_scales_bytes(0, 32, 256) == 0


def test_workspace_bytes_formula(L):
    # one K-block: no split over K, no workspace
    assert api.workspace_bytes(1, 4096, 256) == 0
    assert api.workspace_bytes(4, 4096, 128) == 0
    # KB x min(M, 64) x rows (padded to 32) x 4 B of partial sums
    assert api.workspace_bytes(1, 14336, 4096) == 16 * 1 * 14336 * 4
    assert api.workspace_bytes(8, 14336, 4096) == 16 * 8 * 14336 * 4
    assert api.workspace_bytes(64, 14336, 4096) == 16 * 64 * 14336 * 4
    assert api.workspace_bytes(17, 14336, 4096) == 16 * 17 * 14336 * 4
    assert api.workspace_bytes(2, 33, 640) == 3 * 2 * 64 * 4
    assert api.workspace_bytes(0, 64, 512) == 0
    assert api.workspace_bytes(1, 64, 100) == 0


@pytest.mark.parametrize("M,N,K,p,mixed", [(16, 14336, 4096, 2, False), (5, 4096, 4096, 4, False),
                                           (1, 14336, 4096, 2, False), (1, 14336, 4096, 4, False),
                                           (1, 4096, 14336, 3, False), (2, 4096, 4096, 2, False),
                                           (2, 28672, 8192, 4, True), (1, 256, 512, 4, False),
                                           (1, 1, 128, 1, False), (2, 33, 640, 2, False),
                                           (64, 14336, 4096, 4, False), (33, 4096, 4096, 2, False),
                                           (4, 14336, 4096, 4, False), (3, 4096, 4096, 2, False)])
def test_launch_plans_respect_the_pipeline_rules(L, M, N, K, p, mixed):
    """Plans for a nominal 148-SM B200 (no GPU needed): one CTA per SM at
    most (never more CTAs than units), whole K-blocks per CTA when the CTAs
    divide among them, the 227 KiB of shared memory, and an even ring depth
    (teams alternate stages: a stage's team consumed the stage one ring
    earlier) that is a multiple of the producer warps (each refills only its
    own slots)."""
    pl = api.plan_query(M, N, K, p, mixed=mixed, use_device=False)
    RB, KB = -(-N // 32), -(-K // 256)
    U = RB * KB
    one_row = M == 1 and not mixed
    even = min(U, KB * min(RB, 148 // KB)) if KB <= 148 else None
    if one_row:
        # the one-row kernel keeps whole K-blocks per CTA only while that
        # leaves at most a tenth of the SMs idle, else every SM takes a share
        assert pl["C"] == (even if even is not None and 10 * even >= 9 * min(U, 148)
                           else min(U, 148))
        # planes, scales alpha^(p) and offsets of one row group per stage,
        # two teams of 8 consumer warps alternating stages, a 32 KiB table
        assert pl["stage_bytes"] == 8192 * p + 1024 * p + 1024
        assert pl["consumer_warps"] == 16
        assert pl["dyn_bytes"] <= 232448
        assert pl["dyn_bytes"] >= 32768 + pl["D"] * pl["stage_bytes"]
        # a producer per part of every stage: planes (two halves at four
        # planes), scales, offsets
        assert pl["NP"] == (4 if p >= 4 else 3)
        assert pl["D"] % 2 == 0 and 2 <= pl["D"] <= 20
        assert pl["D"] == 20 or pl["dyn_bytes"] + 2 * pl["stage_bytes"] > 232448
        assert pl["units_max"] == -(-U // pl["C"])
        return
    if KB <= 148:
        assert pl["C"] == even   # whole K-blocks per CTA group
        assert pl["C"] % KB == 0 or pl["C"] == U
    else:
        assert pl["C"] == 148
    assert pl["KB"] == KB
    assert pl["units_max"] == -(-U // pl["C"])
    assert pl["dyn_bytes"] <= 232448
    assert pl["stage_bytes"] == 8192 * p    # the p planes of one row group
    tiles = 2 * (16 if M <= 16 else 64) * 256 * 2        # two activation tiles
    table = 65536 if M <= 2 else 131072 if M <= 4 else tiles  # or the lookup table(s)
    assert pl["dyn_bytes"] >= table + pl["D"] * pl["stage_bytes"]
    assert pl["D"] % 2 == 0 and pl["D"] % pl["NP"] == 0 and 2 <= pl["D"] <= 20
    # as deep as the shared memory allows
    assert pl["D"] == 20 or pl["dyn_bytes"] + 2 * pl["stage_bytes"] > 232448
    assert pl["consumer_warps"] == 16


def test_plan_query_rejects_bad_arguments(L):
    with pytest.raises(api.BcqError):
        api.plan_query(65, 64, 256, 2)            # at most 64 rows per launch
    with pytest.raises(api.BcqError):
        api.plan_query(17, 64, 256, 3, mixed=True)  # mixed launches: 16 rows at most
    pl = api.plan_query(4, 64, 256, 3, mixed=True)  # the mixed tensor-core kernel
    assert pl["stage_bytes"] == 8192 * 3
    with pytest.raises(api.BcqError):
        api.plan_query(1, 64, 200, 2)             # K % 128
    with pytest.raises(api.BcqError):
        api.plan_query(1, 64, 256, 5)             # p_load
    with pytest.raises(api.BcqError):
        api.plan_query(1, 64, 256, 3, mixed=True)  # one row cannot mix


FAKE = 0x10000   # never dereferenced: every call below fails validation first


def _alpha(*present, base=FAKE):
    arr = (ctypes.c_void_p * 4)()
    for q in range(1, 5):
        arr[q - 1] = base if q in present else None
    return ctypes.cast(arr, ctypes.c_void_p)


def _gemm(L, x=FAKE, planes=FAKE, alpha=None, z=None, p=2, p_row=None, M=1,
          N=64, K=256, p_H=4, group=128, y=FAKE, ws=None, ws_bytes=0):
    alpha = _alpha(2, 3, 4) if alpha is None else alpha
    return L.bcq_gemm(x, planes, alpha, z, p, p_row, M, N, K, p_H, group, y, ws, ws_bytes,
                      None)


def test_gemm_rejects_before_launch(L):
    assert _gemm(L, x=None) == api.BCQ_ERR_NULL
    assert _gemm(L, y=None) == api.BCQ_ERR_NULL
    assert _gemm(L, planes=None) == api.BCQ_ERR_NULL
    assert L.bcq_gemm(FAKE, FAKE, None, None, 2, None, 1, 64, 256, 4, 128, FAKE, None, 0,
                      None) == api.BCQ_ERR_NULL
    assert _gemm(L, K=100) == api.BCQ_ERR_SHAPE
    assert _gemm(L, K=0) == api.BCQ_ERR_SHAPE
    assert _gemm(L, N=0) == api.BCQ_ERR_SHAPE
    assert _gemm(L, M=65) == api.BCQ_ERR_SHAPE
    assert _gemm(L, M=-1) == api.BCQ_ERR_SHAPE
    assert _gemm(L, group=64) == api.BCQ_ERR_UNSUPPORTED
    assert _gemm(L, p=5) == api.BCQ_ERR_PRECISION
    assert _gemm(L, p=3, p_H=2) == api.BCQ_ERR_PRECISION
    assert _gemm(L, p_H=0) == api.BCQ_ERR_PRECISION
    assert _gemm(L, p=0, p_row=None) == api.BCQ_ERR_PRECISION
    assert _gemm(L, alpha=_alpha(2, 4), p=3) == api.BCQ_ERR_PRECISION
    pr = (ctypes.c_int32 * 2)(2, 5)
    assert _gemm(L, p=0, p_row=ctypes.cast(pr, ctypes.c_void_p), M=2) == api.BCQ_ERR_PRECISION
    pr = (ctypes.c_int32 * 2)(2, 3)
    assert _gemm(L, p=0, p_row=ctypes.cast(pr, ctypes.c_void_p), M=2,
                 alpha=_alpha(2)) == api.BCQ_ERR_PRECISION
    assert _gemm(L, x=FAKE + 2) == api.BCQ_ERR_ALIGN
    assert _gemm(L, planes=FAKE + 4) == api.BCQ_ERR_ALIGN
    assert _gemm(L, y=FAKE + 1) == api.BCQ_ERR_ALIGN
    assert _gemm(L, z=FAKE + 1) == api.BCQ_ERR_ALIGN
    assert _gemm(L, alpha=_alpha(2, base=FAKE + 2), p=2) == api.BCQ_ERR_ALIGN
    assert _gemm(L, alpha=_alpha(4, base=FAKE + 8), p=4) == api.BCQ_ERR_ALIGN
    assert _gemm(L, z=FAKE + 8) == api.BCQ_ERR_ALIGN
    # K > 256 splits over K: a workspace of bcq_workspace_bytes is required
    need = api.workspace_bytes(1, 64, 512)
    assert need > 0
    assert _gemm(L, K=512) == api.BCQ_ERR_NULL
    assert _gemm(L, K=512, ws=FAKE, ws_bytes=need - 1) == api.BCQ_ERR_NULL
    assert _gemm(L, K=512, ws=FAKE + 8, ws_bytes=need) == api.BCQ_ERR_ALIGN


def test_pack_and_lut_reject_before_launch(L):
    assert L.bcq_pack_planes(None, FAKE, 4, 64, 256, None) == api.BCQ_ERR_NULL
    assert L.bcq_pack_planes(FAKE, FAKE, 5, 64, 256, None) == api.BCQ_ERR_PRECISION
    assert L.bcq_pack_planes(FAKE, FAKE, 4, 64, 200, None) == api.BCQ_ERR_SHAPE
    assert L.bcq_pack_planes(FAKE, FAKE + 4, 4, 64, 256, None) == api.BCQ_ERR_ALIGN
    assert L.bcq_build_lut(None, 1, 256, FAKE, None, None) == api.BCQ_ERR_NULL
    assert L.bcq_build_lut(FAKE, 5, 256, FAKE, None, None) == api.BCQ_ERR_SHAPE
    assert L.bcq_build_lut(FAKE, 1, 250, FAKE, None, None) == api.BCQ_ERR_SHAPE
    assert L.bcq_build_lut(FAKE + 8, 1, 256, FAKE, None, None) == api.BCQ_ERR_ALIGN
    assert L.bcq_pack_scales(None, 2, 64, 256, FAKE, None) == api.BCQ_ERR_NULL
    assert L.bcq_pack_scales(FAKE, 0, 64, 256, FAKE, None) == api.BCQ_ERR_PRECISION
    assert L.bcq_pack_scales(FAKE, 5, 64, 256, FAKE, None) == api.BCQ_ERR_PRECISION
    assert L.bcq_pack_scales(FAKE, 2, 64, 200, FAKE, None) == api.BCQ_ERR_SHAPE
    assert L.bcq_pack_scales(FAKE + 1, 2, 64, 256, FAKE, None) == api.BCQ_ERR_ALIGN
    assert L.bcq_pack_scales(FAKE, 2, 64, 256, FAKE + 8, None) == api.BCQ_ERR_ALIGN
    assert L.bcq_set_pdl(3) == api.BCQ_ERR_UNSUPPORTED
    assert L.bcq_set_pdl(0) == api.BCQ_OK
    assert L.bcq_debug_wait_timeout(0, None) == api.BCQ_ERR_SHAPE
    assert L.bcq_debug_wait_timeout(2000000, None) == api.BCQ_ERR_SHAPE
    assert L.bcq_gemm_host(None, FAKE, _alpha(2), None, 2, None, 1, 64, 256, 4, 128,
                           FAKE, FAKE, FAKE, None, 0, None) == api.BCQ_ERR_NULL


def test_empty_batch_is_a_no_op(L):
    # M = 0: nothing to compute; returns before any CUDA call
    assert _gemm(L, M=0, x=None, y=None) == api.BCQ_OK


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    monkeypatch.setattr(api, "_lib", None)
    monkeypatch.setattr(api, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(api.BcqLibraryError):
        api.lib()


# ---------------------------------------------------------------- routing

def test_mixed_batches_of_up_to_16_rows_are_one_launch(L):
    """Per-request precision (AnyBCQ page, 吞吐量): a batch whose rows use
    different precisions streams the planes once, up to its largest
    precision, in one launch (the mixed tensor-core kernel for 3-16 rows, the
    mixed pair lookup launch for 2)."""
    r = api.route_query(8, 28672, 8192, p_row=[4, 3, 3, 2, 2, 2, 2, 2])
    assert r == [("mma_mixed", 8, 4)]
    assert api.route_query(16, 4096, 4096, p_row=[2, 3, 4, 2] * 4) == [("mma_mixed", 16, 4)]
    assert api.route_query(3, 4096, 4096, p_row=[2, 2, 3]) == [("mma_mixed", 3, 3)]
    assert api.route_query(2, 4096, 4096, p_row=[2, 4]) == [("lut_pair", 2, 4)]


def test_uniform_batches_keep_their_kernels(L):
    assert api.route_query(1, 14336, 4096, p=2) == [("lut_one", 1, 2)]
    assert api.route_query(2, 14336, 4096, p=3) == [("lut_pair", 2, 3)]
    assert api.route_query(4, 14336, 4096, p=4) == [("lut_four", 4, 4)]
    assert api.route_query(8, 14336, 4096, p=2) == [("mma", 8, 2)]
    assert api.route_query(16, 14336, 4096, p=2) == [("mma", 16, 2)]
    assert api.route_query(64, 14336, 4096, p=2) == [("tcgen05", 64, 2)]
    # exactly 32 rows: two 16-row launches at one or two bits, one at three or four
    assert api.route_query(32, 14336, 4096, p=2) == [("mma", 16, 2), ("mma", 16, 2)]
    assert api.route_query(32, 14336, 4096, p=1) == [("mma", 16, 1), ("mma", 16, 1)]
    assert api.route_query(32, 14336, 4096, p=4) == [("tcgen05", 32, 4)]
    assert api.route_query(33, 14336, 4096, p=2) == [("tcgen05", 33, 2)]
    assert api.route_query(17, 14336, 4096, p=2) == [("mma", 16, 2), ("lut_one", 1, 2)]


def test_large_mixed_batches_group_by_precision_and_share_the_rest(L):
    """More than 16 rows: groups of one precision, then the rows left over in
    every group share mixed launches instead of one launch each."""
    p_row = [2] * 18 + [3] * 2 + [4] * 2
    r = api.route_query(22, 4096, 4096, p_row=p_row)
    assert ("mma", 16, 2) in r
    assert ("mma_mixed", 6, 4) in r                   # 2 + 2 + 2 rows left over
    assert sum(n for _, n, _ in r) == 22 and len(r) == 2


def test_routing_follows_the_switches(monkeypatch, L):
    monkeypatch.setenv("BCQ_MMA_MIN_ROWS", "5")
    assert api.route_query(4, 14336, 4096, p=4) == [("lut_pair", 2, 4), ("lut_pair", 2, 4)]
    pl = api.plan_query(4, 14336, 4096, 4)    # a four-row launch is no longer lut_four
    assert pl["stage_bytes"] == 8192 * 4
    monkeypatch.setenv("BCQ_MMA_MIN_ROWS", "3")
    monkeypatch.setenv("BCQ_LUT4_MAX_ROWS", "0")
    assert api.route_query(4, 14336, 4096, p=4) == [("mma", 4, 4)]


def test_route_query_rejects_bad_arguments(L):
    with pytest.raises(api.BcqError):
        api.route_query(0, 64, 256, p=2)
    with pytest.raises(api.BcqError):
        api.route_query(2, 64, 200, p=2)
    with pytest.raises(api.BcqError):
        api.route_query(2, 64, 256, p_row=[2, 5])
