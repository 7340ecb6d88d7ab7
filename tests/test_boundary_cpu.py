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
    assert api.lib().bcq_version() == 100
    for s in range(8):
        assert api.status_string(s).startswith("BCQ_")
    assert api.status_string(99) == "BCQ_ERR_UNKNOWN"


def test_packed_bytes_formula(L):
    # ceil(N/32) row-blocks x p_H x ceil(K/256) K-blocks x 1 KiB
    assert api.packed_planes_bytes(4, 14336, 4096) == 448 * 4 * 16 * 1024
    assert api.packed_planes_bytes(4, 14336, 4096) == 14336 * 4096 * 4 // 8
    assert api.packed_planes_bytes(2, 33, 384) == 2 * 2 * 2 * 1024
    for bad in [(0, 32, 256), (5, 32, 256), (4, 0, 256), (4, 32, 100), (4, 32, 0)]:
        assert api.packed_planes_bytes(*bad) == 0


FAKE = 0x10000   # never dereferenced: every call below fails validation first


def _alpha(*present, base=FAKE):
    arr = (ctypes.c_void_p * 4)()
    for q in range(1, 5):
        arr[q - 1] = base if q in present else None
    return ctypes.cast(arr, ctypes.c_void_p)


def _gemm(L, x=FAKE, planes=FAKE, alpha=None, z=None, p=2, p_row=None, M=1,
          N=64, K=256, p_H=4, group=128, y=FAKE):
    alpha = _alpha(2, 3, 4) if alpha is None else alpha
    return L.bcq_gemm(x, planes, alpha, z, p, p_row, M, N, K, p_H, group, y, None)


def test_gemm_rejects_before_launch(L):
    assert _gemm(L, x=None) == api.BCQ_ERR_NULL
    assert _gemm(L, y=None) == api.BCQ_ERR_NULL
    assert _gemm(L, planes=None) == api.BCQ_ERR_NULL
    assert L.bcq_gemm(FAKE, FAKE, None, None, 2, None, 1, 64, 256, 4, 128, FAKE, None) == api.BCQ_ERR_NULL
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
    assert _gemm(L, alpha=_alpha(4, base=FAKE + 4), p=4) == api.BCQ_ERR_ALIGN


def test_pack_and_lut_reject_before_launch(L):
    assert L.bcq_pack_planes(None, FAKE, 4, 64, 256, None) == api.BCQ_ERR_NULL
    assert L.bcq_pack_planes(FAKE, FAKE, 5, 64, 256, None) == api.BCQ_ERR_PRECISION
    assert L.bcq_pack_planes(FAKE, FAKE, 4, 64, 200, None) == api.BCQ_ERR_SHAPE
    assert L.bcq_pack_planes(FAKE, FAKE + 4, 4, 64, 256, None) == api.BCQ_ERR_ALIGN
    assert L.bcq_build_lut(None, 1, 256, FAKE, None, None) == api.BCQ_ERR_NULL
    assert L.bcq_build_lut(FAKE, 5, 256, FAKE, None, None) == api.BCQ_ERR_SHAPE
    assert L.bcq_build_lut(FAKE, 1, 250, FAKE, None, None) == api.BCQ_ERR_SHAPE
    assert L.bcq_build_lut(FAKE + 8, 1, 256, FAKE, None, None) == api.BCQ_ERR_ALIGN
    assert L.bcq_debug_wait_timeout(0, None) == api.BCQ_ERR_SHAPE
    assert L.bcq_debug_wait_timeout(2000000, None) == api.BCQ_ERR_SHAPE
    assert L.bcq_gemm_host(None, FAKE, _alpha(2), None, 2, None, 1, 64, 256, 4, 128,
                           FAKE, FAKE, FAKE, None) == api.BCQ_ERR_NULL


def test_empty_batch_is_a_no_op(L):
    # M = 0: nothing to compute; returns before any CUDA call
    assert _gemm(L, M=0, x=None, y=None) == api.BCQ_OK


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    monkeypatch.setattr(api, "_lib", None)
    monkeypatch.setattr(api, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(api.BcqLibraryError):
        api.lib()
