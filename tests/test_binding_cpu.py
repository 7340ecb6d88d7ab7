"""The Python binding's marshalling, on the host: what it hands the library.

The binding only marshals arguments (the kernels do all the work), but the
library takes raw pointers and cannot check buffer sizes, so the binding's
checks and the values it passes are host logic worth pinning.  Here the
library is replaced by a recorder, CUDA tensors by CPU tensors (the one check
that needs a device -- "is it a CUDA tensor" -- is switched off; dtype and
contiguity stay) and the current stream by a stand-in.  Every gemm entry point
must pass exactly: the tensors' addresses, the scales of each precision at
index q - 1 of a 4-pointer array, p or the per-row precisions, the sizes, the
workspace and the stream; and refuse a wrong buffer before calling anything.
"""
import contextlib
import ctypes

import numpy as np
import pytest
import torch

from bit_gemv_bcq_b200 import api

N, K = 512, 1024
STREAM = 0x1234


class _Stream:
    def __init__(self, device="cpu"):
        self.cuda_stream = STREAM
        self.device = torch.device(device)


class _Recorder:
    """Stands in for libbcq: records every call, with the pointer arrays and
    the per-row precisions read while the call is running."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def call(*args):
            args = list(args)
            if name.startswith("bcq_gemm"):
                args[2] = _read_ptrs(args[2])
                if name == "bcq_gemm_zp":
                    args[3] = _read_ptrs(args[3])
                if args[5] is not None:
                    rows = ctypes.cast(_addr(args[5]), ctypes.POINTER(ctypes.c_int32))
                    args[5] = [rows[i] for i in range(args[6])]
            args = [a.value if isinstance(a, ctypes.c_void_p) else a for a in args]
            self.calls.append((name, args))
            return api.BCQ_OK
        return call


def _addr(a):
    return a.value if isinstance(a, ctypes.c_void_p) else a


def _read_ptrs(a):
    if isinstance(a, ctypes.Array):
        return [v or 0 for v in a]
    arr = ctypes.cast(_addr(a), ctypes.POINTER(ctypes.c_void_p))
    return [arr[i] or 0 for i in range(4)]


@pytest.fixture
def rec(monkeypatch):
    r = _Recorder()
    ws = torch.zeros(1 << 16, dtype=torch.uint8)

    def need_cuda(t, name, dtype=None):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if dtype is not None and t.dtype != dtype:
            raise ValueError(f"{name} must be {dtype}")

    monkeypatch.setattr(api, "lib", lambda: r)
    monkeypatch.setattr(api, "_need_cuda", need_cuda)
    monkeypatch.setattr(api, "_on", lambda device: contextlib.nullcontext())
    monkeypatch.setattr(api, "workspace", lambda M, N, K, device, stream=None: ws)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda device=None: _Stream())
    r.ws = ws
    return r


def _arrays(p_H=4, qs=(2, 3, 4)):
    packed = torch.zeros(4096, dtype=torch.int32)
    alphas = {q: torch.zeros(N * 8 * q, dtype=torch.float16) for q in qs}
    z = torch.zeros(N * 8, dtype=torch.float16)
    return packed, alphas, z


def _ptrs(alphas):
    return [alphas[q].data_ptr() if q in alphas else 0 for q in (1, 2, 3, 4)]


@pytest.mark.parametrize("M", [1, 3, 16])
def test_gemm_passes_addresses_sizes_and_precisions(rec, M):
    packed, alphas, z = _arrays()
    w = api.BcqWeights(packed=packed, alphas=alphas, z=z, N=N, K=K, p_H=4)
    x = torch.zeros((M, K), dtype=torch.float16)
    y = torch.zeros((M, N), dtype=torch.float16)
    p_row = [2 + (m % 3) for m in range(M)]
    api.gemm(x, w, p=3, out=y)
    api.gemm(x, w, p_row=p_row, out=y)
    api.gemm(x, w, p=2, out=y, stream=_Stream())
    common = [x.data_ptr(), packed.data_ptr(), _ptrs(alphas), z.data_ptr()]
    tail = [M, N, K, 4, 128, y.data_ptr(), rec.ws.data_ptr(), rec.ws.numel(), STREAM]
    assert rec.calls == [("bcq_gemm", common + [3, None] + tail),
                         ("bcq_gemm", common + [0, p_row] + tail),
                         ("bcq_gemm", common + [2, None] + tail)]


def test_gemm_without_offsets_and_allocated_output(rec):
    packed, alphas, _ = _arrays(p_H=2, qs=(2,))
    w = api.BcqWeights(packed=packed, alphas=alphas, z=None, N=N, K=K, p_H=2)
    x = torch.zeros((2, K), dtype=torch.float16)
    y = api.gemm(x, w, p=2)
    assert tuple(y.shape) == (2, N) and y.dtype == torch.float16
    (name, args), = rec.calls
    assert name == "bcq_gemm" and args[2] == [0, alphas[2].data_ptr(), 0, 0] and args[3] is None
    assert args[11] == y.data_ptr()


def test_per_precision_offsets_go_to_the_zp_entry_point(rec):
    packed, alphas, _ = _arrays()
    zq = {q: torch.zeros(N * 8, dtype=torch.float16) for q in (2, 4)}
    w = api.BcqWeights(packed=packed, alphas=alphas, z=None, N=N, K=K, p_H=4, zq=zq)
    x = torch.zeros((4, K), dtype=torch.float16)
    y = torch.zeros((4, N), dtype=torch.float16)
    api.gemm(x, w, p_row=[2, 4, 4, 2], out=y)
    (name, args), = rec.calls
    assert name == "bcq_gemm_zp"
    assert args[2] == _ptrs(alphas)
    assert args[3] == [0, zq[2].data_ptr(), 0, zq[4].data_ptr()]
    assert args[4:6] == [0, [2, 4, 4, 2]]
    with pytest.raises(ValueError):
        api.gemm_noalloc(x, w, p=2)
    with pytest.raises(ValueError):
        api.gemm_host(x, w, y, x, y, p=2)
    assert len(rec.calls) == 1


def test_noalloc_and_host_entry_points(rec):
    packed, alphas, z = _arrays()
    w = api.BcqWeights(packed=packed, alphas=alphas, z=z, N=N, K=K, p_H=4)
    x = torch.zeros((5, K), dtype=torch.float16)
    y = torch.zeros((5, N), dtype=torch.float16)
    x_dev = torch.zeros((16, K), dtype=torch.float16)
    y_dev = torch.zeros((5, N), dtype=torch.float16)
    api.gemm_noalloc(x, w, p=4, out=y)
    api.gemm_host(x, w, y, x_dev[:5], y_dev, p=2)
    head = [x.data_ptr(), packed.data_ptr(), _ptrs(alphas), z.data_ptr()]
    assert rec.calls[0] == ("bcq_gemm_noalloc",
                            head + [4, None, 5, N, K, 4, 128, y.data_ptr(), STREAM])
    assert rec.calls[1] == ("bcq_gemm_host",
                            head + [2, None, 5, N, K, 4, 128, y.data_ptr(), x_dev.data_ptr(),
                                    y_dev.data_ptr(), rec.ws.data_ptr(), rec.ws.numel(),
                                    STREAM])


def test_cached_pointer_arrays_follow_replaced_weights(rec):
    packed, alphas, z = _arrays()
    w = api.BcqWeights(packed=packed, alphas=dict(alphas), z=z, N=N, K=K, p_H=4)
    x = torch.zeros((1, K), dtype=torch.float16)
    y = torch.zeros((1, N), dtype=torch.float16)
    api.gemm(x, w, p=2, out=y)
    api.gemm(x, w, p=2, out=y)
    a2 = torch.zeros_like(alphas[2])
    w.alphas[2] = a2
    api.gemm(x, w, p=2, out=y)
    w.alphas[1] = alphas[3]
    api.gemm(x, w, p=2, out=y)
    w.z = None
    api.gemm(x, w, p=2, out=y)
    arrs = [args[2] for _, args in rec.calls]
    assert arrs[0] == arrs[1] == _ptrs(alphas)
    assert arrs[2][1] == a2.data_ptr() and arrs[3][0] == alphas[3].data_ptr()
    assert [args[3] for _, args in rec.calls] == [z.data_ptr()] * 4 + [None]


def test_wrong_buffers_are_refused_before_any_call(rec):
    packed, alphas, z = _arrays()
    w = api.BcqWeights(packed=packed, alphas=alphas, z=z, N=N, K=K, p_H=4)
    x = torch.zeros((2, K), dtype=torch.float16)
    y = torch.zeros((2, N), dtype=torch.float16)
    bad_calls = [
        lambda: api.gemm(x, w, p=2, out=torch.zeros((2, N - 1), dtype=torch.float16)),
        lambda: api.gemm(x, w, p=2, out=torch.zeros((1, N), dtype=torch.float16)),
        lambda: api.gemm(x, w, p=2, out=torch.zeros((2, N), dtype=torch.float32)),
        lambda: api.gemm(x, w, p=2, out=torch.zeros((N, 2), dtype=torch.float16).t()),
        lambda: api.gemm(x[:, :512].contiguous(), w, p=2),
        lambda: api.gemm(x, w, p=2, p_row=[2, 2]),
        lambda: api.gemm(x, w, p_row=[2, 2, 2]),
        lambda: api.gemm_noalloc(x, w, p=2, out=torch.zeros((2, 8), dtype=torch.float16)),
        lambda: api.gemm(x, w, p=2, stream=_Stream("meta")),
        lambda: api.gemm_host(x, w, torch.zeros((2, N - 1), dtype=torch.float16), x, y, p=2),
        lambda: api.gemm_host(x, w, y, x[:1], y, p=2),
        lambda: api.gemm_host(x, w, y, x, y[:1], p=2),
        lambda: api.gemm_host(x.float(), w, y, x, y, p=2),
    ]
    for i, call in enumerate(bad_calls):
        with pytest.raises(ValueError):
            call()
        assert rec.calls == [], f"case {i} reached the library"
    # an array of the weight on another device than x
    for field in ("packed", "z"):
        w2 = api.BcqWeights(packed=packed, alphas=alphas, z=z, N=N, K=K, p_H=4)
        setattr(w2, field, torch.zeros(16, dtype=getattr(w2, field).dtype, device="meta"))
        with pytest.raises(ValueError):
            api.gemm(x, w2, p=2, out=y)
    w3 = api.BcqWeights(packed=packed, alphas={**alphas, 4: alphas[4].to("meta")}, z=z,
                        N=N, K=K, p_H=4)
    with pytest.raises(ValueError):
        api.gemm(x, w3, p=2, out=y)
    assert rec.calls == []
    np.testing.assert_array_equal(y.numpy(), 0)
