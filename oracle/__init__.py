"""fp64 CPU oracle for the multi-precision BCQ matmul.

TEST INFRASTRUCTURE.  Only tests/, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` import this package.  It shares no code with
the CUDA library (``bit_gemv_bcq_b200``) and never imports it.

The arithmetic lives in ``bcq_oracle.c`` (plain C, fp64); this module only
marshals numpy arrays.  ``quant.py`` holds the quantiser helpers (greedy +-1
decomposition, least-squares scale refit) used by the pins.

What is computed, by page title and section:
  * AnyBCQ (Paper-Notes page), "研究背景与动机 / 切入角度" -- W_hat is a sum of
    scaled +-1 bit-planes; p-bit inference uses p planes.
  * same page, "方法详解 / 训练策略" -- asymmetric, group size 128.
  * same page, "关键设计 / 直接bit-plane运算的CUDA内核" -- planes are +-1, the
    contraction is a signed sum, and only planes 1..p are read.
  * BiLoCo page, "核心思路：修正项只用 +1 和 −1" -- the signed sum of x.

Pins (tests/test_oracle_pins.py): the fp16 decoder against numpy for all
65536 codes; the BiLoCo hand example (3.4); closed forms for the LUT
(T[0xFF] = sum x, T[1<<j] = 2 x_j - sum x, T[~b] = -T[b]); brute-force dense
fp64 matmul on tiny shapes; closed forms for the GEMM (all-ones planes,
alpha = 0); the p-prefix, sign-symmetry, linearity and per-row-precision
invariants; the BiLoCo 3x2 greedy + joint-refit example for ``quant.py``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_HERE = os.path.dirname(os.path.abspath(__file__))
_lib = None
# A deliberately broken build of bcq_oracle.c, used only by the mutation test
# (tests/test_oracle_mutants.py) to show that the pins catch planted mistakes.
_lib_path = os.environ.get("BCQ_ORACLE_LIB") or None


def use_library(path: str | None) -> None:
    """Point this module at another build of bcq_oracle.c (None = default).
    Used by the mutation tests, which compile deliberately broken copies."""
    global _lib, _lib_path
    _lib, _lib_path = None, path


def _load():
    global _lib
    if _lib is None:
        path = _lib_path or _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.bcq_oracle_half_to_double.restype = ctypes.c_double
        lib.bcq_oracle_half_to_double.argtypes = [ctypes.c_uint16]
        lib.bcq_oracle_halves_to_double.restype = None
        lib.bcq_oracle_halves_to_double.argtypes = [P, P, ctypes.c_size_t]
        lib.bcq_oracle_signed_sum.restype = ctypes.c_double
        lib.bcq_oracle_signed_sum.argtypes = [P, P, I]
        lib.bcq_oracle_lut.restype = I
        lib.bcq_oracle_lut.argtypes = [P, I, I, P]
        lib.bcq_oracle_group_sums.restype = I
        lib.bcq_oracle_group_sums.argtypes = [P, I, I, I, P]
        lib.bcq_oracle_gemm.restype = I
        lib.bcq_oracle_gemm.argtypes = [P, P, P, P, I, P, I, I, I, I, I, P, I, P]
        lib.bcq_oracle_num_threads.restype = I
        lib.bcq_oracle_num_threads.argtypes = []
        _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _as_half_bits(a) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype == np.float16:
        a = a.view(np.uint16)
    if a.dtype != np.uint16:
        raise TypeError(f"expected fp16 data, got {a.dtype}")
    return np.ascontiguousarray(a)


def halves_to_double(h) -> np.ndarray:
    """Decode fp16 codes (float16 or uint16 bit patterns) to float64."""
    h = _as_half_bits(h)
    out = np.empty(h.shape, dtype=np.float64)
    _load().bcq_oracle_halves_to_double(_ptr(h), _ptr(out), h.size)
    return out


def signed_sum(x, bits_words) -> float:
    """sum_k (2 bit_k - 1) x_k with bits packed LSB-first in uint32 words."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    w = np.ascontiguousarray(bits_words, dtype=np.uint32)
    if w.size * 32 < x.size:
        raise ValueError("not enough bit words")
    return float(_load().bcq_oracle_signed_sum(_ptr(x), _ptr(w), x.size))


def lut(x) -> np.ndarray:
    """The 256-entry signed-sum table of every 8-column chunk: [M][K/8][256]."""
    x = _as_half_bits(x)
    if x.ndim == 1:
        x = x[None, :]
    M, K = x.shape
    out = np.empty((M, K // 8, 256), dtype=np.float64)
    rc = _load().bcq_oracle_lut(_ptr(x), M, K, _ptr(out))
    if rc:
        raise ValueError(f"bcq_oracle_lut rc={rc}")
    return out


def group_sums(x, group: int = 128) -> np.ndarray:
    """S[m][g] = sum of x[m] over column group g: [M][K/group]."""
    x = _as_half_bits(x)
    if x.ndim == 1:
        x = x[None, :]
    M, K = x.shape
    out = np.empty((M, K // group), dtype=np.float64)
    rc = _load().bcq_oracle_group_sums(_ptr(x), M, K, group, _ptr(out))
    if rc:
        raise ValueError(f"bcq_oracle_group_sums rc={rc}")
    return out


def gemm(x, planes, alphas: dict, z=None, p: int | None = None,
         p_row=None, group: int = 128, rows=None) -> np.ndarray:
    """y = x @ W_hat^T in fp64 (see bcq_oracle.c for the definition).

    x: fp16 [M][K]; planes: uint32 [p_H][N][K/32]; alphas: {q: fp16 [N][G][q]};
    z: fp16 [N][G], or {q: fp16 [N][G]} (offsets per precision: row m uses
    z^(p_m), the variant in which each precision keeps its own offsets, as it
    keeps its own scales -- AnyBCQ page, 渐进式精度扩展), or None; exactly one
    of ``p`` (uniform precision) and ``p_row`` (int per row of x) is given;
    ``rows`` optionally selects output rows n (returns [M][len(rows)]).
    """
    if isinstance(z, dict):
        # the rows of each precision through the same definition, with that
        # precision's offsets
        xa = _as_half_bits(x)
        if xa.ndim == 1:
            xa = xa[None, :]
        pr = np.full(xa.shape[0], int(p)) if p is not None else np.asarray(p_row, dtype=np.int64)
        out = None
        for q in sorted(set(int(v) for v in pr)):
            sel = np.nonzero(pr == q)[0]
            yq = gemm(xa[sel], planes, alphas, z.get(q), p=q, group=group, rows=rows)
            if out is None:
                out = np.empty((xa.shape[0], yq.shape[1]), dtype=np.float64)
            out[sel] = yq
        return out
    x = _as_half_bits(x)
    if x.ndim == 1:
        x = x[None, :]
    M, K = x.shape
    planes = np.ascontiguousarray(planes, dtype=np.uint32)
    p_H, N, KW = planes.shape
    if KW * 32 != K:
        raise ValueError("planes do not match K")
    keep = []
    arr = (ctypes.c_void_p * 4)()
    for q in range(1, 5):
        a = alphas.get(q) if alphas else None
        if a is not None:
            a = _as_half_bits(a)
            keep.append(a)
            arr[q - 1] = a.ctypes.data
        else:
            arr[q - 1] = None
    zz = None if z is None else _as_half_bits(z)
    if (p is None) == (p_row is None):
        raise ValueError("give exactly one of p and p_row")
    pr = None if p_row is None else np.ascontiguousarray(p_row, dtype=np.int32)
    rr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    n_out = N if rr is None else rr.size
    y = np.empty((M, n_out), dtype=np.float64)
    rc = _load().bcq_oracle_gemm(
        _ptr(x), _ptr(planes), ctypes.cast(arr, ctypes.c_void_p), _ptr(zz),
        0 if p is None else int(p), _ptr(pr), M, N, K, p_H, group,
        _ptr(rr), 0 if rr is None else rr.size, _ptr(y))
    if rc:
        raise ValueError(f"bcq_oracle_gemm rc={rc}")
    return y


def num_threads() -> int:
    return int(_load().bcq_oracle_num_threads())
