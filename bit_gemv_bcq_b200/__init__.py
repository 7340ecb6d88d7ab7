"""bit_gemv_bcq_b200 -- multi-precision binary-coded-quantization matmul on B200.

The compute lives in ``libbcq.so`` (hand-written sm_100a CUDA behind a C ABI,
declared in ``include/bcq.h``).  ``api`` is a thin ctypes binding: it marshals
torch CUDA tensors into pointers and calls the library; every step of the
matmul runs in the library's kernels.  There is no CPU fallback: the first
call raises if ``libbcq.so`` is missing.

``synth`` draws the seeded synthetic inputs; it holds none of the method's
arithmetic and is safe to import without a GPU.
"""
from __future__ import annotations

__all__ = ["api", "synth"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
