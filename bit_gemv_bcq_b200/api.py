"""Thin Python binding of libbcq (include/bcq.h).

Argument marshalling only: torch CUDA tensors become raw pointers, the
current torch stream becomes the CUDA stream, and every step of the matmul
runs in the library's kernels.  There is no CPU fallback: a missing
``libbcq.so`` raises ``BcqLibraryError`` on first use.

The same names as the C ABI: ``pack_planes``, ``pack_scales``,
``workspace_bytes``, ``gemm``, ``gemm_host``, ``build_lut``, ``device_error``,
``debug_wait_timeout``; ``BcqWeights`` bundles the packed planes with their
scales and offsets.  The split-K workspace bcq_gemm needs is kept here, one
zero-filled buffer per (device, stream), grown on demand.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
from dataclasses import dataclass, field

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbcq.so")

BCQ_OK = 0
BCQ_ERR_NULL = 1
BCQ_ERR_SHAPE = 2
BCQ_ERR_PRECISION = 3
BCQ_ERR_ALIGN = 4
BCQ_ERR_CUDA = 5
BCQ_ERR_TIMEOUT = 6
BCQ_ERR_UNSUPPORTED = 7
BCQ_ERR_SCRATCH = 8
NOALLOC_SCRATCH_BYTES = 16 << 20   # BCQ_NOALLOC_SCRATCH_BYTES
GROUP = 128
MAX_M = 64

_lib = None


class BcqLibraryError(RuntimeError):
    pass


class BcqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


def lib():
    """Load libbcq.so (built in-tree by bit_gemv_bcq_b200/build.py)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise BcqLibraryError(
                f"{LIB_PATH} is missing: build it with "
                "`python bit_gemv_bcq_b200/build.py` (there is no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.bcq_status_string.restype = ctypes.c_char_p
        L.bcq_status_string.argtypes = [I]
        L.bcq_version.restype = I
        L.bcq_version.argtypes = []
        L.bcq_packed_planes_bytes.restype = S
        L.bcq_packed_planes_bytes.argtypes = [I, I, I]
        L.bcq_pack_planes.restype = I
        L.bcq_pack_planes.argtypes = [P, P, I, I, I, P]
        L.bcq_packed_scales_bytes.restype = S
        L.bcq_packed_scales_bytes.argtypes = [I, I, I]
        L.bcq_pack_scales.restype = I
        L.bcq_pack_scales.argtypes = [P, I, I, I, P, P]
        L.bcq_route_query.restype = I
        L.bcq_route_query.argtypes = [I, I, P, I, I, P, I]
        L.bcq_set_pdl.restype = I
        L.bcq_set_pdl.argtypes = [I]
        L.bcq_workspace_bytes.restype = S
        L.bcq_workspace_bytes.argtypes = [I, I, I]
        L.bcq_plan_query.restype = I
        L.bcq_plan_query.argtypes = [I, I, I, I, I, I, P]
        L.bcq_gemm.restype = I
        L.bcq_gemm.argtypes = [P, P, P, P, I, P, I, I, I, I, I, P, P, S, P]
        L.bcq_gemm_host.restype = I
        L.bcq_gemm_host.argtypes = [P, P, P, P, I, P, I, I, I, I, I, P, P, P, P, S, P]
        L.bcq_gemm_zp.restype = I
        L.bcq_gemm_zp.argtypes = [P, P, P, P, I, P, I, I, I, I, I, P, P, S, P]
        L.bcq_gemm_noalloc.restype = I
        L.bcq_gemm_noalloc.argtypes = [P, P, P, P, I, P, I, I, I, I, I, P, P]
        L.bcq_build_lut.restype = I
        L.bcq_build_lut.argtypes = [P, I, I, P, P, P]
        L.bcq_device_error.restype = I
        L.bcq_device_error.argtypes = [P]
        L.bcq_debug_wait_timeout.restype = I
        L.bcq_debug_wait_timeout.argtypes = [I, P]
        L.bcq_quantize.restype = I
        L.bcq_quantize.argtypes = [P, I, I, I, I, I, P, P, P, P, P]
        L.bcq_quantize_zp.restype = I
        L.bcq_quantize_zp.argtypes = [P, I, I, I, I, I, P, P, P, P, P]
        _lib = L
    return _lib


EXPORTED = ("bcq_status_string", "bcq_version", "bcq_packed_planes_bytes",
            "bcq_pack_planes", "bcq_packed_scales_bytes", "bcq_pack_scales",
            "bcq_workspace_bytes", "bcq_gemm", "bcq_plan_query", "bcq_route_query", "bcq_set_pdl",
            "bcq_gemm_host", "bcq_gemm_noalloc", "bcq_build_lut", "bcq_device_error",
            "bcq_debug_wait_timeout", "bcq_quantize", "bcq_gemm_zp", "bcq_quantize_zp")


def status_string(status: int) -> str:
    return lib().bcq_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != BCQ_OK:
        raise BcqError(status, where)


def _stream(stream=None, device=None):
    """The CUDA stream handle: `stream` (which must belong to `device`), else
    the current stream of `device` (of the current device when None)."""
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    if device is not None and stream.device != device:
        raise ValueError(f"stream is on {stream.device}, the data on {device}")
    return ctypes.c_void_p(stream.cuda_stream)


def _on(device):
    """The C ABI works on the current CUDA device: make `device` current for
    the call when it is not already."""
    if device.index is None or device.index == torch.cuda.current_device():
        return contextlib.nullcontext()
    return torch.cuda.device(device)


def _ptr(t):
    # a plain int: every entry point declares its pointer arguments as void*
    return None if t is None else t.data_ptr()


def _need_cuda(t: torch.Tensor, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def _need_on(t: torch.Tensor, name: str, device) -> None:
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, x on {device}")


def _weights_on(w: "BcqWeights", device) -> None:
    """Every device array of w on `device` (the kernels take raw pointers)."""
    _need_on(w.packed, "planes", device)
    for q, a in w.alphas.items():
        _need_on(a, f"alpha[{q}]", device)
    if w.z is not None:
        _need_on(w.z, "z", device)
    for q, a in (w.zq or {}).items():
        _need_on(a, f"z[{q}]", device)


_data_ptr = torch.Tensor.data_ptr


def _weight_args(w: "BcqWeights", device):
    """(alpha, z) pointer arrays of w for the gemm entry points (z: the
    per-precision offsets, else None), its arrays checked to be on `device`.
    Kept on w while the signature -- device and every array's address --
    stays the same, so repeated calls skip the checks and the marshalling."""
    sig = (device, w.packed.data_ptr(), None if w.z is None else w.z.data_ptr(),
           tuple(w.alphas), tuple(map(_data_ptr, w.alphas.values())),
           None if w.zq is None else (tuple(w.zq), tuple(map(_data_ptr, w.zq.values()))))
    c = w._marshal
    if c is not None and c[0] == sig:
        return c[1], c[2]
    _weights_on(w, device)
    alpha = _alpha_array(w.alphas)
    zarr = None if w.zq is None else _alpha_array(w.zq, "z")
    w._marshal = (sig, alpha, zarr)
    return alpha, zarr


def _need_out(out: torch.Tensor | None, M: int, N: int, device) -> torch.Tensor:
    """The output [M][N] fp16 on `device`: allocated when None, else checked
    (the kernels write M*N values through its pointer)."""
    if out is None:
        return torch.empty((M, N), dtype=torch.float16, device=device)
    _need_cuda(out, "out", torch.float16)
    _need_on(out, "out", device)
    if tuple(out.shape) != (M, N):
        raise ValueError(f"out must be [{M}][{N}], got {list(out.shape)}")
    return out


def _need_x(x: torch.Tensor, K: int) -> int:
    _need_cuda(x, "x", torch.float16)
    if x.dim() != 2 or x.shape[1] != K:
        raise ValueError(f"x must be [M][{K}]")
    return x.shape[0]


def _alpha_array(alphas: dict, what: str = "alpha"):
    arr = (ctypes.c_void_p * 4)()
    for q in range(1, 5):
        a = alphas.get(q) if alphas else None
        if a is not None:
            _need_cuda(a, f"{what}[{q}]", torch.float16)
            arr[q - 1] = a.data_ptr()
        else:
            arr[q - 1] = None
    return arr


def packed_planes_bytes(p_H: int, N: int, K: int) -> int:
    return int(lib().bcq_packed_planes_bytes(p_H, N, K))


def pack_planes(planes_canon: torch.Tensor, stream=None) -> torch.Tensor:
    """Canonical planes (int32/uint32 CUDA tensor [p_H][N][K/32], LSB-first
    bits, 1 = +1) -> packed streaming layout (int32 CUDA tensor)."""
    _need_cuda(planes_canon, "planes")
    if planes_canon.element_size() != 4 or planes_canon.dim() != 3:
        raise ValueError("planes must be a 32-bit [p_H][N][K/32] tensor")
    p_H, N, KW = planes_canon.shape
    K = KW * 32
    nbytes = packed_planes_bytes(p_H, N, K)
    if nbytes == 0:
        raise BcqError(BCQ_ERR_SHAPE, "bcq_packed_planes_bytes")
    dev = planes_canon.device
    out = torch.empty(nbytes // 4, dtype=torch.int32, device=dev)
    with _on(dev):
        _check(lib().bcq_pack_planes(_ptr(planes_canon), _ptr(out), p_H, N, K,
                                     _stream(stream, dev)), "bcq_pack_planes")
    return out


def packed_scales_bytes(q: int, N: int, K: int) -> int:
    return int(lib().bcq_packed_scales_bytes(q, N, K))


def pack_scales(src: torch.Tensor, q: int, stream=None) -> torch.Tensor:
    """Canonical fp16 per-(row, group) array [N][K/128][q] (or [N][K/128] for
    q = 1) -> packed streaming order (fp16 CUDA tensor)."""
    _need_cuda(src, "scales", torch.float16)
    N, G = src.shape[0], src.shape[1]
    if src.numel() != N * G * q:
        raise ValueError("scales must hold q values per (row, group)")
    K = G * GROUP
    nbytes = packed_scales_bytes(q, N, K)
    if nbytes == 0:
        raise BcqError(BCQ_ERR_SHAPE, "bcq_packed_scales_bytes")
    dev = src.device
    out = torch.empty(nbytes // 2, dtype=torch.float16, device=dev)
    with _on(dev):
        _check(lib().bcq_pack_scales(_ptr(src), int(q), N, K, _ptr(out), _stream(stream, dev)),
               "bcq_pack_scales")
    return out


def quantize(w: torch.Tensor, p_L: int = 2, p_H: int = 4, rounds: int = 20,
             with_sse: bool = False, offsets: str = "shared", stream=None):
    """Offline quantiser (bcq_quantize): fp16 CUDA weights [N][K] ->
    (planes int32 [p_H][N][K/32] holding the uint32 words, {p: alpha^(p) fp16
    [N][K/128][p]} for p = p_L..p_H, z fp16 [N][K/128], and with_sse: fp64
    [p_H - p_L + 1][N][K/128] squared error per group, else None).
    offsets="per_precision" (bcq_quantize_zp): z is {p: z^(p) fp16 [N][K/128]}
    for the per-precision offsets of bcq_gemm_zp."""
    if offsets not in ("shared", "per_precision"):
        raise ValueError("offsets must be 'shared' or 'per_precision'")
    _need_cuda(w, "w", torch.float16)
    if w.dim() != 2:
        raise ValueError("w must be [N][K]")
    N, K = w.shape
    G = K // GROUP
    dev = w.device
    planes = torch.empty((p_H, N, K // 32), dtype=torch.int32, device=dev)
    alphas = {p: torch.empty((N, G, p), dtype=torch.float16, device=dev)
              for p in range(p_L, p_H + 1)} if 1 <= p_L <= p_H <= 4 else {}
    sse = (torch.empty((max(p_H - p_L + 1, 0), N, G), dtype=torch.float64, device=dev)
           if with_sse else None)
    if offsets == "per_precision":
        z = {p: torch.empty((N, G), dtype=torch.float16, device=dev) for p in alphas}
        with _on(dev):
            _check(lib().bcq_quantize_zp(_ptr(w), N, K, int(p_L), int(p_H), int(rounds),
                                         _ptr(planes), _alpha_array(alphas),
                                         _alpha_array(z, "z"), _ptr(sse), _stream(stream, dev)),
                   "bcq_quantize_zp")
        return planes, alphas, z, sse
    z = torch.empty((N, G), dtype=torch.float16, device=dev)
    with _on(dev):
        _check(lib().bcq_quantize(_ptr(w), N, K, int(p_L), int(p_H), int(rounds), _ptr(planes),
                                  _alpha_array(alphas), _ptr(z), _ptr(sse),
                                  _stream(stream, dev)), "bcq_quantize")
    return planes, alphas, z, sse


PLAN_FIELDS = ("C", "consumer_warps", "NP", "D", "dyn_bytes", "stage_bytes", "units_max",
               "KB")


def plan_query(M: int, N: int, K: int, p_load: int, mixed: bool = False,
               use_device: bool = False) -> dict:
    """Launch plan of one GEMV launch (see bcq_plan_query)."""
    out = (ctypes.c_int * 8)()
    _check(lib().bcq_plan_query(M, N, K, p_load, int(mixed), int(use_device),
                                ctypes.cast(out, ctypes.c_void_p)), "bcq_plan_query")
    return dict(zip(PLAN_FIELDS, list(out)))


KERNEL_NAMES = {1: "lut_pair", 2: "lut_one", 3: "lut_four", 4: "mma", 5: "mma_mixed",
                6: "tcgen05"}


def route_query(M: int, N: int, K: int, p: int | None = None, p_row=None) -> list:
    """The launches bcq_gemm makes for M rows (see bcq_route_query):
    [(kernel name, rows, planes streamed), ...]."""
    pv, pr_keep, pr_ptr = _prec_args(p, p_row, M)
    out = (ctypes.c_int * (1 + 3 * 64))()
    _check(lib().bcq_route_query(M, pv, pr_ptr, N, K, ctypes.cast(out, ctypes.c_void_p), 64),
           "bcq_route_query")
    del pr_keep
    return [(KERNEL_NAMES[out[1 + 3 * i]], out[2 + 3 * i], out[3 + 3 * i])
            for i in range(min(out[0], 64))]


def workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib().bcq_workspace_bytes(M, N, K))


_WS: dict = {}


def workspace(M: int, N: int, K: int, device, stream=None) -> torch.Tensor | None:
    """The zero-filled workspace of (device, stream), at least
    bcq_workspace_bytes(M, N, K) bytes; None when none is needed.  Every call
    that completes leaves it zero-filled again.  Calls that may run at the
    same time (other streams) get workspaces of their own."""
    need = workspace_bytes(M, N, K)
    if need == 0:
        return None
    s = torch.cuda.current_stream(device) if stream is None else stream
    key = (torch.device(device).index, s.cuda_stream)
    ws = _WS.get(key)
    if ws is None or ws.numel() < need:
        with torch.cuda.stream(s):
            ws = torch.zeros(max(need, 2 * ws.numel() if ws is not None else need),
                             dtype=torch.uint8, device=device)
        _WS[key] = ws
    return ws


def drop_workspaces() -> None:
    """Forget the cached workspaces (after a device error they may hold
    partial sums; new ones are zero-filled)."""
    _WS.clear()


def set_pdl(mode: int) -> None:
    """Programmatic dependent launch for later GEMV launches (see bcq_set_pdl)."""
    _check(lib().bcq_set_pdl(int(mode)), "bcq_set_pdl")


@dataclass
class BcqWeights:
    """One BCQ weight matrix on the device: packed +-1 planes shared by every
    precision, the scales alpha^(q) of each precision q and the offsets z,
    all in the library's streaming order (bcq_pack_planes, bcq_pack_scales)."""
    packed: torch.Tensor        # int32, library layout
    alphas: dict                # {q: packed alpha^(q), fp16}
    z: torch.Tensor | None      # packed offsets (fp16) or None
    N: int
    K: int
    p_H: int
    row_splits: tuple = ()      # rows of each stacked matrix (see stack), else ()
    zq: dict | None = None      # {q: packed offsets z^(q)} when every precision has its own
    # (signature, alpha pointer array, z pointer array) of the last call: see _weight_args
    _marshal: tuple | None = field(default=None, init=False, repr=False, compare=False)

    @classmethod
    def from_canonical(cls, planes, alphas: dict, z=None, device="cuda", stream=None):
        """planes: uint32 [p_H][N][K/32] (numpy or tensor); alphas {q: fp16
        [N][G][q]}; z fp16 [N][G], or {q: fp16 [N][G]} (offsets per precision,
        used through bcq_gemm_zp), or None."""
        if isinstance(planes, np.ndarray):
            planes = torch.from_numpy(np.ascontiguousarray(planes).view(np.int32))
        planes = planes.to(device).contiguous()
        p_H, N, KW = planes.shape
        packed = pack_planes(planes, stream)
        al = {}
        for q, a in alphas.items():
            a = torch.as_tensor(a) if isinstance(a, np.ndarray) else a
            al[int(q)] = pack_scales(a.to(device=device, dtype=torch.float16).contiguous(),
                                     int(q), stream)
        def pack_z(zv):
            zv = torch.as_tensor(zv) if isinstance(zv, np.ndarray) else zv
            return pack_scales(zv.to(device=device, dtype=torch.float16).contiguous(), 1, stream)

        if isinstance(z, dict):
            zq = {int(q): pack_z(zv) for q, zv in z.items() if zv is not None}
            return cls(packed=packed, alphas=al, z=None, N=N, K=KW * 32, p_H=p_H, zq=zq)
        zz = None if z is None else pack_z(z)
        return cls(packed=packed, alphas=al, z=zz, N=N, K=KW * 32, p_H=p_H)

    @classmethod
    def quantize(cls, w: torch.Tensor, p_L: int = 2, p_H: int = 4, rounds: int = 20,
                 offsets: str = "shared", stream=None):
        """Quantise fp16 CUDA weights [N][K] on the device (bcq_quantize, or
        bcq_quantize_zp for offsets="per_precision") and pack the result for
        bcq_gemm (bcq_gemm_zp)."""
        planes, alphas, z, _ = quantize(w, p_L, p_H, rounds, offsets=offsets, stream=stream)
        return cls.from_canonical(planes, alphas, z, device=w.device, stream=stream)

    @classmethod
    def stack(cls, parts, device="cuda", stream=None):
        """Matrices that multiply the same x -- an MLP's gate and up
        projections -- as one weight: their canonical planes, scales and
        offsets stacked along N and packed together.  One call then reads x,
        builds each K-block's lookup table and reduces the split-K partial sums
        once for all of them: the table of cached +-x partial sums depends on x
        only (AnyBCQ Paper-Notes page, 关键设计 / 直接bit-plane运算的CUDA内核),
        and its build is the cost the FluxBin page's "Lookup Table Building
        Approach with Scale Fusion" sets out to keep small.
        parts: sequence of (planes uint32 [p_H][N_i][K/32], {q: alpha fp16
        [N_i][G][q]}, z fp16 [N_i][G] or None); every part has the same p_H,
        K and precisions, and all or none have z.  gemm() returns y
        [M][sum N_i]; split_rows() gives the per-matrix views."""
        parts = list(parts)
        if not parts:
            raise ValueError("nothing to stack")

        def cat(arrays, axis):
            if all(isinstance(a, np.ndarray) for a in arrays):
                return np.concatenate(arrays, axis=axis)
            return torch.cat([torch.as_tensor(a) for a in arrays], dim=axis)

        planes = cat([pl for pl, _, _ in parts], 1)
        qs = set(parts[0][1])
        if any(set(al) != qs for _, al, _ in parts):
            raise ValueError("every stacked matrix needs the same precisions")
        alphas = {q: cat([al[q] for _, al, _ in parts], 0) for q in sorted(qs)}
        zs = [z for _, _, z in parts]
        if any((z is None) != (zs[0] is None) for z in zs):
            raise ValueError("give z for every stacked matrix or for none")
        z = None if zs[0] is None else cat(zs, 0)
        w = cls.from_canonical(planes, alphas, z, device=device, stream=stream)
        w.row_splits = tuple(int(pl.shape[1]) for pl, _, _ in parts)
        return w

    def split_rows(self, y):
        """Per-matrix views [M][N_i] of the output of a stacked weight."""
        if not self.row_splits:
            return [y]
        out, r0 = [], 0
        for n in self.row_splits:
            out.append(y[:, r0:r0 + n])
            r0 += n
        return out

    def gemm(self, x, p=None, p_row=None, out=None, stream=None):
        return gemm(x, self, p=p, p_row=p_row, out=out, stream=stream)


def _prec_args(p, p_row, M):
    if (p is None) == (p_row is None):
        raise ValueError("give exactly one of p and p_row")
    if p is not None:
        return int(p), None, None
    pr = np.ascontiguousarray(np.asarray(p_row, dtype=np.int32))
    if pr.shape != (M,):
        raise ValueError("p_row must have one entry per row of x")
    return 0, pr, pr.ctypes.data_as(ctypes.c_void_p)


def gemm(x: torch.Tensor, w: BcqWeights, p: int | None = None, p_row=None,
         out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y = x . W_hat^T (fp16 [M][N]) with uniform precision p or per-row p_row."""
    M = _need_x(x, w.K)
    dev = x.device
    alpha, zarr = _weight_args(w, dev)   # arrays of 4 device pointers or NULL
    pv, pr_keep, pr_ptr = _prec_args(p, p_row, M)
    out = _need_out(out, M, w.N, dev)
    sh = _stream(stream, dev)
    ws = workspace(M, w.N, w.K, dev, stream)
    with _on(dev):
        if zarr is not None:
            st = lib().bcq_gemm_zp(_ptr(x), _ptr(w.packed), alpha, zarr, pv, pr_ptr, M, w.N,
                                   w.K, w.p_H, GROUP, _ptr(out), _ptr(ws),
                                   0 if ws is None else ws.numel(), sh)
            _check(st, "bcq_gemm_zp")
        else:
            st = lib().bcq_gemm(_ptr(x), _ptr(w.packed), alpha, _ptr(w.z), pv, pr_ptr, M, w.N,
                                w.K, w.p_H, GROUP, _ptr(out), _ptr(ws),
                                0 if ws is None else ws.numel(), sh)
            _check(st, "bcq_gemm")
    del pr_keep
    return out


def gemm_noalloc(x: torch.Tensor, w: BcqWeights, p: int | None = None, p_row=None,
                 out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """bcq_gemm_noalloc: as gemm, but the split-K scratch is the library's own
    static array instead of a workspace, for callers that cannot allocate
    device memory.  Calls that may overlap on the GPU share that array and
    race; shapes needing more than NOALLOC_SCRATCH_BYTES raise
    BcqError(BCQ_ERR_SCRATCH).  `out` should be given by such callers (the
    binding allocates it otherwise)."""
    if w.zq is not None:
        raise ValueError("per-precision offsets: use gemm (bcq_gemm_zp)")
    M = _need_x(x, w.K)
    alpha, _ = _weight_args(w, x.device)
    pv, pr_keep, pr_ptr = _prec_args(p, p_row, M)
    out = _need_out(out, M, w.N, x.device)
    sh = _stream(stream, x.device)
    with _on(x.device):
        st = lib().bcq_gemm_noalloc(_ptr(x), _ptr(w.packed), alpha, _ptr(w.z), pv, pr_ptr, M,
                                    w.N, w.K, w.p_H, GROUP, _ptr(out), sh)
    _check(st, "bcq_gemm_noalloc")
    del pr_keep
    return out


def gemm_host(x_host: torch.Tensor, w: BcqWeights, y_host: torch.Tensor,
              x_dev: torch.Tensor, y_dev: torch.Tensor, p: int | None = None,
              p_row=None, stream=None) -> None:
    """bcq_gemm_host: x and y in (pinned) host memory, copies on the stream.
    The caller synchronises the stream before reading y_host."""
    if w.zq is not None:
        raise ValueError("per-precision offsets: use gemm (bcq_gemm_zp)")
    if x_host.is_cuda or y_host.is_cuda:
        raise ValueError("x_host and y_host must be host tensors")
    for t, name in ((x_host, "x_host"), (y_host, "y_host")):
        if t.dtype != torch.float16 or not t.is_contiguous() or t.dim() != 2:
            raise ValueError(f"{name} must be a contiguous fp16 matrix")
    M = x_host.shape[0]
    if x_host.shape[1] != w.K or tuple(y_host.shape) != (M, w.N):
        raise ValueError(f"x_host must be [M][{w.K}] and y_host [M][{w.N}]")
    for t, name, n in ((x_dev, "x_dev", M * w.K), (y_dev, "y_dev", M * w.N)):
        _need_cuda(t, name, torch.float16)
        if t.numel() < n:
            raise ValueError(f"{name} must hold at least {n} values")
    dev = x_dev.device
    _need_on(y_dev, "y_dev", dev)
    alpha, _ = _weight_args(w, dev)
    pv, pr_keep, pr_ptr = _prec_args(p, p_row, M)
    sh = _stream(stream, dev)
    ws = workspace(M, w.N, w.K, dev, stream)
    with _on(dev):
        st = lib().bcq_gemm_host(_ptr(x_host), _ptr(w.packed), alpha, _ptr(w.z), pv, pr_ptr, M,
                                 w.N, w.K, w.p_H, GROUP, _ptr(y_host), _ptr(x_dev), _ptr(y_dev),
                                 _ptr(ws), 0 if ws is None else ws.numel(), sh)
    _check(st, "bcq_gemm_host")
    del pr_keep


def build_lut(x: torch.Tensor, stream=None):
    """The LUT and group sums as the GEMV kernel builds them:
    (fp32 [M][K/8][256], fp32 [M][K/128])."""
    _need_cuda(x, "x", torch.float16)
    M, K = x.shape
    lut = torch.empty((M, K // 8, 256), dtype=torch.float32, device=x.device)
    gs = torch.empty((M, K // GROUP), dtype=torch.float32, device=x.device)
    with _on(x.device):
        _check(lib().bcq_build_lut(_ptr(x), M, K, _ptr(lut), _ptr(gs), _stream(stream, x.device)),
               "bcq_build_lut")
    return lut, gs


def device_error(stream=None) -> int:
    """Synchronise the stream, return and clear the device error word.  After
    an error the cached workspaces are dropped (they may hold partial sums)."""
    st = int(lib().bcq_device_error(_stream(stream)))
    if st != BCQ_OK:
        drop_workspaces()
    return st


def debug_wait_timeout(limit_us: int, stream=None) -> None:
    _check(lib().bcq_debug_wait_timeout(int(limit_us), _stream(stream)),
           "bcq_debug_wait_timeout")
