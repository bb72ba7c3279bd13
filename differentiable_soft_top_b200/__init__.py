"""Exact-budget LapSum soft top-k on the NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI in ``include/lapsum_topk.h``: it only
marshals tensors, sizes and the current CUDA stream into the native library
``liblapsum_topk.so``; every step of the operator runs in that library's
kernels.  There is no CPU path: CPU tensors are rejected and a missing or
unbuildable library raises.

Operator ("Fast LapSum: Exact Differentiable Top-k at Million Scale",
technical summary section 2.1): p_i = F((r_i - b)/alpha) with F the Laplace
CDF and b chosen so that sum_i p_i = k; backward grad_j = f_j (g_j - lambda),
lambda = sum g f / sum f.

    import torch, differentiable_soft_top_b200 as lt
    p = lt.soft_topk(scores, k=1000.0, alpha=0.1)       # autograd-aware
    res = lt.forward(scores, 1000.0, 0.1, stats=True)   # p, b, sum f, status
    grad, dk = lt.backward(scores, g, res.b, 0.1)
"""
from __future__ import annotations

import ctypes
import math
import os
import threading
from dataclasses import dataclass

import numpy as np

__all__ = [
    "Params", "ForwardResult", "forward", "backward", "forward_into", "backward_into", "soft_topk", "SoftTopK", "workspace_size",
    "status_string", "launch_count", "trace_enable", "trace_collect", "library_path", "STATS_DTYPE", "ROW_CERTIFIED", "ROW_WIDENED",
    "ROW_FALLBACK", "ROW_NONFINITE", "ROW_TIMEOUT", "ROW_OVERFLOW", "ROW_TRUNCATED", "ROW_BADARG",
    "forward_sparse", "SparseResult", "sparse_workspace_size", "FORCE_NONE", "FORCE_FALLBACK",
    "FORCE_STREAMING", "FORCE_TIMEOUT", "LapsumError", "dftopk_forward", "DFTopKResult",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "liblapsum_topk.so")

LAPSUM_OK, LAPSUM_EINVAL, LAPSUM_EBADK, LAPSUM_EBADALPHA, LAPSUM_EWORKSPACE, LAPSUM_ECUDA, LAPSUM_ETOOLARGE = range(7)
NOALLOC_MAX_ROWS, NOALLOC_MAX_N = 65536, 16384  # limits of forward_noalloc_into
ROW_CERTIFIED, ROW_WIDENED, ROW_FALLBACK = 0x01, 0x02, 0x04
ROW_TRUNCATED = 0x40
ROW_BADARG = 0x80  # per-row k or alpha out of range: the row's outputs are NaN
ROW_NONFINITE, ROW_TIMEOUT, ROW_OVERFLOW = 0x08, 0x10, 0x20
FORCE_NONE, FORCE_FALLBACK, FORCE_STREAMING, FORCE_TIMEOUT = 0, 1, 2, 4
DEFAULT_Z = 4.0  # bracket half-width in binomial sigmas that Params.z = 0 selects


class LapsumError(RuntimeError):
    def __init__(self, code: int, where: str):
        msg = f"{where}: {status_string(code)} (code {code})"
        if code == LAPSUM_ECUDA:
            msg += f": {_load().lapsum_last_cuda_error().decode()}"
        super().__init__(msg)
        self.code = code


class _CParams(ctypes.Structure):
    _fields_ = [
        ("sample_m", ctypes.c_uint32),
        ("force_path", ctypes.c_uint32),
        ("z", ctypes.c_double),
        ("seed", ctypes.c_uint64),
        ("band_capacity", ctypes.c_int64),
        ("max_widen", ctypes.c_int32),
        ("spin_limit", ctypes.c_int32),
    ]


STATS_DTYPE = np.dtype([
    ("a_L", np.float32), ("a_R", np.float32),
    ("n_L", np.int64), ("n_R", np.int64), ("band", np.int64),
    ("S_L", np.float64), ("S_R", np.float64),
    ("b", np.float64), ("sum_p", np.float64), ("sum_f", np.float64),
    ("sample_m", np.int32), ("buckets", np.int32),
    ("status", np.uint32), ("reserved", np.int32),
], align=True)
assert STATS_DTYPE.itemsize == 88


@dataclass
class Params:
    """Tuning and test knobs (lapsum_params).  Zero / negative = automatic."""
    sample_m: int = 0
    force_path: int = FORCE_NONE
    z: float = 0.0          # 0 = the library's default (4 binomial sigmas)
    seed: int = 0
    band_capacity: int = 0
    max_widen: int = -1
    spin_limit: int = 0     # polls before a bounded device wait gives up; 0 = about a second

    def _c(self) -> _CParams:
        return _CParams(int(self.sample_m), int(self.force_path), float(self.z),
                        int(self.seed) & (2**64 - 1), int(self.band_capacity), int(self.max_widen),
                        int(self.spin_limit))


_lib = None
_lib_lock = threading.Lock()


def library_path() -> str:
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    with _lib_lock:
        if _lib is None:
            from . import _build
            if _build.stale(_LIB_PATH):
                _build.build()
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(f"native library missing: {_LIB_PATH}")
            lib = ctypes.CDLL(_LIB_PATH)
            P, i64, dbl, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_double, ctypes.c_size_t
            lib.lapsum_default_params.argtypes = [P]
            lib.lapsum_default_params.restype = None
            lib.lapsum_topk_workspace_size.argtypes = [i64, i64, P]
            lib.lapsum_topk_workspace_size.restype = sz
            lib.lapsum_topk_fwd.argtypes = [P, i64, i64, i64, dbl, dbl, P, P, P, P, P, P, sz, P, P]
            lib.lapsum_topk_fwd.restype = ctypes.c_int
            lib.lapsum_topk_bwd.argtypes = [P, P, P, i64, i64, i64, dbl, P, P, P, P, sz, P]
            lib.lapsum_topk_fwd_sparse.argtypes = [P, i64, i64, i64, dbl, dbl, ctypes.c_float, P, P, i64, P, P, P,
                                                   P, P, P, sz, P, P]
            lib.lapsum_topk_fwd_sparse.restype = ctypes.c_int
            lib.lapsum_topk_sparse_workspace_size.argtypes = [i64, i64, P]
            lib.lapsum_topk_sparse_workspace_size.restype = sz
            lib.lapsum_topk_bwd.restype = ctypes.c_int
            lib.lapsum_topk_fwd_noalloc.argtypes = [P, i64, i64, i64, dbl, dbl, P, P, P, P, P, P, P]
            lib.lapsum_topk_fwd_noalloc.restype = ctypes.c_int
            lib.lapsum_topk_fwd_rows.argtypes = [P, i64, i64, i64, P, P, P, P, P, P, P, P, sz, P, P]
            lib.lapsum_topk_fwd_rows.restype = ctypes.c_int
            lib.lapsum_topk_bwd_rows.argtypes = [P, P, P, i64, i64, i64, P, P, P, P, P, sz, P]
            lib.lapsum_topk_bwd_rows.restype = ctypes.c_int
            lib.lapsum_dftopk_fwd.argtypes = [P, i64, i64, i64, i64, dbl, P, P, P, P, P, P, P, sz, P, P]
            lib.lapsum_dftopk_fwd.restype = ctypes.c_int
            lib.lapsum_status_string.argtypes = [ctypes.c_int]
            lib.lapsum_status_string.restype = ctypes.c_char_p
            lib.lapsum_last_cuda_error.argtypes = []
            lib.lapsum_last_cuda_error.restype = ctypes.c_char_p
            lib.lapsum_launch_count.argtypes = []
            lib.lapsum_launch_count.restype = ctypes.c_uint64
            lib.lapsum_trace_enable.argtypes = [ctypes.c_int]
            lib.lapsum_trace_enable.restype = None
            lib.lapsum_trace_collect.argtypes = [ctypes.c_char_p, sz]
            lib.lapsum_trace_collect.restype = ctypes.c_int
            _lib = lib
    return _lib


def status_string(code: int) -> str:
    return _load().lapsum_status_string(int(code)).decode()


def launch_count() -> int:
    """Kernels the native library has launched in this process."""
    return int(_load().lapsum_launch_count())


def trace_enable(on: bool = True) -> None:
    """Bracket every library kernel launch with CUDA events (see trace_collect)."""
    _load().lapsum_trace_enable(1 if on else 0)


def trace_collect() -> dict:
    """{kernel: (launches, total_ms)} of the launches traced since the last call."""
    import json
    lib = _load()
    need = lib.lapsum_trace_collect(None, 0)
    buf = ctypes.create_string_buffer(max(need, 2) + 64)
    n = lib.lapsum_trace_collect(buf, len(buf))
    if n < 0:
        raise RuntimeError("lapsum_trace_collect failed")
    return {k: (int(v[0]), float(v[1])) for k, v in json.loads(buf.value.decode()).items()}


def _params_ptr(params: Params | None):
    if params is None:
        return None, None
    c = params._c()
    return c, ctypes.byref(c)


def workspace_size(rows: int, n: int, params: Params | None = None) -> int:
    c, ptr = _params_ptr(params)
    return int(_load().lapsum_topk_workspace_size(int(rows), int(n), ptr))


# ---------------------------------------------------------------------------
# tensor marshalling (torch is only the owner of device memory and streams)
# ---------------------------------------------------------------------------
def _torch():
    import torch
    return torch


_ws_cache: dict = {}


def _workspace(device, nbytes: int):
    torch = _torch()
    stream = torch.cuda.current_stream(device).cuda_stream
    key = (device.index if device.index is not None else torch.cuda.current_device(), stream)
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        _ws_cache[key] = buf
    return buf


def _rows_view(t, name, *, copy_ok=False):
    """t (CUDA fp32, 1-D or 2-D) as a [rows, n] view with unit column stride.
    An input may be copied to get that stride (copy_ok); an output may not,
    since the kernels would then fill a temporary instead of the caller's
    tensor."""
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor (this library has no CPU path)")
    if t.dtype != torch.float32:
        raise TypeError(f"{name} must be float32")
    if t.dim() == 1:
        t2 = t.view(1, -1)
    elif t.dim() == 2:
        t2 = t
    else:
        raise ValueError(f"{name} must be 1-D or 2-D")
    if t2.stride(1) != 1 and t2.shape[1] > 1:
        if not copy_ok:
            raise ValueError(f"{name} must have unit stride along its rows")
        t2 = t2.contiguous()
    if t2.shape[0] == 1 and t2.stride(0) != t2.shape[1]:
        # one row (a numpy [None, :] view has row stride 0): its row stride
        # is never used, so give it the dense one the C ABI checks
        t2 = t2.as_strided(t2.shape, (max(1, t2.shape[1]), 1))
    return t2


def _as_rows(t, name):
    return _rows_view(t, name, copy_ok=True)


def _check_like(x, t, name):
    """t is laid out as the C ABI reads or writes it beside the scores x: the
    same [rows, n] shape, the same device and x's row stride (one row stride
    serves every array of a call).  Works on any device's tensors."""
    if tuple(t.shape) != tuple(x.shape):
        raise ValueError(f"{name} must have the shape of scores {tuple(x.shape)}, got {tuple(t.shape)}")
    if t.device != x.device:
        raise ValueError(f"{name} must be on the device of scores ({x.device}), got {t.device}")
    if x.shape[0] > 1 and t.stride(0) != x.stride(0):
        raise ValueError(f"{name} must have the row stride of scores ({x.stride(0)}), got {t.stride(0)}")


def _check_vec(t, name, rows, dtype, device, optional=False):
    """A per-row array: `rows` contiguous values of `dtype` on `device`."""
    if t is None:
        if optional:
            return
        raise ValueError(f"{name} is required")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if not t.is_contiguous() or t.numel() < rows:
        raise ValueError(f"{name} must be contiguous with at least {rows} values")


def _like_rows(x):
    """An uninitialised [rows, n] tensor with the row stride of x (the C ABI
    uses one row stride for inputs and outputs) that starts at x's address
    mod 16, so that the kernels move both 16 bytes at a time even when x is
    an offset view."""
    torch = _torch()
    rows, n = x.shape
    s = x.stride(0)
    if rows == 0 or n == 0:  # rejected by the library; nothing to place
        return torch.empty_strided((rows, n), (s, 1), dtype=x.dtype, device=x.device)
    buf = torch.empty((rows - 1) * s + n + 3, dtype=x.dtype, device=x.device)
    off = ((x.data_ptr() - buf.data_ptr()) // x.element_size()) % 4
    return buf.as_strided((rows, n), (s, 1), storage_offset=off)


def _per_row(v, rows, dev):
    """v as a contiguous fp64 [rows] CUDA tensor when it is a 1-D tensor with
    one value per row; None when it is a number or a single-value tensor."""
    torch = _torch()
    if not isinstance(v, torch.Tensor) or v.dim() == 0:
        return None
    if v.dim() != 1 or v.shape[0] != rows:
        raise ValueError(f"a per-row k or alpha must have shape [{rows}], got {tuple(v.shape)}")
    return v.detach().to(device=dev, dtype=torch.float64).contiguous()


def _rows_pair(k, alpha, rows, dev):
    """(k_rows, alpha_rows) for the *_rows entry points, or None when both are
    scalars (a scalar beside a vector is broadcast)."""
    torch = _torch()
    kr, ar = _per_row(k, rows, dev), _per_row(alpha, rows, dev)
    if kr is None and ar is None:
        return None
    if kr is None:
        kr = torch.full((rows,), float(k), dtype=torch.float64, device=dev)
    if ar is None:
        ar = torch.full((rows,), float(alpha), dtype=torch.float64, device=dev)
    return kr, ar


@dataclass
class ForwardResult:
    p: object          # torch.Tensor, same shape as scores
    b: object          # torch.Tensor float64 [rows]
    sumf: object       # torch.Tensor float64 [rows]
    status: object     # torch.Tensor int32 view of uint32 [rows]
    stats: np.ndarray | None = None  # STATS_DTYPE [rows], when requested


def forward(scores, k, alpha, *, params: Params | None = None, workspace=None,
            stats: bool = False, p_out=None) -> ForwardResult:
    """Thresholds and memberships for every row of `scores` (CUDA fp32).  k
    and alpha are numbers, or [rows] tensors giving each row its own value
    (rows with an out-of-range value get ROW_BADARG and NaN outputs)."""
    torch = _torch()
    lib = _load()
    x = _as_rows(scores, "scores")
    rows, n = x.shape
    dev = x.device
    if p_out is None:
        p = _like_rows(x)
    else:
        p = _rows_view(p_out, "p_out")
        _check_like(x, p, "p_out")
    b = torch.empty(rows, dtype=torch.float64, device=dev)
    sumf = torch.empty(rows, dtype=torch.float64, device=dev)
    status = torch.empty(rows, dtype=torch.int32, device=dev)
    st = torch.empty(rows * STATS_DTYPE.itemsize, dtype=torch.uint8, device=dev) if stats else None
    c, pptr = _params_ptr(params)
    need = int(lib.lapsum_topk_workspace_size(rows, n, pptr))
    ws = workspace if workspace is not None else _workspace(dev, need)
    stream = torch.cuda.current_stream(dev).cuda_stream
    pr = _rows_pair(k, alpha, rows, dev)
    if pr is None:
        rc = lib.lapsum_topk_fwd(x.data_ptr(), rows, n, x.stride(0), float(k), float(alpha), p.data_ptr(),
                                 b.data_ptr(), sumf.data_ptr(), status.data_ptr(),
                                 st.data_ptr() if st is not None else None, ws.data_ptr(), ws.numel(), pptr,
                                 stream)
    else:
        rc = lib.lapsum_topk_fwd_rows(x.data_ptr(), rows, n, x.stride(0), pr[0].data_ptr(), pr[1].data_ptr(),
                                      p.data_ptr(), b.data_ptr(), sumf.data_ptr(), status.data_ptr(),
                                      st.data_ptr() if st is not None else None, ws.data_ptr(), ws.numel(), pptr,
                                      stream)
    if rc != LAPSUM_OK:
        raise LapsumError(rc, "lapsum_topk_fwd" if pr is None else "lapsum_topk_fwd_rows")
    stats_np = st.cpu().numpy().view(STATS_DTYPE) if st is not None else None
    return ForwardResult(p.view(scores.shape) if p_out is None and scores.dim() == 1 else (p if p_out is None else p_out),
                         b, sumf, status, stats_np)


@dataclass
class DFTopKResult:
    p: object          # torch.Tensor, same shape as scores
    b: object          # torch.Tensor float64 [rows]: midpoint of the k-th and (k+1)-th largest
    sumf: object       # torch.Tensor float64 [rows]: sum f at alpha
    mass: object       # torch.Tensor float64 [rows]: sum p (drifts from k)
    status: object     # torch.Tensor int32 [rows]


def dftopk_forward(scores, k: int, alpha: float, *, params: Params | None = None,
                   workspace=None) -> DFTopKResult:
    """The DFTopK relaxation of every row of `scores` (CUDA fp32): threshold at
    the midpoint of the k-th and (k+1)-th largest score, Laplace memberships
    at scale alpha around it, and their drifted mass (integer 1 <= k < n)."""
    torch = _torch()
    lib = _load()
    if int(k) != k:
        raise ValueError("k must be an integer for the DFTopK relaxation")
    x = _as_rows(scores, "scores")
    rows, n = x.shape
    dev = x.device
    p = _like_rows(x)
    b = torch.empty(rows, dtype=torch.float64, device=dev)
    sumf = torch.empty(rows, dtype=torch.float64, device=dev)
    mass = torch.empty(rows, dtype=torch.float64, device=dev)
    status = torch.empty(rows, dtype=torch.int32, device=dev)
    c, pptr = _params_ptr(params)
    need = int(lib.lapsum_topk_workspace_size(rows, n, pptr))
    ws = workspace if workspace is not None else _workspace(dev, need)
    stream = torch.cuda.current_stream(dev).cuda_stream
    rc = lib.lapsum_dftopk_fwd(x.data_ptr(), rows, n, x.stride(0), int(k), float(alpha), p.data_ptr(),
                               b.data_ptr(), sumf.data_ptr(), mass.data_ptr(), status.data_ptr(), None,
                               ws.data_ptr(), ws.numel(), pptr, stream)
    if rc != LAPSUM_OK:
        raise LapsumError(rc, "lapsum_dftopk_fwd")
    return DFTopKResult(p.view(scores.shape) if scores.dim() == 1 else p, b, sumf, mass, status)


@dataclass
class SparseResult:
    idx: object        # torch.Tensor int32 [rows, capacity]
    val: object        # torch.Tensor float32 [rows, capacity]
    count: object      # torch.Tensor int64 [rows]: entries with p >= eps (may exceed capacity)
    b: object          # torch.Tensor float64 [rows]
    sumf: object       # torch.Tensor float64 [rows]
    status: object     # torch.Tensor int32 [rows]

    def row(self, r: int):
        """(indices, p) of row r as tensors of its written entries."""
        c = min(int(self.count[r]), self.idx.shape[1])
        return self.idx[r, :c], self.val[r, :c]


def sparse_workspace_size(rows: int, n: int, params: Params | None = None) -> int:
    c, ptr = _params_ptr(params)
    return int(_load().lapsum_topk_sparse_workspace_size(int(rows), int(n), ptr))


def forward_sparse(scores, k: float, alpha: float, eps: float = 2.0 ** -24, *, capacity: int | None = None,
                   params: Params | None = None, workspace=None) -> SparseResult:
    """The entries with p >= eps of every row of `scores` (CUDA fp32) as
    (index, p) pairs; the threshold is that of forward().  With no capacity
    given, 2k + 4096 per row is tried first and, if a row has more entries,
    the call is repeated with the exact count (one host synchronisation)."""
    torch = _torch()
    lib = _load()
    x = _as_rows(scores, "scores")
    rows, n = x.shape
    dev = x.device
    guess = capacity is None
    cap = int(min(n, 2 * math.ceil(k) + 4096)) if guess else int(capacity)
    c, pptr = _params_ptr(params)
    need = int(lib.lapsum_topk_sparse_workspace_size(rows, n, pptr))
    ws = workspace if workspace is not None else _workspace(dev, need)
    stream = torch.cuda.current_stream(dev).cuda_stream
    while True:
        idx = torch.empty((rows, cap), dtype=torch.int32, device=dev)
        val = torch.empty((rows, cap), dtype=torch.float32, device=dev)
        cnt = torch.empty(rows, dtype=torch.int64, device=dev)
        b = torch.empty(rows, dtype=torch.float64, device=dev)
        sumf = torch.empty(rows, dtype=torch.float64, device=dev)
        status = torch.empty(rows, dtype=torch.int32, device=dev)
        rc = lib.lapsum_topk_fwd_sparse(x.data_ptr(), rows, n, x.stride(0), float(k), float(alpha), float(eps),
                                        idx.data_ptr(), val.data_ptr(), cap, cnt.data_ptr(), b.data_ptr(),
                                        sumf.data_ptr(), status.data_ptr(), None, ws.data_ptr(), ws.numel(),
                                        pptr, stream)
        if rc != LAPSUM_OK:
            raise LapsumError(rc, "lapsum_topk_fwd_sparse")
        if not guess:
            break
        top = int(cnt.max())
        if top <= cap:
            break
        cap, guess = top, False
    return SparseResult(idx, val, cnt, b, sumf, status)


def backward(scores, grad_p, b, alpha, *, workspace=None, grad_out=None, want_alpha: bool = False):
    """dL/dscores and dL/dk (per row) for upstream gradient `grad_p` at
    thresholds `b`; with want_alpha also dL/dalpha per row (a third result).
    alpha: a number, or a [rows] tensor (one per row)."""
    torch = _torch()
    lib = _load()
    x = _as_rows(scores, "scores")
    g = _as_rows(grad_p, "grad_p")
    rows, n = x.shape
    if g.shape != x.shape:
        raise ValueError("grad_p must have the shape of scores")
    if g.device != x.device:
        raise ValueError("grad_p must be on the device of scores")
    if b.numel() < rows:
        raise ValueError(f"b must hold one threshold per row ({rows})")
    if g.stride(0) != x.stride(0):  # the C ABI takes one row stride for all arrays
        x, g = x.contiguous(), g.contiguous()
    dev = x.device
    if grad_out is None:
        out = _like_rows(x)
    else:
        out = _rows_view(grad_out, "grad_out")
        _check_like(x, out, "grad_out")
    gk = torch.empty(rows, dtype=torch.float64, device=dev)
    ga = torch.empty(rows, dtype=torch.float64, device=dev) if want_alpha else None
    bb = b.to(device=dev, dtype=torch.float64).contiguous()
    need = int(lib.lapsum_topk_workspace_size(rows, n, None))
    ws = workspace if workspace is not None else _workspace(dev, need)
    stream = torch.cuda.current_stream(dev).cuda_stream
    ar = _per_row(alpha, rows, dev)
    if ar is None:
        rc = lib.lapsum_topk_bwd(x.data_ptr(), g.data_ptr(), bb.data_ptr(), rows, n, x.stride(0), float(alpha),
                                 out.data_ptr(), gk.data_ptr(), ga.data_ptr() if ga is not None else None,
                                 ws.data_ptr(), ws.numel(), stream)
    else:
        rc = lib.lapsum_topk_bwd_rows(x.data_ptr(), g.data_ptr(), bb.data_ptr(), rows, n, x.stride(0),
                                      ar.data_ptr(), out.data_ptr(), gk.data_ptr(),
                                      ga.data_ptr() if ga is not None else None, ws.data_ptr(), ws.numel(), stream)
    if rc != LAPSUM_OK:
        raise LapsumError(rc, "lapsum_topk_bwd" if ar is None else "lapsum_topk_bwd_rows")
    res = (out.view(scores.shape) if grad_out is None else grad_out), gk
    return res + (ga,) if want_alpha else res


def _into_args(scores, p, b, sumf, status, stats):
    """Checks of the preallocated forward outputs against the scores; returns
    the scores as a [rows, n] view."""
    torch = _torch()
    x = _rows_view(scores, "scores")
    rows = x.shape[0]
    pv = _rows_view(p, "p")
    _check_like(x, pv, "p")
    _check_vec(b, "b", rows, torch.float64, x.device)
    _check_vec(sumf, "sumf", rows, torch.float64, x.device, optional=True)
    _check_vec(status, "status", rows, torch.int32, x.device, optional=True)
    if stats is not None:
        _check_vec(stats, "stats", rows * STATS_DTYPE.itemsize, torch.uint8, x.device)
    return x, pv


def forward_into(scores, k: float, alpha: float, p, b, sumf, status, workspace, params: Params | None = None,
                 stats=None) -> None:
    """forward() with every output preallocated (no allocation in the call).
    p has the shape, device and row stride of scores; b (float64), sumf
    (float64) and status (int32) hold one value per row; stats, if given, is
    a uint8 buffer of rows * STATS_DTYPE.itemsize bytes."""
    torch = _torch()
    lib = _load()
    x, pv = _into_args(scores, p, b, sumf, status, stats)
    rows, n = x.shape
    _check_vec(workspace, "workspace", 1, torch.uint8, x.device)
    c, pptr = _params_ptr(params)
    rc = lib.lapsum_topk_fwd(x.data_ptr(), rows, n, x.stride(0), float(k), float(alpha), pv.data_ptr(), b.data_ptr(),
                             sumf.data_ptr() if sumf is not None else None,
                             status.data_ptr() if status is not None else None,
                             stats.data_ptr() if stats is not None else None, workspace.data_ptr(),
                             workspace.numel(), pptr, torch.cuda.current_stream(x.device).cuda_stream)
    if rc != LAPSUM_OK:
        raise LapsumError(rc, "lapsum_topk_fwd")


def forward_noalloc_into(scores, k: float, alpha: float, p, b, sumf=None, status=None,
                         params: Params | None = None, stats=None) -> None:
    """forward_into() without a workspace, for callers that cannot allocate
    device memory during the call (a fixed arena, a fully reserved pool, no
    implicit synchronisation allowed).  Rows of at most NOALLOC_MAX_N scores,
    at most NOALLOC_MAX_ROWS rows.  Its scratch is one static device array
    inside the library, shared by all calls on a device: calls that overlap on
    the GPU race, so serialise them.  The outputs are checked as in
    forward_into()."""
    torch = _torch()
    lib = _load()
    x, pv = _into_args(scores, p, b, sumf, status, stats)
    rows, n = x.shape
    c, pptr = _params_ptr(params)
    rc = lib.lapsum_topk_fwd_noalloc(x.data_ptr(), rows, n, x.stride(0), float(k), float(alpha), pv.data_ptr(),
                                     b.data_ptr(), sumf.data_ptr() if sumf is not None else None,
                                     status.data_ptr() if status is not None else None,
                                     stats.data_ptr() if stats is not None else None, pptr,
                                     torch.cuda.current_stream(x.device).cuda_stream)
    if rc != LAPSUM_OK:
        raise LapsumError(rc, "lapsum_topk_fwd_noalloc")


def backward_into(scores, grad_p, b, alpha: float, grad, workspace, grad_k=None, grad_alpha=None) -> None:
    """backward() with every output preallocated (no allocation in the call).
    grad_p and grad have the shape, device and row stride of scores; b,
    grad_k and grad_alpha are float64 with one value per row."""
    torch = _torch()
    lib = _load()
    x = _rows_view(scores, "scores")
    rows, n = x.shape
    gp = _rows_view(grad_p, "grad_p")
    _check_like(x, gp, "grad_p")
    gv = _rows_view(grad, "grad")
    _check_like(x, gv, "grad")
    _check_vec(b, "b", rows, torch.float64, x.device)
    _check_vec(grad_k, "grad_k", rows, torch.float64, x.device, optional=True)
    _check_vec(grad_alpha, "grad_alpha", rows, torch.float64, x.device, optional=True)
    _check_vec(workspace, "workspace", 1, torch.uint8, x.device)
    rc = lib.lapsum_topk_bwd(x.data_ptr(), gp.data_ptr(), b.data_ptr(), rows, n, x.stride(0), float(alpha),
                             gv.data_ptr(), grad_k.data_ptr() if grad_k is not None else None,
                             grad_alpha.data_ptr() if grad_alpha is not None else None,
                             workspace.data_ptr(), workspace.numel(),
                             torch.cuda.current_stream(x.device).cuda_stream)
    if rc != LAPSUM_OK:
        raise LapsumError(rc, "lapsum_topk_bwd")


class SoftTopK:
    """torch.autograd.Function wrapper: p = soft_topk(scores, k, alpha).  k
    and alpha may be Python numbers, 0-d tensors (shared by all rows) or
    [rows] tensors (one per row); tensors that require grad receive dL/dk
    (lambda per row, summed over the rows for a shared k) and dL/dalpha."""

    _fn = None

    @classmethod
    def fn(cls):
        if cls._fn is None:
            torch = _torch()

            class _F(torch.autograd.Function):
                @staticmethod
                def forward(ctx, scores, k, alpha, params):
                    rows = scores.shape[0] if scores.dim() == 2 else 1
                    kf = k if isinstance(k, torch.Tensor) and k.dim() == 1 else float(k)
                    af = alpha if isinstance(alpha, torch.Tensor) and alpha.dim() == 1 else float(alpha)
                    res = forward(scores, kf, af, params=params)
                    ctx.save_for_backward(scores, res.b)
                    ctx.alpha = af if not isinstance(af, torch.Tensor) else _per_row(af, rows, scores.device)
                    ctx.k_like = k if isinstance(k, torch.Tensor) else None
                    ctx.a_like = alpha if isinstance(alpha, torch.Tensor) else None
                    return res.p.view(scores.shape)

                @staticmethod
                def backward(ctx, gp):
                    scores, b = ctx.saved_tensors
                    sc = scores.contiguous()
                    need_k, need_a = ctx.needs_input_grad[1], ctx.needs_input_grad[2]
                    out = backward(sc, gp.contiguous().view(sc.shape), b, ctx.alpha, want_alpha=need_a)
                    gs, gk = out[0], out[1]

                    def fold(g, like):  # per row for a [rows] input, summed for a shared one
                        return (g if like.dim() == 1 else g.sum()).to(like.dtype).view(like.shape)

                    grad_k = fold(gk, ctx.k_like) if need_k else None
                    grad_a = fold(out[2], ctx.a_like) if need_a else None
                    return gs.view(scores.shape), grad_k, grad_a, None

            cls._fn = _F
        return cls._fn


def soft_topk(scores, k, alpha, params: Params | None = None):
    """Differentiable exact-budget soft top-k memberships of `scores` (CUDA fp32).
    k and alpha: numbers, 0-d tensors, or [rows] tensors (one per row); tensors
    receive their gradients."""
    torch = _torch()
    k = k if isinstance(k, torch.Tensor) else float(k)
    alpha = alpha if isinstance(alpha, torch.Tensor) else float(alpha)
    return SoftTopK.fn().apply(scores, k, alpha, params)
