"""fp64 CPU oracle for the exact-budget LapSum soft top-k.

TEST INFRASTRUCTURE ONLY: imported by tests/, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``.  The product path never imports
it.  It shares no code with the CUDA library; the two meet only in the seeded
input generators of ``differentiable_soft_top_b200.workloads``.

The arithmetic lives in ``lapsum_oracle.c`` (plain C, fp64).  This module
compiles it with gcc on first use (or when the source is newer than the
library) and wraps it with ctypes.

Parity status of each function (see the pin tests in tests/test_oracle_pins.py):
  threshold / forward / S    pinned: closed forms, brute force, bisection,
                             invariants, zero-temperature limit
  backward                   pinned: finite differences, invariants
  sample / bracket / tails   pinned: published splitmix64 vectors, Laplace
                             noise distribution, exact-S identity of the tails,
                             bracket coverage
  sample_ranks               pinned: exact binomial miss probability of the
                             ranks against Phi(-z) (Berry-Esseen band), and
                             the sampled bracket's miss rate per edge
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lapsum_oracle.c")
_LIB = os.path.join(_HERE, "liblapsum_oracle.so")
_lock = threading.Lock()
_lib = None

_i64 = ctypes.c_int64
_u64 = ctypes.c_uint64
_dbl = ctypes.c_double
_P = ctypes.c_void_p


def build(out: str = _LIB, mutant: int = 0, force: bool = False) -> str:
    """Compile the oracle into a shared library (gcc, -O2, IEEE semantics)."""
    if (not force and mutant == 0 and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(_SRC)):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=gnu11", "-fPIC", "-shared", "-fno-fast-math",
           f"-DLO_MUTANT={int(mutant)}", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def _bind(lib):
    sig = {
        "lo_threshold_f64": (ctypes.c_int, [_P, _i64, _dbl, _dbl, _P]),
        "lo_threshold_f32": (ctypes.c_int, [_P, _i64, _dbl, _dbl, _P]),
        "lo_forward_f64": (ctypes.c_int, [_P, _i64, _dbl, _dbl, _P, _P, _P]),
        "lo_forward_f32": (ctypes.c_int, [_P, _i64, _dbl, _dbl, _P, _P, _P]),
        "lo_backward_f64": (ctypes.c_int, [_P, _P, _i64, _dbl, _dbl, _P, _P, _P]),
        "lo_backward_f32": (ctypes.c_int, [_P, _P, _i64, _dbl, _dbl, _P, _P, _P]),
        "lo_backward_alpha_f64": (ctypes.c_int, [_P, _P, _i64, _dbl, _dbl, _P]),
        "lo_backward_alpha_f32": (ctypes.c_int, [_P, _P, _i64, _dbl, _dbl, _P]),
        "lo_S_f64": (_dbl, [_P, _i64, _dbl, _dbl]),
        "lo_S_f32": (_dbl, [_P, _i64, _dbl, _dbl]),
        "lo_sm64_mix": (_u64, [_u64]),
        "lo_sm64_out": (_u64, [_u64, _u64]),
        "lo_row_stream": (_u64, [_u64, _u64]),
        "lo_sample": (None, [_P, _i64, _dbl, _u64, _i64, _i64, _P, _P, _P]),
        "lo_sample_ranks": (None, [_i64, _dbl, _i64, _dbl, _P, _P]),
        "lo_bracket": (ctypes.c_int, [_P, _i64, _dbl, _dbl, _i64, _dbl, _u64, _i64, _P, _P, _P, _P]),
        "lo_tails": (None, [_P, _i64, ctypes.c_float, ctypes.c_float, _dbl, _P, _P, _P, _P, _P]),
        "lo_dftopk_threshold_f32": (ctypes.c_int, [_P, _i64, _i64, _P]),
        "lo_dftopk_forward_f32": (ctypes.c_int, [_P, _i64, _i64, _dbl, _P, _P, _P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def load(path: str | None = None):
    """Load (building if needed) the oracle library; returns the ctypes handle."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
    return _lib


class OracleError(RuntimeError):
    pass


_RC = {1: "EINVAL", 2: "EBADK", 3: "EBADALPHA", 4: "ENOMEM", 5: "ENONFINITE"}


def _check(rc):
    if rc != 0:
        raise OracleError(f"oracle error {_RC.get(rc, rc)}")


def _vec(x, dtype):
    a = np.ascontiguousarray(np.asarray(x, dtype=dtype).reshape(-1))
    return a, a.ctypes.data


class Oracle:
    """Thin numpy front end over one loaded oracle library."""

    def __init__(self, lib=None):
        self.lib = lib if lib is not None else load()

    # -- threshold / forward / backward ---------------------------------
    def threshold(self, r, k, alpha) -> float:
        r = np.asarray(r)
        out = _dbl()
        if r.dtype == np.float64:
            a, p = _vec(r, np.float64)
            _check(self.lib.lo_threshold_f64(p, a.size, float(k), float(alpha), ctypes.byref(out)))
        else:
            a, p = _vec(r, np.float32)
            _check(self.lib.lo_threshold_f32(p, a.size, float(k), float(alpha), ctypes.byref(out)))
        return out.value

    def forward(self, r, k, alpha):
        """Returns (p fp64 array, b, sum_f)."""
        r = np.asarray(r)
        b, sf = _dbl(), _dbl()
        n = r.size
        pout = np.empty(n, np.float64)
        if r.dtype == np.float64:
            a, ptr = _vec(r, np.float64)
            fn = self.lib.lo_forward_f64
        else:
            a, ptr = _vec(r, np.float32)
            fn = self.lib.lo_forward_f32
        _check(fn(ptr, n, float(k), float(alpha), pout.ctypes.data, ctypes.byref(b), ctypes.byref(sf)))
        return pout.reshape(r.shape), b.value, sf.value

    def backward(self, r, g, b, alpha):
        """Returns (grad fp64 array, lambda = dL/dk, sum_f)."""
        r = np.asarray(r)
        n = r.size
        gout = np.empty(n, np.float64)
        lam, sf = _dbl(), _dbl()
        if r.dtype == np.float64:
            a, pa = _vec(r, np.float64)
            c, pc = _vec(g, np.float64)
            fn = self.lib.lo_backward_f64
        else:
            a, pa = _vec(r, np.float32)
            c, pc = _vec(g, np.float32)
            fn = self.lib.lo_backward_f32
        _check(fn(pa, pc, n, float(b), float(alpha), gout.ctypes.data, ctypes.byref(lam), ctypes.byref(sf)))
        return gout.reshape(r.shape), lam.value, sf.value

    def backward_alpha(self, r, g, b, alpha) -> float:
        """dL/dalpha of L = sum g p at the threshold b (b moves with alpha)."""
        r = np.asarray(r)
        out = _dbl()
        if r.dtype == np.float64:
            a, pa = _vec(r, np.float64)
            c, pc = _vec(g, np.float64)
            fn = self.lib.lo_backward_alpha_f64
        else:
            a, pa = _vec(r, np.float32)
            c, pc = _vec(g, np.float32)
            fn = self.lib.lo_backward_alpha_f32
        _check(fn(pa, pc, a.size, float(b), float(alpha), ctypes.byref(out)))
        return out.value

    def S(self, r, b, alpha) -> float:
        r = np.asarray(r)
        if r.dtype == np.float64:
            a, p = _vec(r, np.float64)
            return self.lib.lo_S_f64(p, a.size, float(b), float(alpha))
        a, p = _vec(r, np.float32)
        return self.lib.lo_S_f32(p, a.size, float(b), float(alpha))

    # -- localization ----------------------------------------------------
    def sm64_out(self, s: int, i: int) -> int:
        return int(self.lib.lo_sm64_out(s & (2**64 - 1), i & (2**64 - 1)))

    def row_stream(self, seed: int, row: int) -> int:
        return int(self.lib.lo_row_stream(seed & (2**64 - 1), row))

    def sample(self, r, alpha, seed, row, m):
        a, p = _vec(r, np.float32)
        Y = np.empty(m, np.float32)
        idx = np.empty(m, np.int64)
        eps = np.empty(m, np.float64)
        self.lib.lo_sample(p, a.size, float(alpha), seed & (2**64 - 1), int(row), int(m),
                           Y.ctypes.data, idx.ctypes.data, eps.ctypes.data)
        return Y, idx, eps

    def sample_ranks(self, n, k, m, z):
        lo, hi = _i64(), _i64()
        self.lib.lo_sample_ranks(int(n), float(k), int(m), float(z), ctypes.byref(lo), ctypes.byref(hi))
        return lo.value, hi.value

    def bracket(self, r, k, alpha, m, z, seed, row=0):
        """Returns (a_L, a_R, c_lo, c_hi) as the localization step defines them."""
        a, p = _vec(r, np.float32)
        aL, aR = ctypes.c_float(), ctypes.c_float()
        lo, hi = _i64(), _i64()
        _check(self.lib.lo_bracket(p, a.size, float(k), float(alpha), int(m), float(z),
                                   seed & (2**64 - 1), int(row), ctypes.byref(aL), ctypes.byref(aR),
                                   ctypes.byref(lo), ctypes.byref(hi)))
        return aL.value, aR.value, lo.value, hi.value

    def tails(self, r, aL, aR, alpha):
        """Returns (n_L, S_L, n_R, S_R, M) for the bracket [aL, aR)."""
        a, p = _vec(r, np.float32)
        nL, nR, M = _i64(), _i64(), _i64()
        SL, SR = _dbl(), _dbl()
        self.lib.lo_tails(p, a.size, float(aL), float(aR), float(alpha), ctypes.byref(nL),
                          ctypes.byref(SL), ctypes.byref(nR), ctypes.byref(SR), ctypes.byref(M))
        return nL.value, SL.value, nR.value, SR.value, M.value

    def dftopk_forward(self, r, k: int, alpha: float):
        """DFTopK memberships (fp64), threshold (the midpoint) and mass sum p."""
        a, pa = _vec(r, np.float32)
        p = np.empty(a.size, np.float64)
        b, mass = _dbl(), _dbl()
        _check(self.lib.lo_dftopk_forward_f32(pa, a.size, int(k), float(alpha), p.ctypes.data, ctypes.byref(b),
                                              ctypes.byref(mass)))
        return p, b.value, mass.value

    def dftopk_threshold(self, r, k: int) -> float:
        a, p = _vec(r, np.float32)
        out = _dbl()
        _check(self.lib.lo_dftopk_threshold_f32(p, a.size, int(k), ctypes.byref(out)))
        return out.value


_default = None


def oracle() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default
