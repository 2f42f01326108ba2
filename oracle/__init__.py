"""fp64 CPU oracle for the LUT binary GEMV (ctypes wrapper around oracle.c).

TEST INFRASTRUCTURE ONLY: only tests/, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The library (``lut_binary_gemv_b200``) never imports it, and it
imports nothing from the library.

Every function takes the interchange arrays of ``workloads.Problem`` (see
``workloads/__init__.py``) and returns float64 numpy arrays.  What each C entry
point computes, and which passage of the FluxBin page it follows, is stated at
the top of ``oracle.c``.

Parity status: every function here is pinned by ``tests/test_oracle.py``
(closed forms, exact special cases, invariants, brute force); none is
"parity unpinned".
"""

from __future__ import annotations

import ctypes as C
import os
from typing import Optional, Tuple

import numpy as np

from . import build as _build

_DT = {"f32": 0, "f16": 1, "bf16": 2}


class _Weights(C.Structure):
    _fields_ = [
        ("M", C.c_int64), ("N", C.c_int64), ("K", C.c_int32), ("Ks", C.c_int32),
        ("nS", C.c_int64),
        ("sign_bits", C.c_void_p), ("alpha_r", C.c_void_p), ("alpha_c", C.c_void_p),
        ("s_idx", C.c_void_p), ("s_sign_bits", C.c_void_p), ("s_row_bytes", C.c_int64),
        ("s_alpha_r", C.c_void_p), ("s_alpha_c", C.c_void_p),
    ]


_lib = None


def lib():
    global _lib
    if _lib is None:
        # FB_ORACLE_LIB lets the mutation test load a deliberately broken copy
        # of the oracle, built from a modified oracle.c, to show the pins fail.
        path = os.environ.get("FB_ORACLE_LIB") or _build.build()
        L = C.CDLL(path)
        P = C.c_void_p
        L.oracle_num_threads.restype = C.c_int
        L.oracle_set_num_threads.argtypes = [C.c_int]
        L.oracle_set_num_threads.restype = None
        L.oracle_x_to_f64.argtypes = [C.c_int, P, C.c_int64, P]
        L.oracle_dequant_rows.argtypes = [C.POINTER(_Weights), C.c_int64, P, P]
        L.oracle_gemv.argtypes = [C.POINTER(_Weights), P, C.c_int, C.c_int64, P, P, P, P]
        L.oracle_lut_tables.argtypes = [C.c_int64, C.c_int, C.c_int, P, P, P]
        L.oracle_vcm_gather.argtypes = [P, C.c_int64, P, C.c_int64, C.c_int64, P]
        L.oracle_gemv_lut.argtypes = [C.POINTER(_Weights), C.c_int, P, C.c_int, C.c_int64, P, P]
        for f in ("oracle_x_to_f64", "oracle_dequant_rows", "oracle_gemv",
                  "oracle_lut_tables", "oracle_vcm_gather", "oracle_gemv_lut"):
            getattr(L, f).restype = C.c_int
        _lib = L
    return _lib


def num_threads() -> int:
    return lib().oracle_num_threads()


def set_num_threads(n: int) -> None:
    """Threads the oracle's parallel loops use (timing aid; results do not
    depend on it)."""
    lib().oracle_set_num_threads(int(n))


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"{what} failed with code {rc}")


class OracleWeights:
    """Holds contiguous copies of a problem's weight arrays for the C code."""

    def __init__(self, M, N, K, sign_bits, alpha_r, alpha_c=None, s_idx=None,
                 s_sign_bits=None, s_alpha_r=None, s_alpha_c=None, Ks=0):
        self.arrays = dict(
            sign_bits=np.ascontiguousarray(sign_bits, np.uint8),
            alpha_r=np.ascontiguousarray(alpha_r, np.float32),
            alpha_c=None if alpha_c is None else np.ascontiguousarray(alpha_c, np.float32),
        )
        nS = 0 if s_idx is None else len(s_idx)
        if nS:
            self.arrays.update(
                s_idx=np.ascontiguousarray(s_idx, np.uint32),
                s_sign_bits=np.ascontiguousarray(s_sign_bits, np.uint8),
                s_alpha_r=np.ascontiguousarray(s_alpha_r, np.float32),
                s_alpha_c=np.ascontiguousarray(s_alpha_c, np.float32),
            )
        a = self.arrays
        self.M, self.N, self.K = M, N, K
        self.s = _Weights(
            M=M, N=N, K=K, Ks=Ks if nS else 0, nS=nS,
            sign_bits=_ptr(a["sign_bits"]), alpha_r=_ptr(a["alpha_r"]),
            alpha_c=_ptr(a["alpha_c"]),
            s_idx=_ptr(a.get("s_idx")), s_sign_bits=_ptr(a.get("s_sign_bits")),
            s_row_bytes=a["s_sign_bits"].shape[-1] if nS else 0,
            s_alpha_r=_ptr(a.get("s_alpha_r")), s_alpha_c=_ptr(a.get("s_alpha_c")),
        )

    @classmethod
    def from_problem(cls, p) -> "OracleWeights":
        return cls(p.M, p.N, p.K, p.sign_bits, p.alpha_r, p.alpha_c,
                   p.s_idx if p.nS else None, p.s_sign_bits, p.s_alpha_r,
                   p.s_alpha_c, p.Ks)


def x_to_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    x = np.ascontiguousarray(x)
    out = np.empty(x.shape, np.float64)
    _check(lib().oracle_x_to_f64(_DT[dtype], x.ctypes.data, x.size, out.ctypes.data), "x_to_f64")
    return out


def _rows(rows, M):
    if rows is None:
        return M, None
    r = np.ascontiguousarray(rows, np.int64)
    return len(r), r


def dequant(w: OracleWeights, rows=None) -> np.ndarray:
    n, r = _rows(rows, w.M)
    out = np.empty((n, w.N), np.float64)
    _check(lib().oracle_dequant_rows(C.byref(w.s), n, _ptr(r), out.ctypes.data), "dequant")
    return out


def gemv(w: OracleWeights, x64: np.ndarray, rows=None) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Dense formulation. x64: float64 [batch][N]. Returns (y, d, e), each
    [batch][nrows]."""
    x64 = np.ascontiguousarray(np.atleast_2d(x64), np.float64)
    n, r = _rows(rows, w.M)
    B = x64.shape[0]
    y = np.empty((B, n)); d = np.empty((B, n)); e = np.empty((B, n))
    _check(lib().oracle_gemv(C.byref(w.s), x64.ctypes.data, B, n, _ptr(r), y.ctypes.data,
                             d.ctypes.data, e.ctypes.data), "gemv")
    return y, d, e


def gemv_lut(w: OracleWeights, g: int, x64: np.ndarray, rows=None) -> np.ndarray:
    """LUT formulation with group width g. Returns y [batch][nrows]."""
    x64 = np.ascontiguousarray(np.atleast_2d(x64), np.float64)
    n, r = _rows(rows, w.M)
    B = x64.shape[0]
    y = np.empty((B, n))
    _check(lib().oracle_gemv_lut(C.byref(w.s), g, x64.ctypes.data, B, n, _ptr(r), y.ctypes.data),
           "gemv_lut")
    return y


def lut_tables(x64: np.ndarray, alpha_c: Optional[np.ndarray], K: int, g: int) -> np.ndarray:
    """T[k][q][p] for one activation vector x64 [N]."""
    x64 = np.ascontiguousarray(x64, np.float64)
    N = x64.shape[-1]
    ac = None if alpha_c is None else np.ascontiguousarray(alpha_c, np.float32)
    T = np.empty((K, N // g, 1 << g), np.float64)
    _check(lib().oracle_lut_tables(N, K, g, x64.ctypes.data, _ptr(ac), T.ctypes.data), "lut_tables")
    return T


def vcm_gather(x64: np.ndarray, s_idx: np.ndarray, nS_pad: int) -> np.ndarray:
    x64 = np.ascontiguousarray(x64, np.float64)
    s = np.ascontiguousarray(s_idx, np.uint32)
    out = np.empty(nS_pad, np.float64)
    _check(lib().oracle_vcm_gather(x64.ctypes.data, x64.shape[-1], _ptr(s) if len(s) else None,
                                   len(s), nS_pad, out.ctypes.data), "vcm_gather")
    return out


def problem_reference(p, rows=None):
    """(y, d, e) of the dense formulation for a workloads.Problem."""
    w = OracleWeights.from_problem(p)
    return gemv(w, x_to_f64(p.x, p.x_dtype), rows)
