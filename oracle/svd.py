"""Full SVD of the oracle: one-sided Jacobi in float64 (C helper _jacobi.c).

Test infrastructure only.  The shared library is built from _jacobi.c with
plain `gcc -O2` (no fast-math) on first use, next to this file.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "_jacobi.c")
_LIB = os.path.join(_HERE, "_jacobi.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the Jacobi helper if it is missing or older than its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.oracle_jacobi_svd.restype = ctypes.c_int
        _lib.oracle_jacobi_svd.argtypes = [ctypes.c_int, ctypes.c_int,
                                           ctypes.c_void_p, ctypes.c_void_p,
                                           ctypes.c_double, ctypes.c_int]
    return _lib


class NoConvergence(RuntimeError):
    pass


def jacobi_svd(A: np.ndarray, tol: float = 1e-15, max_sweeps: int = 60):
    """A (m x n, float64) = U diag(s) Vt, singular values sorted descending.

    Thin SVD: U is m x p, s has p entries, Vt is p x n, p = min(m, n).  The
    rotations run on A or A^T, whichever has fewer columns.
    """
    A = np.asarray(A, dtype=np.float64)
    m, n = A.shape
    transpose = n > m
    B = A.T if transpose else A
    mm, nn = B.shape                       # nn <= mm
    work = np.array(B, dtype=np.float64, order="F", copy=True)   # column-major
    V = np.zeros((nn, nn), dtype=np.float64, order="F")
    if nn > 0 and mm > 0:
        sweeps = _load().oracle_jacobi_svd(mm, nn, work.ctypes.data, V.ctypes.data, tol, max_sweeps)
        if sweeps < 0:
            raise NoConvergence(f"Jacobi SVD did not converge in {max_sweeps} sweeps")
    s = np.sqrt((work * work).sum(axis=0))
    order = np.argsort(-s, kind="stable")
    s = s[order]
    US = work[:, order]
    V = V[:, order]
    U = np.zeros_like(US)
    nz = s > 0
    U[:, nz] = US[:, nz] / s[nz]
    # B = U diag(s) V^T
    if transpose:                          # A = B^T = V diag(s) U^T
        return np.ascontiguousarray(V), s, np.ascontiguousarray(U.T)
    return np.ascontiguousarray(U), s, np.ascontiguousarray(V.T)


def lapack_svd(A: np.ndarray):
    """Thin SVD of A by LAPACK (numpy.linalg.svd, a library routine), in the
    same form as jacobi_svd.  For layers too large for the Jacobi sweeps to
    finish in minutes (the benchmark's reference arm and error report); the
    two agree on the truncated product L1 L2 up to rounding (pinned)."""
    A = np.asarray(A, dtype=np.float64)
    U, s, Vt = np.linalg.svd(A, full_matrices=False)
    return U, s, Vt
