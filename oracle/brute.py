"""ctypes loader for the plain-C float64 brute force in ``brute.c``.

TEST INFRASTRUCTURE ONLY.  ``build()`` compiles ``_brute.so`` next to the
source with gcc; ``load()`` compiles on demand if the library is missing.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "brute.c")
_LIB = os.path.join(_HERE, "_brute.so")
_lib = None


def build() -> str:
    """Compile brute.c into oracle/_brute.so (plain C, -O2, no fast-math)."""
    if (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", _SRC, "-o", _LIB, "-lm"])
    return _LIB


def load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        u8p = ctypes.POINTER(ctypes.c_ubyte)
        lib.brute_calibrate.argtypes = [ctypes.c_int, ctypes.c_int, dp, dp, dp, u8p, ctypes.c_double, dp, dp, dp]
        lib.brute_calibrate.restype = ctypes.c_int
        lib.brute_sparse_step.argtypes = [ctypes.c_int, ctypes.c_int, dp, dp, dp, u8p, ctypes.c_double, dp, dp, dp]
        lib.brute_sparse_step.restype = ctypes.c_int
        _lib = lib
    return _lib


def _dp(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def calibrate(q, k, v, keep, scale):
    """One head: q, k, v float64 [L, d]; keep bool [L, L]. Returns (O, rho, R)."""
    L, d = q.shape
    q, k, v = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v))
    keep = np.ascontiguousarray(keep, dtype=np.uint8)
    o = np.zeros((L, d)); r = np.zeros((L, d)); rho = np.zeros(L)
    rc = load().brute_calibrate(L, d, _dp(q), _dp(k), _dp(v),
                                keep.ctypes.data_as(ctypes.POINTER(ctypes.c_ubyte)),
                                float(scale), _dp(o), _dp(rho), _dp(r))
    if rc != 0:
        raise RuntimeError(f"brute_calibrate failed ({rc})")
    return o, rho, r


def sparse_step(q, k, v, keep, scale, rho_hat, r):
    """One head: reshaped sparse step with a given rho_hat [L] and residual R [L, d]."""
    L, d = q.shape
    q, k, v, r = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v, r))
    rho_hat = np.ascontiguousarray(rho_hat, dtype=np.float64)
    keep = np.ascontiguousarray(keep, dtype=np.uint8)
    o = np.zeros((L, d))
    rc = load().brute_sparse_step(L, d, _dp(q), _dp(k), _dp(v),
                                  keep.ctypes.data_as(ctypes.POINTER(ctypes.c_ubyte)),
                                  float(scale), _dp(rho_hat), _dp(r), _dp(o))
    if rc != 0:
        raise RuntimeError(f"brute_sparse_step failed ({rc})")
    return o
