"""Builds and calls the C loop in scan_seq.c (oracle; test infrastructure only)."""
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "scan_seq.c")
_LIB = os.path.join(_HERE, "_scan_seq.so")
_lib = None


def build(force=False):
    """Compile scan_seq.c with gcc into oracle/_scan_seq.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        f = _lib.oracle_selective_scan
        f.restype = None
        f.argtypes = [ctypes.c_void_p] * 10 + [ctypes.c_long] * 4
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def scan(x, dt, A, Bm, Cm, D, z=None, h0=None):
    lib = _load()
    c = lambda a: None if a is None else np.ascontiguousarray(a, dtype=np.float64)
    x, dt, A, Bm, Cm, D, z, h0 = map(c, (x, dt, A, Bm, Cm, D, z, h0))
    nb, L, C = x.shape
    N = A.shape[1]
    y = np.empty((nb, L, C))
    h = np.empty((nb, C, N))
    lib.oracle_selective_scan(_p(x), _p(dt), _p(A), _p(Bm), _p(Cm), _p(D), _p(z),
                              _p(h0), _p(y), _p(h), nb, L, C, N)
    return y, h
