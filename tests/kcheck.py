"""ctypes wrapper of tests/c/kcheck.c (built here with gcc and OpenMP): the
element-wise rotated-K check of the full-size parity tests, the rule of
test_gpu_parity.k_out_of_tolerance in C so that tens of millions of rows
per request are checked in well under a second."""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "c", "kcheck.c")
_LIB = os.path.join(_HERE, "c", "libkcheck.so")
_lib = None


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
            tmp = _LIB + f".tmp{os.getpid()}"
            subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", tmp, _SRC, "-lm"],
                           check=True)
            os.replace(tmp, _LIB)
        lib = ctypes.CDLL(_LIB)
        P, I64 = ctypes.c_void_p, ctypes.c_int64
        lib.kcheck.restype = I64
        lib.kcheck.argtypes = [P, P, P, I64, ctypes.c_double, ctypes.c_double,
                               ctypes.POINTER(I64), ctypes.POINTER(I64), ctypes.POINTER(I64)]
        _lib = lib
    return _lib


def kcheck(got_bits, ref, oracle_bits, rel=2.0 ** -8, abs_tol=1e-3):
    """(number outside the bar, index of the first, bit-identical count,
    compared count) over flattened arrays."""
    g = np.ascontiguousarray(got_bits, np.uint16).reshape(-1)
    r = np.ascontiguousarray(ref, np.float64).reshape(-1)
    o = np.ascontiguousarray(oracle_bits, np.uint16).reshape(-1)
    assert g.size == r.size == o.size
    first, exact, cmp = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    bad = _load().kcheck(g.ctypes.data, r.ctypes.data, o.ctypes.data, g.size, rel, abs_tol,
                         ctypes.byref(first), ctypes.byref(exact), ctypes.byref(cmp))
    return int(bad), int(first.value), int(exact.value), int(cmp.value)
