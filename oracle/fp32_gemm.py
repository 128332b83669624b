"""ctypes loader for the fixed-order fp32 GEMM oracle (fp32_gemm.c). TEST INFRASTRUCTURE ONLY.

``build()`` compiles ``fp32_gemm.c`` with gcc into ``oracle/_build/``; ``gemm_f32_fmaf``
builds it on first use if it is missing.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp32_gemm.c")
_LIB = os.path.join(_HERE, "_build", "liboracle_fp32_gemm.so")
_lib = None


def build() -> str:
    """Compile the C oracle (no fast-math, no contraction: fmaf is the only fused op)."""
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                           "-fno-fast-math", _SRC, "-o", _LIB, "-lm"])
    return _LIB


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
            build()
        lib = ctypes.CDLL(_LIB)
        lib.oracle_gemm_f32_fmaf.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64] * 3
        lib.oracle_gemm_f32_fmaf.restype = None
        _lib = lib
    return _lib


def gemm_f32_fmaf(X: np.ndarray, W: np.ndarray) -> np.ndarray:
    """Y = X·W in fp32, one accumulator per output, k ascending, fmaf steps."""
    X = np.ascontiguousarray(X, dtype=np.float32)
    W = np.ascontiguousarray(W, dtype=np.float32)
    n, d_in = X.shape
    d_in2, d_out = W.shape
    assert d_in == d_in2
    Y = np.empty((n, d_out), dtype=np.float32)
    _load().oracle_gemm_f32_fmaf(X.ctypes.data, W.ctypes.data, Y.ctypes.data, n, d_in, d_out)
    return Y
