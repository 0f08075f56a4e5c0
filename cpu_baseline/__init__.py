"""Multi-threaded CPU Top-k + error-feedback step (OpenMP), the host-core
baseline that ``bench.py`` reports beside the GPU numbers.

The C source ``cpu_topk_ef.c`` is compiled with gcc -fopenmp on first use (or
by ``__graft_entry__.build()``).  It shares no code with the CUDA library or
the oracle; a CPU test checks it against the oracle bit for bit.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "cpu_topk_ef.c")
_LIB = os.path.join(_HERE, "libcpu_topk_ef.so")
GCC_FLAGS = ["-O3", "-std=c11", "-fPIC", "-shared", "-fopenmp",
             "-ffp-contract=off", "-fno-fast-math", "-Wall"]

_lib = None


def build() -> str:
    subprocess.run(["gcc", *GCC_FLAGS, "-o", _LIB, _SRC, "-lm"], check=True)
    return _LIB


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
            build()
        L = ctypes.CDLL(_LIB)
        f32 = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
        i32 = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
        L.cpu_topk_ef.argtypes = [f32, f32, ctypes.c_int64, ctypes.c_float, ctypes.c_int64,
                                  i32, f32, ctypes.c_int]
        L.cpu_topk_ef.restype = ctypes.c_int
        _lib = L
    return _lib


def threads() -> int:
    return os.cpu_count() or 1


def compress(grad: np.ndarray, residual: np.ndarray, lr, k: int, nthreads: int = 0):
    """One EF step on the host cores; residual (float32) is updated in place.
    Returns (idx int32[k], val float32[k]) in ascending index order."""
    k = int(k)
    oi = np.empty(max(k, 1), np.int32)
    ov = np.empty(max(k, 1), np.float32)
    rc = lib().cpu_topk_ef(grad, residual, grad.size, float(np.float32(lr)), k, oi, ov,
                           int(nthreads))
    if rc != 0:
        raise ValueError("cpu_topk_ef: bad arguments or out of memory")
    return oi[:k], ov[:k]
