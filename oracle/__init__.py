"""CPU oracle for Top-k + error feedback and the gTop-k merge (ctypes binding).

TEST INFRASTRUCTURE ONLY.  The arithmetic lives in ``topk_ef_oracle.c``; this
module compiles it with gcc and marshals numpy arrays to it.  Only the tests,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package.  It shares no code with the CUDA library and the library never
calls it.

Every function states the passage it follows in the C source.  All arrays are
numpy; results are returned as new arrays (the residual argument is updated in
place, like the library's).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import tempfile

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "topk_ef_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

GCC_FLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
             "-fno-fast-math", "-Wall"]


def build(out_path: str | None = None, mutant: int = 0) -> str:
    """Compile the oracle (or one planted-mistake variant) with gcc."""
    out = out_path or _LIB
    cmd = ["gcc", *GCC_FLAGS]
    if mutant:
        cmd.append(f"-DORACLE_MUTANT={int(mutant)}")
    cmd += ["-o", out, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _needs_build(path: str) -> bool:
    return (not os.path.exists(path)
            or os.path.getmtime(path) < os.path.getmtime(_SRC))


_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")
_i64 = ctypes.c_int64


class Oracle:
    """Handle on one compiled oracle library (the real one or a mutant)."""

    def __init__(self, lib_path: str | None = None):
        path = lib_path or _LIB
        if lib_path is None and _needs_build(path):
            build(path)
        self.path = path
        lib = ctypes.CDLL(path)
        lib.oracle_accumulate.argtypes = [_f32p, _f32p, _i64, ctypes.c_float, _f32p]
        lib.oracle_accumulate.restype = None
        lib.oracle_select.argtypes = [_f32p, _i64, _i64, ctypes.c_int, _i32p]
        lib.oracle_select.restype = ctypes.c_int
        lib.oracle_compress.argtypes = [_f32p, _f32p, _i64, ctypes.c_float, _i64,
                                        ctypes.c_int, _i32p, _f32p]
        lib.oracle_compress.restype = ctypes.c_int
        lib.oracle_compress_batched.argtypes = [_f32p, _f32p, _i64p, _i64p,
                                                ctypes.c_int32, ctypes.c_float,
                                                ctypes.c_int, _i32p, _f32p]
        lib.oracle_compress_batched.restype = ctypes.c_int
        lib.oracle_gtopk_merge.argtypes = [_i32p, _f32p, ctypes.c_int32, _i64, _i64,
                                           _i64, _i32p, _f32p]
        lib.oracle_gtopk_merge.restype = ctypes.c_int64
        lib.oracle_threshold.argtypes = [_f32p, _f32p, _i64, ctypes.c_float, ctypes.c_float,
                                         _i64, _i32p, _f32p]
        lib.oracle_threshold.restype = ctypes.c_int64
        lib.oracle_residual_return.argtypes = [_i32p, _f32p, ctypes.c_int32, _i64, _i32p,
                                               _i64, _f32p, _i64]
        lib.oracle_residual_return.restype = ctypes.c_int
        lib.oracle_allgather_sum.argtypes = [_i32p, _f32p, ctypes.c_int32, _i64, _i64, _f32p]
        lib.oracle_allgather_sum.restype = ctypes.c_int
        self._lib = lib

    # --- memory update -------------------------------------------------
    def accumulate(self, grad, residual, lr):
        """acc = fmaf(lr, grad, residual) (one fp32 rounding)."""
        grad = np.ascontiguousarray(grad, dtype=np.float32)
        residual = np.ascontiguousarray(residual, dtype=np.float32)
        acc = np.empty_like(grad)
        self._lib.oracle_accumulate(grad, residual, grad.size, np.float32(lr), acc)
        return acc

    # --- selection -------------------------------------------------------
    def select(self, x, k, backend=0):
        """Ascending indices of the top-k of x by (|x| desc, index asc)."""
        x = np.ascontiguousarray(x, dtype=np.float32)
        out = np.empty(max(int(k), 1), dtype=np.int32)
        rc = self._lib.oracle_select(x, x.size, int(k), int(backend), out)
        if rc != 0:
            raise ValueError(f"oracle_select failed: {rc}")
        return out[:int(k)]

    # --- one error-feedback step ----------------------------------------
    def compress(self, grad, residual, lr, k, backend=0):
        """One EF step on a flat tensor; residual (float32 array) is updated
        in place.  Returns (idx int32[k], val float32[k])."""
        grad = np.ascontiguousarray(grad, dtype=np.float32)
        assert residual.dtype == np.float32 and residual.flags.c_contiguous
        k = int(k)
        oi = np.empty(max(k, 1), dtype=np.int32)
        ov = np.empty(max(k, 1), dtype=np.float32)
        rc = self._lib.oracle_compress(grad, residual, grad.size, np.float32(lr), k,
                                       int(backend), oi, ov)
        if rc != 0:
            raise ValueError(f"oracle_compress failed: {rc}")
        return oi[:k], ov[:k]

    def compress_batched(self, grad, residual, offsets, ks, lr, backend=0):
        """Per-tensor EF step over a flat bucket; local indices, packed
        outputs (tensor l's block starts at sum of earlier k)."""
        grad = np.ascontiguousarray(grad, dtype=np.float32)
        assert residual.dtype == np.float32 and residual.flags.c_contiguous
        offsets = np.ascontiguousarray(offsets, dtype=np.int64)
        ks = np.ascontiguousarray(ks, dtype=np.int64)
        total = int(ks.sum())
        oi = np.empty(max(total, 1), dtype=np.int32)
        ov = np.empty(max(total, 1), dtype=np.float32)
        rc = self._lib.oracle_compress_batched(grad, residual, offsets, ks, len(ks),
                                               np.float32(lr), int(backend), oi, ov)
        if rc != 0:
            raise ValueError(f"oracle_compress_batched failed: {rc}")
        return oi[:total], ov[:total]

    # --- gTop-k merge ----------------------------------------------------
    def gtopk_merge(self, in_idx, in_val, k, n):
        """Tournament merge of P index-sorted sets (rows of in_idx/in_val).
        Returns (idx, val) of the result, ascending index."""
        in_idx = np.ascontiguousarray(in_idx, dtype=np.int32)
        in_val = np.ascontiguousarray(in_val, dtype=np.float32)
        P, k_in = in_idx.shape
        k = int(k)
        oi = np.empty(max(k, 1), dtype=np.int32)
        ov = np.empty(max(k, 1), dtype=np.float32)
        flat_i = in_idx.reshape(-1) if in_idx.size else np.zeros(1, np.int32)
        flat_v = in_val.reshape(-1) if in_val.size else np.zeros(1, np.float32)
        m = self._lib.oracle_gtopk_merge(flat_i, flat_v, P, k_in, k, int(n), oi, ov)
        if m < 0:
            raise ValueError(f"oracle_gtopk_merge failed: {m}")
        return oi[:m], ov[:m]


    # --- hard threshold ----------------------------------------------------
    def threshold(self, grad, residual, lr, threshold, max_out):
        """Hard-threshold EF step: sends the first max_out (ascending index)
        of the entries with |acc| >= |threshold|; residual updated in place.
        Returns (idx, val, count) with count = all entries that passed."""
        grad = np.ascontiguousarray(grad, dtype=np.float32)
        assert residual.dtype == np.float32 and residual.flags.c_contiguous
        max_out = int(max_out)
        oi = np.empty(max(max_out, 1), dtype=np.int32)
        ov = np.empty(max(max_out, 1), dtype=np.float32)
        c = self._lib.oracle_threshold(grad, residual, grad.size, np.float32(lr),
                                       np.float32(threshold), max_out, oi, ov)
        if c < 0:
            raise ValueError(f"oracle_threshold failed: {c}")
        m = min(int(c), max_out)
        return oi[:m], ov[:m], int(c)

    # --- residual return after gTop-k ------------------------------------
    def residual_return(self, sent_idx, sent_val, global_idx, residual):
        """Adds back, per worker p (row of sent_*), the sent values whose
        index is not in global_idx; residual is [P][n], updated in place."""
        sent_idx = np.ascontiguousarray(sent_idx, dtype=np.int32)
        sent_val = np.ascontiguousarray(sent_val, dtype=np.float32)
        global_idx = np.ascontiguousarray(global_idx, dtype=np.int32)
        assert residual.dtype == np.float32 and residual.flags.c_contiguous
        P, k_sent = sent_idx.shape
        n = residual.shape[-1]
        si = sent_idx.reshape(-1) if sent_idx.size else np.zeros(1, np.int32)
        sv = sent_val.reshape(-1) if sent_val.size else np.zeros(1, np.float32)
        gi = global_idx if global_idx.size else np.zeros(1, np.int32)
        rc = self._lib.oracle_residual_return(si, sv, P, k_sent, gi, global_idx.size,
                                              residual.reshape(-1), n)
        if rc != 0:
            raise ValueError(f"oracle_residual_return failed: {rc}")

    # --- AllGather aggregation ---------------------------------------------
    def allgather_sum(self, in_idx, in_val, n):
        """Dense sum of the P sets (rows), added in rank order from +0."""
        in_idx = np.ascontiguousarray(in_idx, dtype=np.int32)
        in_val = np.ascontiguousarray(in_val, dtype=np.float32)
        P, k_in = in_idx.shape
        out = np.empty(max(int(n), 1), dtype=np.float32)
        fi = in_idx.reshape(-1) if in_idx.size else np.zeros(1, np.int32)
        fv = in_val.reshape(-1) if in_val.size else np.zeros(1, np.float32)
        rc = self._lib.oracle_allgather_sum(fi, fv, P, k_in, int(n), out)
        if rc != 0:
            raise ValueError(f"oracle_allgather_sum failed: {rc}")
        return out[:int(n)]


_default: Oracle | None = None


def get() -> Oracle:
    """The oracle built from the unmodified source (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def mutant(n: int, workdir: str | None = None) -> Oracle:
    """A build of the oracle with planted mistake number n (tests only)."""
    d = workdir or tempfile.mkdtemp(prefix="oracle_mutant_")
    path = os.path.join(d, f"liboracle_m{n}.so")
    build(path, mutant=n)
    return Oracle(path)
