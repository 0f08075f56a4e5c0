"""B200 Top-k sparsifier with error feedback and gTop-k merge.

Thin ctypes binding over the C ABI in ``include/topk_ef.h``
(``libtopk_ef.so``, built in-tree by ``python -m error_feedback_b200.build``).
The binding only marshals arguments: every step of the computation runs in
the library's CUDA kernels.  PyTorch supplies device memory and the current
stream.  There is no CPU fallback: if the library is missing or the tensors
are not on a CUDA device the calls raise.

Functions mirror the C names:

* ``topk_ef_compress(grad, residual, lr, k)``            -> (idx, val)
* ``topk_ef_compress_batched(grad, residual, offsets, k, lr)`` -> (idx, val)
* ``gtopk_merge(in_idx, in_val, k, n)``                  -> (idx, val, count)
* ``topk_ef_workspace_bytes``, ``topk_ef_batched_workspace_bytes``,
  ``gtopk_merge_workspace_bytes``, ``topk_ef_last_device_status``,
  ``topk_ef_path_info``, ``topk_ef_set_test_flags``.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtopk_ef.so")

OK = 0
ERR_INVALID_ARG = -1
ERR_WORKSPACE = -2
ERR_CUDA = -3
ERR_DEVICE_TIMEOUT = -4
ERR_BAD_INPUT = -5
ERR_INTERNAL = -6


class TopkEfError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {status_string(code)} ({code})")


_lib = None

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_sz = ctypes.c_size_t
_pi64 = ctypes.POINTER(ctypes.c_int64)


def lib() -> ctypes.CDLL:
    """The loaded C-ABI library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run `python -m error_feedback_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.topk_ef_workspace_bytes.argtypes = [_i64, _i64]
        L.topk_ef_workspace_bytes.restype = _sz
        L.topk_ef_compress.argtypes = [_vp, _vp, _i64, ctypes.c_float, _i64, _vp, _vp, _vp, _sz, _vp]
        L.topk_ef_compress.restype = ctypes.c_int
        L.topk_ef_compress_static.argtypes = [_vp, _vp, _i64, ctypes.c_float, _i64, _vp, _vp,
                                              _vp]
        L.topk_ef_compress_static.restype = ctypes.c_int
        L.topk_ef_static_last_device_status.argtypes = [_vp]
        L.topk_ef_static_last_device_status.restype = ctypes.c_int
        L.topk_ef_threshold_workspace_bytes.argtypes = [_i64]
        L.topk_ef_threshold_workspace_bytes.restype = _sz
        L.topk_ef_threshold.argtypes = [_vp, _vp, _i64, ctypes.c_float, ctypes.c_float, _i64,
                                        _vp, _vp, _vp, _vp, _sz, _vp]
        L.topk_ef_threshold.restype = ctypes.c_int
        L.gtopk_residual_return_workspace_bytes.argtypes = []
        L.gtopk_residual_return_workspace_bytes.restype = _sz
        L.gtopk_residual_return.argtypes = [_vp, _vp, _i32, _i64, _vp, _i64, _vp, _i64, _vp,
                                            _sz, _vp]
        L.gtopk_residual_return.restype = ctypes.c_int
        L.topk_allgather_workspace_bytes.argtypes = [_i32, _i64, _i64]
        L.topk_allgather_workspace_bytes.restype = _sz
        L.topk_allgather_sum.argtypes = [_vp, _vp, _i32, _i64, _i64, _vp, _vp, _sz, _vp]
        L.topk_allgather_sum.restype = ctypes.c_int
        L.topk_ef_batched_workspace_bytes.argtypes = [_pi64, _pi64, _i32]
        L.topk_ef_batched_workspace_bytes.restype = _sz
        L.topk_ef_compress_batched.argtypes = [_vp, _vp, _pi64, _pi64, _i32, ctypes.c_float, _vp, _vp,
                                               _vp, _sz, _vp]
        L.topk_ef_compress_batched.restype = ctypes.c_int
        L.gtopk_merge_workspace_bytes.argtypes = [_i32, _i64, _i64]
        L.gtopk_merge_workspace_bytes.restype = _sz
        L.gtopk_merge.argtypes = [_vp, _vp, _i32, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _sz, _vp]
        L.gtopk_merge.restype = ctypes.c_int
        L.topk_ef_last_device_status.argtypes = [_vp, _vp]
        L.topk_ef_last_device_status.restype = ctypes.c_int
        L.topk_ef_last_cuda_error.argtypes = []
        L.topk_ef_last_cuda_error.restype = ctypes.c_int
        L.topk_ef_status_string.argtypes = [ctypes.c_int]
        L.topk_ef_status_string.restype = ctypes.c_char_p
        L.topk_ef_path_info.argtypes = [_vp, _vp, _pi64]
        L.topk_ef_path_info.restype = ctypes.c_int
        L.topk_ef_phase_times.argtypes = [_vp, _vp, _pi64]
        L.topk_ef_phase_times.restype = ctypes.c_int
        L.topk_ef_set_test_flags.argtypes = [ctypes.c_int]
        L.topk_ef_set_test_flags.restype = ctypes.c_int
        L.topk_ef_trace_enable.argtypes = [ctypes.c_int]
        L.topk_ef_trace_enable.restype = ctypes.c_int
        L.topk_ef_trace_read.argtypes = [ctypes.POINTER(ctypes.c_float),
                                         ctypes.POINTER(ctypes.c_char_p), ctypes.c_int,
                                         ctypes.POINTER(ctypes.c_int)]
        L.topk_ef_trace_read.restype = ctypes.c_int
        L.topk_ef_trace_only.argtypes = [ctypes.c_char_p, ctypes.c_int]
        L.topk_ef_trace_only.restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().topk_ef_status_string(int(code)).decode()


def _check(rc: int, what: str) -> None:
    if rc != OK:
        if rc == ERR_CUDA:
            raise TopkEfError(rc, f"{what} (cudaError {lib().topk_ef_last_cuda_error()})")
        raise TopkEfError(rc, what)


def _stream(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _cuda_f32(t: torch.Tensor, name: str) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != torch.float32 or not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous float32")


def _host_i64(a) -> ctypes.Array:
    vals = [int(x) for x in a]
    return (ctypes.c_int64 * max(1, len(vals)))(*vals)


def _workspace(nbytes: int, device, ws):
    if ws is not None:
        if ws.numel() * ws.element_size() < nbytes:
            raise ValueError("workspace too small")
        return ws
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


# ------------------------------------------------------------------ compress

def topk_ef_workspace_bytes(n: int, k: int) -> int:
    return int(lib().topk_ef_workspace_bytes(int(n), int(k)))


def topk_ef_compress(grad, residual, lr, k, out_idx=None, out_val=None, ws=None, stream=None):
    """One EF step: acc = fmaf(lr, grad, residual); send the top-k of |acc|
    (ties to the lower index) in ascending index order; residual becomes acc
    with the sent slots zeroed.  Returns (idx int32[k], val float32[k])."""
    _cuda_f32(grad, "grad")
    _cuda_f32(residual, "residual")
    if grad.numel() != residual.numel():
        raise ValueError("grad and residual differ in size")
    n, k = grad.numel(), int(k)
    dev = grad.device
    if out_idx is None:
        out_idx = torch.empty(k, dtype=torch.int32, device=dev)
    if out_val is None:
        out_val = torch.empty(k, dtype=torch.float32, device=dev)
    nb = topk_ef_workspace_bytes(n, k)
    if nb == 0:
        raise TopkEfError(ERR_INVALID_ARG, "topk_ef_workspace_bytes")
    ws = _workspace(nb, dev, ws)
    rc = lib().topk_ef_compress(grad.data_ptr(), residual.data_ptr(), n, float(lr), k,
                                out_idx.data_ptr(), out_val.data_ptr(), ws.data_ptr(),
                                ws.numel() * ws.element_size(), _stream(stream))
    _check(rc, "topk_ef_compress")
    return out_idx, out_val


def topk_ef_compress_static(grad, residual, lr, k, out_idx=None, out_val=None, stream=None):
    """topk_ef_compress without a caller workspace: for callers that cannot
    allocate device memory.  Uses the library's fixed 32 MiB scratch array
    (shared by all calls; calls whose GPU work overlaps must not be issued)."""
    _cuda_f32(grad, "grad")
    _cuda_f32(residual, "residual")
    if grad.numel() != residual.numel():
        raise ValueError("grad and residual differ in size")
    n, k = grad.numel(), int(k)
    dev = grad.device
    if out_idx is None:
        out_idx = torch.empty(k, dtype=torch.int32, device=dev)
    if out_val is None:
        out_val = torch.empty(k, dtype=torch.float32, device=dev)
    rc = lib().topk_ef_compress_static(grad.data_ptr(), residual.data_ptr(), n, float(lr), k,
                                       out_idx.data_ptr(), out_val.data_ptr(), _stream(stream))
    _check(rc, "topk_ef_compress_static")
    return out_idx, out_val


def topk_ef_static_last_device_status(stream=None) -> int:
    """Device-side status of the last topk_ef_compress_static call on the
    current device (synchronises the stream)."""
    return int(lib().topk_ef_static_last_device_status(_stream(stream)))


def topk_ef_threshold_workspace_bytes(n: int) -> int:
    return int(lib().topk_ef_threshold_workspace_bytes(int(n)))


def topk_ef_threshold(grad, residual, lr, threshold, max_out, out_idx=None, out_val=None,
                      out_count=None, ws=None, stream=None):
    """Hard-threshold EF step: acc = fmaf(lr, grad, residual); the entries
    with |acc| >= |threshold| pass and the first max_out of them (ascending
    index) are sent, their residual zeroed.  Returns (idx int32[max_out],
    val float32[max_out], count int64[1] on the device); only the first
    min(count, max_out) slots of idx / val are written."""
    _cuda_f32(grad, "grad")
    _cuda_f32(residual, "residual")
    if grad.numel() != residual.numel():
        raise ValueError("grad and residual differ in size")
    n, max_out = grad.numel(), int(max_out)
    dev = grad.device
    if out_idx is None:
        out_idx = torch.empty(max(max_out, 1), dtype=torch.int32, device=dev)[:max_out]
    if out_val is None:
        out_val = torch.empty(max(max_out, 1), dtype=torch.float32, device=dev)[:max_out]
    if out_count is None:
        out_count = torch.empty(1, dtype=torch.int64, device=dev)
    nb = topk_ef_threshold_workspace_bytes(n)
    if nb == 0:
        raise TopkEfError(ERR_INVALID_ARG, "topk_ef_threshold_workspace_bytes")
    ws = _workspace(nb, dev, ws)
    rc = lib().topk_ef_threshold(grad.data_ptr(), residual.data_ptr(), n, float(lr),
                                 float(threshold), max_out, out_idx.data_ptr(),
                                 out_val.data_ptr(), out_count.data_ptr(), ws.data_ptr(),
                                 ws.numel() * ws.element_size(), _stream(stream))
    _check(rc, "topk_ef_threshold")
    return out_idx, out_val, out_count


def gtopk_residual_return_workspace_bytes() -> int:
    return int(lib().gtopk_residual_return_workspace_bytes())


def gtopk_residual_return(sent_idx, sent_val, global_idx, residual, ws=None, stream=None):
    """After gTop-k: for every worker p (row of sent_idx / sent_val) and sent
    (i, v) with i not in global_idx, residual[p, i] += v.  residual is a
    [P, n] float32 CUDA tensor, updated in place."""
    for t, name in ((sent_idx, "sent_idx"), (global_idx, "global_idx")):
        if not t.is_cuda or t.dtype != torch.int32 or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous int32 CUDA tensor")
    _cuda_f32(sent_val, "sent_val")
    _cuda_f32(residual, "residual")
    P, k_sent = sent_idx.shape
    if residual.dim() != 2 or residual.shape[0] != P or tuple(sent_val.shape) != (P, k_sent):
        raise ValueError("shapes: sent_idx/sent_val [P, k_sent], residual [P, n]")
    n = residual.shape[1]
    ws = _workspace(gtopk_residual_return_workspace_bytes(), residual.device, ws)
    rc = lib().gtopk_residual_return(sent_idx.data_ptr(), sent_val.data_ptr(), P, k_sent,
                                     global_idx.data_ptr(), global_idx.numel(),
                                     residual.data_ptr(), n, ws.data_ptr(),
                                     ws.numel() * ws.element_size(), _stream(stream))
    _check(rc, "gtopk_residual_return")
    return ws


def topk_allgather_workspace_bytes(P: int, k_in: int, n: int) -> int:
    return int(lib().topk_allgather_workspace_bytes(int(P), int(k_in), int(n)))


def topk_allgather_sum(in_idx, in_val, n, out=None, ws=None, stream=None):
    """Dense rank-order sum of the P sets (rows of in_idx / in_val) into a
    float32[n] CUDA tensor (the AllGather aggregation)."""
    if not in_idx.is_cuda or in_idx.dtype != torch.int32 or not in_idx.is_contiguous():
        raise TypeError("in_idx must be a contiguous int32 CUDA tensor")
    _cuda_f32(in_val, "in_val")
    P, k_in = in_idx.shape
    n = int(n)
    if out is None:
        out = torch.empty(max(n, 1), dtype=torch.float32, device=in_idx.device)[:n]
    nb = topk_allgather_workspace_bytes(P, k_in, n)
    if nb == 0:
        raise TopkEfError(ERR_INVALID_ARG, "topk_allgather_workspace_bytes")
    ws = _workspace(nb, in_idx.device, ws)
    rc = lib().topk_allgather_sum(in_idx.data_ptr(), in_val.data_ptr(), P, k_in, n,
                                  out.data_ptr(), ws.data_ptr(), ws.numel() * ws.element_size(),
                                  _stream(stream))
    _check(rc, "topk_allgather_sum")
    return out


def topk_ef_batched_workspace_bytes(offsets, k) -> int:
    T = len(k)
    return int(lib().topk_ef_batched_workspace_bytes(_host_i64(offsets), _host_i64(k), T))


def topk_ef_compress_batched(grad, residual, offsets, k, lr, out_idx=None, out_val=None,
                             ws=None, stream=None):
    """Per-tensor EF step over a flat bucket (tensor l = [offsets[l],
    offsets[l+1])).  Outputs are packed in tensor order with indices local to
    each tensor.  Returns (idx int32[sum k], val float32[sum k])."""
    _cuda_f32(grad, "grad")
    _cuda_f32(residual, "residual")
    offs = _host_i64(offsets)
    ks = _host_i64(k)
    T = len(k)
    total = int(sum(int(x) for x in k))
    dev = grad.device
    if out_idx is None:
        out_idx = torch.empty(total, dtype=torch.int32, device=dev)
    if out_val is None:
        out_val = torch.empty(total, dtype=torch.float32, device=dev)
    nb = int(lib().topk_ef_batched_workspace_bytes(offs, ks, T))
    if nb == 0:
        raise TopkEfError(ERR_INVALID_ARG, "topk_ef_batched_workspace_bytes")
    ws = _workspace(nb, dev, ws)
    rc = lib().topk_ef_compress_batched(grad.data_ptr(), residual.data_ptr(), offs, ks, T,
                                        float(lr), out_idx.data_ptr(), out_val.data_ptr(),
                                        ws.data_ptr(), ws.numel() * ws.element_size(),
                                        _stream(stream))
    _check(rc, "topk_ef_compress_batched")
    return out_idx, out_val


# --------------------------------------------------------------------- merge

def gtopk_merge_workspace_bytes(P: int, k_in: int, k: int) -> int:
    return int(lib().gtopk_merge_workspace_bytes(int(P), int(k_in), int(k)))


def gtopk_merge(in_idx, in_val, k, n, out_idx=None, out_val=None, out_count=None, ws=None,
                stream=None):
    """gTop-k tournament over the P rows of in_idx (int32, each strictly
    ascending) / in_val (float32).  Returns (idx int32[k], val float32[k],
    count int32[1]); entries past count are -1 / 0."""
    if in_idx.dtype != torch.int32 or not in_idx.is_cuda or not in_idx.is_contiguous():
        raise ValueError("in_idx must be a contiguous int32 CUDA tensor")
    _cuda_f32(in_val, "in_val")
    if in_idx.dim() != 2 or in_idx.shape != in_val.shape:
        raise ValueError("in_idx and in_val must both be [P, k_in]")
    P, k_in = in_idx.shape
    k = int(k)
    dev = in_idx.device
    if out_idx is None:
        out_idx = torch.empty(max(k, 1), dtype=torch.int32, device=dev)[:k]
    if out_val is None:
        out_val = torch.empty(max(k, 1), dtype=torch.float32, device=dev)[:k]
    if out_count is None:
        out_count = torch.empty(1, dtype=torch.int32, device=dev)
    nb = gtopk_merge_workspace_bytes(P, k_in, k)
    if nb == 0:
        raise TopkEfError(ERR_INVALID_ARG, "gtopk_merge_workspace_bytes")
    ws = _workspace(nb, dev, ws)
    rc = lib().gtopk_merge(in_idx.data_ptr(), in_val.data_ptr(), P, k_in, k, int(n),
                           out_idx.data_ptr(), out_val.data_ptr(), out_count.data_ptr(),
                           ws.data_ptr(), ws.numel() * ws.element_size(), _stream(stream))
    _check(rc, "gtopk_merge")
    return out_idx, out_val, out_count


# -------------------------------------------------------------------- status

def topk_ef_last_device_status(ws, stream=None) -> int:
    return int(lib().topk_ef_last_device_status(ws.data_ptr(), _stream(stream)))


def topk_ef_path_info(ws, stream=None) -> dict:
    info = (ctypes.c_int64 * 6)()
    _check(lib().topk_ef_path_info(ws.data_ptr(), _stream(stream), info), "topk_ef_path_info")
    return {"fallback": int(info[0]), "candidates": int(info[1]), "capacity": int(info[2]),
            "kernels": int(info[3]), "crowded_bin": int(info[4])}


def topk_ef_phase_times(ws, stream=None) -> list:
    """Diagnostic timestamps of the last compress call on ws (20 values, ns;
    -1: step not run): select kernel phases, the sampling block, then the
    streaming and select kernels' spans over all blocks."""
    ns = (ctypes.c_int64 * 20)()
    _check(lib().topk_ef_phase_times(ws.data_ptr(), _stream(stream), ns), "topk_ef_phase_times")
    return [int(x) for x in ns]


def topk_ef_set_test_flags(flags: int) -> int:
    return int(lib().topk_ef_set_test_flags(int(flags)))


def topk_ef_trace_enable(on: bool = True, only: str | None = None, every: int = 1) -> None:
    """Record CUDA events around every kernel the library launches, or only
    around the launches of kernel `only`, every `every`-th of them."""
    L = lib()
    _check(L.topk_ef_trace_only(only.encode() if only else None, int(every)),
           "topk_ef_trace_only")
    _check(L.topk_ef_trace_enable(1 if on else 0), "topk_ef_trace_enable")


def topk_ef_trace_read() -> list:
    """[(kernel name, milliseconds)] of the launches recorded since tracing
    was enabled or last read (waits for them to finish), and clears them."""
    ms = (ctypes.c_float * 4096)()
    names = (ctypes.c_char_p * 4096)()
    cnt = ctypes.c_int(0)
    _check(lib().topk_ef_trace_read(ms, names, 4096, ctypes.byref(cnt)), "topk_ef_trace_read")
    return [(names[i].decode(), float(ms[i])) for i in range(cnt.value)]
