"""The C-ABI library on a machine without a GPU: it loads, exports every
function the header declares, and its host-only entry points (workspace
sizes, argument checks, status strings) behave as documented."""
import ctypes
import os
import re

import pytest

import error_feedback_b200 as ef
from error_feedback_b200 import build as efbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "topk_ef.h")


@pytest.fixture(scope="module")
def lib():
    efbuild.build()
    return ef.lib()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", text)) - {"defined"})


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert "topk_ef_compress" in names and "gtopk_merge" in names
    for name in names:
        assert hasattr(lib, name), name
    out = os.popen(f"nm -D --defined-only {ef.LIB_PATH}").read()
    for name in names:
        assert re.search(rf"\bT {name}\b", out), name


def test_workspace_sizes(lib):
    assert ef.topk_ef_workspace_bytes(0, 0) > 0
    assert ef.topk_ef_workspace_bytes(10, 11) == 0
    assert ef.topk_ef_workspace_bytes(-1, 0) == 0
    assert ef.topk_ef_workspace_bytes(2**31, 1) == 0
    a = ef.topk_ef_workspace_bytes(25_557_032, 25_557)
    b = ef.topk_ef_workspace_bytes(25_557_032, 255_570)
    assert 0 < a < b < 64 << 20
    assert ef.topk_ef_batched_workspace_bytes([0, 5, 3], [1, 1]) == 0      # decreasing
    assert ef.topk_ef_batched_workspace_bytes([1, 5], [1]) == 0            # offsets[0] != 0
    assert ef.topk_ef_batched_workspace_bytes([0, 5, 9], [1, 5]) == 0      # k > n
    assert ef.topk_ef_batched_workspace_bytes([0, 5, 9], [1, 4]) > 0
    assert ef.gtopk_merge_workspace_bytes(0, 1, 1) == 0
    assert ef.gtopk_merge_workspace_bytes(32, 25_557, 25_557) > 0


def test_argument_errors_need_no_gpu(lib):
    L = lib
    ws = ctypes.create_string_buffer(1 << 16)
    wsp = (ctypes.addressof(ws) + 255) // 256 * 256
    # k > n, n < 0, n too large: rejected before any CUDA call
    assert L.topk_ef_compress(None, None, 10, ctypes.c_float(0.1), 11, None, None, wsp, 1 << 15, None) == ef.ERR_INVALID_ARG
    assert L.topk_ef_compress(None, None, -1, ctypes.c_float(0.1), 0, None, None, wsp, 1 << 15, None) == ef.ERR_INVALID_ARG
    assert L.topk_ef_compress(None, None, 2**31, ctypes.c_float(0.1), 0, None, None, wsp, 1 << 15, None) == ef.ERR_INVALID_ARG
    # null grad with n > 0
    assert L.topk_ef_compress(None, None, 10, ctypes.c_float(0.1), 1, 16, 16, wsp, 1 << 15, None) == ef.ERR_INVALID_ARG
    # misaligned fp32 pointer
    assert L.topk_ef_compress(17, 32, 10, ctypes.c_float(0.1), 1, 16, 16, wsp, 1 << 15, None) == ef.ERR_INVALID_ARG
    # workspace too small (pointers are never dereferenced on this path)
    assert L.topk_ef_compress(16, 32, 10, ctypes.c_float(0.1), 1, 64, 128, wsp, 16, None) == ef.ERR_WORKSPACE
    # misaligned workspace
    assert L.topk_ef_compress(16, 32, 10, ctypes.c_float(0.1), 1, 64, 128, wsp + 8, 1 << 15, None) == ef.ERR_INVALID_ARG
    # merge: P < 1, k_in > n, null out_count
    assert L.gtopk_merge(16, 32, 0, 1, 1, 10, 64, 128, 256, wsp, 1 << 15, None) == ef.ERR_INVALID_ARG
    assert L.gtopk_merge(16, 32, 2, 11, 1, 10, 64, 128, 256, wsp, 1 << 15, None) == ef.ERR_INVALID_ARG
    assert L.gtopk_merge(16, 32, 2, 1, 1, 10, 64, 128, None, wsp, 1 << 15, None) == ef.ERR_INVALID_ARG
    assert L.gtopk_merge(16, 32, 2, 1, 1, 10, 64, 128, 256, wsp, 8, None) == ef.ERR_WORKSPACE
    # batched: T < 1
    off = (ctypes.c_int64 * 2)(0, 4)
    kk = (ctypes.c_int64 * 1)(1)
    assert L.topk_ef_compress_batched(16, 32, off, kk, 0, ctypes.c_float(0.1), 64, 128, wsp, 1 << 15, None) == ef.ERR_INVALID_ARG


def test_status_strings_and_flags(lib):
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert ef.status_string(code) != "unknown status"
    assert ef.status_string(-99) == "unknown status"
    old = ef.topk_ef_set_test_flags(3)
    assert ef.topk_ef_set_test_flags(old) == 3


def test_binding_rejects_cpu_tensors(lib):
    import torch
    g = torch.zeros(8)
    with pytest.raises(ValueError):
        ef.topk_ef_compress(g, g.clone(), 0.1, 1)
