"""Helpers for the GPU parity tests: run the library and the oracle on the
same seeded inputs and compare bit for bit."""
from __future__ import annotations

import numpy as np
import torch

import error_feedback_b200 as ef
import oracle


def bits(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    return a.view(np.uint32) if a.dtype == np.float32 else a


def to_dev(a: np.ndarray, offset_elems: int = 0) -> torch.Tensor:
    """Copy to cuda:0; with offset_elems > 0 the tensor is a view that starts
    offset_elems elements into a larger buffer (to test misaligned bases)."""
    t = torch.from_numpy(np.ascontiguousarray(a))
    if offset_elems:
        buf = torch.empty(a.size + offset_elems, dtype=t.dtype, device="cuda")
        v = buf[offset_elems:]
        v.copy_(t)
        return v
    return t.to("cuda")


def same_bits(a, b) -> np.ndarray:
    """Elementwise bit equality, where any two NaNs count as equal (NaN
    payloads and signs are implementation-defined; both sides order every
    NaN as one value above +Inf)."""
    a = np.ascontiguousarray(a)
    b = np.ascontiguousarray(b)
    eq = bits(a) == bits(b)
    if a.dtype == np.float32:
        eq |= np.isnan(a) & np.isnan(b)
    return eq


def assert_same_step(step, gi, gv, gres, oi, ov, ores):
    gi = gi.cpu().numpy()
    gv = gv.cpu().numpy()
    gres = gres.cpu().numpy()
    assert gi.shape == oi.shape, (step, gi.shape, oi.shape)
    if not np.array_equal(gi, oi):
        bad = np.nonzero(gi != oi)[0]
        raise AssertionError(f"step {step}: {bad.size} index mismatches, first at {bad[0]}: "
                             f"gpu {gi[bad[0]]} oracle {oi[bad[0]]}")
    eqv = same_bits(gv, ov)
    if not eqv.all():
        bad = np.nonzero(~eqv)[0]
        raise AssertionError(f"step {step}: {bad.size} value mismatches, first at {bad[0]}: "
                             f"gpu {gv[bad[0]]!r} oracle {ov[bad[0]]!r}")
    eqr = same_bits(gres, ores)
    if not eqr.all():
        bad = np.nonzero(~eqr)[0]
        raise AssertionError(f"step {step}: {bad.size} residual mismatches, first at {bad[0]}: "
                             f"gpu {gres[bad[0]]!r} oracle {ores[bad[0]]!r}")


def run_compress_steps(grads, lr, k, res0=None, backend=0, offset_elems=0, ws=None, n=None,
                       paths=None, zero_between=False):
    """EF steps on the GPU and in the oracle; every step compared.
    grads: float32 arrays, one per step (a list, or any iterable when n is
    given, so that full-size sequences need not be held at once).
    paths: a list that receives topk_ef_path_info after every step (needs
    ws).  zero_between: both residuals are set to +0 before every step after
    the first (the caller owns the residual; the workspace, and with it the
    previous call's threshold hint, is kept).  Returns the GPU residual."""
    o = oracle.get()
    if n is None:
        n = grads[0].size
    ores = np.zeros(n, np.float32) if res0 is None else res0.copy()
    dres = to_dev(ores, offset_elems)
    for s, g in enumerate(grads):
        if zero_between and s > 0:
            ores[:] = 0
            dres.zero_()
        dg = to_dev(g, offset_elems)
        gi, gv = ef.topk_ef_compress(dg, dres, lr, k, ws=ws)
        st = ef.topk_ef_last_device_status(ws) if ws is not None else 0
        assert st == 0, ef.status_string(st)
        if paths is not None:
            paths.append(ef.topk_ef_path_info(ws))
        oi, ov = o.compress(g, ores, lr, k, backend)
        assert_same_step(s, gi, gv, dres, oi, ov, ores)
    return dres


def run_batched_steps(grads, offsets, ks, lr, res0=None, backend=0, ws=None):
    """Batched EF steps on the GPU and in the oracle; every step compared.
    grads: any iterable of float32 bucket arrays, one per step."""
    o = oracle.get()
    N = int(offsets[-1])
    ores = np.zeros(N, np.float32) if res0 is None else res0.copy()
    dres = to_dev(ores)
    for s, g in enumerate(grads):
        dg = to_dev(g)
        gi, gv = ef.topk_ef_compress_batched(dg, dres, offsets, ks, lr, ws=ws)
        if ws is not None:
            st = ef.topk_ef_last_device_status(ws)
            assert st == 0, ef.status_string(st)
        oi, ov = o.compress_batched(g, ores, offsets, ks, lr, backend)
        assert_same_step(s, gi, gv, dres, oi, ov, ores)
    return dres


def run_merge(idx, val, k, n, ws=None):
    o = oracle.get()
    di = to_dev(idx)
    dv = to_dev(val)
    gi, gv, gc = ef.gtopk_merge(di, dv, k, n, ws=ws)
    if ws is not None:
        st = ef.topk_ef_last_device_status(ws)
        assert st == 0, ef.status_string(st)
    oi, ov = o.gtopk_merge(idx, val, k, n)
    cnt = int(gc.cpu().item())
    assert cnt == oi.size, (cnt, oi.size)
    gi = gi.cpu().numpy()
    gv = gv.cpu().numpy()
    assert np.array_equal(gi[:cnt], oi), "merge index mismatch"
    assert same_bits(gv[:cnt], ov).all(), "merge value mismatch"
    assert np.all(gi[cnt:] == -1) and np.all(bits(gv[cnt:]) == 0)
    return gi, gv, cnt
