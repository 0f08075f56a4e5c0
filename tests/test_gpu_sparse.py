"""GPU parity of the steps around the gTop-k merge against the CPU oracle,
bit for bit: the residual return of non-surviving sent values, and the
AllGather-style dense rank-order sum of all workers' sets."""
import numpy as np
import pytest
import torch

import datagen
import error_feedback_b200 as ef
import oracle
from gpu_util import bits, same_bits

pytestmark = pytest.mark.gpu


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def check_return(sent_idx, sent_val, global_idx, res0):
    o = oracle.get()
    want = res0.copy()
    o.residual_return(sent_idx, sent_val, global_idx, want)
    dres = _dev(res0)
    ws = ef.gtopk_residual_return(_dev(sent_idx), _dev(sent_val), _dev(global_idx), dres)
    assert ef.topk_ef_last_device_status(ws) == 0
    got = dres.cpu().numpy()
    eq = same_bits(got, want)
    assert eq.all(), f"{(~eq).sum()} residual mismatches"


def check_allgather(idx, val, n):
    o = oracle.get()
    want = o.allgather_sum(idx, val, n)
    out = torch.full((max(n, 1),), 7.0, dtype=torch.float32, device="cuda")[:n]
    ws = torch.empty(ef.topk_allgather_workspace_bytes(idx.shape[0], idx.shape[1], n),
                     dtype=torch.uint8, device="cuda")
    ef.topk_allgather_sum(_dev(idx), _dev(val), n, out=out, ws=ws)
    assert ef.topk_ef_last_device_status(ws) == 0
    got = out.cpu().numpy()
    eq = same_bits(got, want)
    assert eq.all(), f"{(~eq).sum()} mismatches, first at {np.nonzero(~eq)[0][:5]}"


def _sets(rng, P, k, n, pool=None):
    src = n if pool is None else pool
    return np.stack([np.sort(rng.choice(src, k, replace=False)) for _ in range(P)]).astype(np.int32)


# ---------------------------------------------------------- residual return

def test_return_gtopk_p32_full():
    """The gTop-k configuration (P = 32, k = 25,557, n = 25,557,032): the
    global set from the tournament, returned to the first 8 workers'
    memories (random, nonzero)."""
    P, k, n = 32, 25_557, datagen.RESNET50_N
    idx, val = datagen.gtopk_sets(P=P, k=k, n=n, step=0)
    gi, gv = oracle.get().gtopk_merge(idx, val, k, n)
    rng = np.random.default_rng(1)
    res0 = (rng.standard_normal((8, n)) * 1e-3).astype(np.float32)
    check_return(idx[:8], val[:8], gi, res0)


@pytest.mark.parametrize("P,k,n,kg", [(1, 10, 100, 5), (3, 1000, 50_000, 1500),
                                      (8, 4096, 1 << 20, 8192), (5, 1, 10, 0),
                                      (2, 5000, 5000, 5000), (4, 0, 100, 10),
                                      (4, 50_000, 1_000_000, 40_960),
                                      (4, 50_000, 1_000_000, 60_000)])
def test_return_shapes(P, k, n, kg):
    """Global lists from empty to far longer than the kernel's 4,096-entry
    shared-memory sample (long stretches between two samples)."""
    rng = np.random.default_rng(P * 100 + k)
    idx = _sets(rng, P, k, n) if k else np.zeros((P, 0), np.int32)
    val = rng.standard_normal((P, k)).astype(np.float32)
    g = np.sort(rng.choice(n, kg, replace=False)).astype(np.int32)
    res0 = rng.standard_normal((P, n)).astype(np.float32)
    check_return(idx, val, g, res0)


def test_return_global_is_union_and_empty():
    rng = np.random.default_rng(7)
    P, k, n = 6, 300, 20_000
    idx = _sets(rng, P, k, n, pool=1000)         # heavy overlap between rows
    val = rng.standard_normal((P, k)).astype(np.float32)
    res0 = np.zeros((P, n), np.float32)
    check_return(idx, val, np.unique(idx).astype(np.int32), res0)    # nothing returns
    check_return(idx, val, np.zeros(0, np.int32), res0)              # everything returns


def test_return_bad_input_is_reported_and_contained():
    n = 1000
    idx = np.array([[5, 3, 7], [1, 2, 2000]], np.int32)   # row 0 not ascending, 2000 >= n
    val = np.ones((2, 3), np.float32)
    dres = torch.zeros((2, n), dtype=torch.float32, device="cuda")
    ws = ef.gtopk_residual_return(_dev(idx), _dev(val), _dev(np.array([7], np.int32)), dres)
    assert ef.topk_ef_last_device_status(ws) == ef.ERR_BAD_INPUT
    # entries that break the order (3 after 5) or the range (2000) are
    # skipped; the others are handled (5, and 1 and 2 of row 1; 7 survived)
    got = dres.cpu().numpy()
    assert got[0, 5] == 1.0 and got[1, 1] == 1.0 and got[1, 2] == 1.0
    assert got.sum() == 3.0


# ------------------------------------------------------------ AllGather sum

def test_allgather_gtopk_p32_full():
    """All 32 workers' sets of the gTop-k configuration summed into the
    dense n = 25,557,032 gradient."""
    P, k, n = 32, 25_557, datagen.RESNET50_N
    idx, val = datagen.gtopk_sets(P=P, k=k, n=n, step=0)
    check_allgather(idx, val, n)


@pytest.mark.parametrize("P,k,n", [(1, 1, 1), (1, 100, 100), (3, 50, 8191), (7, 2000, 8193),
                                   (32, 512, 100_003), (256, 40, 70_000), (5, 0, 1000),
                                   (2, 9000, 9000)])
def test_allgather_shapes(P, k, n):
    rng = np.random.default_rng(P * 31 + k + n)
    idx = _sets(rng, P, k, n) if k else np.zeros((P, 0), np.int32)
    val = rng.standard_normal((P, k)).astype(np.float32)
    check_allgather(idx, val, n)


def test_allgather_rank_order_and_crowded_chunk():
    """Every row holds the same indices (the adds at an index are ordered by
    rank) with magnitudes that do not add associatively; one chunk holds
    more entries than the shared-memory stage."""
    P, k, n = 32, 3000, 1 << 16
    rng = np.random.default_rng(11)
    base = np.sort(rng.choice(8192, k, replace=False)).astype(np.int32)
    idx = np.tile(base, (P, 1))
    mags = np.array([1e8, 1.0, -1e8, 3.0, 0.5, -0.0, 1e-30], np.float32)
    val = rng.choice(mags, (P, k)).astype(np.float32)
    check_allgather(idx, val, n)


def test_allgather_bad_input_is_reported():
    n = 20_000
    idx = np.array([[10, 5, 30], [1, 2, 3]], np.int32)
    val = np.ones((2, 3), np.float32)
    out = torch.zeros(n, dtype=torch.float32, device="cuda")
    ws = torch.empty(ef.topk_allgather_workspace_bytes(2, 3, n), dtype=torch.uint8, device="cuda")
    ef.topk_allgather_sum(_dev(idx), _dev(val), n, out=out, ws=ws)
    assert ef.topk_ef_last_device_status(ws) == ef.ERR_BAD_INPUT


def test_allgather_rows_with_long_gaps():
    """Rows crowded into narrow index ranges, far apart: most chunk bounds
    lie in gaps of thousands of chunks (filled by search, not by the entry
    scan)."""
    n = 3_000_000
    rng = np.random.default_rng(13)
    rows = []
    for p in range(6):
        lo = int(rng.integers(0, n - 5000))
        a = rng.choice(np.arange(lo, lo + 5000), 300, replace=False)
        b = rng.choice(n, 100, replace=False) if p % 2 else rng.choice(np.arange(n - 2000, n), 100, replace=False)
        rows.append(np.sort(np.unique(np.concatenate([a, b]))[:350]))
    k = min(len(r) for r in rows)
    idx = np.stack([r[:k] for r in rows]).astype(np.int32)
    val = rng.standard_normal(idx.shape).astype(np.float32)
    check_allgather(idx, val, n)
