"""The multi-threaded CPU baseline computes exactly what the oracle computes
(indices, values and the residual bit for bit), for several thread counts."""
import numpy as np
import pytest

import cpu_baseline
import oracle

LR = np.float32(0.1)


def _same(a, b):
    a, b = np.ascontiguousarray(a), np.ascontiguousarray(b)
    eq = a.view(np.uint32) == b.view(np.uint32) if a.dtype == np.float32 else a == b
    if a.dtype == np.float32:
        eq |= np.isnan(a) & np.isnan(b)
    return bool(eq.all())


@pytest.mark.parametrize("n,k,threads", [(1, 1, 1), (10, 0, 2), (1000, 1000, 3), (100_003, 100, 0),
                                         (300_000, 7_000, 5), (2_000_000, 2_000, 8)])
def test_matches_oracle(n, k, threads):
    rng = np.random.default_rng(n + k)
    o = oracle.get()
    r1 = (rng.standard_normal(n) * 0.05).astype(np.float32)
    r2 = r1.copy()
    for step in range(2):
        g = rng.laplace(0, 1e-3, n).astype(np.float32)
        ci, cv = cpu_baseline.compress(g, r1, LR, k, threads)
        oi, ov = o.compress(g, r2, LR, k)
        assert np.array_equal(ci, oi), step
        assert _same(cv, ov) and _same(r1, r2), step


def test_ties_and_specials():
    rng = np.random.default_rng(4)
    n, k = 50_000, 3_000
    g = rng.choice(np.array([0.5, -0.5, 1.0, 0.0, -0.0, np.inf, -np.inf, np.nan, 1e-45],
                            np.float32), n)
    r1 = np.zeros(n, np.float32)
    r2 = r1.copy()
    ci, cv = cpu_baseline.compress(g, r1, np.float32(1.0), k, 4)
    oi, ov = oracle.get().compress(g, r2, np.float32(1.0), k)
    assert np.array_equal(ci, oi)
    assert _same(cv, ov) and _same(r1, r2)
