"""Checks that pin the CPU oracle to something other than itself.

Each ``pin_*`` function raises AssertionError when the oracle it is given
breaks the property.  The real oracle must pass all of them; every build of
the oracle with a planted mistake must fail at least one
(``test_oracle_mutants.py``).  The pins are:

* exact arithmetic: the memory update equals lr*grad + residual computed in
  exact rational arithmetic and rounded once to fp32 (nearest even);
* brute force: for n <= 12 the chosen set is the only k-subset S with
  |x_s| > |x_u| or (|x_s| == |x_u| and s < u) for every s in S, u not in S;
* invariants of one step (exactly k outputs, ascending index, val == acc,
  sent + residual == acc, nothing unselected above the selected minimum);
* special cases (k = 0, k = n, lr = 1 with zero memory, all magnitudes equal);
* hand-worked examples under tests/golden/ (one EF run, one merge tournament);
* merge special cases: P = 1 identity, disjoint supports give the plain union,
  and with k >= |union| the tournament is the dense pairwise tree sum;
* hard threshold: hand-worked run, special thresholds (0, +Inf, a negative
  threshold, max_out = 0) and agreement with the top-k step at k = count;
* residual return: hand-worked example, a global set that holds every sent
  index (nothing returned) and one that holds none (everything returned);
* AllGather sum: hand-worked example (rank order visible in fp32), and on
  values whose sums are exact it equals the gTop-k merge with k >= |union|.
"""
from __future__ import annotations

import itertools
import json
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _bits(x):
    return np.asarray(x, dtype=np.float32).view(np.uint32)


def f32_round(q: Fraction) -> np.float32:
    """Round a nonzero rational to float32, nearest with ties to even."""
    f = np.float32(float(q))
    best = None
    for c in (np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))):
        if not np.isfinite(c):
            continue
        d = abs(Fraction(float(c)) - q)
        if (best is None or d < best[0]
                or (d == best[0] and (int(np.float32(c).view(np.uint32)) & 1) == 0)):
            best = (d, np.float32(c))
    return best[1]


# ------------------------------------------------------------------ compress

def pin_fmaf_exact(o, seed=11):
    rng = np.random.default_rng(seed)
    m = 3000
    lr = np.float32(0.1)
    g = rng.standard_normal(m).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 20, m).astype(np.float32)
    r = rng.standard_normal(m).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 20, m).astype(np.float32)
    # cancellation cases: memory equal to minus the rounded product, where one
    # rounding and two roundings differ
    c = rng.integers(0, m, m // 3)
    r[c] = -(lr * g[c])
    # subnormal results
    s = rng.integers(0, m, 50)
    g[s] = np.float32(1e-38) * rng.standard_normal(50).astype(np.float32)
    r[s] = np.float32(1e-39) * rng.standard_normal(50).astype(np.float32)
    for lrv in (np.float32(0.1), np.float32(1.0), np.float32(-0.37), np.float32(3.0e-3)):
        acc = o.accumulate(g, r, lrv)
        for i in range(m):
            q = Fraction(float(lrv)) * Fraction(float(g[i])) + Fraction(float(r[i]))
            if q == 0:
                assert acc[i] == 0.0, (i, acc[i])
                continue
            want = f32_round(q)
            assert _bits(acc[i]) == _bits(want), (float(lrv), g[i], r[i], acc[i], want)


def _dominates_all(x, S, n):
    Sset = set(S)
    a = np.abs(x.astype(np.float64))
    for s in S:
        for u in range(n):
            if u in Sset:
                continue
            if not (a[s] > a[u] or (a[s] == a[u] and s < u)):
                return False
    return True


def pin_bruteforce_select(o, seed=12, trials=160):
    rng = np.random.default_rng(seed)
    pool = np.array([0.0, -0.0, 0.5, -0.5, 1.0, -1.0, 2.0, -2.0, 3.0], dtype=np.float32)
    for t in range(trials):
        n = int(rng.integers(1, 13))
        if t % 2:
            x = rng.choice(pool, n).astype(np.float32)
        else:
            x = rng.standard_normal(n).astype(np.float32)
        k = int(rng.integers(0, n + 1))
        hits = [S for S in itertools.combinations(range(n), k) if _dominates_all(x, S, n)]
        assert len(hits) == 1, (x, k, hits)
        got = o.select(x, k, 0).tolist()
        assert got == list(hits[0]), (x.tolist(), k, got, hits[0])
        got_h = o.select(x, k, 1).tolist()
        assert got_h == list(hits[0]), (x.tolist(), k, got_h, hits[0])


def check_step(grad, res_before, lr, k, idx, val, res_after, acc_exact=None):
    """Invariants of one EF step (used by the oracle pins and the GPU tests).
    acc is recomputed here in exact arithmetic only when acc_exact is None
    and the arrays are small; otherwise acc_exact must be given."""
    n = grad.size
    acc = acc_exact
    assert acc is not None
    assert idx.size == k and val.size == k
    if k:
        assert np.all(np.diff(idx.astype(np.int64)) > 0), "indices not strictly ascending"
        assert idx.min() >= 0 and idx.max() < n
        assert np.array_equal(_bits(val), _bits(acc[idx])), "val != acc at the selected slots"
    sel = np.zeros(n, dtype=bool)
    sel[idx] = True
    assert np.all(_bits(res_after[sel]) == 0), "selected residual not +0.0"
    assert np.array_equal(_bits(res_after[~sel]), _bits(acc[~sel])), "unselected residual != acc"
    sent = np.zeros(n, dtype=np.float32)
    sent[idx] = val
    tot = sent + res_after
    same = (tot == acc) | (np.isnan(tot) & np.isnan(acc))
    assert np.all(same), "sent + residual != acc"
    if 0 < k < n:
        key = _bits(acc) & np.uint32(0x7FFFFFFF)
        kmin = key[sel].min()
        kmax = key[~sel].max()
        assert kmin >= kmax, "an unselected |acc| exceeds a selected one"
        if kmin == kmax:
            tie_sel = np.nonzero(sel & (key == kmin))[0]
            tie_uns = np.nonzero(~sel & (key == kmin))[0]
            assert tie_sel.max() < tie_uns.min(), "tie not broken by lower index"


def _exact_acc(grad, res, lr):
    out = np.empty_like(grad)
    for i in range(grad.size):
        q = Fraction(float(np.float32(lr))) * Fraction(float(grad[i])) + Fraction(float(res[i]))
        out[i] = np.float32(0.0) if q == 0 else f32_round(q)
    return out


def pin_compress_invariants(o, seed=13):
    rng = np.random.default_rng(seed)
    for trial in range(12):
        n = int(rng.integers(1, 3000))
        k = int(rng.integers(0, n + 1))
        if trial % 3 == 0:
            grad = rng.choice(np.array([1.0, -1.0, 2.0, 0.5, -0.5, 4.0], np.float32), n)
            res = rng.choice(np.array([0.0, 0.5, -0.5, 1.0], np.float32), n)
        else:
            grad = rng.standard_normal(n).astype(np.float32)
            res = (rng.standard_normal(n) * 0.1).astype(np.float32)
        lr = np.float32(0.1)
        acc = _exact_acc(grad, res, lr)
        r = res.copy()
        idx, val = o.compress(grad, r, lr, k)
        check_step(grad, res, lr, k, idx, val, r, acc_exact=acc)


def pin_special_cases(o, seed=14):
    rng = np.random.default_rng(seed)
    n = 257
    grad = rng.standard_normal(n).astype(np.float32)
    grad[grad == 0] = 1.0
    res = (rng.standard_normal(n) * 0.1).astype(np.float32)
    acc = _exact_acc(grad, res, np.float32(0.1))
    # k = 0: nothing sent, memory becomes acc
    r = res.copy()
    idx, val = o.compress(grad, r, 0.1, 0)
    assert idx.size == 0 and np.array_equal(_bits(r), _bits(acc))
    # k = n: everything sent, memory all +0
    r = res.copy()
    idx, val = o.compress(grad, r, 0.1, n)
    assert idx.tolist() == list(range(n))
    assert np.array_equal(_bits(val), _bits(acc)) and np.all(_bits(r) == 0)
    # lr = 1 with empty memory: acc is the gradient itself
    r = np.zeros(n, np.float32)
    k = 40
    idx, val = o.compress(grad, r, 1.0, k)
    order = sorted(range(n), key=lambda i: (-abs(float(grad[i])), i))[:k]
    assert idx.tolist() == sorted(order)
    assert np.array_equal(_bits(val), _bits(grad[idx]))
    # all magnitudes equal (mixed signs): the k lowest indices
    g = np.where(rng.random(n) < 0.5, np.float32(0.75), np.float32(-0.75)).astype(np.float32)
    r = np.zeros(n, np.float32)
    idx, val = o.compress(g, r, 1.0, 33)
    assert idx.tolist() == list(range(33))
    # NaN sorts above +Inf (magnitude key)
    x = np.array([1.0, np.inf, np.nan, -np.inf, 2.0], np.float32)
    assert o.select(x, 1).tolist() == [2]
    assert o.select(x, 3).tolist() == [1, 2, 3]
    # every NaN is one value whatever its payload or sign: ties go to the
    # lower index
    nans = np.array([0x7FC00001, 0xFFC00000, 0x7FFFFFFF, 0xFF800001], np.uint32).view(np.float32)
    x = np.array([5.0, nans[0], 7.0, nans[1], nans[2], nans[3]], np.float32)
    assert o.select(x, 1).tolist() == [1]
    assert o.select(x, 4).tolist() == [1, 3, 4, 5]


def pin_backends_agree(o, seed=15):
    rng = np.random.default_rng(seed)
    for n, k in ((10_000, 10), (50_000, 5_000), (100_000, 99_999), (30_000, 1)):
        x = rng.standard_normal(n).astype(np.float32)
        x[rng.integers(0, n, n // 4)] = np.float32(0.25)  # many ties
        a = o.select(x, k, 0)
        b = o.select(x, k, 1)
        assert np.array_equal(a, b)


def pin_golden_compress(o):
    with open(os.path.join(GOLDEN, "compress_small.json")) as f:
        g = json.load(f)
    r = np.array(g["residual0"], np.float32)
    for st in g["steps"]:
        grad = np.array(st["grad"], np.float32)
        idx, val = o.compress(grad, r, g["lr"], g["k"])
        assert idx.tolist() == st["idx"], (idx, st["idx"])
        assert val.tolist() == st["val"], (val, st["val"])
        assert r.tolist() == st["residual"], (r, st["residual"])


def pin_batched_matches_flat(o, seed=16):
    rng = np.random.default_rng(seed)
    sizes = [5, 0, 300, 1, 1000]
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    ks = np.array([2, 0, 30, 1, 7], np.int64)
    grad = rng.standard_normal(offsets[-1]).astype(np.float32)
    res = rng.standard_normal(offsets[-1]).astype(np.float32) * np.float32(0.1)
    r1 = res.copy()
    bi, bv = o.compress_batched(grad, r1, offsets, ks, 0.1)
    base = 0
    for l in range(len(sizes)):
        lo, hi = offsets[l], offsets[l + 1]
        acc = _exact_acc(grad[lo:hi], res[lo:hi], np.float32(0.1))
        check_step(grad[lo:hi], res[lo:hi], 0.1, int(ks[l]), bi[base:base + ks[l]],
                   bv[base:base + ks[l]], r1[lo:hi], acc_exact=acc)
        base += int(ks[l])


# --------------------------------------------------------------------- merge

def pin_golden_merge(o):
    with open(os.path.join(GOLDEN, "merge_small.json")) as f:
        g = json.load(f)
    idx = np.array(g["idx"], np.int32)
    val = np.array(g["val"], np.float32)
    oi, ov = o.gtopk_merge(idx, val, g["k"], g["n"])
    assert oi.tolist() == g["out_idx"], (oi, g["out_idx"])
    assert ov.tolist() == g["out_val"], (ov, g["out_val"])


def _random_sets(rng, P, k_in, n, hot=None):
    idx = np.empty((P, k_in), np.int32)
    for p in range(P):
        pool = hot if hot is not None else n
        idx[p] = np.sort(rng.choice(pool, k_in, replace=False))
    val = rng.standard_normal((P, k_in)).astype(np.float32)
    return idx, val


def pin_merge_identity(o, seed=17):
    rng = np.random.default_rng(seed)
    idx, val = _random_sets(rng, 1, 50, 1000)
    oi, ov = o.gtopk_merge(idx, val, 50, 1000)
    assert np.array_equal(oi, idx[0]) and np.array_equal(_bits(ov), _bits(val[0]))
    oi, ov = o.gtopk_merge(idx, val, 80, 1000)
    assert np.array_equal(oi, idx[0]) and np.array_equal(_bits(ov), _bits(val[0]))


def pin_merge_disjoint_union(o, seed=18):
    rng = np.random.default_rng(seed)
    P, k_in, n = 8, 20, 4000
    perm = rng.permutation(n)[:P * k_in].reshape(P, k_in)
    idx = np.sort(perm, axis=1).astype(np.int32)
    val = rng.standard_normal((P, k_in)).astype(np.float32)
    oi, ov = o.gtopk_merge(idx, val, P * k_in, n)
    order = np.argsort(idx.reshape(-1))
    assert np.array_equal(oi, idx.reshape(-1)[order])
    assert np.array_equal(_bits(ov), _bits(val.reshape(-1)[order]))


def _dense_tree_sum(idx, val, n):
    """Pairwise tree sum of P sparse vectors on dense float32 arrays with a
    presence mask: vector i absorbs vector i + 2^r in round r."""
    P = idx.shape[0]
    d = np.zeros((P, n), np.float32)
    pres = np.zeros((P, n), bool)
    for p in range(P):
        d[p, idx[p]] = val[p]
        pres[p, idx[p]] = True
    step = 1
    while step < P:
        for i in range(0, P - step, 2 * step):
            j = i + step
            both = pres[i] & pres[j]
            only_j = pres[j] & ~pres[i]
            d[i, both] = d[i, both] + d[j, both]
            d[i, only_j] = d[j, only_j]
            pres[i] |= pres[j]
        step *= 2
    nz = np.nonzero(pres[0])[0]
    return nz.astype(np.int32), d[0, nz]


def pin_merge_dense_tree_sum(o, seed=19):
    rng = np.random.default_rng(seed)
    for P in (2, 3, 5, 8, 13):
        n, k_in = 300, 25
        idx, val = _random_sets(rng, P, k_in, n, hot=60)  # many common indices
        want_i, want_v = _dense_tree_sum(idx, val, n)
        oi, ov = o.gtopk_merge(idx, val, P * k_in, n)
        assert np.array_equal(oi, want_i), P
        assert np.array_equal(_bits(ov), _bits(want_v)), P


def pin_merge_bruteforce_select(o, seed=20):
    """P = 2 with a selection: the kept set is the unique dominating k-subset
    of the union (brute force over subsets, |union| <= 12)."""
    rng = np.random.default_rng(seed)
    for t in range(60):
        n = 16
        k_in = int(rng.integers(1, 7))
        idx, _ = _random_sets(rng, 2, k_in, n)
        val = rng.choice(np.array([0.5, -0.5, 1.0, -1.0, 2.0, 0.25], np.float32), (2, k_in))
        ui, uv = _dense_tree_sum(idx, val, n)
        k = int(rng.integers(0, len(ui) + 1))
        hits = [S for S in itertools.combinations(range(len(ui)), k)
                if _dominates_all_ids(uv, ui, S)]
        assert len(hits) == 1
        want = sorted(ui[list(hits[0])].tolist())
        oi, ov = o.gtopk_merge(idx, val, k, n)
        assert oi.tolist() == want, (idx, val, k, oi, want)


def _dominates_all_ids(v, ids, S):
    a = np.abs(v.astype(np.float64))
    Sset = set(S)
    for s in S:
        for u in range(len(v)):
            if u in Sset:
                continue
            if not (a[s] > a[u] or (a[s] == a[u] and ids[s] < ids[u])):
                return False
    return True


# ------------------------------------------------------------ hard threshold

def pin_golden_threshold(o):
    with open(os.path.join(GOLDEN, "threshold_small.json")) as f:
        g = json.load(f)
    r = np.array(g["residual0"], np.float32)
    for st in g["steps"]:
        idx, val, cnt = o.threshold(np.array(st["grad"], np.float32), r, g["lr"],
                                    g["threshold"], g["max_out"])
        assert cnt == st["count"], (cnt, st["count"])
        assert idx.tolist() == st["idx"], (idx, st["idx"])
        assert val.tolist() == st["val"], (val, st["val"])
        assert r.tolist() == st["residual"], (r, st["residual"])


def pin_threshold_special(o, seed=21):
    rng = np.random.default_rng(seed)
    n = 300
    grad = rng.standard_normal(n).astype(np.float32)
    res = (rng.standard_normal(n) * 0.5).astype(np.float32)
    acc = _exact_acc(grad, res, np.float32(0.5))
    # threshold 0: every entry passes; the first max_out are sent
    r = res.copy()
    idx, val, cnt = o.threshold(grad, r, 0.5, 0.0, 40)
    assert cnt == n and idx.tolist() == list(range(40))
    assert np.array_equal(_bits(val), _bits(acc[:40]))
    assert np.all(_bits(r[:40]) == 0) and np.array_equal(_bits(r[40:]), _bits(acc[40:]))
    # max_out = 0: nothing sent, the count is still reported
    r = res.copy()
    idx, val, cnt = o.threshold(grad, r, 0.5, 0.0, 0)
    assert cnt == n and idx.size == 0 and np.array_equal(_bits(r), _bits(acc))
    # +Inf: only infinities and NaNs pass; a negative threshold acts by magnitude
    x = np.array([1.0, -np.inf, 3.0, np.nan, np.inf, -3.0], np.float32)
    z = np.zeros(6, np.float32)
    idx, val, cnt = o.threshold(x, z.copy(), 1.0, np.inf, 10)
    assert cnt == 3 and idx.tolist() == [1, 3, 4]
    idx, val, cnt = o.threshold(x, z.copy(), 1.0, -3.0, 10)
    assert idx.tolist() == [1, 2, 3, 4, 5]


def pin_threshold_matches_topk(o, seed=22):
    """With room for every passing entry, the sent set is the top-k set for
    k = count (nothing outside it has a magnitude at or above the threshold),
    so the two steps agree bit for bit."""
    rng = np.random.default_rng(seed)
    for n, thr in ((5_000, 1.5), (20_000, 2.5), (777, 0.25)):
        grad = rng.standard_normal(n).astype(np.float32)
        res = (rng.standard_normal(n) * 0.1).astype(np.float32)
        at = rng.integers(0, n, n // 10)
        grad[at] = np.float32(thr) * 2          # acc = 0.5 * 2 thr exactly at the threshold
        res[at] = 0.0
        r1, r2 = res.copy(), res.copy()
        idx, val, cnt = o.threshold(grad, r1, 0.5, thr, n)
        ti, tv = o.compress(grad, r2, 0.5, cnt)
        assert np.array_equal(idx, ti) and np.array_equal(_bits(val), _bits(tv))
        assert np.array_equal(_bits(r1), _bits(r2))


# ----------------------------------------------------------- residual return

def pin_golden_residual_return(o):
    with open(os.path.join(GOLDEN, "residual_return_small.json")) as f:
        g = json.load(f)
    r = np.array(g["residual0"], np.float32)
    o.residual_return(np.array(g["sent_idx"], np.int32), np.array(g["sent_val"], np.float32),
                      np.array(g["global_idx"], np.int32), r)
    assert r.tolist() == g["residual"], (r, g["residual"])


def pin_residual_return_special(o, seed=23):
    rng = np.random.default_rng(seed)
    P, k, n = 4, 50, 1000
    idx = np.stack([np.sort(rng.choice(n, k, replace=False)) for _ in range(P)]).astype(np.int32)
    val = rng.standard_normal((P, k)).astype(np.float32)
    res = rng.standard_normal((P, n)).astype(np.float32)
    # every sent index survived: nothing comes back
    r = res.copy()
    o.residual_return(idx, val, np.unique(idx).astype(np.int32), r)
    assert np.array_equal(_bits(r), _bits(res))
    # no sent index survived: every sent value comes back (memory was +0 there)
    r = res.copy()
    for p in range(P):
        r[p, idx[p]] = 0.0
    want = r.copy()
    for p in range(P):
        want[p, idx[p]] = val[p]
    rest = np.setdiff1d(np.arange(n), np.unique(idx))[:30].astype(np.int32)
    o.residual_return(idx, val, rest, r)
    assert np.array_equal(_bits(r), _bits(want))


# ------------------------------------------------------------ AllGather sum

def pin_golden_allgather(o):
    with open(os.path.join(GOLDEN, "allgather_small.json")) as f:
        g = json.load(f)
    out = o.allgather_sum(np.array(g["idx"], np.int32), np.array(g["val"], np.float32), g["n"])
    assert out.tolist() == g["out"], (out, g["out"])


def pin_allgather_matches_merge(o, seed=24):
    """Small integer values add exactly in any order, so the dense sum equals
    the gTop-k tournament kept whole (k >= |union|) scattered into zeros."""
    rng = np.random.default_rng(seed)
    for P, k, n in ((5, 40, 200), (8, 100, 5000), (1, 10, 10)):
        idx = np.stack([np.sort(rng.choice(n, k, replace=False)) for _ in range(P)]).astype(np.int32)
        val = rng.integers(-50, 51, (P, k)).astype(np.float32)
        dense = o.allgather_sum(idx, val, n)
        mi, mv = o.gtopk_merge(idx, val, P * k, n)
        want = np.zeros(n, np.float32)
        want[mi] = mv
        assert np.array_equal(dense, want)
        assert np.count_nonzero(np.isin(np.arange(n), mi)) == np.unique(idx).size


ALL_PINS = [
    pin_fmaf_exact, pin_bruteforce_select, pin_compress_invariants,
    pin_special_cases, pin_backends_agree, pin_golden_compress,
    pin_batched_matches_flat, pin_golden_merge, pin_merge_identity,
    pin_merge_disjoint_union, pin_merge_dense_tree_sum,
    pin_merge_bruteforce_select, pin_golden_threshold, pin_threshold_special,
    pin_threshold_matches_topk, pin_golden_residual_return,
    pin_residual_return_special, pin_golden_allgather, pin_allgather_matches_merge,
]
