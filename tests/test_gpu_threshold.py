"""GPU parity of topk_ef_threshold (the hard-threshold sparsifier under error
feedback) against the CPU oracle: the count of passing entries, the sent
indices and values, and the residual, bit for bit at every step."""
import numpy as np
import pytest
import torch

import datagen
import error_feedback_b200 as ef
import oracle
from gpu_util import assert_same_step, to_dev

pytestmark = pytest.mark.gpu

LR = np.float32(0.1)


def run_threshold_steps(grads, lr, thr, max_out, res0=None, offset_elems=0):
    o = oracle.get()
    n = grads[0].size
    ores = np.zeros(n, np.float32) if res0 is None else res0.copy()
    dres = to_dev(ores, offset_elems)
    ws = torch.empty(ef.topk_ef_threshold_workspace_bytes(n), dtype=torch.uint8, device="cuda")
    counts = []
    for s, g in enumerate(grads):
        dg = to_dev(g, offset_elems)
        gi, gv, gc = ef.topk_ef_threshold(dg, dres, lr, thr, max_out, ws=ws)
        oi, ov, oc = o.threshold(g, ores, lr, thr, max_out)
        cnt = int(gc.cpu().item())
        assert cnt == oc, (s, cnt, oc)
        m = min(cnt, max_out)
        assert_same_step(s, gi[:m], gv[:m], dres, oi, ov, ores)
        counts.append(cnt)
    return counts


def test_flat_normal_1m():
    """1M N(0,1) gradients, lr 0.1, threshold 0.33 (about 0.1% pass at the
    first step, more as the memory grows), room for all."""
    n = 1 << 20
    grads = [datagen.flat_normal(s) for s in range(4)]
    counts = run_threshold_steps(grads, LR, 0.33, n)
    assert counts[0] > 500 and counts[-1] > counts[0]


@pytest.mark.parametrize("n,thr,max_out", [
    (1, 0.0, 1), (1, 5.0, 1), (31, 0.1, 4), (1000, 0.2, 1000), (8193, 0.15, 50),
    (65537, 0.2, 65537), (100003, 0.25, 10), (300001, 0.3, 0), (2_000_003, 0.35, 700),
])
def test_shapes(n, thr, max_out):
    rng = np.random.default_rng(n + int(thr * 100))
    grads = [rng.standard_normal(n).astype(np.float32) for _ in range(2)]
    res0 = (rng.standard_normal(n) * 0.05).astype(np.float32)
    run_threshold_steps(grads, LR, thr, max_out, res0=res0)


def test_threshold_zero_all_pass():
    """Every entry passes: every warp tile has more candidates than it can
    stage and is rescanned; only the first max_out are sent."""
    n = 500_000
    rng = np.random.default_rng(3)
    grads = [rng.standard_normal(n).astype(np.float32) for _ in range(2)]
    counts = run_threshold_steps(grads, LR, 0.0, 123_456)
    assert counts == [n, n]
    counts = run_threshold_steps(grads, LR, 0.0, n)
    assert counts == [n, n]


def test_dense_tiles_past_queue():
    """More dense warp tiles than the rescan queue holds (3,906 > 3,072): the
    overflow is rescanned by the blocks that found it."""
    n = 4_000_000
    rng = np.random.default_rng(5)
    grads = [rng.standard_normal(n).astype(np.float32) for _ in range(2)]
    counts = run_threshold_steps(grads, LR, 0.0, n)
    assert counts == [n, n]


def test_dense_block_region():
    """Passing entries crowded into one contiguous region (as when the
    entries past the cap keep growing): the region's tiles are rescanned by
    warps all over the grid."""
    n = 3_000_000
    rng = np.random.default_rng(6)
    grads = []
    for _ in range(2):
        g = (rng.standard_normal(n) * 0.01).astype(np.float32)
        g[1_000_000:1_200_000] = rng.uniform(1.0, 2.0, 200_000).astype(np.float32)
        grads.append(g)
    counts = run_threshold_steps(grads, LR, 0.05, 150_000)
    assert counts[0] >= 200_000


def test_ties_at_threshold_and_specials():
    """Magnitudes exactly at the threshold pass; NaN, +-Inf and -0 follow the
    magnitude order; a negative threshold acts by magnitude."""
    n = 200_003
    rng = np.random.default_rng(5)
    pool = np.array([0.5, -0.5, 0.25, -0.25, 1.0, 0.0, -0.0, 0.125], np.float32)
    g = rng.choice(pool, n)
    g[rng.integers(0, n, 50)] = np.nan
    g[rng.integers(0, n, 50)] = np.inf
    g[rng.integers(0, n, 50)] = -np.inf
    for thr, mo in ((0.5, n), (-0.5, 1000), (0.25, 70_000), (np.inf, n), (np.nan, n)):
        run_threshold_steps([g, g[::-1].copy()], np.float32(1.0), thr, mo)


def test_unaligned_base():
    """Bases that are not 16-byte aligned take the scalar streaming path."""
    n = 333_333
    rng = np.random.default_rng(9)
    grads = [rng.standard_normal(n).astype(np.float32) for _ in range(2)]
    run_threshold_steps(grads, LR, 0.3, n, offset_elems=1)


def test_empty():
    ws = torch.empty(ef.topk_ef_threshold_workspace_bytes(0), dtype=torch.uint8, device="cuda")
    g = torch.empty(0, dtype=torch.float32, device="cuda")
    r = torch.empty(0, dtype=torch.float32, device="cuda")
    i, v, c = ef.topk_ef_threshold(g, r, LR, 0.5, 0, ws=ws)
    assert int(c.cpu().item()) == 0


def test_resnet50_mix_full():
    """The ResNet-50-sized mixed gradient (n = 25,557,032), threshold 6e-3
    (about 0.1% pass at the first step), max_out = 1% of n, three steps."""
    n = datagen.RESNET50_N
    grads = [datagen.resnet50_mix(s) for s in range(3)]
    counts = run_threshold_steps(grads, LR, 6e-3, n // 100)
    assert counts[0] > 5_000
