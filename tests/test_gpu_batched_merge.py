"""GPU parity of topk_ef_compress_batched and gtopk_merge against the oracle."""
import json
import os

import numpy as np
import pytest
import torch

import datagen
import error_feedback_b200 as ef
from gpu_util import run_batched_steps, run_merge, to_dev

pytestmark = pytest.mark.gpu

LR = np.float32(0.1)
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _bucket(sizes, seed, scales=None):
    rng = np.random.default_rng(seed)
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    g = np.empty(int(offsets[-1]), np.float32)
    for l, nl in enumerate(sizes):
        s = scales[l] if scales is not None else 10.0 ** rng.uniform(-4, -1)
        g[offsets[l]:offsets[l + 1]] = rng.laplace(0, s, nl).astype(np.float32)
    return g, offsets


def _wsb(offsets, ks):
    return torch.empty(ef.topk_ef_batched_workspace_bytes(offsets, ks), dtype=torch.uint8,
                       device="cuda")


def test_batched_small_mixed():
    sizes = [1, 0, 7, 8192, 8193, 100_000, 3, 70_001, 0, 5]
    ks = [1, 0, 0, 8192, 9, 100, 3, 71, 0, 2]
    grads = []
    for s in range(3):
        g, offsets = _bucket(sizes, 100 + s)
        grads.append(g)
    run_batched_steps(grads, offsets, ks, LR, ws=_wsb(offsets, ks))


def test_batched_vgg16_scaled_down():
    """VGG-16 layer structure with every tensor 1/64 of its size."""
    sizes = [max(1, n // 64) for n in datagen.VGG16_SIZES]
    ks = [(n + 999) // 1000 for n in sizes]
    b = datagen.vgg16_scales()
    grads = [_bucket(sizes, 200 + s, b)[0] for s in range(3)]
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    run_batched_steps(grads, offsets, ks, LR, ws=_wsb(offsets, ks))


def test_batched_dense_tiles():
    """Tiles of the streaming pass with far more than 32 candidates, which
    the select rescans: four small tensors of equal magnitudes (random
    signs, a few doubled), sharing tiles, where every element is a
    candidate and the ties at the k-th magnitude go to the lower indices;
    and a large tensor whose 25,000 largest entries sit in one contiguous
    block.  The candidate path must hold (no rescan of the residual)."""
    rng = np.random.default_rng(21)
    sizes = [700, 1500, 3000, 5001, 130_000, 9]
    ks = [50, 1500, 100, 2600, 20_000, 0]
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    grads = []
    for s in range(2):
        g = np.empty(int(offsets[-1]), np.float32)
        for l in range(4):
            a, b = int(offsets[l]), int(offsets[l + 1])
            m = np.where(rng.random(b - a) < 0.5, -1.0, 1.0).astype(np.float32)
            m[rng.choice(b - a, max(1, (b - a) // 100), replace=False)] *= np.float32(2.0)
            g[a:b] = m
        a, b = int(offsets[4]), int(offsets[5])
        g[a:b] = rng.laplace(0, 1e-3, b - a).astype(np.float32)
        g[a + 40_000:a + 65_000] = (rng.uniform(0.5, 1.5, 25_000) *
                                    np.where(rng.random(25_000) < 0.5, -1, 1)).astype(np.float32)
        g[offsets[5]:] = rng.laplace(0, 1.0, sizes[5]).astype(np.float32)
        grads.append(g)
    ws = _wsb(offsets, ks)
    run_batched_steps(grads, offsets, ks, LR, ws=ws)
    assert ef.topk_ef_path_info(ws)["fallback"] == 0


def test_batched_many_tensors():
    """More tensors than one launch group holds (600 > 256)."""
    rng = np.random.default_rng(9)
    sizes = rng.integers(0, 3000, 600).tolist()
    sizes[17] = 200_000
    ks = [int(rng.integers(0, n + 1)) if n else 0 for n in sizes]
    grads = [_bucket(sizes, 300 + s)[0] for s in range(2)]
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    run_batched_steps(grads, offsets, ks, LR, ws=_wsb(offsets, ks))


def test_batched_vgg16_full():
    """The full VGG-16 bucket (16 tensors, 138,344,128 elements), per-tensor
    k = ceil(n_l / 1000); all 5 EF steps of the workload, every one compared
    bit for bit."""
    _, offsets, ks = datagen.vgg16_bucket(0)
    ws = _wsb(offsets, ks)
    run_batched_steps((datagen.vgg16_bucket(s)[0] for s in range(5)), offsets, ks, LR,
                      backend=1, ws=ws)
    assert ef.topk_ef_path_info(ws)["fallback"] == 0


# --------------------------------------------------------------------- merge

def _mws(P, k_in, k):
    return torch.empty(ef.gtopk_merge_workspace_bytes(P, k_in, k), dtype=torch.uint8,
                       device="cuda")


def test_merge_golden():
    with open(os.path.join(GOLDEN, "merge_small.json")) as f:
        g = json.load(f)
    idx = np.array(g["idx"], np.int32)
    val = np.array(g["val"], np.float32)
    gi, gv, cnt = run_merge(idx, val, g["k"], g["n"], ws=_mws(4, 3, g["k"]))
    assert gi[:cnt].tolist() == g["out_idx"] and gv[:cnt].tolist() == g["out_val"]


@pytest.mark.parametrize("P,k_in,k,n", [
    (1, 100, 50, 1000), (1, 100, 200, 1000), (2, 1000, 1000, 5000), (3, 500, 700, 3000),
    (5, 800, 300, 4000), (8, 2000, 2000, 100_000), (13, 1000, 4000, 20_000),
    (32, 3000, 3000, 1_000_000), (4, 0, 10, 100), (6, 10, 0, 100), (7, 5000, 100, 6000),
    (2, 5000, 10_000, 10_000),
])
def test_merge_shapes(P, k_in, k, n):
    idx, val = datagen.gtopk_sets(P=P, k=k_in, n=n, step=P + k) if k_in else (
        np.zeros((P, 0), np.int32), np.zeros((P, 0), np.float32))
    run_merge(idx, val, k, n, ws=_mws(P, k_in, k))


def test_merge_heavy_overlap():
    """Every set drawn from one small pool: most indices collide."""
    rng = np.random.default_rng(21)
    P, k_in, n = 16, 900, 1000
    idx = np.stack([np.sort(rng.choice(n, k_in, replace=False)) for _ in range(P)]).astype(np.int32)
    val = rng.choice(np.array([0.5, -0.5, 1.0, 0.25], np.float32), (P, k_in))
    run_merge(idx, val, 400, n, ws=_mws(P, k_in, 400))


def test_merge_resnet50_32_workers():
    """P = 32 workers, k = 25,557 of n = 25,557,032 each, half from a shared
    hot set of 2k indices; 5 rounds."""
    idx, val = datagen.gtopk_sets()
    ws = _mws(32, idx.shape[1], 25_557)
    run_merge(idx, val, 25_557, datagen.RESNET50_N, ws=ws)


def test_merge_bad_input_flagged():
    idx = np.array([[1, 5, 3], [0, 2, 4]], np.int32)   # row 0 not ascending
    val = np.ones((2, 3), np.float32)
    ws = _mws(2, 3, 3)
    ef.gtopk_merge(to_dev(idx), to_dev(val), 3, 10, ws=ws)
    assert ef.topk_ef_last_device_status(ws) == ef.ERR_BAD_INPUT
    idx2 = np.array([[1, 5, 30], [0, 2, 4]], np.int32)  # index >= n
    ef.gtopk_merge(to_dev(idx2), to_dev(val), 3, 10, ws=ws)
    assert ef.topk_ef_last_device_status(ws) == ef.ERR_BAD_INPUT
    good = np.array([[1, 3, 5], [0, 2, 4]], np.int32)
    ef.gtopk_merge(to_dev(good), to_dev(val), 3, 10, ws=ws)
    assert ef.topk_ef_last_device_status(ws) == 0


@pytest.mark.parametrize("P,k_in,k,n,cluster", [
    (32, 25_557, 25_557, datagen.RESNET50_N, True),    # one cluster kernel per round
    (4, 40_000, 40_000, 2_000_000, False),             # merged lists too long: merge + select
    (32, 8_000, 40_000, 1_000_000, False),             # sets grow past the cluster size
    (16, 30_000, 30_000, 500_000, True),
])
def test_merge_paths(P, k_in, k, n, cluster):
    """Both round implementations: the cluster kernel (merge, select and
    emission of a pair in one thread-block cluster) and the merge kernel +
    grid-wide select; the launch count tells which one ran."""
    idx, val = datagen.gtopk_sets(P=P, k=k_in, n=n, step=7)
    ws = _mws(P, k_in, k)
    run_merge(idx, val, k, n, ws=ws)
    rounds = (P - 1).bit_length()
    kernels = ef.topk_ef_path_info(ws)["kernels"]
    assert kernels == (1 + rounds if cluster else 1 + 2 * rounds), kernels


@pytest.mark.parametrize("case", ["cancel", "grow"])
def test_merge_relative_digit_falls_back(case):
    """After the first round the cluster kernel bins digit 1 relative to the
    lower of the two sets' lowest keys, two octaves wide; a k-th key below
    it (values that cancel at common indices) or above it (values that add
    up to more than four times it) repeats the digit over the whole key.
    P = 4: round 0 builds two sets on the same indices, round 1 merges them."""
    rng = np.random.default_rng(41)
    n, k = 10_000, 1000
    I = np.sort(rng.choice(n, k, replace=False))
    J = np.sort(np.setdiff1d(rng.choice(n, 3 * k, replace=False), I)[:k])
    x = rng.uniform(1.0, 1.1, k).astype(np.float32)
    y = rng.uniform(0.5, 0.6, k).astype(np.float32)
    if case == "cancel":
        vals = [x, y, -x, -y]
    else:
        vals = [x, y, (np.float32(7.0) * x).astype(np.float32), y]
    idx = np.stack([I, J, I, J]).astype(np.int32)
    val = np.stack(vals).astype(np.float32)
    run_merge(idx, val, k, n, ws=_mws(4, k, k))


@pytest.mark.parametrize("size", [16, 14, 12, 8])
@pytest.mark.parametrize("P,k_in,k,n", [
    (32, 25_557, 25_557, datagen.RESNET50_N),
    (13, 3_001, 2_500, 200_000),
])
def test_merge_cluster_sizes(size, P, k_in, k, n):
    """Every cluster size of the cluster kernel (one pair per cluster of
    16, 14, 12 or 8 CTAs; 16, 14 and 12 divide digit 1's 2,048 bins into
    slices of 128, 148 and 172, the last slice shorter), forced through the
    test flag for every round."""
    idx, val = datagen.gtopk_sets(P=P, k=k_in, n=n, step=size)
    ws = _mws(P, k_in, k)
    old = ef.topk_ef_set_test_flags({16: 1, 14: 2, 12: 3, 8: 4}[size] << 3)
    try:
        run_merge(idx, val, k, n, ws=ws)
    finally:
        ef.topk_ef_set_test_flags(old)
    assert ef.topk_ef_path_info(ws)["kernels"] == 1 + (P - 1).bit_length()
