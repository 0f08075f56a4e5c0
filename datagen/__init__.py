"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module only draws inputs; it holds none of the method's arithmetic.
Every array is produced on the host with numpy ``Generator(PCG64)`` streams:
an array of n elements is drawn in fixed chunks of ``CHUNK`` elements, chunk j
from ``SeedSequence([seed, j])``, so the values do not depend on the number of
threads used to draw them.  Floating-point draws are made in float64 and
rounded to float32 (round to nearest even).

Workloads (the stand-ins for the pages' ResNet-50 / VGG-16 training
gradients; no dataset or model is involved):

* ``flat_normal``      grad ~ N(0, 1)                         (1M elements)
* ``vgg16_bucket``     16 VGG-16 weight tensors, grad_l ~ Laplace(0, b_l),
                       b_l = 10**U(-4, -1) drawn once per run
* ``resnet50_mix``     n = 25,557,032; Laplace(0, 1e-3) everywhere, then
                       exactly round(0.1 n) positions (without replacement,
                       redrawn every step) replaced by 1e-2 * Student-t(3)
* ``gtopk_sets``       P index-sorted sparse sets of k entries over [0, n):
                       floor(k/2) indices from a shared hot set of 2k indices,
                       the rest uniform over the other indices; val ~ N(0, 1e-2)
* ``bf16_normal``      grad ~ N(0, 1e-3) rounded to bfloat16 (nearest even)
                       and widened back to float32, so |acc| has heavy ties

Seeds: ``seed = 1000 * config + step`` (config numbered 1..5, step from 0).
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

CHUNK = 1 << 24

# VGG-16 weight tensors (conv 3x3 stacks 64..512 channels, FC 25088x4096,
# 4096x4096, 4096x1000), in layer order.
VGG16_SIZES = [
    3 * 64 * 9, 64 * 64 * 9,
    64 * 128 * 9, 128 * 128 * 9,
    128 * 256 * 9, 256 * 256 * 9, 256 * 256 * 9,
    256 * 512 * 9, 512 * 512 * 9, 512 * 512 * 9,
    512 * 512 * 9, 512 * 512 * 9, 512 * 512 * 9,
    25088 * 4096, 4096 * 4096, 4096 * 1000,
]

RESNET50_N = 25_557_032
LARGE_N = 1_500_000_000


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def _chunked(n: int, seed: int, fill) -> np.ndarray:
    """float32[n]; fill(rng, m) returns float64[m] for one chunk."""
    out = np.empty(n, dtype=np.float32)
    nchunks = (n + CHUNK - 1) // CHUNK

    def work(j):
        lo = j * CHUNK
        hi = min(n, lo + CHUNK)
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, j])))
        out[lo:hi] = fill(rng, hi - lo)

    if nchunks <= 1:
        for j in range(nchunks):
            work(j)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(work, range(nchunks)))
    return out


def normal(n: int, seed: int, sigma: float = 1.0) -> np.ndarray:
    return _chunked(n, seed, lambda rng, m: rng.normal(0.0, sigma, m))


def laplace(n: int, seed: int, scale: float) -> np.ndarray:
    return _chunked(n, seed, lambda rng, m: rng.laplace(0.0, scale, m))


def to_bf16_rne(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest even) and widen back."""
    u = x.view(np.uint32)
    out = np.empty_like(u)
    step = CHUNK
    for lo in range(0, u.size, step):
        s = u[lo:lo + step]
        lsb = (s >> np.uint32(16)) & np.uint32(1)
        out[lo:lo + step] = (s + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)
    return out.view(np.float32)


# ---------------------------------------------------------------- workloads

def flat_normal(step: int, n: int = 1 << 20, config: int = 1) -> np.ndarray:
    """grad ~ N(0, 1), fresh every step."""
    return normal(n, 1000 * config + step, 1.0)


def vgg16_scales(config: int = 2) -> np.ndarray:
    """b_l = 10**U(-4, -1), one per tensor, drawn once per run."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([1000 * config, 999])))
    return 10.0 ** rng.uniform(-4.0, -1.0, len(VGG16_SIZES))


def vgg16_bucket(step: int, sizes=None, config: int = 2):
    """Flat bucket of per-tensor Laplace(0, b_l) gradients.
    Returns (grad float32[sum n_l], offsets int64[T+1], k int64[T])."""
    sizes = list(VGG16_SIZES if sizes is None else sizes)
    b = vgg16_scales(config)
    offsets = np.zeros(len(sizes) + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(sizes)
    grad = np.empty(int(offsets[-1]), dtype=np.float32)
    for l, nl in enumerate(sizes):
        seed = 1000 * config + step
        grad[offsets[l]:offsets[l + 1]] = _chunked(
            nl, seed * 100 + l, lambda rng, m, s=b[l % len(b)]: rng.laplace(0.0, s, m))
    ks = np.array([(nl + 999) // 1000 for nl in sizes], dtype=np.int64)
    return grad, offsets, ks


def resnet50_mix(step: int, n: int = RESNET50_N, config: int = 3) -> np.ndarray:
    """90% Laplace(0, 1e-3) plus exactly round(0.1 n) positions (drawn
    without replacement, fresh each step) of 1e-2 * Student-t(3)."""
    seed = 1000 * config + step
    grad = laplace(n, seed, 1e-3)
    m = int(round(0.1 * n))
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 1 << 20])))
    pos = rng.choice(n, size=m, replace=False)
    grad[pos] = (1e-2 * rng.standard_t(3.0, m)).astype(np.float32)
    return grad


def density_k(n: int, density: float) -> int:
    """k = floor(density * n), computed without binary rounding surprises."""
    # density is one of 1e-2, 1e-3, 1e-4: use the exact decimal ratio.
    inv = round(1.0 / density)
    return n // inv


def gtopk_sets(P: int = 32, k: int = 25_557, n: int = RESNET50_N, config: int = 4,
               step: int = 0):
    """P index-sorted sets of k (int32 idx, float32 val) over [0, n)."""
    seed = 1000 * config + step
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 0])))
    nhot = min(2 * k, n)
    hot = rng.choice(n, size=nhot, replace=False)
    hot_mask = np.zeros(n, dtype=bool)
    hot_mask[hot] = True
    idx = np.empty((P, k), dtype=np.int32)
    val = np.empty((P, k), dtype=np.float32)
    if k > n:
        raise ValueError("k > n")
    khot = min(k // 2, nhot)
    for p in range(P):
        r = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 1 + p])))
        a = r.choice(hot, size=khot, replace=False)
        need = k - khot
        if n - nhot >= 4 * need:
            # rejection sampling over the indices outside the hot set
            rest = np.empty(0, dtype=np.int64)
            while rest.size < need:
                cand = r.integers(0, n, size=2 * (need - rest.size) + 16)
                cand = cand[~hot_mask[cand]]
                rest = np.unique(np.concatenate([rest, cand]))
        else:
            # small index space: draw from every index not taken yet
            taken = np.zeros(n, dtype=bool)
            taken[a] = True
            rest = np.nonzero(~taken)[0]
        if rest.size > need:
            rest = r.choice(rest, size=need, replace=False)
        s = np.sort(np.concatenate([a.astype(np.int64), rest]))
        idx[p] = s.astype(np.int32)
        val[p] = r.normal(0.0, 1e-2, k).astype(np.float32)
    return idx, val


def bf16_normal(step: int, n: int = LARGE_N, config: int = 5) -> np.ndarray:
    """grad = bf16-RNE(N(0, 1e-3)) widened to float32."""
    x = normal(n, 1000 * config + step, 1e-3)
    return to_bf16_rne(x)


def sizes_check() -> int:
    return int(sum(VGG16_SIZES))


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


__all__ = [
    "CHUNK", "VGG16_SIZES", "RESNET50_N", "LARGE_N", "normal", "laplace",
    "to_bf16_rne", "flat_normal", "vgg16_scales", "vgg16_bucket",
    "resnet50_mix", "density_k", "gtopk_sets", "bf16_normal", "ceil_div",
    "math",
]
