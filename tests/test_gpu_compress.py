"""GPU parity of topk_ef_compress against the CPU oracle (bit-exact: identical
index sets, values and residuals at 0 ULP, every error-feedback step)."""
import numpy as np
import pytest
import torch

import datagen
import error_feedback_b200 as ef
from gpu_util import bits, run_compress_steps, to_dev

pytestmark = pytest.mark.gpu

LR = np.float32(0.1)


def _ws(n, k):
    return torch.empty(ef.topk_ef_workspace_bytes(n, k), dtype=torch.uint8, device="cuda")


def test_flat_normal_1m():
    """1,048,576 elements, N(0,1), k = 1,048, three EF steps with fresh
    gradients (the 1M flat workload)."""
    n, k = 1 << 20, 1048
    grads = [datagen.flat_normal(s) for s in range(3)]
    ws = _ws(n, k)
    run_compress_steps(grads, LR, k, ws=ws)
    info = ef.topk_ef_path_info(ws)
    # a tensor this small takes one launch (small_kernel, no setup)
    assert info["kernels"] == 1, info


# Small tensors (one wave of blocks): small_kernel lists the elements that
# reach the previous call's threshold and, when that list decides the top k
# (at least k and at most 8,192 of them), every block selects from that list
# after one exchange ("fallback" 0); otherwise every block runs the exact
# two-exchange select ("fallback" 1).  Both must give the oracle's answer bit for bit.
SK_CAP1 = 8192


def test_small_bench_sequence():
    """The 1M flat workload's own sequence: one residual through 32 EF steps
    whose gradients cycle through a pool of 4, as the benchmark runs it.
    Early steps widen |acc| too fast for the previous threshold; later ones
    take it."""
    n, k = 1 << 20, 1048
    pool = [datagen.flat_normal(s) for s in range(4)]
    ws = _ws(n, k)
    paths = []
    run_compress_steps([pool[i % 4] for i in range(32)], LR, k, ws=ws, paths=paths)
    assert paths[0]["fallback"] == 1            # no threshold yet
    late = [p["fallback"] for p in paths[16:]]
    assert late.count(0) >= 14, [(p["fallback"], p["candidates"]) for p in paths]
    for p in paths:
        assert p["kernels"] == 1
        assert p["fallback"] == 1 or k <= p["candidates"] <= SK_CAP1, p


def test_small_threshold_misses_both_ways():
    """The threshold hint stays valid while the caller zeroes the residual,
    so acc = lr * grad: steady gradients take it; a step with gradients 1000x
    smaller leaves fewer than k above it, the next step at full scale puts
    almost every element above the small step's threshold; both fall back to
    the exact path and the step after takes the hint again."""
    n, k = 1 << 20, 1048
    rng = np.random.default_rng(5)
    scale = [1, 1, 1, 1, 1e-3, 1, 1, 1]
    grads = [(rng.standard_normal(n) * s).astype(np.float32) for s in scale]
    ws = _ws(n, k)
    paths = []
    run_compress_steps(grads, LR, k, ws=ws, paths=paths, zero_between=True)
    got = [p["fallback"] for p in paths]
    assert got == [1, 0, 0, 0, 1, 1, 0, 0], [(p["fallback"], p["candidates"]) for p in paths]
    assert paths[4]["candidates"] < k and paths[5]["candidates"] > SK_CAP1


def test_small_hint_ties():
    """3,000 entries of magnitude exactly 1.0 among values below 0.4: the k-th
    key is shared by all of them, the threshold path sees exactly those
    3,000 and must keep the k lowest indices."""
    n, k = 100_000, 1000
    rng = np.random.default_rng(8)
    grads = []
    for _ in range(4):
        g = rng.uniform(-0.4, 0.4, n).astype(np.float32)
        pos = rng.choice(n, 3000, replace=False)
        g[pos] = rng.choice(np.array([1.0, -1.0], np.float32), 3000)
        grads.append(g)
    ws = _ws(n, k)
    paths = []
    run_compress_steps(grads, np.float32(1.0), k, ws=ws, paths=paths, zero_between=True)
    assert [p["fallback"] for p in paths] == [1, 0, 0, 0], paths
    assert all(p["candidates"] == 3000 for p in paths[1:]), paths


@pytest.mark.parametrize("k,paths", [(200, [1, 0, 0, 0]), (50, None)])
def test_small_hint_special_values(k, paths):
    """NaN, +-Inf and -0 among small normal values: the NaNs rank first (one
    key above +Inf).  With k = 200 the k-th key is a normal value and the
    threshold path counts the specials in its open top bin; with k = 50 the
    infinities share the k-th key, far above the threshold's bins, and the
    lower indices must win (the exact path takes that case)."""
    n = 50_000
    rng = np.random.default_rng(9)
    grads = []
    for _ in range(4):
        g = (rng.standard_normal(n) * 1e-3).astype(np.float32)
        pos = rng.choice(n, 100, replace=False)
        g[pos[:30]] = np.float32(np.nan)
        g[pos[30:50]] = np.float32(np.inf)
        g[pos[50:70]] = np.float32(-np.inf)
        g[pos[70:]] = np.float32(-0.0)
        grads.append(g)
    ws = _ws(n, k)
    got = []
    run_compress_steps(grads, np.float32(1.0), k, ws=ws, paths=got, zero_between=True)
    if paths is not None:
        assert [p["fallback"] for p in got] == paths, got


@pytest.mark.parametrize("offset", [1, 2, 3])
def test_small_hint_unaligned(offset):
    """grad/residual not 16-byte aligned on the threshold path."""
    n, k = 300_007, 301
    rng = np.random.default_rng(20 + offset)
    grads = [rng.standard_normal(n).astype(np.float32) for _ in range(4)]
    ws = _ws(n, k)
    paths = []
    run_compress_steps(grads, LR, k, offset_elems=offset, ws=ws, paths=paths, zero_between=True)
    assert [p["fallback"] for p in paths][1:] == [0, 0, 0], paths


@pytest.mark.parametrize("n,k,path", [(5000, 100, 0), (8192, 8192, 0), (8192, 5, 0),
                                      (8193, 5, 1), (20_000, 100, 1)])
def test_small_threshold_zero(n, k, path):
    """Test flag bit 1 (threshold 0): every element is a candidate, so a
    tensor of at most 8,192 elements takes the threshold path over its whole
    key range and a larger one the exact path."""
    rng = np.random.default_rng(n)
    grads = [rng.standard_normal(n).astype(np.float32) for _ in range(2)]
    ws = _ws(n, k)
    paths = []
    old = ef.topk_ef_set_test_flags(2)
    try:
        run_compress_steps(grads, LR, k, ws=ws, paths=paths)
    finally:
        ef.topk_ef_set_test_flags(old)
    assert [p["fallback"] for p in paths] == [path, path], paths


@pytest.mark.parametrize("fill", [0x00, 0xFF, 0xA5])
def test_small_workspace_contents(fill):
    """The kernel needs no cleared state: a workspace of zeros, of ones or of
    a pattern gives exact results from the first call on."""
    n, k = 1 << 20, 1048
    ws = torch.full((ef.topk_ef_workspace_bytes(n, k),), fill, dtype=torch.uint8, device="cuda")
    rng = np.random.default_rng(fill)
    grads = [rng.standard_normal(n).astype(np.float32) for _ in range(3)]
    run_compress_steps(grads, LR, k, ws=ws, zero_between=True)


def test_small_two_residuals_one_workspace():
    """Two tensors' steps interleaved on one workspace: each call's hint is
    tagged with its residual, so neither takes the other's threshold."""
    import oracle
    o = oracle.get()
    n, k = 400_000, 400
    rng = np.random.default_rng(31)
    ws = _ws(n, k)
    ores = [np.zeros(n, np.float32), np.zeros(n, np.float32)]
    dres = [torch.zeros(n, dtype=torch.float32, device="cuda") for _ in range(2)]
    for step in range(6):
        t = step % 2
        g = (rng.standard_normal(n) * (1.0 if t == 0 else 1e-4)).astype(np.float32)
        gi, gv = ef.topk_ef_compress(to_dev(g), dres[t], LR, k, ws=ws)
        assert ef.topk_ef_last_device_status(ws) == 0
        oi, ov = o.compress(g, ores[t], LR, k, 0)
        from gpu_util import assert_same_step
        assert_same_step(step, gi, gv, dres[t], oi, ov, ores[t])


def test_small_graph_replay():
    """One compress call captured in a CUDA graph and replayed with new
    gradients: every replay is exact (the launch parameters repeat, the
    workspace's call counter keeps the replays apart)."""
    import oracle
    o = oracle.get()
    n, k = 1 << 20, 1048
    pool = [datagen.flat_normal(s) for s in range(4)]
    ws = _ws(n, k)
    g = torch.empty(n, dtype=torch.float32, device="cuda")
    dres = torch.zeros(n, dtype=torch.float32, device="cuda")
    oi_ = torch.empty(k, dtype=torch.int32, device="cuda")
    ov_ = torch.empty(k, dtype=torch.float32, device="cuda")
    ores = np.zeros(n, np.float32)
    # two eager steps (the library's one-time device queries happen here)
    for step in range(2):
        g.copy_(torch.from_numpy(pool[step]))
        ef.topk_ef_compress(g, dres, LR, k, oi_, ov_, ws=ws)
        oi, ov = o.compress(pool[step], ores, LR, k, 0)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            ef.topk_ef_compress(g, dres, LR, k, oi_, ov_, ws=ws)
    torch.cuda.current_stream().wait_stream(s)
    paths = []
    from gpu_util import assert_same_step
    for step in range(2, 14):
        g.copy_(torch.from_numpy(pool[step % 4]))
        graph.replay()
        torch.cuda.synchronize()
        assert ef.topk_ef_last_device_status(ws) == 0
        paths.append(ef.topk_ef_path_info(ws)["fallback"])
        oi, ov = o.compress(pool[step % 4], ores, LR, k, 0)
        assert_same_step(step, oi_, ov_, dres, oi, ov, ores)
    del graph
    assert 0 in paths, paths


@pytest.mark.parametrize("n,k", [
    (1, 1), (1, 0), (2, 1), (5, 5), (31, 7), (1000, 1), (1000, 999), (8191, 100),
    (8192, 8192), (8193, 3), (65535, 65), (65537, 66), (100003, 100), (300001, 3000),
    (2_000_003, 2), (777_777, 77_777),
])
def test_shapes(n, k):
    rng = np.random.default_rng(n * 7 + k)
    grads = [rng.standard_normal(n).astype(np.float32) for _ in range(2)]
    res0 = (rng.standard_normal(n) * 0.05).astype(np.float32)
    run_compress_steps(grads, LR, k, res0=res0, ws=_ws(n, k))


def test_empty():
    ws = _ws(0, 0)
    g = torch.empty(0, dtype=torch.float32, device="cuda")
    r = torch.empty(0, dtype=torch.float32, device="cuda")
    i, v = ef.topk_ef_compress(g, r, LR, 0, ws=ws)
    assert i.numel() == 0 and ef.topk_ef_last_device_status(ws) == 0


@pytest.mark.parametrize("n,k", [(200_001, 5000), (1_000_000, 123_457), (70_000, 1),
                                 (3_000_001, 30_000), (2_600_000, 1)])
def test_heavy_ties(n, k):
    """Magnitudes from a handful of values: the threshold is shared by
    thousands of entries and the lower indices must win."""
    rng = np.random.default_rng(n + k)
    pool = np.array([0.5, -0.5, 1.0, -1.0, 0.25, 2.0, -2.0, 0.0], np.float32)
    grads = [rng.choice(pool, n) for _ in range(3)]
    run_compress_steps(grads, np.float32(1.0), k, ws=_ws(n, k))


def test_concentrated_candidates():
    """n = 3,000,017 with k = 25,000 and 30,000 large values in one
    contiguous run: the candidates crowd into one or two select blocks'
    ranges (more than one shared-memory staging round there) and into tiles
    of more than 32 candidates (rescanned from the residual).  Three EF
    steps; the streaming pass + select path, no rescan of the whole residual."""
    n, k = 3_000_017, 25_000
    rng = np.random.default_rng(77)
    grads = []
    for s in range(3):
        g = rng.laplace(0, 1e-3, n).astype(np.float32)
        a = 1_234_567 + 1000 * s
        g[a:a + 30_000] = (rng.uniform(1.0, 2.0, 30_000) *
                           np.where(rng.random(30_000) < 0.5, -1, 1)).astype(np.float32)
        grads.append(g)
    ws = _ws(n, k)
    run_compress_steps(grads, LR, k, backend=1, ws=ws)
    info = ef.topk_ef_path_info(ws)
    assert info["fallback"] == 0 and info["kernels"] == 3, info


def test_all_equal_magnitude():
    n, k = 150_000, 4321
    rng = np.random.default_rng(3)
    g = np.where(rng.random(n) < 0.5, np.float32(0.75), np.float32(-0.75)).astype(np.float32)
    run_compress_steps([g], np.float32(1.0), k, ws=_ws(n, k))


@pytest.mark.parametrize("n,k", [(120_001, 1200), (2_500_001, 2500)])
def test_special_values(n, k):
    """NaN, +-Inf, +-0 and subnormals mixed into a normal gradient (one size
    for the one-kernel path, one for the streaming pass + select)."""
    rng = np.random.default_rng(5)
    g = rng.standard_normal(n).astype(np.float32)
    sp = np.array([np.nan, np.inf, -np.inf, 0.0, -0.0, 1e-45, -1e-45, 1e-40, 3e38, -3e38],
                  np.float32)
    pos = rng.choice(n, 500, replace=False)
    g[pos] = rng.choice(sp, 500)
    res0 = np.zeros(n, np.float32)
    res0[rng.choice(n, 100, replace=False)] = np.float32(-0.0)
    run_compress_steps([g, g], np.float32(1.0), k, res0=res0, ws=_ws(n, k))


@pytest.mark.parametrize("offset,n,k", [(1, 300_007, 301), (2, 300_007, 301), (3, 300_007, 301),
                                        (1, 2_600_003, 2600), (3, 2_600_003, 2600)])
def test_unaligned_base(offset, n, k):
    """grad/residual not 16-byte aligned: the scalar paths must agree."""
    rng = np.random.default_rng(offset)
    grads = [rng.standard_normal(n).astype(np.float32) for _ in range(2)]
    run_compress_steps(grads, LR, k, offset_elems=offset, ws=_ws(n, k))


@pytest.mark.parametrize("flags", [1, 2])
def test_forced_fallback(flags):
    """bit 0: force the residual rescan; bit 1: prefilter threshold 0, which
    overflows the candidate capacity and so also ends in the rescan."""
    n, k = 3_000_017, 3000
    rng = np.random.default_rng(11 + flags)
    grads = [rng.laplace(0, 1e-3, n).astype(np.float32) for _ in range(2)]
    ws = _ws(n, k)
    old = ef.topk_ef_set_test_flags(flags)
    try:
        run_compress_steps(grads, LR, k, ws=ws)
        info = ef.topk_ef_path_info(ws)
    finally:
        ef.topk_ef_set_test_flags(old)
    assert info["fallback"] == 1, info


def test_sampler_defeated():
    """Only the prefilter's sample positions hold large values (the library
    samples 128 evenly spread runs of 64 consecutive elements), so the
    threshold estimate sits above the k-th magnitude and fewer than k elements
    pass it: the rescan fallback must give the exact answer."""
    n, k = 4_000_000, 20_000
    g = np.full(n, 1e-6, np.float32)
    starts = (np.arange(128, dtype=np.int64) * n) >> 7
    sampled = (starts[:, None] + np.arange(64)[None, :]).reshape(-1)
    mask = np.ones(n, bool)
    mask[sampled] = False
    pos = np.nonzero(mask)[0][::7][:50_000]
    g[pos] = np.float32(1.0) + np.arange(pos.size, dtype=np.float32) * np.float32(1e-4)
    g[sampled] = np.float32(10.0)
    ws = _ws(n, k)
    run_compress_steps([g], np.float32(1.0), k, ws=ws)
    info = ef.topk_ef_path_info(ws)
    assert info["fallback"] == 1 and info["candidates"] < k, info


def test_deterministic():
    n, k = 5_000_000, 5000
    g = datagen.laplace(n, 77, 1e-3)
    out = []
    for _ in range(2):
        dg = to_dev(g)
        dr = torch.zeros(n, dtype=torch.float32, device="cuda")
        i, v = ef.topk_ef_compress(dg, dr, LR, k)
        out.append((i.cpu().numpy(), bits(v.cpu().numpy()), bits(dr.cpu().numpy())))
    for a, b in zip(out[0], out[1]):
        assert np.array_equal(a, b)


@pytest.mark.parametrize("density", [1e-2, 1e-3, 1e-4])
def test_resnet50_mix_full(density):
    """n = 25,557,032 (ResNet-50 sized) mixed Laplace / Student-t gradient,
    k = floor(density * n); all 10 EF steps of the workload, every one
    compared bit for bit (later steps carry larger memories and more
    candidates, and take the previous step's prefilter threshold)."""
    n = datagen.RESNET50_N
    k = datagen.density_k(n, density)
    ws = _ws(n, k)
    run_compress_steps((datagen.resnet50_mix(s) for s in range(10)), LR, k, backend=1, ws=ws,
                       n=n)
    info = ef.topk_ef_path_info(ws)
    assert info["fallback"] == 0, info


def test_bench_sequence_64_steps():
    """The benchmark's own sequence at the headline size (n = 25,557,032,
    k = 25,557): one residual carried through 64 EF steps whose gradients
    cycle through the same pool of 4 the benchmark uses; every step compared
    with the oracle."""
    n = datagen.RESNET50_N
    k = datagen.density_k(n, 1e-3)
    pool = [datagen.resnet50_mix(s) for s in range(4)]
    ws = _ws(n, k)
    run_compress_steps((pool[i % 4] for i in range(64)), LR, k, backend=1, ws=ws, n=n)
    assert ef.topk_ef_path_info(ws)["fallback"] == 0


@pytest.mark.slow
def test_bf16_ties_1p5b_full():
    """n = 1.5e9 (6 GB gradient + 6 GB residual), grad = bf16-rounded
    N(0, 1e-3) so |acc| has heavy ties, k = 1,500,000, three EF steps; every
    step compared bit for bit with the oracle (bounded-heap back-end).  The
    oracle's residual is compared on the device to keep host memory down."""
    import oracle
    n, k = datagen.LARGE_N, 1_500_000
    o = oracle.get()
    ores = np.zeros(n, np.float32)
    dres = torch.zeros(n, dtype=torch.float32, device="cuda")
    ws = _ws(n, k)
    for step in range(3):
        g = datagen.bf16_normal(step)
        dg = torch.from_numpy(g).cuda()
        gi, gv = ef.topk_ef_compress(dg, dres, LR, k, ws=ws)
        assert ef.topk_ef_last_device_status(ws) == 0
        del dg
        oi, ov = o.compress(g, ores, LR, k, 1)
        del g
        assert np.array_equal(gi.cpu().numpy(), oi), f"step {step}: index sets differ"
        assert np.array_equal(bits(gv.cpu().numpy()), bits(ov)), f"step {step}: values differ"
        dor = torch.from_numpy(ores).cuda()
        same = torch.equal(dor.view(torch.int32), dres.view(torch.int32))
        del dor
        assert same, f"step {step}: residuals differ"
    info = ef.topk_ef_path_info(ws)
    assert info["fallback"] == 0, info


def test_index_width_boundary():
    """n = 2^31 - 1, the largest n the int32 indices allow (indices up to
    2^31 - 2; the last warp tile holds 1,023 elements).  The gradient, drawn
    on the device, is small everywhere (|g| in [1e-4, 1e-2]) except the last
    1,000 elements (|g| in [1, 2]), so the top k = 600 lie in that tail and the
    oracle on the tail alone gives the expected output; the residual must be
    RN(lr * g) = fmaf(lr, g, 0) everywhere except the 600 sent slots (+0),
    checked in full on the device and on a 2^20-element sample against the
    oracle's own accumulate.  One EF step from a zero residual."""
    import oracle
    n, k, tail = (1 << 31) - 1, 600, 1000
    gen = torch.Generator(device="cuda")
    gen.manual_seed(2_147_483_647)
    g = torch.empty(n, dtype=torch.float32, device="cuda")
    g.uniform_(1e-4, 1e-2, generator=gen)
    sign = torch.empty(n, dtype=torch.float32, device="cuda").bernoulli_(0.5, generator=gen)
    g.mul_(sign.mul_(2).sub_(1))
    del sign
    rng = np.random.default_rng(31)
    gt = (rng.uniform(1.0, 2.0, tail) * np.where(rng.random(tail) < 0.5, -1, 1)).astype(np.float32)
    g[n - tail:] = torch.from_numpy(gt).cuda()
    res = torch.zeros(n, dtype=torch.float32, device="cuda")
    ws = _ws(n, k)
    gi, gv = ef.topk_ef_compress(g, res, LR, k, ws=ws)
    assert ef.topk_ef_last_device_status(ws) == 0
    o = oracle.get()
    rt = np.zeros(tail, np.float32)
    oi, ov = o.compress(gt, rt, LR, k, 1)
    assert np.array_equal(gi.cpu().numpy(), oi.astype(np.int64) + (n - tail))
    assert np.array_equal(bits(gv.cpu().numpy()), bits(ov))
    # the sample, against the oracle's accumulate (fmaf(lr, g, 0))
    pos = torch.from_numpy(np.sort(rng.choice(n - tail, 1 << 20, replace=False))).cuda()
    acc = o.accumulate(g[pos].cpu().numpy(), np.zeros(1 << 20, np.float32), LR)
    assert np.array_equal(bits(res[pos].cpu().numpy()), bits(acc))
    assert np.array_equal(bits(res[n - tail:].cpu().numpy()), bits(rt))
    # everywhere: fmaf(lr, g, +0) = RN(lr * g) for these magnitudes (no
    # product rounds to zero), +0 at the sent slots
    want = g.mul_(LR)
    want[gi.long()] = 0.0
    assert torch.equal(want.view(torch.int32), res.view(torch.int32))


@pytest.mark.parametrize("seed", range(8))
def test_small_random_sequences(seed):
    """Random small tensors (one wave of blocks, so small_kernel) with k
    small enough for the threshold hint, eight EF steps each over gradients
    whose scale drifts, some steps from a zeroed memory: both paths and their
    switches, every step compared bit for bit."""
    rng = np.random.default_rng(1000 + seed)
    n = int(rng.integers(1, 2_400_000))
    k = int(rng.integers(1, min(n, 2048) + 1))
    offset = int(rng.integers(0, 4))
    scales = np.exp(rng.normal(0.0, 0.3, 8)).astype(np.float32)
    grads = [(rng.standard_normal(n) * s).astype(np.float32) for s in scales]
    ws = _ws(n, k)
    paths = []
    run_compress_steps(grads, LR, k, offset_elems=offset, ws=ws, paths=paths,
                       zero_between=bool(seed % 2))
    assert all(p["kernels"] == 1 for p in paths), paths
