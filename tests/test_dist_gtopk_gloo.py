"""Host logic of the multi-rank gTopKAllReduce (error_feedback_b200.dist) on
CPU: the exchange schedule, and whole runs over gloo with 1-5 ranks whose
local merges are the oracle's, compared with the oracle's single-device
tournament over all the ranks' sets (the result must be the same, bit for
bit, on every rank)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from error_feedback_b200.dist import tree_schedule  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", range(1, 18))
def test_tree_schedule_is_the_tournament(world):
    """Replaying every rank's schedule merges the same pairs, in the same
    rounds and with the same left/right order, as the tournament of the
    gTop-k merge: worker i with i + 2^r for i = 0 mod 2^(r+1)."""
    sched = {r: tree_schedule(r, world) for r in range(world)}
    # each non-zero rank sends exactly once, as its last step; rank 0 never sends
    for r in range(world):
        kinds = [k for k, _ in sched[r]]
        assert kinds.count("send") == (0 if r == 0 else 1)
        if r:
            assert kinds[-1] == "send"
    # receives of rank i, in order, against the tournament's pairs
    rounds = []
    s = 1
    while s < world:
        rounds.append([(i, i + s) for i in range(0, world, 2 * s) if i + s < world])
        s *= 2
    for i in range(world):
        mine = [p for kind, p in sched[i] if kind == "recv"]
        want = [b for pairs in rounds for a, b in pairs if a == i]
        assert mine == want
    # every receive is matched by the partner's send to this rank, made after
    # the partner's own receives (its set is complete when sent)
    for i in range(world):
        for kind, p in sched[i]:
            if kind == "recv":
                assert sched[p][-1] == ("send", i)
    # replay: the leaves rank 0 ends with, in tournament order
    sets = {r: [r] for r in range(world)}
    for pairs in rounds:
        for a, b in pairs:
            sets[a] = sets[a] + sets[b]
    assert sorted(sets[0]) == list(range(world))


def _rank_main(rank, world, port, k, n, q):
    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import datagen
    import oracle
    from error_feedback_b200.dist import gtopk_allreduce

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        o = oracle.get()
        idx, val = datagen.gtopk_sets(P=world, k=k, n=n, step=world)

        def merge(in_idx, in_val, kk, nn):
            oi, ov = o.gtopk_merge(in_idx.numpy(), in_val.numpy(), kk, nn)
            assert oi.size == kk
            return torch.from_numpy(oi.copy()), torch.from_numpy(ov.copy())

        gi, gv = gtopk_allreduce(torch.from_numpy(idx[rank].copy()),
                                 torch.from_numpy(val[rank].copy()), k, n, merge=merge)
        q.put((rank, gi.numpy().copy(), gv.numpy().copy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [1, 2, 3, 4, 5])
def test_allreduce_matches_single_device_tournament(world):
    sys.path.insert(0, ROOT)
    import datagen
    import oracle

    k, n = 300, 20_000
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, k, n, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        r, gi, gv = q.get(timeout=180)
        got[r] = (gi, gv)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    idx, val = datagen.gtopk_sets(P=world, k=k, n=n, step=world)
    oi, ov = oracle.get().gtopk_merge(idx, val, k, n)
    for r in range(world):
        gi, gv = got[r]
        assert np.array_equal(gi, oi), r
        assert np.array_equal(gv.view(np.uint32), ov.view(np.uint32)), r


def _single_rank_checks(port, q):
    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    from error_feedback_b200.dist import gtopk_allreduce

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=0, world_size=1)
    errs = []
    try:
        i = torch.arange(4, dtype=torch.int32)
        v = torch.ones(4, dtype=torch.float32)
        for bad in [(i.long(), v, 4), (i, v.double(), 4), (i, v, 3), (i[:3], v, 3)]:
            try:
                gtopk_allreduce(*bad, n=10)
                errs.append("accepted a bad argument")
            except ValueError:
                pass
        # one rank: no exchange, the set comes back as a new tensor
        gi, gv = gtopk_allreduce(i, v, 4, 10)
        if not (torch.equal(gi, i) and torch.equal(gv, v)) or gi.data_ptr() == i.data_ptr():
            errs.append("single rank result")
    finally:
        dist.destroy_process_group()
    q.put(errs)


def test_argument_checks_and_single_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_single_rank_checks, args=(_free_port(), q))
    p.start()
    errs = q.get(timeout=120)
    p.join(60)
    assert p.exitcode == 0 and errs == []
