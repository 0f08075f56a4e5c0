"""The device side of the multi-rank gTopKAllReduce (error_feedback_b200.dist)
on the one GPU a run has.

- The tree replayed in one process: every "rank" is a row on the device, a
  send is the partner's row, and each merge is ``_device_merge`` (the
  library's gtopk_merge with P = 2, as a real rank runs it).  Rank 0's set
  must equal the oracle's tournament over all rows, bit for bit.
- gloo ranks (processes exchanging CPU tensors, receives posted ahead of the
  merges) whose merges copy the two sets to cuda:0, run ``_device_merge`` and
  copy the result back: every rank must end with the oracle's set.
The merges of different ranks never wait on one another on the device."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import datagen
import error_feedback_b200 as ef
import oracle
from error_feedback_b200.dist import _device_merge, tree_schedule

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,k,n", [(2, 1000, 50_000), (3, 2000, 100_000), (5, 3000, 200_000),
                                       (8, 4000, 1_000_000), (32, 25_557, datagen.RESNET50_N)])
def test_tree_replay_with_device_merges(world, k, n):
    idx, val = datagen.gtopk_sets(P=world, k=k, n=n, step=world + 11)
    ws = torch.empty(ef.gtopk_merge_workspace_bytes(2, k, k), dtype=torch.uint8, device="cuda")
    merge = _device_merge(ws)
    cur = {r: (torch.from_numpy(idx[r].copy()).cuda(), torch.from_numpy(val[r].copy()).cuda())
           for r in range(world)}
    sent = set()
    # rounds in order: all ranks' r-th steps
    sched = {r: tree_schedule(r, world) for r in range(world)}
    for rnd in range(max((len(s) for s in sched.values()), default=0)):
        for r in range(world):
            if rnd < len(sched[r]) and sched[r][rnd][0] == "recv":
                p = sched[r][rnd][1]
                assert sched[p][-1] == ("send", r) and p not in sent
                sent.add(p)
                ai, av = cur[r]
                bi, bv = cur[p]
                oi, ov = merge(torch.stack([ai, bi]), torch.stack([av, bv]), k, n)
                assert oi.numel() == k
                cur[r] = (oi, ov)
    gi, gv = cur[0]
    oi, ov = oracle.get().gtopk_merge(idx, val, k, n)
    assert np.array_equal(gi.cpu().numpy(), oi)
    assert np.array_equal(gv.cpu().numpy().view(np.uint32), ov.view(np.uint32))
    assert ef.topk_ef_last_device_status(ws) == 0


def _rank_main(rank, world, port, k, n, q):
    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import datagen
    import error_feedback_b200 as ef
    from error_feedback_b200.dist import _device_merge, gtopk_allreduce

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        torch.cuda.set_device(0)
        ws = torch.empty(ef.gtopk_merge_workspace_bytes(2, k, k), dtype=torch.uint8,
                         device="cuda")
        dev_merge = _device_merge(ws)

        def merge(in_idx, in_val, kk, nn):
            oi, ov = dev_merge(in_idx.cuda(), in_val.cuda(), kk, nn)
            st = ef.topk_ef_last_device_status(ws)
            assert st == 0, ef.status_string(st)
            return oi.cpu(), ov.cpu()

        idx, val = datagen.gtopk_sets(P=world, k=k, n=n, step=world)
        gi, gv = gtopk_allreduce(torch.from_numpy(idx[rank].copy()),
                                 torch.from_numpy(val[rank].copy()), k, n, merge=merge)
        q.put((rank, gi.numpy().copy(), gv.numpy().copy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 5])
def test_gloo_ranks_with_device_merges(world):
    k, n = 2000, 300_000
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, k, n, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        r, gi, gv = q.get(timeout=300)
        got[r] = (gi, gv)
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    idx, val = datagen.gtopk_sets(P=world, k=k, n=n, step=world)
    oi, ov = oracle.get().gtopk_merge(idx, val, k, n)
    for r in range(world):
        gi, gv = got[r]
        assert np.array_equal(gi, oi), r
        assert np.array_equal(gv.view(np.uint32), ov.view(np.uint32)), r
