"""Multi-process host logic of the benchmark on CPU (gloo, world size 2).

The compress path has no data exchange between ranks (each rank compresses
its own gradient), so the only cross-rank logic is the barrier and the
max-over-ranks of the device time; the reference arm runs on rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench
    got = bench.reduce_max(10.0 * (rank + 1) + 0.5)
    dist.barrier()
    q.put((rank, got))
    dist.destroy_process_group()


def test_reduce_max_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res == {0: 20.5, 1: 20.5}


def test_reduce_max_single_process():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.25) == 3.25


def test_reference_arm_under_torchrun():
    """torchrun with 2 ranks: rank 0 alone prints the reference line."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={port}", "bench.py", "--gpus", "2",
           "--steps", "3", "--warmup", "3", "--impl", "reference", "--ref-elems", "200000"]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
