#!/usr/bin/env python
"""Throughput of the Top-k + error-feedback compress on B200.

Default workload: one error-feedback step on the ResNet-50-sized flat fp32
gradient (n = 25,557,032, 90% Laplace(0, 1e-3) + 10% 1e-2 * Student-t(3) at
random positions) with k = 25,557 (density 0.1%), lr = 0.1, the residual
carried from step to step.  A "step" is one topk_ef_compress call: the fused
accumulate pass, the threshold resolution and the ordered compaction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

Prints ONE JSON line (rank 0).  value = algorithmic GB/s of the whole job:
(12 B per element + 8 B per emitted pair) x elements of all ranks / device
time, max over ranks.  Device time is one CUDA-event interval around the K
back-to-back steps on the launching stream when a step's inputs (grad +
residual) exceed the 126 MB L2; for smaller inputs L2 is flushed (256 MiB
write) before each step and the device time is the sum of per-step event
intervals, the flush outside them.  Multi-GPU: every rank
compresses its own gradient (data-parallel replicas, no collective on the
data path); torch.distributed is used only for the barrier and the max.

--impl reference times the CPU oracle (oracle/, single thread) on a bounded
sample of the same workload and prints the same line with "impl":
"reference"; under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import datagen  # noqa: E402

METRIC = "Top-k+EF compress GB/s & elems/s at n=25.6M, density 0.1% (% of HBM peak)"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20
L2_BYTES = 126 << 20       # B200 L2; step inputs above this run back to back
TRACE_BRACKETS = 4         # timed region: events around at most this many dominant launches
LR = np.float32(0.1)
POOL = 4          # distinct gradients cycled through the steps
KERNEL_SOURCES = ["error_feedback_b200/csrc/kernels_stream.cuh",
                  "error_feedback_b200/csrc/kernels_compress.cuh",
                  "error_feedback_b200/csrc/common.cuh"]


# ------------------------------------------------------------------ helpers

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_max(x: float, device=None) -> float:
    """Max of x over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def sources_sha():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def traffic_per_launch(kernel: str, workload: str):
    """DRAM bytes (read + write) per launch of `kernel` from the committed ncu
    summary, for the workload it was captured on only; None if absent, for
    another workload, or if the kernel's sources changed since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)[kernel]
    except (OSError, KeyError, ValueError):
        return None
    if t.get("src_sha256") != sources_sha() or t.get("bench_workload") != workload:
        return None
    return float(t["dram_bytes"])


_SAMPLER_CHILD = r"""
import select, sys, time
import pynvml
pynvml.nvmlInit()
h = pynvml.nvmlDeviceGetHandleByUUID(sys.argv[1])
period = float(sys.argv[2])
reasons = (getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None)
           or pynvml.nvmlDeviceGetCurrentClocksThrottleReasons)
print("max", pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM), flush=True)
rows = []
while True:
    t = time.monotonic()
    rows.append((t, pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM), int(reasons(h))))
    if len(rows) == 1:
        print("ready", flush=True)
    r, _, _ = select.select([sys.stdin], [], [], period)
    if r and not sys.stdin.read(1):
        break
for t, m, rs in rows:
    print(t, m, rs)
"""


class ClockSampler:
    """Polls SM clock and throttle reasons through NVML while running.

    The polling runs in a child process: a thread of this process would take
    the interpreter lock from the loop that launches the timed steps and
    delay them.  Samples are stamped with the host's monotonic clock, and
    only those taken between entry and exit are kept."""

    def __init__(self, torch_dev: int, period_s: float = 0.0005, uuid: str | None = None):
        self.samples = []
        self.max_mhz = None
        self.err = None
        self.period = period_s
        self.proc = None
        self.uuid = uuid
        if uuid is None:
            try:
                import torch
                u = str(torch.cuda.get_device_properties(torch_dev).uuid)
                self.uuid = u if u.startswith("GPU-") else "GPU-" + u
            except Exception as e:  # noqa: BLE001
                self.err = f"{type(e).__name__}: {e}"

    def start(self):
        """Start polling (a child process: its start-up takes a fraction of a
        second, so start it before the warm-up, not just before timing)."""
        import select
        import subprocess
        self.t0 = time.monotonic()
        if self.uuid is None:
            return self
        try:
            self.proc = subprocess.Popen(
                [sys.executable, "-c", _SAMPLER_CHILD, self.uuid, str(self.period)],
                stdin=subprocess.PIPE, stdout=subprocess.PIPE, stderr=subprocess.PIPE)
            # unbuffered reads of the child's first lines (a buffered reader
            # would swallow lines that select() then never reports)
            fd = self.proc.stdout.fileno()
            head = b""
            deadline = time.monotonic() + 60
            while b"ready\n" not in head:
                left = deadline - time.monotonic()
                if left <= 0 or not select.select([fd], [], [], left)[0]:
                    raise RuntimeError("NVML sampler did not start")
                chunk = os.read(fd, 4096)
                if not chunk:
                    raise RuntimeError("NVML sampler exited: "
                                       + self.proc.stderr.read().decode(errors="replace")[-300:])
                head += chunk
            for line in head.decode().splitlines():
                if line.startswith("max "):
                    self.max_mhz = int(line.split()[1])
        except Exception as e:  # noqa: BLE001
            self.err = f"{type(e).__name__}: {e}"
            self._end()
        self.t0 = time.monotonic()
        return self

    def mark(self):
        """Keep only the samples taken from now on."""
        self.t0 = time.monotonic()

    def __enter__(self):
        return self.start()

    def _end(self):
        import subprocess
        if self.proc is None:
            return ""
        out = b""
        try:
            out, _ = self.proc.communicate(input=b"", timeout=30)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            self.proc.communicate()
            self.err = "NVML sampler did not stop"
        self.proc = None
        return out.decode(errors="replace")

    def __exit__(self, *a):
        self.stop()

    def stop(self):
        """Stop polling; keeps the samples taken since start() or mark()."""
        t1 = time.monotonic()
        rows = []
        for line in self._end().splitlines():
            f = line.split()
            if len(f) == 3:
                try:
                    rows.append((float(f[0]), int(f[1]), int(f[2])))
                except ValueError:
                    pass
        inside = [(m, r) for t, m, r in rows if self.t0 <= t <= t1]
        if not inside and rows:
            # a region shorter than the polling interval: the nearest sample
            t_mid = 0.5 * (self.t0 + t1)
            _, m, r = min(rows, key=lambda x: abs(x[0] - t_mid))
            inside = [(m, r)]
        self.samples = inside

    def summary(self):
        names = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
                 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
                 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0, "note": self.err or "no samples"}
        mask = 0
        for _, r in self.samples:
            mask |= r
        reasons = [v for k, v in names.items() if mask & k and v != "gpu_idle"]
        return {"sm_mhz": statistics.median(m for m, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples)}


# ---------------------------------------------------------------- workloads

def l2_note(flush: bool, input_bytes: int) -> str:
    if flush:
        return (f"flushed between steps (256 MiB write, not timed); step inputs "
                f"{input_bytes / 1e6:.0f} MB")
    return (f"no flush: step inputs {input_bytes / 1e6:.0f} MB (grad + residual) exceed the "
            f"126 MB L2; steps run back to back")


def hbm_bar(wl, frac):
    """The 60%-of-HBM bar set for the Top-k + EF compress of n >= 25.6M
    elements, measured on the whole call; other workloads are not held to it."""
    if isinstance(wl, (FlatCompress, BatchedCompress)) and wl.n >= datagen.RESNET50_N:
        return {"measured_on": "whole call (hbm_frac_whole_step): setup, streaming pass "
                               "and select", "bar": 0.60, "met": bool(frac >= 0.60)}
    return {"applies": False,
            "why": "the bar is set for the Top-k + EF compress of n >= 25.6M elements"}


class FlatCompress:
    """One EF step of topk_ef_compress on a flat gradient."""

    def __init__(self, name, n, k, make_grad, label):
        self.name, self.n, self.k, self.make_grad, self.label = name, n, k, make_grad, label
        self.bytes_per_step = 12 * n + 8 * k
        self.elems_per_step = n
        self.dominant = "stream_kernel"
        self.dominant_bytes = 12 * n     # read grad + read residual + write residual
        self.flush = 8 * n <= L2_BYTES

    def config(self):
        return {"workload": self.label, "n": self.n, "k": self.k, "lr": float(LR),
                "l2": l2_note(self.flush, 8 * self.n),
                "parallelism": "replicas (one independent EF step per GPU)"}

    def setup(self, rank, steps_needed):
        import torch
        import error_feedback_b200 as ef
        self.ef = ef
        # distinct gradients cycled through the steps (fewer for huge tensors)
        npool = min(POOL, max(1, steps_needed), max(1, int(16e9 // (4 * self.n))))
        self.host = [self.make_grad(100 * rank + s) for s in range(npool)]
        self.dev = [torch.from_numpy(g).cuda() for g in self.host]
        self.res = torch.zeros(self.n, dtype=torch.float32, device="cuda")
        self.oi = torch.empty(max(self.k, 1), dtype=torch.int32, device="cuda")[:self.k]
        self.ov = torch.empty(max(self.k, 1), dtype=torch.float32, device="cuda")[:self.k]
        self.ws = torch.empty(ef.topk_ef_workspace_bytes(self.n, self.k), dtype=torch.uint8,
                              device="cuda")
        # host-buffer path: pinned gradient, device staging, pinned outputs
        self.hpin = [torch.from_numpy(g).pin_memory() for g in self.host]
        self.stage = torch.empty(self.n, dtype=torch.float32, device="cuda")
        self.hoi = torch.empty(max(self.k, 1), dtype=torch.int32).pin_memory()[:self.k]
        self.hov = torch.empty(max(self.k, 1), dtype=torch.float32).pin_memory()[:self.k]
        self.h2d_bytes = 4 * self.n
        self.d2h_bytes = 8 * self.k

    def step(self, i):
        self.ef.topk_ef_compress(self.dev[i % len(self.dev)], self.res, LR, self.k,
                                 self.oi, self.ov, self.ws)

    def e2e_step(self, i):
        self.stage.copy_(self.hpin[i % len(self.hpin)], non_blocking=True)
        self.ef.topk_ef_compress(self.stage, self.res, LR, self.k, self.oi, self.ov, self.ws)
        self.hoi.copy_(self.oi, non_blocking=True)
        self.hov.copy_(self.ov, non_blocking=True)

    def status(self):
        return self.ef.topk_ef_last_device_status(self.ws)

    def path(self):
        return self.ef.topk_ef_path_info(self.ws)

    # CPU oracle on a bounded sample of the workload
    def oracle_sample(self, budget_elems):
        ns = int(min(self.n, max(1 << 16, budget_elems)))
        ks = ns // max(1, round(self.n / max(self.k, 1))) if self.k else 0
        ks = min(ks, ns)
        g = self.make_grad(0)[:ns].copy()
        return ns, ks, g


class BatchedCompress:
    """One EF step of topk_ef_compress_batched on the VGG-16 bucket."""

    def __init__(self):
        g, off, ks = datagen.vgg16_bucket(0)
        self.offsets, self.ks = off, ks
        self.n = int(off[-1])
        self.k = int(ks.sum())
        self.bytes_per_step = 12 * self.n + 8 * self.k
        self.elems_per_step = self.n
        self.dominant = "stream_kernel"
        self.dominant_bytes = 12 * self.n
        self.flush = 8 * self.n <= L2_BYTES
        self._first = g

    def config(self):
        return {"workload": "vgg16_bucket: 16 VGG-16 weight tensors, Laplace(0, b_l), "
                            "k_l = ceil(n_l/1000)", "n": self.n, "k": self.k, "lr": float(LR),
                "l2": l2_note(self.flush, 8 * self.n),
                "parallelism": "replicas (one independent EF step per GPU)"}

    def setup(self, rank, steps_needed):
        import torch
        import error_feedback_b200 as ef
        self.ef = ef
        npool = min(2, max(1, steps_needed))
        host = [self._first] + [datagen.vgg16_bucket(s)[0] for s in range(1, npool)]
        self.dev = [torch.from_numpy(g).cuda() for g in host]
        self.hpin = [torch.from_numpy(g).pin_memory() for g in host]
        self.res = torch.zeros(self.n, dtype=torch.float32, device="cuda")
        self.oi = torch.empty(self.k, dtype=torch.int32, device="cuda")
        self.ov = torch.empty(self.k, dtype=torch.float32, device="cuda")
        self.ws = torch.empty(ef.topk_ef_batched_workspace_bytes(self.offsets, self.ks),
                              dtype=torch.uint8, device="cuda")
        self.stage = torch.empty(self.n, dtype=torch.float32, device="cuda")
        self.hoi = torch.empty(self.k, dtype=torch.int32).pin_memory()
        self.hov = torch.empty(self.k, dtype=torch.float32).pin_memory()
        self.h2d_bytes = 4 * self.n
        self.d2h_bytes = 8 * self.k

    def step(self, i):
        self.ef.topk_ef_compress_batched(self.dev[i % len(self.dev)], self.res, self.offsets,
                                         self.ks, LR, self.oi, self.ov, self.ws)

    def e2e_step(self, i):
        self.stage.copy_(self.hpin[i % len(self.hpin)], non_blocking=True)
        self.ef.topk_ef_compress_batched(self.stage, self.res, self.offsets, self.ks, LR,
                                         self.oi, self.ov, self.ws)
        self.hoi.copy_(self.oi, non_blocking=True)
        self.hov.copy_(self.ov, non_blocking=True)

    def status(self):
        return self.ef.topk_ef_last_device_status(self.ws)

    def path(self):
        return self.ef.topk_ef_path_info(self.ws)


class Merge:
    """One gTop-k tournament: P = 32 sets of k = 25,557 over n = 25,557,032."""

    def __init__(self, P=32, k=25_557, n=datagen.RESNET50_N):
        self.P, self.kin, self.k, self.nidx = P, k, k, n
        rounds = (P - 1).bit_length()
        # algorithmic bytes: every pair merge reads two sets and writes one
        merges = P - 1
        self.bytes_per_step = merges * 3 * 8 * k
        self.elems_per_step = P * k
        self.dominant = "merge_cluster_kernel"
        self.dominant_bytes = None
        self.flush = True
        self.rounds = rounds

    def config(self):
        return {"workload": f"gtopk_merge P={self.P} k={self.kin} n={self.nidx}",
                "P": self.P, "k": self.k, "n": self.nidx,
                "l2": "flushed between steps (256 MiB write); working set is L2-resident",
                "parallelism": "P workers simulated on each GPU"}

    def setup(self, rank, steps_needed):
        import torch
        import error_feedback_b200 as ef
        self.ef = ef
        idx, val = datagen.gtopk_sets(P=self.P, k=self.kin, n=self.nidx, step=rank)
        self.di = torch.from_numpy(idx).cuda()
        self.dv = torch.from_numpy(val).cuda()
        self.hi = torch.from_numpy(idx).pin_memory()
        self.hv = torch.from_numpy(val).pin_memory()
        self.oi = torch.empty(self.k, dtype=torch.int32, device="cuda")
        self.ov = torch.empty(self.k, dtype=torch.float32, device="cuda")
        self.oc = torch.empty(1, dtype=torch.int32, device="cuda")
        self.ws = torch.empty(ef.gtopk_merge_workspace_bytes(self.P, self.kin, self.k),
                              dtype=torch.uint8, device="cuda")
        self.si = torch.empty_like(self.di)
        self.sv = torch.empty_like(self.dv)
        self.hoi = torch.empty(self.k, dtype=torch.int32).pin_memory()
        self.hov = torch.empty(self.k, dtype=torch.float32).pin_memory()
        self.h2d_bytes = 8 * self.P * self.kin
        self.d2h_bytes = 8 * self.k

    def step(self, i):
        self.ef.gtopk_merge(self.di, self.dv, self.k, self.nidx, self.oi, self.ov, self.oc,
                            self.ws)

    def e2e_step(self, i):
        self.si.copy_(self.hi, non_blocking=True)
        self.sv.copy_(self.hv, non_blocking=True)
        self.ef.gtopk_merge(self.si, self.sv, self.k, self.nidx, self.oi, self.ov, self.oc,
                            self.ws)
        self.hoi.copy_(self.oi, non_blocking=True)
        self.hov.copy_(self.ov, non_blocking=True)

    def status(self):
        return self.ef.topk_ef_last_device_status(self.ws)

    def path(self):
        return {}


class ThresholdCompress:
    """One hard-threshold EF step (topk_ef_threshold) on the ResNet-50-sized
    mixed gradient, threshold 6e-3 (about 0.1% pass at the first step),
    max_out = 1% of n."""

    def __init__(self, thr=6e-3):
        self.n = datagen.RESNET50_N
        self.thr = thr
        self.max_out = self.n // 100
        self.elems_per_step = self.n
        self.dominant = "stream_kernel"
        self.dominant_bytes = 12 * self.n
        self.flush = False
        self.bytes_per_step = 12 * self.n      # + 8 per sent pair, set after warm-up

    def config(self):
        return {"workload": f"hard_threshold: resnet50_mix n={self.n:,}, |acc| >= {self.thr}, "
                            f"max_out={self.max_out:,}", "n": self.n, "lr": float(LR),
                "l2": l2_note(self.flush, 8 * self.n),
                "parallelism": "replicas (one independent EF step per GPU)"}

    def setup(self, rank, steps_needed):
        import torch
        import error_feedback_b200 as ef
        self.ef = ef
        npool = min(POOL, max(1, steps_needed))
        host = [datagen.resnet50_mix(100 * rank + s) for s in range(npool)]
        self.dev = [torch.from_numpy(g).cuda() for g in host]
        self.hpin = [torch.from_numpy(g).pin_memory() for g in host]
        self.res = torch.zeros(self.n, dtype=torch.float32, device="cuda")
        self.oi = torch.empty(self.max_out, dtype=torch.int32, device="cuda")
        self.ov = torch.empty(self.max_out, dtype=torch.float32, device="cuda")
        self.oc = torch.empty(1, dtype=torch.int64, device="cuda")
        self.ws = torch.empty(ef.topk_ef_threshold_workspace_bytes(self.n), dtype=torch.uint8,
                              device="cuda")
        self.stage = torch.empty(self.n, dtype=torch.float32, device="cuda")
        self.hoi = torch.empty(self.max_out, dtype=torch.int32).pin_memory()
        self.hov = torch.empty(self.max_out, dtype=torch.float32).pin_memory()
        self.hoc = torch.empty(1, dtype=torch.int64).pin_memory()
        self.h2d_bytes = 4 * self.n
        self.d2h_bytes = 8 * self.max_out + 8

    def after_warmup(self):
        sent = min(int(self.oc.cpu().item()), self.max_out)
        self.bytes_per_step = 12 * self.n + 8 * sent
        self.sent = sent

    def step(self, i):
        self.ef.topk_ef_threshold(self.dev[i % len(self.dev)], self.res, LR, self.thr,
                                  self.max_out, self.oi, self.ov, self.oc, self.ws)

    def e2e_step(self, i):
        self.stage.copy_(self.hpin[i % len(self.hpin)], non_blocking=True)
        self.ef.topk_ef_threshold(self.stage, self.res, LR, self.thr, self.max_out, self.oi,
                                  self.ov, self.oc, self.ws)
        self.hoc.copy_(self.oc, non_blocking=True)
        self.hoi.copy_(self.oi, non_blocking=True)
        self.hov.copy_(self.ov, non_blocking=True)

    def status(self):
        return self.ef.topk_ef_last_device_status(self.ws)

    def path(self):
        return {"sent_per_step_after_warmup": getattr(self, "sent", None)}


class SparseAfterMerge:
    """The steps around the gTop-k merge on its configuration (P = 32 sets of
    k = 25,557 over n = 25,557,032): the residual return of the non-surviving
    sent values to all 32 workers' memories ([32][n] fp32), or the AllGather
    dense rank-order sum of all sets."""

    def __init__(self, kind, P=32, k=25_557, n=datagen.RESNET50_N):
        self.kind, self.P, self.k, self.n = kind, P, k, n
        self.elems_per_step = P * k
        self.flush = True
        self.dominant = "return_kernel" if kind == "return" else "ag_sum_kernel"

    def config(self):
        what = ("gtopk_residual_return: 32 workers' memories [32][n]" if self.kind == "return"
                else "topk_allgather_sum: dense rank-order sum of 32 sets")
        return {"workload": f"{what}, P={self.P} k={self.k} n={self.n}", "P": self.P,
                "k": self.k, "n": self.n,
                "l2": "flushed between steps (256 MiB write, not timed)",
                "parallelism": "P workers simulated on each GPU"}

    def setup(self, rank, steps_needed):
        import torch
        import error_feedback_b200 as ef
        self.ef = ef
        idx, val = datagen.gtopk_sets(P=self.P, k=self.k, n=self.n, step=rank)
        self.di = torch.from_numpy(idx).cuda()
        self.dv = torch.from_numpy(val).cuda()
        self.hi = torch.from_numpy(idx).pin_memory()
        self.hv = torch.from_numpy(val).pin_memory()
        self.si = torch.empty_like(self.di)
        self.sv = torch.empty_like(self.dv)
        if self.kind == "return":
            gi = torch.empty(self.k, dtype=torch.int32, device="cuda")
            gv = torch.empty(self.k, dtype=torch.float32, device="cuda")
            gc = torch.empty(1, dtype=torch.int32, device="cuda")
            ef.gtopk_merge(self.di, self.dv, self.k, self.n, gi, gv, gc)
            self.gidx = gi[:int(gc.cpu().item())].contiguous()
            self.res = torch.zeros((self.P, self.n), dtype=torch.float32, device="cuda")
            self.ws = torch.empty(ef.gtopk_residual_return_workspace_bytes(), dtype=torch.uint8,
                                  device="cuda")
            returned = int((~np.isin(idx, self.gidx.cpu().numpy())).sum())
            # read the sent sets and the global list, read and write each returned value
            self.bytes_per_step = 8 * self.P * self.k + 4 * self.gidx.numel() + 8 * returned
            self.h2d_bytes = 8 * self.P * self.k
            self.d2h_bytes = 0
        else:
            self.out = torch.empty(self.n, dtype=torch.float32, device="cuda")
            self.hout = torch.empty(self.n, dtype=torch.float32).pin_memory()
            self.ws = torch.empty(ef.topk_allgather_workspace_bytes(self.P, self.k, self.n),
                                  dtype=torch.uint8, device="cuda")
            # read the sets, write the dense sum
            self.bytes_per_step = 8 * self.P * self.k + 4 * self.n
            self.h2d_bytes = 8 * self.P * self.k
            self.d2h_bytes = 4 * self.n
        self.dominant_bytes = self.bytes_per_step

    def _run(self, i, si, sv):
        if self.kind == "return":
            self.ef.gtopk_residual_return(si, sv, self.gidx, self.res, ws=self.ws)
        else:
            self.ef.topk_allgather_sum(si, sv, self.n, out=self.out, ws=self.ws)

    def step(self, i):
        self._run(i, self.di, self.dv)

    def e2e_step(self, i):
        self.si.copy_(self.hi, non_blocking=True)
        self.sv.copy_(self.hv, non_blocking=True)
        self._run(i, self.si, self.sv)
        if self.kind != "return":
            self.hout.copy_(self.out, non_blocking=True)

    def status(self):
        return self.ef.topk_ef_last_device_status(self.ws)

    def path(self):
        return {}


def make_workload(name):
    n3 = datagen.RESNET50_N
    if name in ("resnet50_mix", "resnet50_mix_0.1pct"):
        return FlatCompress(name, n3, datagen.density_k(n3, 1e-3), datagen.resnet50_mix,
                            "resnet50_mix: n=25,557,032, 90% Laplace(0,1e-3) + 10% "
                            "1e-2*Student-t(3), k=25,557 (density 0.1%)")
    if name == "resnet50_mix_1pct":
        return FlatCompress(name, n3, datagen.density_k(n3, 1e-2), datagen.resnet50_mix,
                            "resnet50_mix n=25,557,032 k=255,570 (density 1%)")
    if name == "resnet50_mix_0.01pct":
        return FlatCompress(name, n3, datagen.density_k(n3, 1e-4), datagen.resnet50_mix,
                            "resnet50_mix n=25,557,032 k=2,555 (density 0.01%)")
    if name == "flat_normal_1m":
        return FlatCompress(name, 1 << 20, 1048, datagen.flat_normal,
                            "flat_normal: n=1,048,576 N(0,1), k=1,048")
    if name == "bf16_normal_1.5b":
        return FlatCompress(name, datagen.LARGE_N, 1_500_000, datagen.bf16_normal,
                            "bf16_normal: n=1.5e9, bf16-rounded N(0,1e-3), k=1.5e6")
    if name == "vgg16_bucket":
        return BatchedCompress()
    if name == "gtopk_merge_p32":
        return Merge()
    if name == "hard_threshold_resnet50":
        return ThresholdCompress()
    if name == "gtopk_return_p32":
        return SparseAfterMerge("return")
    if name == "allgather_sum_p32":
        return SparseAfterMerge("allgather")
    raise SystemExit(f"unknown workload {name}")


# --------------------------------------------------------------------- arms

def run_ours(args):
    import torch
    import torch.distributed as dist
    import error_feedback_b200 as ef

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    wl = make_workload(args.workload)
    if args.no_flush and wl.flush:
        wl.flush = False
        wl.l2_kept = True
    wl.setup(rank, args.steps + args.warmup)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()

    # clock polling starts before the warm-up, so that its start-up does not
    # leave the GPU idle just before the timed region
    clk = ClockSampler(local).start()
    for w in range(args.warmup):
        if wl.flush:
            flush.fill_(float(w))
        wl.step(w)
    barrier()
    st = wl.status()
    if st != 0:
        clk.stop()
        raise SystemExit(f"device status after warm-up: {ef.status_string(st)}")
    if hasattr(wl, "after_warmup"):
        wl.after_warmup()

    # launches per step and per-kernel times: a short fully traced run before
    # the timed region (tracing every launch breaks the overlap between them)
    nt = min(args.steps, 20)
    ef.topk_ef_trace_enable(True)
    for i in range(nt):
        if wl.flush:
            flush.fill_(float(i))
        wl.step(args.warmup + i)
    trace_all = ef.topk_ef_trace_read()
    ef.topk_ef_trace_enable(False)
    launches_per_step = len(trace_all) / nt

    # timed region: K steps; inputs larger than L2 run back to back, smaller
    # ones get an L2 flush before each step (outside the timed intervals).
    # Only the dominant kernel is bracketed by events, and only a few of its
    # launches spread over the region (one per twenty, at least one, at most
    # TRACE_BRACKETS):
    # events between two launches stop the second from starting early, so
    # every bracket slows the step it falls in.
    dom_launches = sum(1 for name, _ in trace_all if name == wl.dominant) * args.steps // nt
    brackets = min(TRACE_BRACKETS, max(1, dom_launches // 20))
    every = max(1, -(-dom_launches // brackets))
    ef.topk_ef_trace_enable(True, only=wl.dominant, every=every)
    barrier()
    clk.mark()
    if wl.flush:
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for i in range(args.steps):
            flush.fill_(float(i))
            ev[i][0].record(stream)
            wl.step(args.warmup + i)
            ev[i][1].record(stream)
    else:
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))]
        ev[0][0].record(stream)
        for i in range(args.steps):
            wl.step(args.warmup + i)
        ev[0][1].record(stream)
    barrier()
    clk.stop()
    trace = ef.topk_ef_trace_read()
    ef.topk_ef_trace_enable(False)
    st = wl.status()
    if st != 0:
        raise SystemExit(f"device status after timing: {ef.status_string(st)}")
    path = wl.path()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = reduce_max(float(sum(step_ms)), "cuda")
    units = world * args.steps
    gbs = units * wl.bytes_per_step / (total_ms * 1e-3) / 1e9
    eps = units * wl.elems_per_step / (total_ms * 1e-3)

    # dominant kernel, timed by the library's events on the launch stream
    dom = [ms for name, ms in trace if name == wl.dominant]
    launches = int(round(launches_per_step * args.steps))
    roof = None
    peak, peak_src = peaks()
    if dom and wl.dominant_bytes:
        avg = sum(dom) / len(dom)
        ach = wl.dominant_bytes / (avg * 1e-3) / 1e9
        roof = {"bound": "hbm", "kernel": wl.dominant, "achieved": round(ach, 1),
                "peak": peak, "unit": "GB/s", "frac": round(ach / peak, 4),
                "peak_source": f"{peak_src} (hbm_gbs, burst copy)",
                "traffic": traffic_per_launch(wl.dominant, args.workload),
                "algorithmic_bytes_per_launch": wl.dominant_bytes,
                "avg_launch_ms": round(avg, 5), "launches": len(dom)}
    per_kernel = {}
    for name, ms in trace_all:
        d = per_kernel.setdefault(name, [0, 0.0])
        d[0] += 1
        d[1] += ms

    # end to end through the C ABI with host buffers (pinned), copies timed
    e2e = None
    if not args.no_e2e:
        ke = min(args.steps, 50)
        ee = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(ke)]
        for w in range(2):
            wl.e2e_step(w)
        barrier()
        for i in range(ke):
            ee[i][0].record(stream)
            wl.e2e_step(i)
            ee[i][1].record(stream)
        barrier()
        e_ms = reduce_max(float(sum(a.elapsed_time(b) for a, b in ee)), "cuda")
        e2e = {"value": round(world * ke * wl.bytes_per_step / (e_ms * 1e-3) / 1e9, 2),
               "unit": "GB/s", "h2d_bytes_per_step": wl.h2d_bytes,
               "d2h_bytes_per_step": wl.d2h_bytes, "steps": ke,
               "ms_per_step": round(e_ms / ke, 4)}

    clocks = clk.summary()
    if world > 1:
        dist.barrier()
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(gbs, 2), "unit": "GB/s",
            "elems_per_s": round(eps, 1),
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total_ms / args.steps, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": wl.config(),
            "roofline": roof,
            "hbm_frac_whole_step": round(gbs / world / peak, 4),
            "hbm_bar": hbm_bar(wl, gbs / world / peak),
            "gpu_launches": launches,
            "kernels": {k: {"launches": v[0], "avg_ms": round(v[1] / v[0], 5)}
                        for k, v in per_kernel.items()},
            "path": path,
            "e2e": e2e,
            "clocks": clocks,
        }
        if getattr(wl, "l2_kept", False):
            line["config"]["l2"] = ("not flushed (--no-flush): the step's inputs stay in L2 and "
                                    "the steps run back to back")
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(wl, args)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def time_oracle(wl, steps, budget_elems):
    """Run the oracle (full-sort back-end, one thread) for `steps` EF steps on
    a bounded sample of the workload; returns (seconds, sample description,
    bytes per step, elems per step)."""
    import oracle
    o = oracle.get()
    if isinstance(wl, FlatCompress):
        ns, ks, g = wl.oracle_sample(budget_elems)
        res = np.zeros(ns, np.float32)
        t0 = time.perf_counter()
        for _ in range(steps):
            o.compress(g, res, LR, ks, 0)
        dt = time.perf_counter() - t0
        return dt, f"{steps} EF steps on the first {ns} elements (k={ks})", 12 * ns + 8 * ks, ns
    if isinstance(wl, BatchedCompress):
        g, off, ks = datagen.vgg16_bucket(0)
        res = np.zeros(g.size, np.float32)
        t0 = time.perf_counter()
        for _ in range(steps):
            o.compress_batched(g, res, off, ks, LR, 0)
        dt = time.perf_counter() - t0
        return dt, f"{steps} EF steps on the full bucket", wl.bytes_per_step, wl.elems_per_step
    if isinstance(wl, Merge):
        idx, val = datagen.gtopk_sets(P=wl.P, k=wl.kin, n=wl.nidx)
        t0 = time.perf_counter()
        for _ in range(steps):
            o.gtopk_merge(idx, val, wl.k, wl.nidx)
        dt = time.perf_counter() - t0
        return dt, f"{steps} full tournaments", wl.bytes_per_step, wl.elems_per_step
    if isinstance(wl, ThresholdCompress):
        ns = int(min(wl.n, budget_elems or wl.n))
        g = datagen.resnet50_mix(0)[:ns].copy()
        res = np.zeros(ns, np.float32)
        t0 = time.perf_counter()
        sent = 0
        for _ in range(steps):
            _, _, c = o.threshold(g, res, LR, wl.thr, ns // 100)
            sent += min(c, ns // 100)
        dt = time.perf_counter() - t0
        return (dt, f"{steps} hard-threshold steps on the first {ns} elements",
                12 * ns + 8 * sent // max(1, steps), ns)
    if isinstance(wl, SparseAfterMerge):
        idx, val = datagen.gtopk_sets(P=wl.P, k=wl.k, n=wl.n)
        if wl.kind == "return":
            gi, _ = o.gtopk_merge(idx, val, wl.k, wl.n)
            rows = 4                     # memories of 4 of the 32 workers (host RAM)
            res = np.zeros((rows, wl.n), np.float32)
            t0 = time.perf_counter()
            for _ in range(steps):
                o.residual_return(idx[:rows], val[:rows], gi, res)
            dt = time.perf_counter() - t0
            frac = rows / wl.P
            return (dt, f"{steps} residual returns to {rows} of the {wl.P} workers",
                    wl.bytes_per_step * frac if hasattr(wl, "bytes_per_step") else 8 * rows * wl.k,
                    rows * wl.k)
        t0 = time.perf_counter()
        for _ in range(steps):
            o.allgather_sum(idx, val, wl.n)
        dt = time.perf_counter() - t0
        return (dt, f"{steps} dense sums of all {wl.P} sets", 8 * wl.P * wl.k + 4 * wl.n,
                wl.elems_per_step)
    raise SystemExit("no oracle sample for this workload")


def time_multithreaded(wl, budget_s=3.0):
    """The OpenMP CPU baseline (cpu_baseline/, all host cores) on the same
    workload: fused fmaf, per-thread bounded heaps, a merge of the heaps.
    Returns None for workloads it does not cover."""
    import cpu_baseline as mtb
    nth = mtb.threads()
    if isinstance(wl, FlatCompress):
        ns = int(min(wl.n, 256 << 20))
        ks = ns // max(1, round(wl.n / max(wl.k, 1))) if wl.k else 0
        g = wl.make_grad(0)[:ns].copy()
        res = np.zeros(ns, np.float32)
        mtb.compress(g, res, LR, ks, nth)          # warm-up (page faults, threads)
        steps, t0 = 0, time.perf_counter()
        while True:
            mtb.compress(g, res, LR, ks, nth)
            steps += 1
            dt = time.perf_counter() - t0
            if dt > budget_s or steps >= 200:
                break
        sample = f"{steps} EF steps on the first {ns} elements (k={ks}), {nth} threads"
        return steps * (12 * ns + 8 * ks) / dt, steps * ns / dt, nth, sample, dt
    if isinstance(wl, BatchedCompress):
        g, off, ks = datagen.vgg16_bucket(0)
        res = np.zeros(g.size, np.float32)
        steps, t0 = 0, time.perf_counter()
        while True:
            for l in range(len(ks)):
                a, b = int(off[l]), int(off[l + 1])
                r = res[a:b]
                mtb.compress(g[a:b], r, LR, int(ks[l]), nth)
            steps += 1
            dt = time.perf_counter() - t0
            if dt > budget_s:
                break
        return (steps * wl.bytes_per_step / dt, steps * wl.elems_per_step / dt, nth,
                f"{steps} EF steps on the full bucket, {nth} threads", dt)
    return None


def cpu_baseline(wl, args):
    budget = wl.elems_per_step if isinstance(wl, FlatCompress) else None
    if isinstance(wl, FlatCompress):
        # about 15 s of single-thread work at ~5M elements/s
        steps = max(1, min(3, int(75e6 // max(1, min(wl.n, 64 << 20)))))
        dt, sample, bps, eps = time_oracle(wl, steps, min(wl.n, 64 << 20))
    else:
        steps = 1
        dt, sample, bps, eps = time_oracle(wl, steps, budget)
    out = {"value": round(steps * bps / dt / 1e9, 4), "unit": "GB/s",
           "elems_per_s": round(steps * eps / dt, 1), "cores": 1, "kind": "oracle",
           "sample": sample, "seconds": round(dt, 3)}
    mt = time_multithreaded(wl)
    if mt is not None:
        gbs, eps_mt, nth, sample_mt, dt_mt = mt
        out["multithreaded"] = {"value": round(gbs / 1e9, 4), "unit": "GB/s",
                                "elems_per_s": round(eps_mt, 1), "cores": nth,
                                "kind": "openmp fmaf + per-thread heaps (cpu_baseline/)",
                                "sample": sample_mt, "seconds": round(dt_mt, 3)}
    return out


def run_reference(args):
    world, rank, local = dist_env()
    if rank != 0:
        return
    wl = make_workload(args.workload)
    # each step a bounded sample: the whole run stays near a minute
    per_step_elems = int(max(1 << 16, min(getattr(wl, "n", 1 << 20),
                                          300e6 / max(1, args.steps + args.warmup))))
    if args.ref_elems:
        per_step_elems = args.ref_elems
    if isinstance(wl, FlatCompress):
        ns, ks, g = wl.oracle_sample(per_step_elems)
        import oracle
        o = oracle.get()
        res = np.zeros(ns, np.float32)
        for _ in range(args.warmup):
            o.compress(g, res, LR, ks, 0)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            o.compress(g, res, LR, ks, 0)
        dt = time.perf_counter() - t0
        bps, eps = 12 * ns + 8 * ks, ns
        sample = f"each step: one EF step on the first {ns} elements (k={ks})"
    else:
        dt, sample, bps, eps = time_oracle(wl, args.steps, None)
    gbs = args.steps * bps / dt / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
        "elems_per_s": round(args.steps * eps / dt, 1),
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3 / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": wl.config(),
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="resnet50_mix")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-flush", action="store_true",
                    help="do not flush L2 between steps of a workload smaller than L2 "
                         "(steps then run back to back from L2)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-elems", type=int, default=0,
                    help="reference arm: elements per step (default: sized to ~1 min)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    world, _, _ = dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}: launch N>1 with torchrun")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
