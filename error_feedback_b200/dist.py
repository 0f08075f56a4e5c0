"""gTopKAllReduce across the ranks of a torch.distributed process group.

"A Distributed Synchronous SGD Algorithm with Global Top-k Sparsification
for Low Bandwidth Networks" (review page, method section 提出的方法: the
global top-k is found by a tournament in O(log P) rounds, each worker
exchanging one k-pair set per round; ABSTRACT: O(k log P) communication):
after each worker has sparsified its gradient to k (index, value) pairs, the
workers reduce their sets along a binary tree in log2 P rounds and the
result, the global top-k set, is broadcast to all of them.

Round r (step s = 2^r): rank i with i mod 2s == s sends its set to rank
i - s and leaves the tree; rank i with i mod 2s == 0 and a partner i + s < P
receives the partner's set and merges the two with the library's gTop-k
merge (P = 2: values summed at coinciding indices, then the k largest |value|,
lower index first, index-ascending).  These are the pairs and the round order
of the single-device tournament (``gtopk_merge`` over P rows), so rank 0 ends
with the same set, bit for bit.  Rank 0 then broadcasts it.

Only the exchange happens here (torch.distributed point-to-point and
broadcast: NCCL for CUDA tensors, one k-pair set per message); every merge
runs in the library's kernels.  A rank posts the receives of all its rounds
before its first merge, so a partner's set travels while this rank is still
merging earlier rounds: each round's transfer overlaps the merge before it.
``merge`` may be replaced by a callable with the same contract, which the
CPU tests use to check the exchange schedule with gloo.
"""
import torch

__all__ = ["gtopk_allreduce", "tree_schedule"]


def tree_schedule(rank: int, world: int):
    """The rounds of ``rank`` in the reduction tree, in order: a list of
    ("recv", partner) and ("send", partner) steps; a sender leaves the tree
    after its send."""
    steps = []
    s = 1
    while s < world:
        if rank % (2 * s) == s:
            steps.append(("send", rank - s))
            break
        if rank % (2 * s) == 0 and rank + s < world:
            steps.append(("recv", rank + s))
        s *= 2
    return steps


def _device_merge(ws):
    from . import gtopk_merge

    def merge(in_idx, in_val, k, n):
        oi, ov, _ = gtopk_merge(in_idx, in_val, k, n, ws=ws)
        return oi, ov

    return merge


def gtopk_allreduce(idx, val, k, n, group=None, merge=None, ws=None):
    """Global top-k of the ranks' sparse sets.

    idx: int32[k] strictly ascending indices in [0, n); val: float32[k]; both
    contiguous, on the device the group communicates from (CUDA for NCCL).
    Every rank passes the same k and n.  Returns (idx, val) of the global set
    on every rank (new tensors; the inputs are not modified).  ws: optional
    workspace for the merges (``gtopk_merge_workspace_bytes(2, k, k)``
    bytes).  Collective: every rank of the group must call it.
    """
    import torch.distributed as dist

    k = int(k)
    if idx.dim() != 1 or idx.shape != val.shape or idx.numel() != k:
        raise ValueError("idx and val must both be [k]")
    if idx.dtype != torch.int32 or val.dtype != torch.float32:
        raise ValueError("idx must be int32 and val float32")
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)

    def glob(r):
        return r if group is None else dist.get_global_rank(group, r)

    if merge is None:
        merge = _device_merge(ws)
    cur_i, cur_v = idx.contiguous(), val.contiguous()
    steps = tree_schedule(rank, world)
    # every receive of this rank's tree, posted before the first merge
    recvs = []
    for kind, partner in steps:
        if kind == "recv":
            ri = torch.empty_like(cur_i)
            rv = torch.empty_like(cur_v)
            works = [dist.irecv(ri, src=glob(partner), group=group),
                     dist.irecv(rv, src=glob(partner), group=group)]
            recvs.append((ri, rv, works))
    nr = 0
    for kind, partner in steps:
        if kind == "send":
            dist.send(cur_i, dst=glob(partner), group=group)
            dist.send(cur_v, dst=glob(partner), group=group)
        else:
            ri, rv, works = recvs[nr]
            nr += 1
            for w in works:
                w.wait()
            cur_i, cur_v = merge(torch.stack([cur_i, ri]), torch.stack([cur_v, rv]), k, n)
    out_i = cur_i.clone() if rank == 0 else torch.empty_like(idx)
    out_v = cur_v.clone() if rank == 0 else torch.empty_like(val)
    dist.broadcast(out_i, src=glob(0), group=group)
    dist.broadcast(out_v, src=glob(0), group=group)
    return out_i, out_v
