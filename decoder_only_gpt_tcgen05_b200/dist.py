"""Data-parallel plumbing over torch.distributed (NCCL on GPUs, gloo in CPU tests).

Each rank runs forward + backward on its own rows of the global batch; the
gradient of the global mean loss is the average of the ranks' gradients of
their local mean losses (every rank holds the same number of tokens), and the
bits-per-byte sums add over ranks.  These helpers only move data between ranks:
all arithmetic of the step runs in the library's kernels.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_rows(n_rows: int, rank: int, world: int) -> slice:
    """The rows of an n_rows global batch that `rank` processes (equal shards)."""
    if n_rows % world:
        raise ValueError(f"global batch of {n_rows} rows does not split over {world} ranks")
    per = n_rows // world
    return slice(rank * per, (rank + 1) * per)


def allreduce_grads_(grads: torch.Tensor, group=None) -> torch.Tensor:
    """In place: grads <- mean over ranks (the gradient of the global mean loss)."""
    world = dist.get_world_size(group)
    if world > 1:
        dist.all_reduce(grads, op=dist.ReduceOp.SUM, group=group)
        grads.div_(world)
    return grads


def allreduce_bpb(sum_nats: torch.Tensor, sum_bytes: torch.Tensor, group=None):
    """Global (sum_nats, sum_bytes) from the ranks' sums; returns the tensors reduced in place."""
    if dist.get_world_size(group) > 1:
        dist.all_reduce(sum_nats, op=dist.ReduceOp.SUM, group=group)
        dist.all_reduce(sum_bytes, op=dist.ReduceOp.SUM, group=group)
    return sum_nats, sum_bytes
