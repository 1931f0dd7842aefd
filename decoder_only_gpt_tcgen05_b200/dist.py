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


# ------------------------------------------------------------------ overlapped gradient exchange
#
# "Train your own ChatGPT", read the source optim.py: DistMuonAdamW (1) launches every gradient
# reduce_scatter at once so that communication overlaps compute, (2) updates only the slice of
# each parameter group a rank owns (the optimizer state is sharded the same way, ZeRO-2 style),
# (3) all-gathers the updated weights.  Here the backward marks each gradient bucket final with a
# CUDA event (gpt_backward_bucketed) and a communication stream reduces the bucket as soon as its
# event fires, while the backward goes on with the layers below.


def grad_buckets(cfg):
    """[(begin, end)] of the flat gradient, in the order the backward completes them."""
    import ctypes as C
    from ._lib import lib
    c = cfg.c()
    n = C.c_int32()
    rc = lib().gpt_grad_buckets(C.byref(c), 0, C.byref(n), None, None)
    if rc:
        raise RuntimeError(lib().gpt_last_error().decode())
    b = (C.c_int64 * n.value)()
    e = (C.c_int64 * n.value)()
    if lib().gpt_grad_buckets(C.byref(c), n.value, C.byref(n), b, e):
        raise RuntimeError(lib().gpt_last_error().decode())
    return [(int(b[k]), int(e[k])) for k in range(n.value)]


def shard_of(begin: int, end: int, rank: int, world: int):
    """The slice [b, e) of bucket [begin, end) that `rank` owns: equal parts, in rank order."""
    n = end - begin
    if n % world:
        raise ValueError(f"bucket of {n} elements does not split over {world} ranks")
    per = n // world
    return begin + rank * per, begin + (rank + 1) * per


def shard_plan(buckets, rank: int, world: int):
    """[(param_begin, param_end, state_begin)]: the owned slice of every non-empty bucket and where
    its optimizer state lives in this rank's (1 / world sized) state buffers."""
    plan, s = [], 0
    for b, e in buckets:
        if e <= b:
            continue
        lo, hi = shard_of(b, e, rank, world)
        plan.append((lo, hi, s))
        s += hi - lo
    return plan


def decay_runs(tensors, lo: int, hi: int):
    """Weight-decay run table of the element range [lo, hi): (starts relative to lo, flags), from
    [(name, offset, rows, cols)] of the layout (2-D tensors decay, as AdamW's groups do)."""
    starts, flags = [], []
    for _, off, rows, cols in tensors:
        a, z = max(off, lo), min(off + rows * cols, hi)
        if a >= z:
            continue
        d = cols > 1
        if not flags or flags[-1] != d:
            starts.append(a - lo)
            flags.append(d)
    return starts, flags


def _reduce_scatter_mean_(flat: torch.Tensor, lo: int, hi: int, rank: int, world: int, group=None):
    """flat[lo:hi] of this rank <- the mean over ranks of that slice; the rest of the bucket is left
    as it is (its owners hold it).  NCCL reduces in place; backends without reduce_scatter (gloo)
    all-reduce the bucket."""
    n = hi - lo
    b = lo - rank * n
    bucket = flat[b:b + world * n]
    if dist.get_backend(group) == "nccl":
        dist.reduce_scatter_tensor(flat[lo:hi], bucket, op=dist.ReduceOp.SUM, group=group)
    else:
        dist.all_reduce(bucket, op=dist.ReduceOp.SUM, group=group)
    flat[lo:hi].div_(world)


def _all_gather_(flat: torch.Tensor, lo: int, hi: int, rank: int, world: int, group=None):
    """Every rank's flat[bucket] <- the owners' slices (in place)."""
    n = hi - lo
    b = lo - rank * n
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(flat[b:b + world * n], flat[lo:hi], group=group)
    else:
        parts = [torch.empty_like(flat[lo:hi]) for _ in range(world)]
        dist.all_gather(parts, flat[lo:hi].contiguous(), group=group)
        for r in range(world):
            flat[b + r * n:b + (r + 1) * n].copy_(parts[r])


def reduce_bucket_(g: torch.Tensor, b: int, e: int, mode: str, rank: int, world: int, group=None):
    """One bucket [b, e) of the flat gradient: averaged over ranks (mode "allreduce"), or this rank's
    slice of it averaged (mode "reduce_scatter"; the rest of the bucket is then unspecified)."""
    if e <= b:
        return
    if mode == "allreduce":
        dist.all_reduce(g[b:e], op=dist.ReduceOp.SUM, group=group)
        g[b:e].div_(world)
    else:
        lo, hi = shard_of(b, e, rank, world)
        _reduce_scatter_mean_(g, lo, hi, rank, world, group)


class OverlappedGradSync:
    """Gradient exchange that overlaps the backward.

    mode "allreduce": every bucket is averaged over ranks (DDP: every rank then holds the whole
    mean gradient).  mode "reduce_scatter": each rank receives the mean of its own slice of every
    bucket only (ZeRO-2; see ShardedAdamW for the update and the all-gather of the weights)."""

    def __init__(self, model, mode: str = "allreduce", group=None):
        assert mode in ("allreduce", "reduce_scatter")
        self.model, self.mode, self.group = model, mode, group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.buckets = grad_buckets(model.cfg)
        self.plan = shard_plan(self.buckets, self.rank, self.world)
        self.events = [torch.cuda.Event() for _ in self.buckets]
        self.comm = torch.cuda.Stream(model.device)
        main = torch.cuda.current_stream(model.device)
        for ev in self.events:        # an event has a CUDA handle only once it has been recorded
            ev.record(main)

    def backward(self, accumulate: bool = False) -> torch.Tensor:
        """gpt_backward with each bucket reduced on the communication stream as soon as it is final;
        the current stream waits for the last reduction before it returns."""
        import ctypes as C
        from ._lib import call
        mdl = self.model
        main = torch.cuda.current_stream(mdl.device)
        handles = (C.c_void_p * len(self.events))(*[ev.cuda_event for ev in self.events])
        call("gpt_backward_bucketed", C.byref(mdl._c), mdl.params.data_ptr(), mdl.B, mdl.T, mdl.workspace.data_ptr(),
             mdl.ws_bytes, mdl.grads.data_ptr(), int(accumulate), handles, len(self.events), main.cuda_stream)
        g = mdl.grads
        with torch.cuda.stream(self.comm):
            for (b, e), ev in zip(self.buckets, self.events):
                self.comm.wait_event(ev)
                reduce_bucket_(g, b, e, self.mode, self.rank, self.world, self.group)
        main.wait_stream(self.comm)
        return g


class ShardedAdamW:
    """AdamW on this rank's slices of the parameter buffer only (gpt_op_adamw per slice, with the
    layout's weight-decay runs), the optimizer state sized 1 / world, then the weights all-gathered
    bucket by bucket: phases 2 and 3 of DistMuonAdamW's choreography for the AdamW groups.
    Gradient clipping is left out (a global norm would need one more reduction before the update)."""

    def __init__(self, sync: OverlappedGradSync, lr: float = 6e-4, betas=(0.9, 0.95), eps: float = 1e-8,
                 weight_decay: float = 0.1):
        assert sync.mode == "reduce_scatter"
        from .model import param_tensors
        self.sync, self.lr, self.betas, self.eps, self.wd = sync, lr, betas, eps, weight_decay
        mdl = sync.model
        n_state = sum(hi - lo for lo, hi, _ in sync.plan)
        self.m = torch.zeros(n_state, dtype=torch.float32, device=mdl.device)
        self.v = torch.zeros_like(self.m)
        tensors = param_tensors(mdl.cfg)
        self.runs = [decay_runs(tensors, lo, hi) for lo, hi, _ in sync.plan]
        self.step_count = 0
        from ._lib import lib
        self.scratch = torch.empty(int(lib().gpt_op_adamw_scratch_bytes()), dtype=torch.uint8, device=mdl.device)

    def step(self):
        from .ops import adamw
        mdl = self.sync.model
        self.step_count += 1
        for (lo, hi, s), (starts, flags) in zip(self.sync.plan, self.runs):
            n = hi - lo
            adamw(mdl.params[lo:hi], mdl.grads[lo:hi], self.m[s:s + n], self.v[s:s + n], starts, flags,
                  self.step_count, lr=self.lr, beta1=self.betas[0], beta2=self.betas[1], eps=self.eps,
                  weight_decay=self.wd, scratch=self.scratch)
        for lo, hi, _ in self.sync.plan:
            _all_gather_(mdl.params, lo, hi, self.sync.rank, self.sync.world, self.sync.group)
