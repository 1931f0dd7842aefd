"""The overlapped, bucketed gradient exchange on the GPU path.

- gpt_backward_bucketed writes bitwise the gradients of gpt_backward and records one event per
  bucket of gpt_grad_buckets.
- Two ranks (processes) on one GPU with gloo for the host-side exchange (no kernel of one rank
  waits for the other): each takes half of the batch; the bucket-by-bucket average, issued on a
  communication stream while the backward runs, equals the full batch's gradient (the loss is a
  mean, so the halves' mean gradients average to it), and after a ZeRO-2 style step (reduce-scatter
  of the gradient, AdamW on the owned slices, all-gather of the weights) both ranks hold the same
  weights, those of one AdamW step on the full-batch gradient."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import synth

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")
CFG = dict(n_layer=3, n_embd=128, n_head=1, vocab_size=512, block_size=256)


def _cos_rel(a, b):
    a, b = a.reshape(-1), b.reshape(-1)
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b))), float(np.linalg.norm(a - b) / np.linalg.norm(b))


def test_bucketed_backward_equals_plain_backward():
    import decoder_only_gpt_tcgen05_b200 as g
    from decoder_only_gpt_tcgen05_b200 import dist as D
    cfg = g.preset("gpt2", **CFG)
    model = g.GPT(cfg, 2, 256, device=DEV, seed=1)
    idx, tgt = synth.next_token_batch(2, 256, cfg.vocab_size, seed=2)
    idx, tgt = torch.from_numpy(idx).to(DEV), torch.from_numpy(tgt).to(DEV)
    model.forward_loss(idx, tgt)
    ref = model.backward().clone()
    events = [torch.cuda.Event() for _ in D.grad_buckets(cfg)]
    for ev in events:
        ev.record()
    import ctypes as C
    from decoder_only_gpt_tcgen05_b200._lib import call
    model.forward_loss(idx, tgt)
    h = (C.c_void_p * len(events))(*[ev.cuda_event for ev in events])
    call("gpt_backward_bucketed", C.byref(model._c), model.params.data_ptr(), model.B, model.T,
         model.workspace.data_ptr(), model.ws_bytes, model.grads.data_ptr(), 0, h, len(events),
         torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert torch.equal(model.grads, ref)
    assert all(ev.query() for ev in events)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=120))
    import decoder_only_gpt_tcgen05_b200 as g
    from decoder_only_gpt_tcgen05_b200 import dist as D
    torch.cuda.set_device(0)
    cfg = g.preset("gpt2", **CFG)
    B, T = 4, 256
    idx, tgt = synth.next_token_batch(B, T, cfg.vocab_size, seed=3)
    rows = D.shard_rows(B, rank, world)
    half = g.GPT(cfg, B // world, T, device=DEV, seed=4)
    params0 = half.params.clone()
    i_d = torch.from_numpy(idx[rows].copy()).to(DEV)
    t_d = torch.from_numpy(tgt[rows].copy()).to(DEV)
    res = {}
    # DDP style: every bucket averaged
    sync = D.OverlappedGradSync(half, "allreduce")
    half.forward_loss(i_d, t_d)
    res["allreduce"] = sync.backward().cpu().numpy().copy()
    # ZeRO-2 style: reduce-scatter, AdamW on the owned slices, all-gather the weights
    zs = D.OverlappedGradSync(half, "reduce_scatter")
    opt = D.ShardedAdamW(zs, lr=1e-3, betas=(0.9, 0.95), eps=1e-8, weight_decay=0.1)
    half.forward_loss(i_d, t_d)
    zs.backward()
    opt.step()
    torch.cuda.synchronize()
    res["params_after"] = half.params.cpu().numpy().copy()
    # the full batch on one rank: gradient and one AdamW step without clipping
    full = g.GPT(cfg, B, T, device=DEV, params=params0.clone())
    full.forward_loss(torch.from_numpy(idx).to(DEV), torch.from_numpy(tgt).to(DEV))
    res["full_grad"] = full.backward().cpu().numpy().copy()
    ad = g.AdamW(full, lr=1e-3, betas=(0.9, 0.95), eps=1e-8, weight_decay=0.1, grad_clip=0.0)
    ad.step()
    torch.cuda.synchronize()
    res["full_params_after"] = full.params.cpu().numpy().copy()
    out[rank] = res
    dist.destroy_process_group()


def test_two_ranks_on_one_gpu_match_the_full_batch():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for pr in procs:
        pr.start()
    for pr in procs:
        pr.join(timeout=300)
        assert pr.exitcode == 0
    r0, r1 = out[0], out[1]
    # the averaged gradient: the full batch's, up to the order of the fp32 sums
    for r in (r0, r1):
        cos, rel = _cos_rel(r["allreduce"], r["full_grad"])
        assert cos >= 0.99999 and rel <= 1e-4, (cos, rel)
    assert np.array_equal(r0["allreduce"], r1["allreduce"])
    # after the sharded step both ranks hold the same weights, those of the full-batch step
    assert np.array_equal(r0["params_after"], r1["params_after"])
    # AdamW's first step moves each weight by about lr * g / (|g| + eps): where |g| is far above
    # eps the two gradients' rounding differences vanish in it; near zero the step may differ, but
    # never by more than its size, 2 lr
    d = np.abs(r0["params_after"] - r0["full_params_after"])
    big = np.abs(r0["full_grad"]) > 1e-6
    assert d[big].max() <= 1e-5, d[big].max()
    assert d.max() <= 2e-3 + 1e-6, d.max()
