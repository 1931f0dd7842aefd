"""Data-parallel host logic with two gloo ranks on CPU.

Per-rank work is the oracle (the GPU path is not available here); what is
tested is the sharding and the reductions that bench.py and a training loop
use around the library: averaged per-rank gradients must equal the full-batch
gradient, and the reduced bpb sums must equal the full-batch bpb."""
import math
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
import synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from decoder_only_gpt_tcgen05_b200 import dist as D
    cfg = O.preset("tiny")
    p = O.init_params(cfg, 3) * 10
    idx, tgt = synth.next_token_batch(4, 16, cfg.vocab_size, dist="uniform", seed=7)
    tb = synth.byte_table(cfg.vocab_size, 1, 4, seed=8, n_zero=2)
    rows = D.shard_rows(idx.shape[0], rank, world)
    f = O.forward(cfg, p, idx[rows], tgt[rows])
    g = torch.from_numpy(O.backward(cfg, p, f))
    D.allreduce_grads_(g)
    s, b, _, _ = O.bits_per_byte(f["ell"], tgt[rows], tb)
    sn = torch.tensor([s], dtype=torch.float64)
    sb = torch.tensor([b], dtype=torch.int64)
    D.allreduce_bpb(sn, sb)
    out[rank] = (g.numpy(), float(sn.item()), int(sb.item()))
    dist.destroy_process_group()


def test_two_rank_gradient_average_and_bpb_sums():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for pr in procs:
        pr.start()
    for pr in procs:
        pr.join(timeout=120)
        assert pr.exitcode == 0
    cfg = O.preset("tiny")
    p = O.init_params(cfg, 3) * 10
    idx, tgt = synth.next_token_batch(4, 16, cfg.vocab_size, dist="uniform", seed=7)
    tb = synth.byte_table(cfg.vocab_size, 1, 4, seed=8, n_zero=2)
    f = O.forward(cfg, p, idx, tgt)
    g_full = O.backward(cfg, p, f)
    s, b, _, bpb = O.bits_per_byte(f["ell"], tgt, tb)
    for r in range(2):
        g, sn, sb = out[r]
        assert np.allclose(g, g_full, rtol=1e-12, atol=1e-15)
        assert sb == b and math.isclose(sn, s, rel_tol=1e-12)
        assert math.isclose(sn / (math.log(2) * sb), bpb, rel_tol=1e-12)


def test_shard_rows_partitions_the_batch():
    from decoder_only_gpt_tcgen05_b200 import dist as D
    seen = []
    for r in range(4):
        s = D.shard_rows(16, r, 4)
        seen += list(range(16))[s]
    assert seen == list(range(16))
    try:
        D.shard_rows(10, 0, 4)
        assert False
    except ValueError:
        pass
