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


# ------------------------------------------------------------ bucketed, overlapped exchange

PRESET_NAMES = ("tiny", "gpt2", "d20", "d26")


def _lib_cfgs():
    import decoder_only_gpt_tcgen05_b200 as g
    cfgs = {n: g.preset(n) for n in PRESET_NAMES}
    cfgs["tied_ln_odd"] = g.preset("gpt2", n_layer=3, n_embd=64, n_head=2, vocab_size=100, block_size=32)
    cfgs["untied_rms_odd"] = g.preset("d20", n_layer=5, n_embd=64, n_head=1, vocab_size=100, block_size=32)
    return cfgs


def test_grad_buckets_cover_every_parameter_in_backward_order():
    """The buckets tile [0, P) exactly once; the head (final norm, untied lm_head) comes first, then
    the layers from the top down in the pairs the weight-gradient launches use, the embeddings last;
    every size is a multiple of 16, so any world size dividing 16 shards every bucket evenly."""
    from decoder_only_gpt_tcgen05_b200 import dist as D
    from decoder_only_gpt_tcgen05_b200.model import param_count, param_tensors
    for name, cfg in _lib_cfgs().items():
        bk = D.grad_buckets(cfg)
        P = param_count(cfg)
        spans = sorted((b, e) for b, e in bk if e > b)
        assert spans[0][0] == 0 and spans[-1][1] == P, name
        assert all(a[1] == b[0] for a, b in zip(spans, spans[1:])), name
        assert all((e - b) % 16 == 0 for b, e in bk), name
        layer_of = {}
        for t in param_tensors(cfg):
            if t[0].startswith("h"):
                layer_of.setdefault(t[0].split(".")[0], t[1])   # the layer's first tensor
        starts = [layer_of[f"h{l}"] for l in range(cfg.n_layer)]
        # completion order: descending positions, the embeddings (position 0) last
        mids = [b for b, e in bk[1:-1]]
        assert mids == sorted(mids, reverse=True) and bk[-1] == (0, starts[0]), name
        expected_layers = [l for l in range(cfg.n_layer - 1, -1, -1) if not (l & 1 and l > 0)]
        assert mids == [starts[l] for l in expected_layers], name


def test_shard_plan_partitions_buckets_and_decay_runs_follow_the_layout():
    from decoder_only_gpt_tcgen05_b200 import dist as D
    from decoder_only_gpt_tcgen05_b200.model import param_tensors
    for name, cfg in _lib_cfgs().items():
        bk = D.grad_buckets(cfg)
        mask = O.optim.decay_mask(O.Config(**__import__("dataclasses").asdict(cfg)))
        tensors = param_tensors(cfg)
        for world in (1, 2, 4, 8):
            owned = np.zeros(mask.size, np.int32)
            for rank in range(world):
                plan = D.shard_plan(bk, rank, world)
                s = 0
                for lo, hi, st in plan:
                    assert st == s
                    s += hi - lo
                    owned[lo:hi] += 1
                    starts, flags = D.decay_runs(tensors, lo, hi)
                    rebuilt = np.zeros(hi - lo, bool)
                    bounds = starts + [hi - lo]
                    for k, f in enumerate(flags):
                        rebuilt[bounds[k]:bounds[k + 1]] = f
                    assert starts[0] == 0 and np.array_equal(rebuilt, mask[lo:hi]), (name, world, rank)
                assert s * world == mask.size
            assert np.all(owned == 1), (name, world)


def _bucket_rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from decoder_only_gpt_tcgen05_b200 import dist as D
    import decoder_only_gpt_tcgen05_b200 as g
    cfg = g.preset("gpt2", n_layer=3, n_embd=64, n_head=2, vocab_size=100, block_size=32)
    bk = D.grad_buckets(cfg)
    P = max(e for _, e in bk)
    local = torch.from_numpy(synth.normal(P, 100 + rank)).float()
    whole = local.clone()
    dist.all_reduce(whole)
    whole.div_(world)
    res = {}
    for mode in ("allreduce", "reduce_scatter"):
        gb = local.clone()
        for b, e in bk:
            D.reduce_bucket_(gb, b, e, mode, rank, world)
        res[mode] = gb.numpy()
    out[rank] = (whole.numpy(), res)
    dist.destroy_process_group()


def test_bucketed_exchange_equals_one_whole_buffer_reduction():
    """Two gloo ranks: averaging bucket by bucket, in the backward's completion order, gives bitwise
    the whole-buffer average; in reduce_scatter mode each rank's owned slices are bitwise it too."""
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_bucket_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for pr in procs:
        pr.start()
    for pr in procs:
        pr.join(timeout=120)
        assert pr.exitcode == 0
    from decoder_only_gpt_tcgen05_b200 import dist as D
    import decoder_only_gpt_tcgen05_b200 as g
    bk = D.grad_buckets(g.preset("gpt2", n_layer=3, n_embd=64, n_head=2, vocab_size=100, block_size=32))
    for r in range(2):
        whole, res = out[r]
        assert np.array_equal(res["allreduce"], whole)
        for lo, hi, _ in D.shard_plan(bk, r, 2):
            assert np.array_equal(res["reduce_scatter"][lo:hi], whole[lo:hi])
