"""A training step captured in a CUDA graph.

forward_loss + backward captured once and replayed must compute exactly what the eager calls
compute: every kernel argument (pointers, sizes, tensor maps) is fixed at capture, and the backward
has no atomics, so loss and gradients agree bit for bit, also after new tokens are copied into
the captured input buffers."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")

CASES = {
    "d20_small": ("d20", dict(n_layer=2, n_embd=256, n_head=2, vocab_size=2048, block_size=512), 2, 256),
    "gpt2_ragged": ("gpt2", dict(n_layer=1, n_embd=64, n_head=1, vocab_size=300, block_size=256), 3, 200),
}


@pytest.mark.parametrize("name", list(CASES))
def test_graph_replay_matches_eager_step(name):
    import decoder_only_gpt_tcgen05_b200 as g
    base, over, B, T = CASES[name]
    cfg = g.preset(base, **over)
    model = g.GPT(cfg, B, T, device=DEV, seed=0)
    batches = [synth.next_token_batch(B, T, cfg.vocab_size, seed=s) for s in (1, 2)]
    idx_d = torch.from_numpy(batches[0][0]).to(DEV)
    tgt_d = torch.from_numpy(batches[0][1]).to(DEV)

    def eager(k):
        idx_d.copy_(torch.from_numpy(batches[k][0]))
        tgt_d.copy_(torch.from_numpy(batches[k][1]))
        loss = model.forward_loss(idx_d, tgt_d).clone()
        return loss, model.backward().clone()

    ref = [eager(0), eager(1)]
    stream = torch.cuda.current_stream(DEV)
    side = torch.cuda.Stream(DEV)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        model.forward_loss(idx_d, tgt_d)
        model.backward()
    stream.wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        model.forward_loss(idx_d, tgt_d)
        model.backward()
    for k in (0, 1, 0):
        idx_d.copy_(torch.from_numpy(batches[k][0]))
        tgt_d.copy_(torch.from_numpy(batches[k][1]))
        model.grads.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize(DEV)
        assert torch.equal(model.loss, ref[k][0]), (k, model.loss.item(), ref[k][0].item())
        assert torch.equal(model.grads, ref[k][1]), k
    g.model.sync_status()
    del graph
    assert np.isfinite(ref[0][0].item())
