"""Parity of the optimizer step (gpt_adamw_step, gpt_op_adamw) with the optimizer oracle.

The oracle runs in float64 from the same fp32 starting values; the library computes in fp32 with an
fp64 gradient norm.  Bar: the norm within 1e-12 relative; parameters within 1e-6 |p| + 1e-5 lr over
three steps (fp32 rounding of p and of the update, which is of order lr); moments within 1e-5
relative.  The weight-decay split and the decay table's run boundaries are exact (a decayed element
that should not be, or the reverse, moves by lr * wd * |p|, far outside the bar)."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")
OPT = O.optim
HP = dict(lr=3e-3, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1)


def _pkg():
    import decoder_only_gpt_tcgen05_b200 as g
    return g


def _check(p, m, v, rp, rm, rv, lr):
    """m = beta1 m + (1 - beta1) g cancels where the two terms have opposite signs: there the fp32
    rounding of the terms (a few ulps of the moment's typical size) dominates, so each moment's
    bound carries an absolute part of 2e-6 of its largest magnitude next to the relative 1e-5."""
    p, m, v = (t.double().cpu().numpy() for t in (p, m, v))
    assert np.all(np.abs(p - rp) <= 1e-6 * np.abs(rp) + 1e-5 * lr), np.abs(p - rp).max()
    assert np.all(np.abs(m - rm) <= 1e-5 * np.abs(rm) + 2e-6 * np.abs(rm).max()), np.abs(m - rm).max()
    assert np.all(np.abs(v - rv) <= 1e-5 * np.abs(rv) + 2e-6 * np.abs(rv).max()), np.abs(v - rv).max()


CASES = {
    # LayerNorm + biases: 1-D and 2-D tensors alternate (many decay runs)
    "gpt2_small": ("gpt2", dict(n_layer=2, n_embd=128, n_head=2, vocab_size=1000, block_size=256)),
    # nanochat shape: every tensor decayed
    "d20_small": ("d20", dict(n_layer=2, n_embd=256, n_head=2, vocab_size=2048, block_size=512)),
}


@pytest.mark.parametrize("grad_clip,grad_scale", [(0.0, 1.0), (0.05, 1.0), (1e4, 0.5), (0.5, 0.25)])
@pytest.mark.parametrize("name", list(CASES))
def test_adamw_step_matches_oracle(name, grad_clip, grad_scale):
    g = _pkg()
    base, over = CASES[name]
    cfg = g.preset(base, **over)
    ocfg = O.Config(**dataclasses.asdict(cfg))
    model = g.GPT(cfg, 1, 16, device=DEV, seed=3)
    n = model.params.numel()
    model.params.copy_(torch.from_numpy(synth.normal(n, 5, std=0.3)))
    opt = g.AdamW(model, lr=HP["lr"], betas=(HP["beta1"], HP["beta2"]), eps=HP["eps"],
                  weight_decay=HP["weight_decay"], grad_clip=grad_clip)
    mask = OPT.decay_mask(ocfg)
    rp = model.params.double().cpu().numpy()
    rm, rv = np.zeros(n), np.zeros(n)
    for t in range(1, 4):
        gr = synth.normal(n, 20 + t, std=0.05)
        model.grads.copy_(torch.from_numpy(gr))
        norm = opt.step(grad_scale=grad_scale).item()
        rp, rm, rv, rnorm = OPT.adamw_step(rp, gr.astype(np.float64), rm, rv, t, HP["lr"], HP["beta1"], HP["beta2"],
                                           HP["eps"], HP["weight_decay"], mask, grad_scale=grad_scale,
                                           grad_clip=grad_clip)
        assert norm == pytest.approx(rnorm, rel=1e-12)
        _check(model.params, opt.m, opt.v, rp, rm, rv, HP["lr"])
    g.model.sync_status()


def _runs_to_mask(n, starts, decay):
    mask = np.zeros(n, dtype=bool)
    ends = list(starts[1:]) + [n]
    for s, e, d in zip(starts, ends, decay):
        mask[s:e] = bool(d)
    return mask


@pytest.mark.parametrize("n,starts", [
    (1001, [0, 3, 17, 18, 500, 997]),                      # runs cut float4 vectors, a 1-element run
    (5, [0, 1, 2, 3, 4]),                                  # every element its own run
    (4099, None),                                          # 300 random runs: several launches of the table
])
def test_adamw_op_decay_runs_match_oracle(n, starts):
    g = _pkg()
    rng = np.random.default_rng(n)
    if starts is None:
        starts = [0] + sorted(rng.choice(np.arange(1, n), size=299, replace=False).tolist())
    decay = [(i * 7 + 3) % 2 for i in range(len(starts))]
    p = torch.from_numpy(synth.normal(n, 31, std=0.5)).to(DEV)
    m0 = synth.normal(n, 32, std=0.01)
    m = torch.from_numpy(m0).to(DEV)
    # a second moment that could follow from such a first moment: v >= m^2
    v = torch.from_numpy((m0 * m0 + np.abs(synth.normal(n, 33, std=1e-4))).astype(np.float32)).to(DEV)
    gr = synth.normal(n, 34, std=0.1)
    grads = torch.from_numpy(gr).to(DEV)
    rp, rm, rv = (t.double().cpu().numpy() for t in (p, m, v))
    mask = _runs_to_mask(n, starts, decay)
    for t in (4, 5):                                       # a resumed state: step numbers above 1
        norm = g.ops.adamw(p, grads, m, v, starts, decay, t, lr=HP["lr"], beta1=HP["beta1"], beta2=HP["beta2"],
                           eps=HP["eps"], weight_decay=HP["weight_decay"], grad_clip=0.2).item()
        rp, rm, rv, rnorm = OPT.adamw_step(rp, gr.astype(np.float64), rm, rv, t, HP["lr"], HP["beta1"], HP["beta2"],
                                           HP["eps"], HP["weight_decay"], mask, grad_clip=0.2)
        assert norm == pytest.approx(rnorm, rel=1e-12)
        _check(p, m, v, rp, rm, rv, HP["lr"])


def test_adamw_is_deterministic_and_handles_empty_buffers():
    g = _pkg()
    n = 100_003
    base = torch.from_numpy(synth.normal(n, 41, std=0.5)).to(DEV)
    grads = torch.from_numpy(synth.normal(n, 42, std=0.1)).to(DEV)
    outs = []
    for _ in range(2):
        p, m, v = base.clone(), torch.zeros_like(base), torch.zeros_like(base)
        norm = g.ops.adamw(p, grads, m, v, [0, 50_000], [1, 0], 1, lr=1e-3, weight_decay=0.1, grad_clip=1.0)
        outs.append((p, m, v, norm.clone()))
    for a, b in zip(outs[0], outs[1]):
        assert torch.equal(a, b)
    e = torch.empty(0, dtype=torch.float32, device=DEV)
    norm = torch.full((), 7.0, dtype=torch.float64, device=DEV)
    g.ops.adamw(e, e, e, e, [], [], 1, lr=1e-3, grad_norm=norm)
    assert norm.item() == 0.0
