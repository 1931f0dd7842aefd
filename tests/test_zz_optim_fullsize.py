"""The optimizer step at full size: GPT-2 124M (124,475,904 parameters) through gpt_adamw_step.

Kept apart from tests/test_gpu_optim.py: it holds the largest buffers of the optimizer tests and
is the last to run.  Same bar as there: the norm to 1e-12 relative (here against a float64 sum over
the whole buffer), and on 200,000 sampled elements parameters to 1e-6 |p| + 1e-5 lr, moments to
1e-5 relative plus 2e-6 of their largest magnitude."""
import numpy as np
import pytest
import torch

import oracle as O
from test_gpu_optim import DEV, OPT, _check, _pkg

pytestmark = pytest.mark.gpu


def test_adamw_full_size_gpt2_sampled():
    """GPT-2 124M (124,475,904 parameters): the norm against a float64 sum over the whole buffer,
    and 200,000 sampled elements against the oracle's elementwise step."""
    g = _pkg()
    cfg = g.preset("gpt2")
    ocfg = O.preset("gpt2")
    model = g.GPT(cfg, 1, 16, device=DEV, seed=0)
    n = model.params.numel()
    gen = torch.Generator(device=DEV).manual_seed(5)
    model.grads.copy_(torch.randn(n, generator=gen, device=DEV) * 1e-3)
    p0 = model.params.clone()
    opt = g.AdamW(model, lr=6e-4, betas=(0.9, 0.95), weight_decay=0.1, grad_clip=1.0)
    norm = opt.step().item()
    gd = model.grads.double()
    ref_norm = float(torch.sqrt((gd * gd).sum()))
    assert norm == pytest.approx(ref_norm, rel=1e-12)
    idx = np.sort(np.random.default_rng(0).choice(n, size=200_000, replace=False))
    ii = torch.from_numpy(idx).to(DEV)
    mask = OPT.decay_mask(ocfg)[idx]
    gs = model.grads[ii].double().cpu().numpy()
    factor = OPT.clip_coefficient(ref_norm, 1.0)
    # the step restricted to the sample, with the global norm's clip factor (grad_clip off inside)
    rp, rm, rv, _ = OPT.adamw_step(p0[ii].double().cpu().numpy(), gs * factor, np.zeros(idx.size), np.zeros(idx.size),
                                   1, 6e-4, 0.9, 0.95, 1e-8, 0.1, mask)
    _check(model.params[ii], opt.m[ii], opt.v[ii], rp, rm, rv, 6e-4)
    g.model.sync_status()
