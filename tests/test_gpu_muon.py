"""Parity of the split optimizer step (gpt_muon_step: Muon on the block matrices, AdamW on the rest)
with the optimizer oracle, over three steps with different gradients.

The oracle runs in float64 from the same fp32 starting values.  The library's Muon runs the
Newton-Schulz iteration in bf16 on the tensor cores, as the published Muon does, so each block
matrix's update (the parameter change of one step) is held to the bar of every gradient in this
suite: cosine >= 0.999 and relative L2 <= 3e-2 against the oracle's update, and the update's
singular values stay in the band the iteration lands them in.  The momentum buffer is plain fp32
arithmetic: within 1e-5 relative of the oracle's.  The other tensors take the AdamW step, with the
bar of the AdamW suite."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")
OPT = O.optim
HP = dict(lr=0.02, momentum=0.95, adam_lr=3e-3, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1)

CASES = {
    # LayerNorm + biases, tied: AdamW ranges between the matrices of every layer
    "gpt2_small": ("gpt2", dict(n_layer=2, n_embd=128, n_head=2, vocab_size=1000, block_size=256)),
    # nanochat shape: AdamW on wte and lm_head only; four matrix shapes, two of them transposed
    "d20_small": ("d20", dict(n_layer=3, n_embd=256, n_head=2, vocab_size=2048, block_size=512)),
    # more same-shape matrices than one grouped launch takes (8 per chunk)
    "d20_deep": ("d20", dict(n_layer=10, n_embd=128, n_head=1, vocab_size=512, block_size=512)),
    # 512-wide matrices: the symmetric products X X^T and A A skip the tiles below their diagonal
    # (128 x 256 tiles: 6 of 8 computed) and the lower triangles are copied from the upper ones
    "d20_wide": ("d20", dict(n_layer=1, n_embd=512, n_head=4, vocab_size=1024, block_size=256)),
}


def _cos_rel(a, b):
    a, b = a.reshape(-1), b.reshape(-1)
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b))), float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.mark.parametrize("nesterov", [True, False])
@pytest.mark.parametrize("name", list(CASES))
def test_muon_step_matches_oracle(name, nesterov):
    import decoder_only_gpt_tcgen05_b200 as g
    base, over = CASES[name]
    cfg = g.preset(base, **over)
    ocfg = O.Config(**dataclasses.asdict(cfg))
    model = g.GPT(cfg, 1, 16, device=DEV, seed=3)
    n = model.params.numel()
    model.params.copy_(torch.from_numpy(synth.normal(n, 5, std=0.3)))
    opt = g.MuonAdamW(model, lr=HP["lr"], momentum=HP["momentum"], nesterov=nesterov, ns_steps=5,
                      adam_lr=HP["adam_lr"], betas=(HP["beta1"], HP["beta2"]), eps=HP["eps"],
                      weight_decay=HP["weight_decay"])
    rp = model.params.double().cpu().numpy()
    rm = np.zeros(n)
    rv = np.zeros(n)
    offsets = O.param_offsets(ocfg)
    for t in (1, 2, 3):
        grads = synth.normal(n, 10 + t, std=0.01)
        model.grads.copy_(torch.from_numpy(grads))
        p_prev = model.params.double().cpu().numpy()
        opt.step()
        torch.cuda.synchronize()
        g.model.sync_status(DEV)
        rp_prev = rp
        rp, rm, rv = OPT.muon_adamw_step(ocfg, rp, grads.astype(np.float64), rm, rv, t, HP["lr"], HP["momentum"],
                                         nesterov, HP["adam_lr"], HP["beta1"], HP["beta2"], HP["eps"],
                                         HP["weight_decay"])
        p = model.params.double().cpu().numpy()
        mom = opt.mom.double().cpu().numpy()
        v = opt.v.double().cpu().numpy()
        for nm, (off, shape) in offsets.items():
            sl = slice(off, off + int(np.prod(shape)))
            if OPT.is_muon_tensor(nm):
                upd, ref = (p[sl] - p_prev[sl]).reshape(shape), (rp[sl] - rp_prev[sl]).reshape(shape)
                cos, rel = _cos_rel(upd, ref)
                assert cos >= 0.999 and rel <= 3e-2, (t, nm, cos, rel)
                sv = np.linalg.svd(upd / (-HP["lr"] * np.sqrt(max(1.0, shape[0] / shape[1]))), compute_uv=False)
                assert sv.max() <= 1.25, (t, nm, sv.max())
                # mu buf + (1 - mu) g cancels where the terms have opposite signs (as for AdamW's moments)
                assert np.all(np.abs(mom[sl] - rm[sl]) <= 1e-5 * np.abs(rm[sl]) + 2e-6 * np.abs(rm[sl]).max()), nm
                assert np.all(v[sl] == 0), nm
            else:
                lr = HP["adam_lr"]
                assert np.all(np.abs(p[sl] - rp[sl]) <= 1e-6 * np.abs(rp[sl]) + 1e-5 * lr), (t, nm)
                for a, b in ((mom[sl], rm[sl]), (v[sl], rv[sl])):
                    assert np.all(np.abs(a - b) <= 1e-5 * np.abs(b) + 2e-6 * np.abs(b).max()), (t, nm)
        # keep both sides on the same parameters: the next step starts from the library's values
        rp = p.copy()
        rm = mom.copy()
        rv = v.copy()


def test_muon_upper_triangle_tiles_in_cta_pairs():
    """The d20_wide case again with 256 x 256 CTA-pair tiles forced (GPT_GEMM_PAIR=1, read once per
    process, hence a child process): 3 of the 4 tiles of each symmetric product are computed."""
    import os
    import subprocess
    import sys
    env = dict(os.environ, GPT_GEMM_PAIR="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", "-m", "gpu",
                        f"{__file__}::test_muon_step_matches_oracle[d20_wide-True]"],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "1 passed" in r.stdout, r.stdout[-2000:]
