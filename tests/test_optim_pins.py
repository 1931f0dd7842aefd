"""Pins of the optimizer oracle (oracle/optim_oracle.py) to outside facts.

The nanoGPT page names the routines of its step: PyTorch's fused AdamW with two parameter groups
(2-D tensors decayed, 1-D not) and clip_grad_norm_ before it.  Those library routines, run in
float64 on the CPU, are the reference for the oracle's step; the learning-rate schedule is pinned to
the closed-form values of the page's warmup + cosine formula.  No GPU."""
import math

import numpy as np
import pytest
import torch

import oracle as O
import synth

OPT = O.optim


def _cfg(**kw):
    base = dict(n_layer=2, n_embd=16, n_head=2, block_size=16, vocab_size=19, norm=O.NORM_LN, linear_bias=1,
                tie_embed=1, act=O.ACT_GELU, pos=O.POS_LEARNED)
    base.update(kw)
    return O.Config(**base)


@pytest.mark.parametrize("grad_clip,grad_scale", [(0.0, 1.0), (0.05, 1.0), (1e3, 0.25), (0.3, 0.5)])
def test_adamw_matches_torch_adamw_with_clip_grad_norm(grad_clip, grad_scale):
    cfg = _cfg()
    n = O.param_count(cfg)
    shapes = O.param_shapes(cfg)
    p0 = synth.normal(n, 1, std=0.5).astype(np.float64)
    grads = [synth.normal(n, 10 + k, std=0.1).astype(np.float64) for k in range(3)]
    lr, b1, b2, eps, wd = 3e-3, 0.9, 0.95, 1e-8, 0.1

    # library: one tensor per parameter, 2-D ones decayed
    ts, off = [], 0
    for _, s in shapes:
        k = int(np.prod(s))
        ts.append(torch.tensor(p0[off:off + k].reshape(s), dtype=torch.float64, requires_grad=True))
        off += k
    groups = [{"params": [t for t in ts if t.dim() == 2], "weight_decay": wd},
              {"params": [t for t in ts if t.dim() < 2], "weight_decay": 0.0}]
    opt = torch.optim.AdamW(groups, lr=lr, betas=(b1, b2), eps=eps, foreach=False)

    mask = OPT.decay_mask(cfg)
    p, m, v = p0.copy(), np.zeros(n), np.zeros(n)
    for t, g in enumerate(grads, start=1):
        off = 0
        for tt in ts:
            k = tt.numel()
            tt.grad = torch.tensor(g[off:off + k].reshape(tt.shape) * grad_scale, dtype=torch.float64)
            off += k
        lib_norm = None
        if grad_clip > 0:
            lib_norm = float(torch.nn.utils.clip_grad_norm_(ts, grad_clip))
        opt.step()
        p, m, v, norm = OPT.adamw_step(p, g, m, v, t, lr, b1, b2, eps, wd, mask, grad_scale=grad_scale,
                                       grad_clip=grad_clip)
        if lib_norm is not None:
            assert norm == pytest.approx(lib_norm, rel=1e-13)
        got = np.concatenate([tt.detach().numpy().reshape(-1) for tt in ts])
        ea = np.concatenate([opt.state[tt]["exp_avg"].numpy().reshape(-1) for tt in ts])
        es = np.concatenate([opt.state[tt]["exp_avg_sq"].numpy().reshape(-1) for tt in ts])
        assert np.allclose(p, got, rtol=0, atol=1e-13)
        assert np.allclose(m, ea, rtol=1e-12, atol=1e-18)
        assert np.allclose(v, es, rtol=1e-12, atol=1e-20)
    # something moved, and the 1-D tensors were not decayed (a zero gradient leaves them in place)
    assert not np.allclose(p, p0)


def test_zero_gradient_moves_only_decayed_tensors():
    cfg = _cfg()
    n = O.param_count(cfg)
    p0 = synth.normal(n, 2, std=0.5).astype(np.float64)
    mask = OPT.decay_mask(cfg)
    p, m, v, norm = OPT.adamw_step(p0, np.zeros(n), np.zeros(n), np.zeros(n), 1, 1e-2, 0.9, 0.95, 1e-8, 0.1, mask,
                                   grad_clip=1.0)
    assert norm == 0.0 and not np.any(m) and not np.any(v)
    assert np.array_equal(p[~mask], p0[~mask])
    assert np.allclose(p[mask], p0[mask] * (1 - 1e-3), rtol=1e-15)


def test_decay_mask_counts():
    # GPT-2 124M: the 1-D tensors are ln1 (g, b), b_qkv, b_o, ln2 (g, b), b_up, b_down per layer = 13 D,
    # plus the final LayerNorm's 2 D
    gpt2 = O.preset("gpt2")
    mask = OPT.decay_mask(gpt2)
    D, L = 768, 12
    assert mask.size == 124_475_904
    assert int((~mask).sum()) == 13 * D * L + 2 * D == 121_344
    assert int(mask.sum()) == 124_354_560
    # the nanochat shapes have no 1-D tensors (parameter-free RMSNorm, no biases)
    assert OPT.decay_mask(O.preset("d20")).all()


def test_lr_schedule_closed_forms():
    # the page's values: warmup_iters 2000, lr_decay_iters 600000, learning_rate 6e-4, min_lr 6e-5
    f = lambda it: OPT.lr_schedule(it, 2000, 600_000, 6e-4, 6e-5)  # noqa: E731
    assert f(0) == 0.0
    assert f(1000) == pytest.approx(3e-4, rel=1e-15)
    assert f(2000) == pytest.approx(6e-4, rel=1e-15)
    assert f(301_000) == pytest.approx(0.5 * (6e-4 + 6e-5), rel=1e-12)       # decay_ratio 1/2: cos = 0
    assert f(600_000) == pytest.approx(6e-5, rel=1e-12)
    assert f(10**7) == 6e-5
    # decay_ratio 1/3: coeff = 0.5 (1 + cos(pi/3)) = 3/4
    assert f(2000 + 199_333) == pytest.approx(6e-5 + 0.75 * (6e-4 - 6e-5), rel=1e-5)
    seq = [f(it) for it in range(2000, 600_001, 997)]
    assert all(a >= b for a, b in zip(seq, seq[1:]))
    assert OPT.lr_schedule(5, 0, 0, 1e-3, 1e-4) == 1e-4 and OPT.lr_schedule(0, 0, 0, 1e-3, 1e-4) == 1e-3


# ------------------------------------------------------------ Muon

def _spectrum_matrix(rows, cols, svals, seed):
    """A matrix with the given singular values and random orthogonal factors."""
    rng = np.random.default_rng(seed)
    k = min(rows, cols)
    U, _ = np.linalg.qr(rng.standard_normal((rows, k)))
    V, _ = np.linalg.qr(rng.standard_normal((cols, k)))
    return (U * np.asarray(svals)) @ V.T


@pytest.mark.parametrize("shape", [(24, 40), (40, 24), (32, 32)])
def test_newton_schulz_acts_on_singular_values(shape):
    """Five quintic steps map X = G / ||G||_F to U phi^5(S / ||G||_F) V^T, phi(s) = a s + b s^3 + c s^5:
    the same result reached through the SVD and the scalar polynomial instead of matrix products
    (a transposed operand, a wrong coefficient or a dropped normalization differs)."""
    G = synth.normal(shape, 61).astype(np.float64)
    U, S, Vt = np.linalg.svd(G, full_matrices=False)
    s = S / (np.linalg.norm(G) + 1e-7)
    a, b, c = OPT.NS_COEFFS
    for _ in range(5):
        s = a * s + b * s ** 3 + c * s ** 5
    assert np.allclose(OPT.newton_schulz5(G), (U * s) @ Vt, rtol=1e-10, atol=1e-12)


def test_newton_schulz_equalizes_singular_values():
    """The page's description: the update's singular values become (nearly) equal.  For inputs
    whose normalized singular values span [3e-3, 1] the five steps land them in [0.68, 1.21]."""
    for shape, seed in (((64, 96), 62), ((96, 64), 63)):
        k = min(shape)
        sv = np.geomspace(1.0, 3e-3 * np.sqrt(k), k)       # ||G||_F ~ sqrt(sum s^2)
        G = _spectrum_matrix(*shape, sv, seed)
        out = np.linalg.svd(OPT.newton_schulz5(G), compute_uv=False)
        assert out.min() >= 0.68 and out.max() <= 1.21, (out.min(), out.max())
        # the spread of the input (hundreds) collapses to under 2
        assert out.max() / out.min() < 1.8


def test_newton_schulz_invariances():
    G = synth.normal((20, 36), 64).astype(np.float64)
    X = OPT.newton_schulz5(G)
    assert np.allclose(OPT.newton_schulz5(7.5 * G), X, rtol=1e-6, atol=1e-9)     # scale (up to eps)
    assert np.allclose(OPT.newton_schulz5(G.T), X.T, rtol=1e-12, atol=1e-14)    # orientation
    rng = np.random.default_rng(65)
    Q1, _ = np.linalg.qr(rng.standard_normal((20, 20)))
    Q2, _ = np.linalg.qr(rng.standard_normal((36, 36)))
    assert np.allclose(OPT.newton_schulz5(Q1 @ G @ Q2), Q1 @ X @ Q2, rtol=1e-9, atol=1e-11)


def test_muon_momentum_closed_form():
    """A constant gradient g: the average after t steps is (1 - mu^t) g and the update is the
    orthogonalized g scaled by sqrt(max(1, rows/cols)) (the normalization removes the scale, up
    to the 1e-7 guard, which the steep start of phi^5 amplifies to ~1e-5).  Two different
    gradients g1, g2: the Nesterov input of step 2 points along (1 + mu) g2 + mu^2 g1, the plain
    average along g2 + mu g1."""
    g = synth.normal((12, 8), 66).astype(np.float64)
    buf = np.zeros_like(g)
    mu = 0.95
    for t in range(1, 6):
        upd, buf = OPT.muon_update(g, buf, mu, True)
        assert np.allclose(buf, (1 - mu ** t) * g, rtol=1e-13)
        assert np.allclose(upd, OPT.newton_schulz5(g) * np.sqrt(12 / 8), rtol=1e-4, atol=1e-6)
    g1, g2 = (synth.normal((10, 30), s).astype(np.float64) for s in (69, 70))
    for nesterov, direction in ((True, (1 + mu) * g2 + mu ** 2 * g1), (False, g2 + mu * g1)):
        _, b1 = OPT.muon_update(g1, np.zeros_like(g1), mu, nesterov)
        upd, _ = OPT.muon_update(g2, b1, mu, nesterov)
        assert np.allclose(upd, OPT.newton_schulz5(direction), rtol=1e-4, atol=1e-6)


def test_muon_adamw_step_routes_tensors():
    """Block matrices move by -lr * (orthogonalized update); every other tensor takes the AdamW
    step of its own slice."""
    cfg = O.Config(n_layer=2, n_embd=16, n_head=2, block_size=8, vocab_size=11, norm=O.NORM_LN, linear_bias=1,
                   tie_embed=0)
    n = O.param_count(cfg)
    p, g = (synth.normal(n, s).astype(np.float64) for s in (67, 68))
    mom, v = np.zeros(n), np.zeros(n)
    p2, mom2, v2 = OPT.muon_adamw_step(cfg, p, g, mom, v, 1, 0.02, 0.95, True, 1e-3, 0.9, 0.95, 1e-8, 0.1)
    seen = set()
    for name, (off, shape) in O.param_offsets(cfg).items():
        sl = slice(off, off + int(np.prod(shape)))
        if OPT.is_muon_tensor(name):
            seen.add(name.split(".")[-1])
            upd, _ = OPT.muon_update(g[sl].reshape(shape), np.zeros(shape))
            assert np.allclose(p2[sl], p[sl] - 0.02 * upd.reshape(-1), rtol=1e-13)
            assert np.all(v2[sl] == 0)
        else:
            ref = OPT.adamw_step(p[sl], g[sl], mom[sl], v[sl], 1, 1e-3, 0.9, 0.95, 1e-8, 0.1,
                                 np.full(sl.stop - sl.start, len(shape) == 2))
            assert np.allclose(p2[sl], ref[0], rtol=1e-15) and np.allclose(v2[sl], ref[2], rtol=1e-15)
    assert seen == set(OPT.MUON_TENSORS)
