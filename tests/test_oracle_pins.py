"""Pins of the oracle to facts outside itself: numbers the pages print, closed
forms, invariants, library routines for special cases, and central finite
differences.  No GPU; no call into the CUDA library."""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as O
import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _cfg(**kw):
    base = dict(n_layer=2, n_embd=16, n_head=2, block_size=16, vocab_size=23)
    base.update(kw)
    return O.Config(**base)


SMALL_CONFIGS = {
    # the tiny oracle check exactly: 1 layer, 16 wide, 4 heads, 27 tokens, tied, GELU, RMSNorm, wpe
    "tiny": O.preset("tiny"),
    # GPT-2 block shape at toy size: LayerNorm with bias, biases everywhere, tied, scaled init
    "gpt2ish": _cfg(norm=O.NORM_LN, linear_bias=1, tie_embed=1, act=O.ACT_GELU,
                    pos=O.POS_LEARNED, scale_resid_init=1, vocab_size=19),
    # nanochat block shape at toy size: RoPE, QK-norm, ReLU^2, untied, RMSNorm
    "d20ish": _cfg(norm=O.NORM_RMS, pos=O.POS_ROPE, qk_norm=1, act=O.ACT_RELU2, tie_embed=0),
    # the same with sliding-window layers in the "SSSL" pattern (short window of 3 keys back)
    "d20ish_sssl": _cfg(n_layer=4, norm=O.NORM_RMS, pos=O.POS_ROPE, qk_norm=1, act=O.ACT_RELU2, tie_embed=0,
                        window_short=3, window_pattern=O.pattern_bits("SSSL"), window_period=4),
}


def _random_params(cfg, seed, std=0.5):
    """Large random parameters (so every nonlinearity is exercised), with
    LayerNorm gains near 1 and nonzero biases."""
    p = synth.normal(O.param_count(cfg), seed, std=std).astype(np.float64)
    pr = O.unflatten(cfg, p)
    for name, v in pr.items():
        if name.endswith("_g"):
            v += 1.0
    return p


# ------------------------------------------------------------ parameter counts

def test_param_counts_match_pages():
    facts = _gold("page_facts.json")
    tiny_untied = O.preset("tiny", tie_embed=0)
    assert O.param_count(tiny_untied) == facts["microgpt_params"]["value"] == 4192
    assert O.param_count(O.preset("tiny")) == 4192 - 27 * 16 == 3760
    g = O.preset("gpt2")
    n = O.param_count(g)
    assert n == 124_475_904
    assert abs(n - facts["gpt2_params_approx"]["value"]) / 124e6 < 0.01
    assert O.param_count(O.preset("gpt2", vocab_size=facts["gpt2_vocab_raw"]["value"])) == 124_439_808
    saved = O.param_count(O.preset("gpt2", tie_embed=0)) - n
    assert saved == 50304 * 768 == 38_633_472
    assert abs(saved - facts["gpt2_tying_saves_approx"]["value"]) < 1e6
    d20 = O.preset("d20")
    transformer = d20.n_layer * 12 * d20.n_embd ** 2
    assert transformer == 393_216_000
    assert abs(transformer - facts["d20_transformer_params_approx"]["value"]) < 1e6
    assert O.param_count(d20) == transformer + 2 * 32768 * 1280 == 477_102_080
    # the card's 897M adds per-layer value embeddings: 12 tables of V x D in total
    assert abs(transformer + 12 * 32768 * 1280 - facts["d20_total_params_approx"]["value"]) < 1e6


# ------------------------------------------------------------ loss closed forms

@pytest.mark.parametrize("V", [27, 32768, 50304])
def test_uniform_logits_give_ln_v(V):
    cfg = _cfg(vocab_size=V, tie_embed=0, n_layer=1)
    p = _random_params(cfg, 3, std=0.3)
    O.unflatten(cfg, p)["lm_head"][:] = 0.0
    idx, tg = synth.next_token_batch(2, 8, V, dist="uniform", seed=4)
    f = O.forward(cfg, p, idx, tg)
    assert f["loss"] == pytest.approx(math.log(V), abs=1e-12)
    assert np.allclose(f["ell"], math.log(V), atol=1e-12)


def test_tied_zero_embedding_gives_ln_v():
    cfg = O.preset("tiny")
    p = _random_params(cfg, 5)
    O.unflatten(cfg, p)["wte"][:] = 0.0
    idx, tg = synth.next_token_batch(4, 16, 27, dist="uniform", seed=1)
    assert O.forward(cfg, p, idx, tg)["loss"] == pytest.approx(math.log(27), abs=1e-12)


def test_step0_loss_near_ln_v():
    """At init N(0, 0.02^2) the logits are tiny, so the loss starts near ln V
    (the page's step-0 log line, 9.21 for an 8192 vocabulary, sits just above
    ln 8192 = 9.011)."""
    facts = _gold("page_facts.json")
    V = facts["step0_loss_vocab8192"]["vocab"]
    cfg = _cfg(vocab_size=V, n_embd=64, n_head=2, pos=O.POS_ROPE, qk_norm=1,
               act=O.ACT_RELU2, tie_embed=0)
    p = O.init_params(cfg, seed=0)
    idx, tg = synth.next_token_batch(2, 16, V, seed=1)
    loss = O.forward(cfg, p, idx, tg)["loss"]
    assert abs(loss - math.log(V)) < 0.2
    assert abs(facts["step0_loss_vocab8192"]["value"] - math.log(V)) < 0.25


def test_cross_entropy_matches_library():
    z = synth.normal((7, 11), 8).astype(np.float64) * 3
    y = np.array([0, 3, 10, 5, 5, 1, 2])
    ell, lse = O.cross_entropy(z, y)
    ref = F.cross_entropy(torch.from_numpy(z), torch.from_numpy(y), reduction="none").numpy()
    assert np.allclose(ell, ref, rtol=1e-13, atol=1e-13)
    assert np.allclose(lse, torch.logsumexp(torch.from_numpy(z), -1).numpy(), rtol=1e-13)


# ------------------------------------------------------------ bits per byte

def test_bpb_worked_example():
    g = _gold("bpb_worked_example.json")
    s, b, n, bpb = O.bits_per_byte(g["ell"], g["targets"], g["token_bytes"])
    assert s == g["sum_nats"] and b == g["sum_bytes"] and n == g["n_tokens"]
    assert bpb == pytest.approx(g["bpb"], rel=1e-15)


def test_bpb_one_byte_tokens_is_loss_over_ln2():
    cfg = O.preset("tiny")
    p = O.init_params(cfg, 0)
    idx, tg = synth.next_token_batch(4, 16, 27, dist="uniform", seed=1)
    f = O.forward(cfg, p, idx, tg)
    s, b, n, bpb = O.bits_per_byte(f["ell"], tg, np.ones(27, np.int32))
    assert b == n == 64
    assert bpb == pytest.approx(f["loss"] / math.log(2), rel=1e-14)


def test_bpb_scales_inversely_with_bytes():
    ell = synth.normal(50, 3).astype(np.float64) ** 2
    tg = synth.uniform_tokens(50, 9, seed=4)
    tb = synth.byte_table(9, 1, 5, seed=5)
    s1, b1, _, r1 = O.bits_per_byte(ell, tg, tb)
    s2, b2, _, r2 = O.bits_per_byte(ell, tg, 3 * tb)
    assert s1 == s2 and b2 == 3 * b1 and r2 == pytest.approx(r1 / 3, rel=1e-14)


def test_bpb_zero_byte_targets_do_not_count():
    """Changing the loss at a 0-byte target changes neither sum."""
    ell = np.abs(synth.normal(40, 6).astype(np.float64))
    tg = synth.uniform_tokens(40, 10, seed=7)
    tb = synth.byte_table(10, 1, 4, seed=8)
    tb[tg[3]] = 0
    a = O.bits_per_byte(ell, tg, tb)
    ell2 = ell.copy()
    ell2[tg == tg[3]] += 100.0
    assert O.bits_per_byte(ell2, tg, tb) == a


# ------------------------------------------------------------ causality

@pytest.mark.parametrize("name", list(SMALL_CONFIGS))
def test_causality_future_tokens_do_not_change_past(name):
    cfg = SMALL_CONFIGS[name]
    p = _random_params(cfg, 11)
    B, T = 2, 12
    idx, tg = synth.next_token_batch(B, T, cfg.vocab_size, dist="uniform", seed=12)
    f1 = O.forward(cfg, p, idx, tg, return_logits=True)
    t0 = 7
    idx2 = idx.copy()
    idx2[:, t0 + 1:] = (idx2[:, t0 + 1:] + 5) % cfg.vocab_size
    f2 = O.forward(cfg, p, idx2, tg, return_logits=True)
    z1 = f1["logits"].reshape(B, T, -1)
    z2 = f2["logits"].reshape(B, T, -1)
    assert np.array_equal(z1[:, :t0 + 1], z2[:, :t0 + 1])
    assert not np.allclose(z1[:, t0 + 1:], z2[:, t0 + 1:])


# ------------------------------------------------------------ attention

def test_attention_matches_library_sdpa():
    q, k, v = (synth.normal((2, 3, 17, 8), s).astype(np.float64) for s in (1, 2, 3))
    o, p = O.causal_attention(q, k, v)
    ref = F.scaled_dot_product_attention(*(torch.from_numpy(t) for t in (q, k, v)), is_causal=True)
    assert np.allclose(o, ref.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(p.sum(-1), 1.0)
    assert np.all(np.triu(p[0, 0], 1) == 0.0)


def test_attention_backward_matches_library_autograd():
    q, k, v, do = (synth.normal((1, 2, 9, 4), s).astype(np.float64) for s in (5, 6, 7, 8))
    o, p = O.causal_attention(q, k, v)
    dq, dk, dv = O.causal_attention_bwd(do, q, k, v, p)
    tq, tk, tv = (torch.from_numpy(t).requires_grad_() for t in (q, k, v))
    F.scaled_dot_product_attention(tq, tk, tv, is_causal=True).backward(torch.from_numpy(do))
    for a, b in ((dq, tq), (dk, tk), (dv, tv)):
        assert np.allclose(a, b.grad.numpy(), rtol=1e-11, atol=1e-12)


def _brute_force_window_attention(q, k, v, w):
    """Row by row: softmax over the keys j with i - w <= j <= i only, then the weighted sum."""
    B, H, T, hd = q.shape
    o = np.zeros_like(q)
    for b in range(B):
        for h in range(H):
            for i in range(T):
                js = [j for j in range(T) if j <= i and (w is None or j >= i - w)]
                sc = np.array([q[b, h, i] @ k[b, h, j] for j in js]) / np.sqrt(hd)
                e = np.exp(sc - sc.max())
                a = e / e.sum()
                o[b, h, i] = sum(a[n] * v[b, h, j] for n, j in enumerate(js))
    return o


@pytest.mark.parametrize("w", [0, 1, 3, 7, None])
def test_window_attention_matches_brute_force(w):
    q, k, v = (synth.normal((1, 2, 11, 4), s).astype(np.float64) for s in (21, 22, 23))
    o, p = O.causal_attention(q, k, v, w)
    assert np.allclose(o, _brute_force_window_attention(q, k, v, w), rtol=1e-12, atol=1e-12)
    i, j = np.indices((11, 11))
    outside = (j > i) if w is None else ((j > i) | (j < i - w))
    assert np.all(p[:, :, outside] == 0.0) and np.allclose(p.sum(-1), 1.0)


def test_window_special_cases():
    q, k, v = (synth.normal((2, 2, 13, 8), s).astype(np.float64) for s in (24, 25, 26))
    full, _ = O.causal_attention(q, k, v)
    for w in (12, 13, 100):   # a window reaching back to key 0 from every query is the full causal mask
        assert np.array_equal(O.causal_attention(q, k, v, w)[0], full)
    assert np.array_equal(O.causal_attention(q, k, v, 0)[0], v)   # each query sees only itself


def test_window_pattern_expands_per_layer():
    cfg = O.Config(n_layer=9, n_embd=16, n_head=2, block_size=16, vocab_size=10, window_short=5,
                   window_pattern=O.pattern_bits("SSSL"), window_period=4)
    assert [O.layer_window(cfg, l) for l in range(9)] == [5, 5, 5, None, 5, 5, 5, None, 5]
    off = O.Config(**{**cfg.__dict__, "window_short": 0})
    assert all(O.layer_window(off, l) is None for l in range(9))


def test_window_layer_sees_only_its_band():
    """One short-window layer of width w: the logits at position i depend on tokens i - w .. i
    only, so changing token t0 leaves every position outside [t0, t0 + w] bitwise unchanged."""
    w = 3
    cfg = _cfg(n_layer=1, norm=O.NORM_RMS, pos=O.POS_ROPE, qk_norm=1, act=O.ACT_RELU2, tie_embed=0,
               window_short=w, window_pattern=1, window_period=1)
    p = _random_params(cfg, 27)
    idx, tg = synth.next_token_batch(1, 14, cfg.vocab_size, dist="uniform", seed=28)
    t0 = 5
    idx2 = idx.copy()
    idx2[0, t0] = (idx2[0, t0] + 7) % cfg.vocab_size
    z1 = O.forward(cfg, p, idx, tg, return_logits=True)["logits"]
    z2 = O.forward(cfg, p, idx2, tg, return_logits=True)["logits"]
    changed = np.any(z1 != z2, axis=1)
    assert changed[t0:t0 + w + 1].all() and not changed[:t0].any() and not changed[t0 + w + 1:].any()


def test_uniform_attention_closed_form():
    """q = k = 0 gives equal weights over the causal prefix, so the attention
    sublayer becomes a running mean of v; with a non-symmetric w_o this also
    fixes the orientation of the output projection (y = x W^T)."""
    cfg = _cfg(n_layer=1, vocab_size=13, tie_embed=0)
    D = cfg.n_embd
    p = _random_params(cfg, 21)
    pr = O.unflatten(cfg, p)
    pr["h0.w_qkv"][:2 * D] = 0.0
    pr["h0.w_qkv"][2 * D:] = np.eye(D)
    A = synth.normal((D, D), 22).astype(np.float64)
    pr["h0.w_o"][:] = A
    pr["h0.w_down"][:] = 0.0
    B, T = 2, 10
    idx, tg = synth.next_token_batch(B, T, 13, dist="uniform", seed=23)
    f = O.forward(cfg, p, idx, tg, return_logits=True)
    x0 = (pr["wte"][idx] + pr["wpe"][:T][None]).reshape(B, T, D)
    a1 = x0 / np.sqrt(np.mean(x0 ** 2, -1, keepdims=True) + cfg.norm_eps)
    run_mean = np.cumsum(a1, axis=1) / np.arange(1, T + 1)[None, :, None]
    x1 = x0 + run_mean @ A.T
    af = x1 / np.sqrt(np.mean(x1 ** 2, -1, keepdims=True) + cfg.norm_eps)
    z = af.reshape(B * T, D) @ pr["lm_head"].T
    assert np.allclose(f["logits"], z, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------ RoPE, QK-norm, norms, activations

def test_rope_is_complex_rotation():
    T, hd = 9, 8
    x = synth.normal((2, T, hd), 31).astype(np.float64)
    phi = O.rope_angles(T, hd, 10000.0)
    y = O.rope(x, phi)
    zc = (x[..., :hd // 2] + 1j * x[..., hd // 2:]) * np.exp(1j * phi)
    assert np.allclose(y[..., :hd // 2], zc.real, atol=1e-14)
    assert np.allclose(y[..., hd // 2:], zc.imag, atol=1e-14)
    assert np.allclose(phi[3, 1], 3 * 10000.0 ** (-2.0 / hd))


def test_rope_scores_depend_only_on_offset():
    T, hd = 12, 16
    q = synth.normal(hd, 32).astype(np.float64)
    k = synth.normal(hd, 33).astype(np.float64)
    phi = O.rope_angles(T, hd, 10000.0)
    qr = O.rope(np.tile(q, (T, 1)), phi)
    kr = O.rope(np.tile(k, (T, 1)), phi)
    s = qr @ kr.T
    for d in range(-3, 4):
        vals = np.diagonal(s, offset=d)
        assert np.allclose(vals, vals[0], atol=1e-12)
    assert np.allclose(O.rope_bwd(qr, phi), np.tile(q, (T, 1)), atol=1e-13)


def test_qk_norm_unit_rms():
    x = synth.normal((3, 5, 32), 34).astype(np.float64) * 7
    y, r = O.rmsnorm(x, 1e-5)
    rms = np.sqrt(np.mean(y * y, -1))
    assert np.allclose(rms, np.sqrt(np.mean(x * x, -1) / (np.mean(x * x, -1) + 1e-5)), rtol=1e-14)
    assert np.allclose(rms, 1.0, atol=1e-6)


def test_norm_constant_rows_and_library():
    eps = 1e-5
    c = 0.37
    y, _ = O.rmsnorm(np.full((2, 8), c), eps)
    assert np.allclose(y, c / math.sqrt(c * c + eps), rtol=1e-15)
    g = synth.normal(8, 35).astype(np.float64)
    b = synth.normal(8, 36).astype(np.float64)
    y, _, _ = O.layernorm(np.full((3, 8), -2.5), g, b, eps)
    assert np.allclose(y, b[None], atol=1e-15)
    x = synth.normal((4, 24), 37).astype(np.float64) * 3 + 1
    g24 = synth.normal(24, 38).astype(np.float64)
    b24 = synth.normal(24, 39).astype(np.float64)
    y, _, _ = O.layernorm(x, g24, b24, eps)
    ref = F.layer_norm(torch.from_numpy(x), (24,), torch.from_numpy(g24), torch.from_numpy(b24), eps)
    assert np.allclose(y, ref.numpy(), rtol=1e-12, atol=1e-12)
    y, _ = O.rmsnorm(x, eps)
    ref = F.rms_norm(torch.from_numpy(x), (24,), eps=eps)
    assert np.allclose(y, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_activations_match_library():
    u = np.linspace(-6, 6, 101)
    assert np.allclose(O.gelu(u), F.gelu(torch.from_numpy(u), approximate="none").numpy(), atol=1e-15)
    assert np.allclose(O.relu2(u), np.where(u > 0, u * u, 0.0))
    tu = torch.from_numpy(u).requires_grad_()
    F.gelu(tu).sum().backward()
    assert np.allclose(O.gelu_grad(u), tu.grad.numpy(), atol=1e-14)
    tu = torch.from_numpy(u).requires_grad_()
    torch.relu(tu).square().sum().backward()
    assert np.allclose(O.relu2_grad(u), tu.grad.numpy(), atol=1e-14)


# ------------------------------------------------------------ gradients

def test_dlogits_rows_sum_to_zero():
    cfg = SMALL_CONFIGS["d20ish"]
    p = _random_params(cfg, 41)
    idx, tg = synth.next_token_batch(2, 8, cfg.vocab_size, seed=42)
    f = O.forward(cfg, p, idx, tg)
    z = f["cache"]["z"]
    dz = np.exp(z - f["lse"][:, None])
    dz[np.arange(len(tg.reshape(-1))), tg.reshape(-1)] -= 1
    assert np.allclose(dz.sum(-1), 0, atol=1e-14)
    # the lm_head gradient equals dz^T af / M: check against the oracle's backward
    g = O.backward(cfg, p, f)
    M = z.shape[0]
    assert np.allclose(O.unflatten(cfg, g)["lm_head"], dz.T @ f["cache"]["af"] / M, atol=1e-14)


def test_embedding_gradient_rows_follow_the_inputs():
    """x0[m] = wte[idx[m]] (+ wpe[t]): the embedding gradient scatters into the rows of the INPUT
    ids and positions only.  Untied, the rows of ids absent from idx are exactly zero (ids that
    occur only as targets included), and wpe rows at positions >= T are zero.  Tied, the absent
    rows carry the lm_head part alone, which equals the untied model's lm_head gradient."""
    B, T, V = 2, 6, 40
    rng = np.random.default_rng(7)
    idx = rng.integers(0, 10, size=(B, T)).astype(np.int32)        # inputs use ids 0..9 only
    tgt = rng.integers(20, V, size=(B, T)).astype(np.int32)        # targets 20..39 only
    absent = np.setdiff1d(np.arange(V), idx)
    present = np.unique(idx)
    grads = {}
    for tie in (0, 1):
        cfg = _cfg(vocab_size=V, tie_embed=tie, pos=O.POS_LEARNED, block_size=16)
        p = _random_params(cfg, 43, std=0.3)
        gr = O.unflatten(cfg, O.backward(cfg, p, O.forward(cfg, p, idx, tgt)))
        grads[tie] = (cfg, p, gr)
        assert not np.any(gr["wpe"][T:]) and np.all(np.abs(gr["wpe"][:T]).sum(-1) > 0)
    cfg0, p0, g0 = grads[0]
    assert not np.any(g0["wte"][absent])
    assert np.all(np.abs(g0["wte"][present]).sum(-1) > 0)
    # tied: same weights with lm_head := wte; the absent rows hold only the lm_head gradient
    cfg1 = grads[1][0]
    p1 = O.unflatten(cfg1, np.zeros(O.param_count(cfg1)))
    for name, v in O.unflatten(cfg0, p0).items():
        if name in p1:
            p1[name][...] = v
    pu = O.unflatten(cfg0, p0.copy())
    pu["lm_head"][...] = pu["wte"]
    flat_u = np.concatenate([pu[n].reshape(-1) for n, _ in O.param_shapes(cfg0)])
    flat_t = np.concatenate([p1[n].reshape(-1) for n, _ in O.param_shapes(cfg1)])
    gu = O.unflatten(cfg0, O.backward(cfg0, flat_u, O.forward(cfg0, flat_u, idx, tgt)))
    gt = O.unflatten(cfg1, O.backward(cfg1, flat_t, O.forward(cfg1, flat_t, idx, tgt)))
    assert np.allclose(gt["wte"][absent], gu["lm_head"][absent], rtol=0, atol=1e-15)
    assert np.allclose(gt["wte"], gu["wte"] + gu["lm_head"], rtol=0, atol=1e-14)


@pytest.mark.parametrize("name", list(SMALL_CONFIGS))
def test_gradients_match_central_differences(name):
    """fp64 central differences, h = 1e-5 (about 1e-4 relative to the
    parameter scale 0.5 and below), on a sample of entries of every tensor."""
    cfg = SMALL_CONFIGS[name]
    p = _random_params(cfg, 51)
    B, T = (4, 16) if name == "tiny" else (2, 8)
    idx, tg = synth.next_token_batch(B, T, cfg.vocab_size, dist="uniform", seed=52)
    loss, g = O.loss_and_grad(cfg, p, idx, tg)
    rng = np.random.default_rng(53)
    h = 1e-5
    for pname, (off, shape) in O.param_offsets(cfg).items():
        n = int(np.prod(shape))
        picks = np.arange(n) if n <= 24 else rng.choice(n, size=24, replace=False)
        fd = np.empty(len(picks))
        for j, i in enumerate(picks):
            pp = p.copy()
            pp[off + i] += h
            lp = O.forward(cfg, pp, idx, tg, keep_cache=False)["loss"]
            pp[off + i] -= 2 * h
            lm = O.forward(cfg, pp, idx, tg, keep_cache=False)["loss"]
            fd[j] = (lp - lm) / (2 * h)
        an = g[off + picks]
        err = np.linalg.norm(fd - an) / max(np.linalg.norm(an), 1e-12)
        assert err < 1e-6, (pname, err)
        assert np.linalg.norm(an) > 0, pname


# ------------------------------------------------------------ initialisation

def test_splitmix64_published_vector():
    g = _gold("splitmix64.json")
    # the generator seeded with state s outputs mix(s + gamma) first
    assert O.splitmix64((g["seed"] + 0x9E3779B97F4A7C15) & ((1 << 64) - 1)) == int(g["first_output_hex"], 16)
    assert int(O.splitmix64_stream(g["seed"], np.array([0], np.uint64))[0]) == int(g["first_output_hex"], 16)


def test_init_statistics():
    from scipy import stats
    cfg = O.preset("gpt2", n_layer=2, n_embd=128, n_head=2, vocab_size=1000, block_size=64)
    p = O.init_params(cfg, seed=7)
    pr = O.unflatten(cfg, p)
    w = pr["wte"].reshape(-1)
    assert abs(np.std(w) - 0.02) < 0.02 * 0.01
    assert abs(np.mean(w)) < 0.02 * 0.01
    assert stats.kstest(w / 0.02, "norm").pvalue > 1e-3
    wo = pr["h1.w_o"].reshape(-1)
    assert abs(np.std(wo) - 0.02 / math.sqrt(4)) < 0.02 / 2 * 0.03
    assert np.all(pr["h0.ln1_g"] == 1) and np.all(pr["h0.b_qkv"] == 0)
    q = O.init_params(cfg, seed=8)
    assert not np.allclose(p, q)
    assert np.array_equal(p, O.init_params(cfg, seed=7))


# ------------------------------------------------------------ FLOP accounting

def test_flop_counts():
    d20 = O.preset("d20")
    assert O.matmul_params(d20) == 435_159_040
    assert O.step_flops(d20, 16, 2048) == pytest.approx(95.864e12, rel=1e-4)
    assert O.step_flops(d20, 16, 2048, causal=False) == pytest.approx(106.17e12, rel=1e-4)
