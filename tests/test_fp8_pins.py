"""Pins of the FP8 oracle ("Train your own ChatGPT", read the source fp8.py) against what fixes it:
the format definitions (every code of each format, decoded from its bits by the OCP layout, is a
fixed point of the rounding; midpoints round to even; saturation), the library's own casts
(torch.float8_e4m3fn / float8_e5m2) on values inside the range, and exact products of small
integers."""
import numpy as np
import pytest
import torch

import oracle as O

F = O.fp8


def _decode_all(fmt):
    """Every finite value of the format from its bit layout (sign, exponent, mantissa, bias)."""
    eb, mb, bias, fmax = F.FORMATS[fmt]
    vals = []
    for e in range(2 ** eb):
        for m in range(2 ** mb):
            if e == 0:
                v = m / 2 ** mb * 2.0 ** (1 - bias)
            else:
                v = (1 + m / 2 ** mb) * 2.0 ** (e - bias)
            if v <= fmax:
                vals += [v, -v]
    return np.unique(np.array(vals))


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_codes_are_fixed_points_and_midpoints_round_to_even(fmt):
    v = _decode_all(fmt)
    assert np.array_equal(F.quantize(v, fmt), v)
    assert v.max() == F.FORMATS[fmt][3]
    pos = v[v >= 0]
    mid = (pos[:-1] + pos[1:]) / 2
    q = F.quantize(mid, fmt)
    # a midpoint goes to the neighbour whose last mantissa bit is 0
    eb, mb, bias, _ = F.FORMATS[fmt]
    def even(x):
        x = np.abs(x)
        e = np.maximum(np.floor(np.log2(np.where(x > 0, x, 1.0))), 1 - bias)
        return (np.round(x / 2.0 ** (e - mb)) % 2) == 0
    assert np.all(even(q))
    assert np.all((q == pos[:-1]) | (q == pos[1:]))
    # saturation above the largest value, and the sign
    assert F.quantize(1e9, fmt) == F.FORMATS[fmt][3] and F.quantize(-1e9, fmt) == -F.FORMATS[fmt][3]


@pytest.mark.parametrize("fmt,tdt", [("e4m3", torch.float8_e4m3fn), ("e5m2", torch.float8_e5m2)])
def test_quantize_matches_library_cast_in_range(fmt, tdt):
    fmax = F.FORMATS[fmt][3]
    x = np.concatenate([np.linspace(-fmax, fmax, 100001), np.geomspace(1e-7, 1, 5001), -np.geomspace(1e-7, 1, 5001)])
    x = x.astype(np.float32).astype(np.float64)
    ref = torch.from_numpy(x).float().to(tdt).double().numpy()
    assert np.array_equal(F.quantize(x, fmt), ref)


def test_scaled_matmul_exact_on_small_integers():
    rng = np.random.default_rng(0)
    a = rng.integers(-8, 9, (7, 32)).astype(np.float64)
    b = rng.integers(-8, 9, (5, 32)).astype(np.float64)
    # with scale 1 the integers up to 16 are e4m3 codes: the product is exact
    assert np.array_equal(F.scaled_matmul(a, b, s_a=1.0, s_b=1.0), a @ b.T)
    # a power-of-two scale moves the codes without rounding
    assert np.array_equal(F.scaled_matmul(a, b, s_a=4.0, s_b=0.5), a @ b.T)
    # the dynamic scale maps the largest magnitude onto FP8_MAX
    assert F.scale_of(a, "e4m3") == 448.0 / 8.0


def test_kernel_precision_cast():
    x = np.float32([0.1, -3.7, 2.5e-3, 0.0, 11.0])
    q, amax, s, inv = F.quantize_tensor_fp32(x, "e4m3")
    assert amax == np.float32(11.0) and s == np.float32(448.0) / np.float32(11.0)
    assert q[4] == 448.0 and q[3] == 0.0
    assert np.array_equal(q, F.quantize((x * s).astype(np.float32), "e4m3"))


def test_fp8_model_forward_casts_the_four_projections():
    """With fp8 = 1 the oracle's forward runs its four block projections through the scaled product:
    the loss moves by the casts' noise only (well under 1 % here).  Causality no longer holds
    bitwise: a per-tensor scale is the maximum over every token, so a future token that changes
    the maximum changes how earlier tokens are cast (a property of the method, kept by the GPU)."""
    import synth
    cfg = O.Config(n_layer=2, n_embd=32, n_head=2, block_size=16, vocab_size=29, pos=O.POS_ROPE, qk_norm=1,
                   act=O.ACT_RELU2, tie_embed=0, fp8=1)
    p = synth.normal(O.param_count(cfg), 5, std=0.2).astype(np.float64)
    idx, tg = synth.next_token_batch(2, 12, cfg.vocab_size, dist="uniform", seed=6)
    f8 = O.forward(cfg, p, idx, tg, return_logits=True)
    hi = O.forward(O.Config(**{**cfg.__dict__, "fp8": 0}), p, idx, tg, keep_cache=False)
    assert f8["loss"] != hi["loss"] and abs(f8["loss"] - hi["loss"]) < 1e-2 * hi["loss"]
    idx2 = idx.copy()
    idx2[:, 8:] = (idx2[:, 8:] + 3) % cfg.vocab_size
    z2 = O.forward(cfg, p, idx2, tg, return_logits=True)["logits"].reshape(2, 12, -1)
    z1 = f8["logits"].reshape(2, 12, -1)[:, :8]
    assert np.abs(z2[:, :8] - z1).max() < 0.2 * np.abs(z1).max()     # changed only by the casts
