"""The logits deviation that bf16 matmul operands alone cause in the fp64 oracle (bf16_floor.py),
on the model suite's shapes at initialisation: below the target's 2e-2 of the RMS on the GPT-2
shape, above it on the d20 shape (RoPE + QK-norm + ReLU^2), which is why the GPU logits bar is
the larger of the two."""
import dataclasses

import numpy as np

import oracle as O
import synth
from bf16_floor import logits_floor


def _floor(base, over, B, T):
    cfg = O.preset(base, **over)
    p = O.init_params(cfg, 0)
    idx, tgt = synth.next_token_batch(B, T, cfg.vocab_size, seed=1)
    z = O.forward(cfg, p, idx, tgt, return_logits=True, keep_cache=False)["logits"]
    f_max, f_rms = logits_floor(cfg, p, idx, tgt, z)
    rms = float(np.sqrt(np.mean(z ** 2)))
    return f_max / rms, f_rms / rms


def test_bf16_operand_floor_of_the_logits():
    g_max, g_rms = _floor("gpt2", dict(n_layer=2, n_embd=128, n_head=2, vocab_size=1000, block_size=256), 2, 128)
    d_max, d_rms = _floor("d20", dict(n_layer=2, n_embd=256, n_head=2, vocab_size=2048, block_size=512), 2, 256)
    assert g_max < 2e-2 < d_max, (g_max, d_max)
    assert 1e-3 < g_rms < 1e-2 and 1e-3 < d_rms < 1e-2, (g_rms, d_rms)


def test_floor_includes_the_lm_head_operands():
    """On the one-layer toy model (D = 16) the rounding of the lm_head's own two operands dominates:
    0.07 % of the RMS without it, 0.22 % with it."""
    _, t_rms = _floor("tiny", {}, 4, 16)
    assert 1.5e-3 < t_rms < 4e-3, t_rms
