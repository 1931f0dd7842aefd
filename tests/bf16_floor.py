"""How far bf16 operands alone move the oracle's logits: the scale of the logits bar.

A tensor-core path must round every matmul operand to bf16 (activations and weights of each linear
layer, and q, k, v of attention).  Running the fp64 oracle with exactly those operands rounded, and
nothing else changed, gives the deviation that arithmetic alone produces; the GPU's logits are held
to twice it (and never to less than the target's 2e-2 of their RMS).  On the d20-shaped test models
this floor is 2-4 % of the logits' RMS at the largest element (0.4-0.6 % RMS), above the target's
2e-2 bar; on GPT-2 shapes it is below it.

Test helper: it patches the oracle's module functions for one call and restores them."""
from unittest import mock

import numpy as np
import torch

import oracle.gpt_oracle as G


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64)).float().bfloat16().double().numpy()


def bf16_operand_forward(ocfg, p, idx, tgt):
    """The oracle forward with every linear-layer operand and q, k, v rounded to bf16."""
    lin, attn = G._linear, G.causal_attention
    with mock.patch.object(G, "_linear", lambda x, w, b, fp8=False: lin(_bf16(x), _bf16(w), b, fp8)), \
         mock.patch.object(G, "causal_attention", lambda q, k, v, w=None: attn(_bf16(q), _bf16(k), _bf16(v), w)):
        return G.forward(ocfg, p, idx, tgt, return_logits=True, keep_cache=False)


def logits_floor(ocfg, p, idx, tgt, z_exact):
    """(max |dz|, rms dz) of the bf16-operand oracle against the exact one."""
    zb = bf16_operand_forward(ocfg, p, idx, tgt)["logits"]
    d = zb - z_exact
    return float(np.abs(d).max()), float(np.sqrt(np.mean(d * d)))
