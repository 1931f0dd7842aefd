"""Oracle for the optimizer step of nanoGPT's training loop: plain fp64 numpy.

TEST INFRASTRUCTURE ONLY, like the model oracle: imported by the test suite
alone.  It shares no code with the CUDA library.

Source: "nanoGPT - Karpathy's minimal GPT pretraining repo", How it works:
  - model.py, configure_optimizers: AdamW with two parameter groups; every 2-D
    tensor (matmuls, embeddings) gets weight decay, every 1-D tensor (biases,
    LayerNorm gains) none;
  - train.py, the loop: gradient clipping at grad_clip via clip_grad_norm_
    before the step; the loss (hence the gradient) divided by the number of
    accumulated micro-steps; learning rate by linear warmup over warmup_iters
    to learning_rate, then cosine decay over lr_decay_iters down to min_lr,
    coeff = 0.5 (1 + cos(pi * decay_ratio)), lr = min_lr + coeff (learning_rate - min_lr).

Readings where the page is silent:
  - AdamW is the decoupled-weight-decay Adam the page names (the fused AdamW
    of PyTorch): p <- p (1 - lr wd) for decayed tensors, then the Adam moments
    and the bias-corrected step; beta1, beta2, eps and the decay are arguments.
  - clip_grad_norm_ is PyTorch's routine the page names: the global L2 norm
    over every gradient, and a scale of min(1, max_norm / (norm + 1e-6)).
  - The micro-step division is a grad_scale factor applied to the gradient
    before the norm is taken.
  - Linear warmup rises from 0 at it = 0 to learning_rate at it = warmup_iters;
    decay_ratio = (it - warmup_iters) / (lr_decay_iters - warmup_iters); past
    lr_decay_iters the rate stays min_lr.
"""
from __future__ import annotations

import math

import numpy as np

from .gpt_oracle import param_offsets, param_shapes


def decay_mask(cfg) -> np.ndarray:
    """True for every element of a 2-D parameter tensor, False for 1-D ones."""
    parts = [np.full(int(np.prod(s)), len(s) == 2) for _, s in param_shapes(cfg)]
    return np.concatenate(parts)


def global_grad_norm(grads: np.ndarray, grad_scale: float = 1.0) -> float:
    g = np.asarray(grads, dtype=np.float64) * grad_scale
    return math.sqrt(float(np.sum(g * g)))


def clip_coefficient(norm: float, max_norm: float) -> float:
    """clip_grad_norm_'s factor: every gradient is multiplied by it (1 when clipping is off)."""
    if max_norm <= 0:
        return 1.0
    return min(1.0, max_norm / (norm + 1e-6))


def adamw_step(p, g, m, v, t: int, lr: float, beta1: float, beta2: float, eps: float, weight_decay: float,
               mask, grad_scale: float = 1.0, grad_clip: float = 0.0):
    """One AdamW step at step number t >= 1 (bias corrections use t).  Returns new
    (p, m, v) and the global gradient norm taken before clipping."""
    p = np.asarray(p, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64) * grad_scale
    m = np.asarray(m, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    norm = math.sqrt(float(np.sum(g * g)))
    g = g * clip_coefficient(norm, grad_clip)
    p = np.where(mask, p * (1.0 - lr * weight_decay), p)
    m = beta1 * m + (1.0 - beta1) * g
    v = beta2 * v + (1.0 - beta2) * g * g
    m_hat = m / (1.0 - beta1 ** t)
    v_hat = v / (1.0 - beta2 ** t)
    p = p - lr * m_hat / (np.sqrt(v_hat) + eps)
    return p, m, v, norm


def lr_schedule(it: int, warmup_iters: int, lr_decay_iters: int, learning_rate: float, min_lr: float) -> float:
    if it < warmup_iters:
        return learning_rate * it / warmup_iters
    if it > lr_decay_iters:
        return min_lr
    if lr_decay_iters == warmup_iters:
        return learning_rate
    decay_ratio = (it - warmup_iters) / (lr_decay_iters - warmup_iters)
    coeff = 0.5 * (1.0 + math.cos(math.pi * decay_ratio))
    return min_lr + coeff * (learning_rate - min_lr)


# ------------------------------------------------------------------ Muon + AdamW
#
# Source: "Train your own ChatGPT", read the source optim.py -- Muon + AdamW: the transformer's
# 2-D weight matrices go to Muon, an optimizer that orthogonalizes each update (making all its
# singular values equal); embeddings, the lm_head and the per-layer scalars go to AdamW.
#
# Readings where the page is silent (the published Muon of its authors, K. Jordan et al.,
# "Muon: An optimizer for hidden layers in neural networks", 2024):
#   - momentum as an exponential average, buf <- mu buf + (1 - mu) g, with the Nesterov form
#     u = (1 - mu) g + mu buf (mu = 0.95);
#   - the orthogonalization is five steps of the quintic Newton-Schulz iteration
#     X <- a X + (b A + c A^2) X, A = X X^T, (a, b, c) = (3.4445, -4.7750, 2.0315), started from
#     X = u / (||u||_F + 1e-7) on the wide orientation (the matrix is transposed first when it
#     has more rows than columns, and back afterwards); it maps every singular value s of X to
#     phi^5(s), phi(s) = a s + b s^3 + c s^5, which lies in [0.68, 1.21] for s >= 3e-3;
#   - the update is scaled by sqrt(max(1, rows / cols)) and applied as p <- p - lr * update,
#     with no weight decay on the Muon matrices;
#   - AdamW as above on every other tensor (no clipping: the page names none for this loop).

NS_COEFFS = (3.4445, -4.7750, 2.0315)
MUON_TENSORS = ("w_qkv", "w_o", "w_up", "w_down")


def is_muon_tensor(name: str) -> bool:
    return name.split(".")[-1] in MUON_TENSORS


def newton_schulz5(G, steps: int = 5, eps: float = 1e-7) -> np.ndarray:
    """The quintic Newton-Schulz orthogonalization of a 2-D matrix, in the published order."""
    X = np.asarray(G, dtype=np.float64)
    wide = X.shape[0] <= X.shape[1]
    if not wide:
        X = X.T
    X = X / (np.linalg.norm(X) + eps)
    a, b, c = NS_COEFFS
    for _ in range(steps):
        A = X @ X.T
        B = b * A + c * (A @ A)
        X = a * X + B @ X
    return X if wide else X.T


def muon_update(g, buf, momentum: float = 0.95, nesterov: bool = True):
    """(update, new momentum buffer) of one Muon step on one matrix."""
    g = np.asarray(g, dtype=np.float64)
    buf = momentum * np.asarray(buf, dtype=np.float64) + (1.0 - momentum) * g
    u = (1.0 - momentum) * g + momentum * buf if nesterov else buf
    rows, cols = g.shape
    return newton_schulz5(u) * math.sqrt(max(1.0, rows / cols)), buf


def muon_adamw_step(cfg, p, g, mom, v, t: int, muon_lr: float, muon_momentum: float, nesterov: bool,
                    adam_lr: float, beta1: float, beta2: float, eps: float, weight_decay: float):
    """One step of the split optimizer over the flat parameter buffer: Muon on the block
    matrices (mom holds their momentum), AdamW on every other tensor (mom holds its first
    moment, v its second; weight decay on the 2-D ones).  Returns new (p, mom, v)."""
    p = np.array(p, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    mom = np.array(mom, dtype=np.float64)
    v = np.array(v, dtype=np.float64)
    for name, (off, shape) in param_offsets(cfg).items():
        n = int(np.prod(shape))
        sl = slice(off, off + n)
        if is_muon_tensor(name):
            upd, buf = muon_update(g[sl].reshape(shape), mom[sl].reshape(shape), muon_momentum, nesterov)
            p[sl] -= muon_lr * upd.reshape(-1)
            mom[sl] = buf.reshape(-1)
        else:
            mask = np.full(n, len(shape) == 2)
            p[sl], mom[sl], v[sl], _ = adamw_step(p[sl], g[sl], mom[sl], v[sl], t, adam_lr, beta1, beta2, eps,
                                                  weight_decay, mask)
    return p, mom, v
