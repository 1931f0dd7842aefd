"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module only draws random numbers: it holds none of the model's arithmetic.
The datasets the pages train and evaluate on (ClimbMix, OpenWebText,
FineWeb-Edu) and their tokenizers are not available here, so these generators
stand in for them with the same shapes and a Zipf-like token distribution.

Every generator takes an explicit seed and returns a fresh numpy array; the
same seed always gives byte-identical output (numpy PCG64).
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "zipf_tokens",
    "uniform_tokens",
    "byte_table",
    "normal",
    "next_token_batch",
]


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(int(seed)))


def zipf_tokens(n: int, vocab: int, s: float = 1.1, seed: int = 1) -> np.ndarray:
    """n token ids drawn from a truncated Zipf law over ``vocab`` ids.

    p(k) is proportional to k^-s for rank k = 1..vocab, and the token id is
    k - 1 (so id 0 is the most frequent).  Sampling is by inverse CDF in fp64.
    """
    k = np.arange(1, vocab + 1, dtype=np.float64)
    w = k ** (-float(s))
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    u = _rng(seed).random(n)
    ids = np.searchsorted(cdf, u, side="right")
    return np.minimum(ids, vocab - 1).astype(np.int32)


def uniform_tokens(n: int, vocab: int, seed: int = 1) -> np.ndarray:
    """n token ids uniform in [0, vocab)."""
    return _rng(seed).integers(0, vocab, size=n, dtype=np.int64).astype(np.int32)


def next_token_batch(B: int, T: int, vocab: int, dist: str = "zipf", seed: int = 1,
                     s: float = 1.1):
    """(idx, targets) int32 arrays of shape [B, T]: one draw of B*(T+1) ids,
    reshaped to [B, T+1]; inputs are the first T columns and targets the last T
    (targets are the inputs shifted by one position)."""
    n = B * (T + 1)
    if dist == "zipf":
        flat = zipf_tokens(n, vocab, s=s, seed=seed)
    elif dist == "uniform":
        flat = uniform_tokens(n, vocab, seed=seed)
    else:
        raise ValueError(f"unknown token distribution {dist!r}")
    seq = flat.reshape(B, T + 1)
    return np.ascontiguousarray(seq[:, :T]), np.ascontiguousarray(seq[:, 1:])


def byte_table(vocab: int, lo: int, hi: int, seed: int = 2, n_zero: int = 0) -> np.ndarray:
    """int32[vocab] UTF-8 byte length per token id, uniform integers in [lo, hi].

    ``n_zero`` ids (chosen at random) get length 0, the way special tokens do.
    """
    g = _rng(seed)
    t = g.integers(lo, hi + 1, size=vocab, dtype=np.int64).astype(np.int32)
    if n_zero:
        t[g.choice(vocab, size=n_zero, replace=False)] = 0
    return t


def normal(shape, seed: int, std: float = 1.0, dtype=np.float32) -> np.ndarray:
    """Array of N(0, std^2) draws."""
    return (_rng(seed).standard_normal(size=shape) * std).astype(dtype)
