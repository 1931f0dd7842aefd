"""B200-native decoder-only GPT hot path: forward + backward of next-token
cross-entropy and bits-per-byte evaluation (plus nanoGPT's AdamW step), as
hand-written sm_100a kernels behind a C ABI (include/gpt.h, include/gpt_ops.h).

This package is the thin Python binding: it passes torch tensors' device
pointers and the current CUDA stream to the library and does nothing else.
"""
from ._lib import GptError, LIB_PATH, lib  # noqa: F401
from . import ops  # noqa: F401
from . import model  # noqa: F401
from .model import GPT, GPTConfig, PRESETS, preset  # noqa: F401
from . import optim  # noqa: F401
from .optim import AdamW, MuonAdamW, lr_schedule  # noqa: F401
