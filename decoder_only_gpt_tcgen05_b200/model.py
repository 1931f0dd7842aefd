"""Model-level calls (include/gpt.h) on torch tensors.

``GPTConfig`` mirrors the C struct ``gpt_config``.  ``GPT`` bundles a config
with its device buffers (parameters, gradients, workspace) and forwards every
call to the library; all the arithmetic runs in the CUDA kernels.
"""
from __future__ import annotations

import ctypes as C
import dataclasses

import torch

from ._lib import call, lib

NORM_RMS, NORM_LN = 0, 1
POS_LEARNED, POS_ROPE = 0, 1
ACT_GELU, ACT_RELU2 = 0, 1


class _CConfig(C.Structure):
    _fields_ = [(n, C.c_int32) for n in ("n_layer", "n_embd", "n_head", "block_size", "vocab_size", "norm", "pos",
                                         "act", "tie_embed", "qk_norm", "linear_bias", "scale_resid_init")] + \
               [("rope_base", C.c_float), ("norm_eps", C.c_float)] + \
               [(n, C.c_int32) for n in ("window_short", "window_pattern", "window_period", "fp8")]


@dataclasses.dataclass(frozen=True)
class GPTConfig:
    n_layer: int
    n_embd: int
    n_head: int
    block_size: int
    vocab_size: int
    norm: int = NORM_RMS
    pos: int = POS_LEARNED
    act: int = ACT_GELU
    tie_embed: int = 1
    qk_norm: int = 0
    linear_bias: int = 0
    scale_resid_init: int = 0
    rope_base: float = 10000.0
    norm_eps: float = 1e-5
    window_short: int = 0     # > 0: left window of the short-window ('S') layers
    window_pattern: int = 0   # bit (l mod window_period) set: layer l is a short-window layer
    window_period: int = 1
    fp8: int = 0              # 1: the forward's block projections on e4m3 operands

    def c(self) -> _CConfig:
        return _CConfig(**dataclasses.asdict(self))


# Named shapes: the GPT-2 124M GPTConfig defaults, the nanochat d20 card, d26 (width 64*26),
# and the 27-token, 1-layer toy model.
PRESETS = {
    "tiny": GPTConfig(n_layer=1, n_embd=16, n_head=4, block_size=16, vocab_size=27, norm=NORM_RMS,
                      pos=POS_LEARNED, act=ACT_GELU, tie_embed=1),
    "gpt2": GPTConfig(n_layer=12, n_embd=768, n_head=12, block_size=1024, vocab_size=50304, norm=NORM_LN,
                      pos=POS_LEARNED, act=ACT_GELU, tie_embed=1, linear_bias=1, scale_resid_init=1),
    "d20": GPTConfig(n_layer=20, n_embd=1280, n_head=10, block_size=2048, vocab_size=32768, norm=NORM_RMS,
                     pos=POS_ROPE, act=ACT_RELU2, tie_embed=0, qk_norm=1),
    "d26": GPTConfig(n_layer=26, n_embd=1664, n_head=13, block_size=2048, vocab_size=32768, norm=NORM_RMS,
                     pos=POS_ROPE, act=ACT_RELU2, tie_embed=0, qk_norm=1),
}


def pattern_bits(pattern: str) -> int:
    """window_pattern of a layer pattern string such as "SSSL" (bit i set for an 'S')."""
    return sum(1 << i for i, ch in enumerate(pattern) if ch == "S")


def preset(name: str, **over) -> GPTConfig:
    return dataclasses.replace(PRESETS[name], **over)


def _stream(dev=None):
    return torch.cuda.current_stream(dev).cuda_stream


def param_count(cfg: GPTConfig) -> int:
    n = C.c_int64()
    c = cfg.c()
    call("gpt_param_count", C.byref(c), C.byref(n))
    return n.value


def param_tensors(cfg: GPTConfig):
    """[(name, offset, rows, cols)] of the flat parameter buffer."""
    c = cfg.c()
    cnt = C.c_int32()
    call("gpt_param_tensor_count", C.byref(c), C.byref(cnt))
    out = []
    buf = C.create_string_buffer(64)
    off, r, k = C.c_int64(), C.c_int64(), C.c_int64()
    for i in range(cnt.value):
        call("gpt_param_tensor", C.byref(c), i, buf, 64, C.byref(off), C.byref(r), C.byref(k))
        out.append((buf.value.decode(), off.value, r.value, k.value))
    return out


def workspace_size(cfg: GPTConfig, B: int, T: int) -> int:
    n = C.c_size_t()
    c = cfg.c()
    call("gpt_workspace_size", C.byref(c), B, T, C.byref(n))
    return n.value


def sync_status(dev=None) -> None:
    call("gpt_sync_status", _stream(dev))


def set_wait_timeout_ns(ns: int) -> None:
    call("gpt_set_wait_timeout_ns", int(ns))


class GPT:
    """A config plus its device buffers for a fixed batch shape (B, T)."""

    def __init__(self, cfg: GPTConfig, B: int, T: int, device="cuda:0", params: torch.Tensor | None = None,
                 seed: int = 0):
        self.cfg, self.B, self.T = cfg, B, T
        self.device = torch.device(device)
        self._c = cfg.c()
        n = param_count(cfg)
        if params is None:
            params = torch.empty(n, dtype=torch.float32, device=self.device)
            self.init_weights(seed, params)
        assert params.numel() == n and params.dtype == torch.float32 and params.is_contiguous()
        self.params = params
        self.grads = torch.zeros(n, dtype=torch.float32, device=self.device)
        self.ws_bytes = workspace_size(cfg, B, T)
        self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8, device=self.device)
        self.loss = torch.zeros(1, dtype=torch.float32, device=self.device)
        self.sum_nats = torch.zeros(1, dtype=torch.float64, device=self.device)
        self.sum_bytes = torch.zeros(1, dtype=torch.int64, device=self.device)
        self.bpb = torch.zeros(1, dtype=torch.float32, device=self.device)

    def init_weights(self, seed: int, params: torch.Tensor | None = None) -> None:
        p = self.params if params is None else params
        call("gpt_init_weights", C.byref(self._c), int(seed), p.data_ptr(), _stream(self.device))

    def forward_loss(self, idx: torch.Tensor, targets: torch.Tensor) -> torch.Tensor:
        """Mean next-token loss (device scalar); keeps activations for backward()."""
        self._check_tokens(idx, targets)
        call("gpt_forward_loss", C.byref(self._c), self.params.data_ptr(), idx.data_ptr(), targets.data_ptr(),
             self.B, self.T, self.workspace.data_ptr(), self.ws_bytes, self.loss.data_ptr(), _stream(self.device))
        return self.loss

    def backward(self, accumulate: bool = False) -> torch.Tensor:
        call("gpt_backward", C.byref(self._c), self.params.data_ptr(), self.B, self.T, self.workspace.data_ptr(),
             self.ws_bytes, self.grads.data_ptr(), int(accumulate), _stream(self.device))
        return self.grads

    def eval_bpb(self, idx: torch.Tensor, targets: torch.Tensor, token_bytes: torch.Tensor):
        """(sum_nats fp64, sum_bytes int64, bpb fp32) device scalars."""
        self._check_tokens(idx, targets)
        assert token_bytes.dtype == torch.int32 and token_bytes.numel() == self.cfg.vocab_size
        call("gpt_eval_bpb", C.byref(self._c), self.params.data_ptr(), idx.data_ptr(), targets.data_ptr(),
             token_bytes.data_ptr(), self.B, self.T, self.workspace.data_ptr(), self.ws_bytes,
             self.sum_nats.data_ptr(), self.sum_bytes.data_ptr(), self.bpb.data_ptr(), _stream(self.device))
        return self.sum_nats, self.sum_bytes, self.bpb

    def token_losses(self):
        """(ell, lse): fp32 [B*T] per-token loss and logsumexp of the last forward_loss / eval_bpb."""
        ell = torch.empty(self.B * self.T, dtype=torch.float32, device=self.device)
        lse = torch.empty_like(ell)
        call("gpt_token_losses", C.byref(self._c), self.B, self.T, self.workspace.data_ptr(), self.ws_bytes,
             ell.data_ptr(), lse.data_ptr(), _stream(self.device))
        return ell, lse

    def debug_logits(self) -> torch.Tensor:
        """fp32 [B*T, V] logits of the last forward (recomputed by the lm_head GEMM; small batches only)."""
        z = torch.empty((self.B * self.T, self.cfg.vocab_size), dtype=torch.float32, device=self.device)
        call("gpt_debug_logits", C.byref(self._c), self.B, self.T, self.workspace.data_ptr(), self.ws_bytes,
             z.data_ptr(), _stream(self.device))
        return z

    def _check_tokens(self, idx, targets):
        for t in (idx, targets):
            assert t.dtype == torch.int32 and t.is_contiguous() and t.numel() == self.B * self.T, \
                "token tensors must be contiguous int32 [B, T]"
            assert t.device == self.device
