"""nanoGPT's optimizer step on a GPT's buffers (include/gpt.h: gpt_adamw_step, gpt_lr_schedule).

``AdamW`` owns the two moment buffers and the step count and calls the library's fused step:
global-norm clipping as clip_grad_norm_ does it, then AdamW with weight decay on the 2-D tensors
("nanoGPT - Karpathy's minimal GPT pretraining repo", How it works: configure_optimizers, train.py).
The defaults of betas, eps and weight_decay are those of PyTorch's AdamW, the routine the page
names; learning_rate and grad_clip default to the page's 6e-4 and 1.0."""
from __future__ import annotations

import ctypes as C

import torch

from ._lib import AdamWParams, MuonParams, call


def lr_schedule(it: int, warmup_iters: int, lr_decay_iters: int, learning_rate: float, min_lr: float) -> float:
    """Linear warmup, then cosine decay to min_lr (computed by the library on the host)."""
    out = C.c_double()
    call("gpt_lr_schedule", it, warmup_iters, lr_decay_iters, learning_rate, min_lr, C.byref(out))
    return out.value


class AdamW:
    def __init__(self, model, lr: float = 6e-4, betas=(0.9, 0.999), eps: float = 1e-8, weight_decay: float = 0.01,
                 grad_clip: float = 1.0):
        self.model = model
        self.lr, self.betas, self.eps, self.weight_decay, self.grad_clip = lr, tuple(betas), eps, weight_decay, grad_clip
        self.m = torch.zeros_like(model.params)
        self.v = torch.zeros_like(model.params)
        n = C.c_size_t()
        call("gpt_adamw_scratch_size", C.byref(n))
        self.scratch = torch.empty(n.value, dtype=torch.uint8, device=model.device)
        self.grad_norm = torch.zeros((), dtype=torch.float64, device=model.device)
        self.step_count = 0

    def step(self, lr: float | None = None, grad_scale: float = 1.0) -> torch.Tensor:
        """One step from model.grads (grad_scale multiplies them first, e.g. 1 / micro-steps).
        Returns the pre-clipping gradient norm as a device scalar (no synchronisation)."""
        self.step_count += 1
        h = AdamWParams(self.lr if lr is None else lr, self.betas[0], self.betas[1], self.eps, self.weight_decay,
                        grad_scale, self.grad_clip)
        mdl = self.model
        call("gpt_adamw_step", C.byref(mdl._c), mdl.params.data_ptr(), mdl.grads.data_ptr(), self.m.data_ptr(),
             self.v.data_ptr(), self.step_count, C.byref(h), self.scratch.data_ptr(), self.grad_norm.data_ptr(),
             torch.cuda.current_stream(mdl.device).cuda_stream)
        return self.grad_norm


class MuonAdamW:
    """nanochat's split optimizer ("Train your own ChatGPT", read the source optim.py): Muon on the
    block matrices, AdamW on everything else (include/gpt.h: gpt_muon_step).  Owns the momentum /
    first-moment buffer, the second-moment buffer, the scratch and the step count."""

    def __init__(self, model, lr: float = 0.02, momentum: float = 0.95, nesterov: bool = True, ns_steps: int = 5,
                 adam_lr: float = 3e-4, betas=(0.9, 0.95), eps: float = 1e-8, weight_decay: float = 0.0):
        self.model = model
        self.h = MuonParams(lr, momentum, int(nesterov), ns_steps, adam_lr, betas[0], betas[1], eps, weight_decay)
        self.mom = torch.zeros_like(model.params)
        self.v = torch.zeros_like(model.params)
        n = C.c_size_t()
        call("gpt_muon_scratch_size", C.byref(model._c), C.byref(n))
        self.scratch = torch.empty(n.value, dtype=torch.uint8, device=model.device)
        self.step_count = 0

    def step(self) -> None:
        self.step_count += 1
        mdl = self.model
        call("gpt_muon_step", C.byref(mdl._c), mdl.params.data_ptr(), mdl.grads.data_ptr(), self.mom.data_ptr(),
             self.v.data_ptr(), self.step_count, C.byref(self.h), self.scratch.data_ptr(),
             torch.cuda.current_stream(mdl.device).cuda_stream)
