"""Op-level calls (include/gpt_ops.h) on torch tensors."""
from __future__ import annotations

import torch

from ._lib import AdamWParams, call

GEMM_OUT_BF16 = 0
GEMM_OUT_F32 = 1


def _stream(t: torch.Tensor):
    return torch.cuda.current_stream(t.device).cuda_stream


def gemm(a: torch.Tensor, b: torch.Tensor, out: torch.Tensor, *, a_mn: bool = False, b_mn: bool = False,
         bias: torch.Tensor | None = None, accumulate: bool = False, bn: int = 256,
         M: int | None = None, N: int | None = None, K: int | None = None) -> torch.Tensor:
    """out[M,N] = A[M,K] B[N,K]^T.  ``a`` is [M,K] (or [K,M] when a_mn), ``b``
    is [N,K] (or [K,N] when b_mn), both bf16; ``out`` is bf16 or fp32 with at
    least N columns.  M, N, K default to the tensors' logical shapes; pass them
    when the storage is wider than the matrix (padded pitches)."""
    assert a.dtype == torch.bfloat16 and b.dtype == torch.bfloat16
    M = M if M is not None else (a.shape[1] if a_mn else a.shape[0])
    K = K if K is not None else (a.shape[0] if a_mn else a.shape[1])
    N = N if N is not None else (b.shape[1] if b_mn else b.shape[0])
    epi = GEMM_OUT_F32 if out.dtype == torch.float32 else GEMM_OUT_BF16
    call("gpt_op_gemm", epi, bn, a.data_ptr(), a.stride(0), int(a_mn), b.data_ptr(), b.stride(0), int(b_mn),
         M, N, K, out.data_ptr(), out.stride(0), bias.data_ptr() if bias is not None else None,
         int(accumulate), _stream(out))
    return out


FP8_E4M3, FP8_E5M2 = 0, 1


def fp8_quantize(x: torch.Tensor, fmt: int = FP8_E4M3, out: torch.Tensor | None = None):
    """(q uint8 same shape as x, amax fp32 [1], inv_scale fp32 [1]): x cast to 8-bit floats with the
    per-tensor scale FP8_MAX / max|x|.  x: contiguous bf16 or fp32."""
    assert x.is_contiguous() and x.dtype in (torch.bfloat16, torch.float32)
    q = torch.empty(x.shape, dtype=torch.uint8, device=x.device) if out is None else out
    assert q.dtype == torch.uint8 and q.is_contiguous() and q.numel() == x.numel()
    amax = torch.empty(1, dtype=torch.float32, device=x.device)
    inv = torch.empty(1, dtype=torch.float32, device=x.device)
    call("gpt_op_fp8_quantize", x.data_ptr(), int(x.dtype == torch.float32), x.numel(), fmt, q.data_ptr(),
         amax.data_ptr(), inv.data_ptr(), _stream(x))
    return q, amax, inv


def gemm_fp8(a: torch.Tensor, fmt_a: int, inv_a: torch.Tensor, b: torch.Tensor, fmt_b: int, inv_b: torch.Tensor,
             out: torch.Tensor, *, bias: torch.Tensor | None = None, accumulate: bool = False, bn: int = 256):
    """out[M,N] = (A B^T) inv_a inv_b for 8-bit (uint8-stored) A [M,K], B [N,K], both K-major."""
    assert a.dtype == torch.uint8 and b.dtype == torch.uint8 and a.shape[1] == b.shape[1]
    M, K = a.shape
    N = b.shape[0]
    epi = GEMM_OUT_F32 if out.dtype == torch.float32 else GEMM_OUT_BF16
    call("gpt_op_gemm_fp8", epi, bn, a.data_ptr(), a.stride(0), fmt_a, b.data_ptr(), b.stride(0), fmt_b, M, N, K,
         inv_a.data_ptr(), inv_b.data_ptr(), out.data_ptr(), out.stride(0),
         bias.data_ptr() if bias is not None else None, int(accumulate), _stream(out))
    return out


def _ptr(t):
    return t.data_ptr() if t is not None else None


def attention_fwd(qkv: torch.Tensor, B: int, T: int, H: int, hd: int, *, rope: bool = True, qk_norm: bool = True,
                  window: int = -1, rope_base: float = 10000.0, eps: float = 1e-5, out: dict | None = None):
    """RoPE + QK-norm + causal attention.  qkv: bf16 [B*T, 3*H*hd] (raw).  window >= 0 limits
    query i to keys i - window .. i (-1: every earlier key).
    Returns a dict with qkv_norm, rstd_q, rstd_k, rope_cs, o, lse; ``out``, a
    dict returned by an earlier call with the same sizes, is written again
    instead of allocating."""
    dev = qkv.device
    M = B * T
    r = out if out is not None else {
        "qkv_norm": torch.empty((M, 3 * H * hd), dtype=torch.bfloat16, device=dev),
        "rstd_q": torch.empty((M, H), dtype=torch.float32, device=dev) if qk_norm else None,
        "rstd_k": torch.empty((M, H), dtype=torch.float32, device=dev) if qk_norm else None,
        "rope_cs": torch.empty((T, hd // 2, 2), dtype=torch.float32, device=dev) if rope else None,
        "o": torch.empty((M, H * hd), dtype=torch.bfloat16, device=dev),
        "lse": torch.empty((B, H, T), dtype=torch.float32, device=dev),
    }
    assert r["qkv_norm"].numel() >= M * 3 * H * hd and r["o"].numel() >= M * H * hd and r["lse"].numel() >= M * H
    assert not rope or r["rope_cs"].numel() >= T * hd
    assert not qk_norm or (r["rstd_q"].numel() >= M * H and r["rstd_k"].numel() >= M * H)
    call("gpt_op_attention_fwd", qkv.data_ptr(), B, T, H, hd, int(rope), int(qk_norm), int(window), rope_base, eps,
         r["qkv_norm"].data_ptr(), _ptr(r["rstd_q"]), _ptr(r["rstd_k"]), _ptr(r["rope_cs"]), r["o"].data_ptr(),
         r["lse"].data_ptr(), _stream(qkv))
    return r


def attention_bwd(fwd: dict, dout: torch.Tensor, B: int, T: int, H: int, hd: int, *, rope: bool = True,
                  qk_norm: bool = True, window: int = -1, delta: torch.Tensor | None = None,
                  dqkv: torch.Tensor | None = None) -> torch.Tensor:
    """dL/dqkv (bf16 [B*T, 3*H*hd]) from dout = dL/do (bf16 [B*T, H*hd]).
    ``delta`` (fp32 [B, H, T] scratch) and ``dqkv`` may be passed in to avoid
    allocating them."""
    dev = dout.device
    if delta is None:
        delta = torch.empty((B, H, T), dtype=torch.float32, device=dev)
    if dqkv is None:
        dqkv = torch.empty((B * T, 3 * H * hd), dtype=torch.bfloat16, device=dev)
    assert delta.numel() >= B * H * T and dqkv.numel() >= B * T * 3 * H * hd
    call("gpt_op_attention_bwd", fwd["qkv_norm"].data_ptr(), _ptr(fwd["rstd_q"]), _ptr(fwd["rstd_k"]),
         _ptr(fwd["rope_cs"]), fwd["o"].data_ptr(), fwd["lse"].data_ptr(), dout.data_ptr(), B, T, H, hd, int(rope),
         int(qk_norm), int(window), delta.data_ptr(), dqkv.data_ptr(), _stream(dout))
    return dqkv


def _check_lmhead(x, w, targets, ell=None, lse=None):
    assert x.dim() == 2 and w.dim() == 2 and x.shape[1] == w.shape[1], "x [M, D] and w [V, D]"
    for t in (x, w):
        assert t.dtype == torch.bfloat16 and t.is_contiguous() and t.device == x.device, "x, w: contiguous bf16"
    assert targets.dtype == torch.int32 and targets.is_contiguous() and targets.device == x.device, \
        "targets: contiguous int32 on the device of x"
    assert targets.numel() >= x.shape[0], "one target per row of x"
    for t in (ell, lse):
        if t is not None:
            assert t.dtype == torch.float32 and t.is_contiguous() and t.device == x.device and \
                t.numel() >= x.shape[0], "ell, lse: contiguous fp32 with at least M elements"


def lmhead_ce_fwd(x: torch.Tensor, w: torch.Tensor, targets: torch.Tensor):
    """Per-row (loss, logsumexp) of logits x w^T without storing them.
    x bf16 [M, D], w bf16 [V, D], targets int32 [M]."""
    from ._lib import lib
    _check_lmhead(x, w, targets)
    M, D = x.shape
    V = w.shape[0]
    ell = torch.empty(M, dtype=torch.float32, device=x.device)
    lse = torch.empty(M, dtype=torch.float32, device=x.device)
    scratch = torch.empty(lib().gpt_op_lmhead_ce_scratch_bytes(M, V), dtype=torch.uint8, device=x.device)
    call("gpt_op_lmhead_ce_fwd", x.data_ptr(), w.data_ptr(), targets.data_ptr(), M, D, V, ell.data_ptr(),
         lse.data_ptr(), scratch.data_ptr(), _stream(x))
    return ell, lse


def lmhead_ce_fwd_noalloc(x: torch.Tensor, w: torch.Tensor, targets: torch.Tensor,
                          ell: torch.Tensor | None = None, lse: torch.Tensor | None = None):
    """lmhead_ce_fwd without caller scratch: the library keeps its scratch in a
    fixed device array, so only the outputs are passed (pre-allocate them to
    make the call itself allocation-free)."""
    _check_lmhead(x, w, targets, ell, lse)
    M, D = x.shape
    V = w.shape[0]
    ell = torch.empty(M, dtype=torch.float32, device=x.device) if ell is None else ell
    lse = torch.empty(M, dtype=torch.float32, device=x.device) if lse is None else lse
    call("gpt_op_lmhead_ce_fwd_noalloc", x.data_ptr(), w.data_ptr(), targets.data_ptr(), M, D, V, ell.data_ptr(),
         lse.data_ptr(), _stream(x))
    return ell, lse


PROFILE_FAMILIES = ["gemm", "attn_fwd", "attn_bwd_dkv", "attn_bwd_dq", "norm_fwd", "norm_bwd", "embed_fwd",
                    "embed_bwd", "cast", "ce_combine", "loss", "qk", "delta", "colsum", "misc",
                    "gemm_qkv", "gemm_o", "gemm_up", "gemm_down", "gemm_lm_fwd", "gemm_lm_bwd", "gemm_dgrad",
                    "gemm_wgrad", "optim", "gemm_muon"]
GEMM_FAMILIES = [f for f in PROFILE_FAMILIES if f.startswith("gemm")]


def launch_count() -> int:
    from ._lib import lib
    return int(lib().gpt_launch_count())


def profile_start() -> None:
    call("gpt_profile_start")


def profile_stop() -> dict:
    """{family: (ms, launches, flops, bytes)} summed over the launches since profile_start()."""
    import ctypes as C
    from ._lib import lib
    n = len(PROFILE_FAMILIES)
    ms = (C.c_double * n)()
    cnt = (C.c_longlong * n)()
    fl = (C.c_double * n)()
    by = (C.c_double * n)()
    rc = lib().gpt_profile_stop(n, ms, cnt, fl, by)
    if rc != n:
        raise RuntimeError(lib().gpt_last_error().decode())
    return {f: (ms[i], cnt[i], fl[i], by[i]) for i, f in enumerate(PROFILE_FAMILIES)}


def adamw(params: torch.Tensor, grads: torch.Tensor, m: torch.Tensor, v: torch.Tensor, run_start, run_decay,
          step: int, *, lr: float, beta1: float = 0.9, beta2: float = 0.999, eps: float = 1e-8,
          weight_decay: float = 0.0, grad_scale: float = 1.0, grad_clip: float = 0.0,
          scratch: torch.Tensor | None = None, grad_norm: torch.Tensor | None = None) -> torch.Tensor:
    """clip_grad_norm_ + AdamW over flat fp32 buffers (gpt_op_adamw).  run_start / run_decay: the
    weight-decay table (run r covers [run_start[r], run_start[r+1]), decayed when run_decay[r]).
    Returns the fp64 gradient norm (device scalar)."""
    import ctypes as C
    from ._lib import lib
    n = params.numel()
    for t in (params, grads, m, v):
        assert t.dtype == torch.float32 and t.is_contiguous() and t.numel() == n and t.device == params.device
    dev = params.device
    if scratch is None:
        scratch = torch.empty(int(lib().gpt_op_adamw_scratch_bytes()), dtype=torch.uint8, device=dev)
    if grad_norm is None:
        grad_norm = torch.empty((), dtype=torch.float64, device=dev)
    rs = (C.c_int64 * len(run_start))(*[int(x) for x in run_start])
    rd = (C.c_uint8 * len(run_decay))(*[1 if x else 0 for x in run_decay])
    h = AdamWParams(lr, beta1, beta2, eps, weight_decay, grad_scale, grad_clip)
    call("gpt_op_adamw", params.data_ptr(), grads.data_ptr(), m.data_ptr(), v.data_ptr(), n, rs, rd, len(run_start),
         step, C.byref(h), scratch.data_ptr(), grad_norm.data_ptr(), _stream(params))
    return grad_norm
