"""Op-level calls (include/gpt_ops.h) on torch tensors."""
from __future__ import annotations

import torch

from ._lib import call

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


def _ptr(t):
    return t.data_ptr() if t is not None else None


def attention_fwd(qkv: torch.Tensor, B: int, T: int, H: int, hd: int, *, rope: bool = True, qk_norm: bool = True,
                  rope_base: float = 10000.0, eps: float = 1e-5):
    """RoPE + QK-norm + causal attention.  qkv: bf16 [B*T, 3*H*hd] (raw).
    Returns a dict with qkv_norm, rstd_q, rstd_k, rope_cs, o, lse."""
    dev = qkv.device
    M = B * T
    r = {
        "qkv_norm": torch.empty((M, 3 * H * hd), dtype=torch.bfloat16, device=dev),
        "rstd_q": torch.empty((M, H), dtype=torch.float32, device=dev) if qk_norm else None,
        "rstd_k": torch.empty((M, H), dtype=torch.float32, device=dev) if qk_norm else None,
        "rope_cs": torch.empty((T, hd // 2, 2), dtype=torch.float32, device=dev) if rope else None,
        "o": torch.empty((M, H * hd), dtype=torch.bfloat16, device=dev),
        "lse": torch.empty((B, H, T), dtype=torch.float32, device=dev),
    }
    call("gpt_op_attention_fwd", qkv.data_ptr(), B, T, H, hd, int(rope), int(qk_norm), rope_base, eps,
         r["qkv_norm"].data_ptr(), _ptr(r["rstd_q"]), _ptr(r["rstd_k"]), _ptr(r["rope_cs"]), r["o"].data_ptr(),
         r["lse"].data_ptr(), _stream(qkv))
    return r


def attention_bwd(fwd: dict, dout: torch.Tensor, B: int, T: int, H: int, hd: int, *, rope: bool = True,
                  qk_norm: bool = True) -> torch.Tensor:
    """dL/dqkv (bf16 [B*T, 3*H*hd]) from dout = dL/do (bf16 [B*T, H*hd])."""
    dev = dout.device
    delta = torch.empty((B, H, T), dtype=torch.float32, device=dev)
    dqkv = torch.empty((B * T, 3 * H * hd), dtype=torch.bfloat16, device=dev)
    call("gpt_op_attention_bwd", fwd["qkv_norm"].data_ptr(), _ptr(fwd["rstd_q"]), _ptr(fwd["rstd_k"]),
         _ptr(fwd["rope_cs"]), fwd["o"].data_ptr(), fwd["lse"].data_ptr(), dout.data_ptr(), B, T, H, hd, int(rope),
         int(qk_norm), delta.data_ptr(), dqkv.data_ptr(), _stream(dout))
    return dqkv
