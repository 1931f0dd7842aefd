"""ctypes loader for libgpt_b200.so: argument marshalling only.

Every call goes straight to the C ABI declared in include/gpt.h and
include/gpt_ops.h; there is no Python or CPU fallback.  If the library has not
been built, importing the binding raises.
"""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libgpt_b200.so")

_lib = None


class GptError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"gpt status {code}: {msg}")
        self.code = code


_P = C.c_void_p
_I = C.c_int
_LL = C.c_longlong
_F = C.c_float

# name -> argument types (restype is int for all but gpt_last_error)
SIGNATURES = {
    "gpt_op_gemm": [_I, _I, _P, _LL, _I, _P, _LL, _I, _I, _I, _I, _P, _LL, _P, _I, _P],
    "gpt_op_attention_fwd": [_P, _I, _I, _I, _I, _I, _I, _I, _F, _F, _P, _P, _P, _P, _P, _P, _P],
    "gpt_op_attention_bwd": [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P],
    "gpt_op_lmhead_ce_fwd": [_P, _P, _P, _I, _I, _I, _P, _P, _P, _P],
    "gpt_op_lmhead_ce_fwd_noalloc": [_P, _P, _P, _I, _I, _I, _P, _P, _P],
    "gpt_op_wait_probe": [C.c_ulonglong, _P],
    "gpt_op_exp2": [_P, C.c_longlong, C.c_int, _P, _P],
    "gpt_profile_start": [],
    "gpt_profile_stop": [_I, _P, _P, _P, _P],
    "gpt_param_count": [_P, _P],
    "gpt_param_tensor_count": [_P, _P],
    "gpt_param_tensor": [_P, _I, _P, _I, _P, _P, _P],
    "gpt_workspace_size": [_P, _I, _I, _P],
    "gpt_init_weights": [_P, C.c_uint64, _P, _P],
    "gpt_forward_loss": [_P, _P, _P, _P, _I, _I, _P, C.c_size_t, _P, _P],
    "gpt_backward": [_P, _P, _I, _I, _P, C.c_size_t, _P, _I, _P],
    "gpt_eval_bpb": [_P, _P, _P, _P, _P, _I, _I, _P, C.c_size_t, _P, _P, _P, _P],
    "gpt_token_losses": [_P, _I, _I, _P, C.c_size_t, _P, _P, _P],
    "gpt_debug_logits": [_P, _I, _I, _P, C.c_size_t, _P, _P],
    "gpt_sync_status": [_P],
    "gpt_set_wait_timeout_ns": [C.c_uint64],
    "gpt_adamw_scratch_size": [_P],
    "gpt_adamw_step": [_P, _P, _P, _P, _P, _LL, _P, _P, _P, _P],
    "gpt_lr_schedule": [_LL, _LL, _LL, C.c_double, C.c_double, _P],
    "gpt_op_adamw": [_P, _P, _P, _P, _LL, _P, _P, _I, _LL, _P, _P, _P, _P],
    "gpt_op_fp8_quantize": [_P, _I, _LL, _I, _P, _P, _P, _P],
    "gpt_op_gemm_fp8": [_I, _I, _P, _LL, _I, _P, _LL, _I, _I, _I, _I, _P, _P, _P, _LL, _P, _I, _P],
    "gpt_muon_scratch_size": [_P, _P],
    "gpt_grad_buckets": [_P, C.c_int32, _P, _P, _P],
    "gpt_backward_bucketed": [_P, _P, _I, _I, _P, C.c_size_t, _P, _I, _P, _I, _P],
    "gpt_muon_step": [_P, _P, _P, _P, _P, _LL, _P, _P, _P],
}


class MuonParams(C.Structure):
    """gpt_muon of include/gpt.h."""
    _fields_ = [("lr", C.c_float), ("momentum", C.c_float), ("nesterov", C.c_int32), ("ns_steps", C.c_int32),
                ("adam_lr", C.c_float), ("beta1", C.c_float), ("beta2", C.c_float), ("eps", C.c_float),
                ("weight_decay", C.c_float)]


class AdamWParams(C.Structure):
    """gpt_adamw of include/gpt.h."""
    _fields_ = [("lr", C.c_float), ("beta1", C.c_float), ("beta2", C.c_float), ("eps", C.c_float),
                ("weight_decay", C.c_float), ("grad_scale", C.c_float), ("grad_clip", C.c_float)]


def lib():
    """The loaded library (loaded on first use)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m decoder_only_gpt_tcgen05_b200.build`")
        L = C.CDLL(LIB_PATH)
        L.gpt_last_error.restype = C.c_char_p
        L.gpt_last_error.argtypes = []
        L.gpt_launch_count.restype = C.c_ulonglong
        L.gpt_launch_count.argtypes = []
        L.gpt_op_lmhead_ce_scratch_bytes.restype = C.c_size_t
        L.gpt_op_lmhead_ce_scratch_bytes.argtypes = [_I, _I]
        L.gpt_op_lmhead_ce_noalloc_max_scratch_bytes.restype = C.c_size_t
        L.gpt_op_lmhead_ce_noalloc_max_scratch_bytes.argtypes = []
        L.gpt_op_adamw_scratch_bytes.restype = C.c_size_t
        L.gpt_op_adamw_scratch_bytes.argtypes = []
        for name, args in SIGNATURES.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = C.c_int
        _lib = L
    return _lib


def check(rc: int) -> None:
    if rc != 0:
        raise GptError(rc, lib().gpt_last_error().decode())


def call(name: str, *args) -> None:
    check(getattr(lib(), name)(*args))
