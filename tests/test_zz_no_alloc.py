"""The allocation-free lm_head + cross-entropy entry point.

Callers that cannot allocate device memory on this path (a loop whose device
memory is all reserved by its own pool, or that cannot take the device-wide
synchronisation of a cudaMalloc mid-step) use gpt_op_lmhead_ce_fwd_noalloc,
which keeps its scratch in a fixed device array.  Its results must equal
those of gpt_op_lmhead_ce_fwd (caller scratch) on the same inputs, call after
call, although every call reuses the same array.

This file is collected last on purpose, and must pass alone or after the rest."""
import ctypes as C

import numpy as np
import pytest
import torch

import synth

DEV = torch.device("cuda:0")


@pytest.mark.gpu
def test_noalloc_matches_scratch_entry_point_twice():
    import decoder_only_gpt_tcgen05_b200 as g
    M, D, V = 3000, 256, 5000
    x = torch.from_numpy(synth.normal((M, D), 31)).bfloat16().to(DEV)
    w = torch.from_numpy(synth.normal((V, D), 32, std=0.1)).bfloat16().to(DEV)
    ell = torch.empty(M, dtype=torch.float32, device=DEV)
    lse = torch.empty(M, dtype=torch.float32, device=DEV)
    for call_no, seed in enumerate((33, 34)):
        tg = torch.from_numpy(synth.zipf_tokens(M, V, seed=seed)).to(DEV)
        ref_ell, ref_lse = g.ops.lmhead_ce_fwd(x, w, tg)
        g.ops.lmhead_ce_fwd_noalloc(x, w, tg, ell=ell, lse=lse)
        torch.cuda.synchronize()
        for a, b in ((ell, ref_ell), (lse, ref_lse)):
            a, b = a.double().cpu().numpy(), b.double().cpu().numpy()
            assert np.all(np.isfinite(a))
            assert np.abs(a - b).max() <= 2e-3 * np.abs(b).max(), (call_no, np.abs(a - b).max())


@pytest.mark.gpu
def test_noalloc_rejects_sizes_beyond_its_array():
    import decoder_only_gpt_tcgen05_b200 as g
    L = g.lib()
    cap = L.gpt_op_lmhead_ce_noalloc_max_scratch_bytes()
    M, V = 40000, 32768
    assert L.gpt_op_lmhead_ce_scratch_bytes(M, V) > cap
    fake = C.c_void_p(1 << 20)
    assert L.gpt_op_lmhead_ce_fwd_noalloc(fake, fake, fake, M, 256, V, fake, fake, None) == 1
    assert b"scratch" in L.gpt_last_error()
