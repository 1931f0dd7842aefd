"""The allocation-free lm_head + cross-entropy entry point.

Callers that cannot allocate device memory on this path (a loop whose device
memory is all reserved by its own pool, or that cannot take the device-wide
synchronisation of a cudaMalloc mid-step) use gpt_op_lmhead_ce_fwd_noalloc,
which keeps its scratch in a fixed device array.  Its results must match the
oracle's cross-entropy of the fp64 product of the same bf16 operands, and equal
those of gpt_op_lmhead_ce_fwd (caller scratch) on the same inputs, call after
call, although every call reuses the same array.

This file is collected last on purpose, and must pass alone or after the rest."""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle as O
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
    z = x.double().cpu().numpy() @ w.double().cpu().numpy().T
    z_rms = float(np.sqrt(np.mean(z ** 2)))
    for call_no, seed in enumerate((33, 34)):
        tg_np = synth.zipf_tokens(M, V, seed=seed)
        tg = torch.from_numpy(tg_np).to(DEV)
        ref_ell, ref_lse = g.ops.lmhead_ce_fwd(x, w, tg)
        g.ops.lmhead_ce_fwd_noalloc(x, w, tg, ell=ell, lse=lse)
        torch.cuda.synchronize()
        or_ell, or_lse = O.cross_entropy(z, tg_np)
        for a, b, o, bar in ((ell, ref_ell, or_ell, 4e-2), (lse, ref_lse, or_lse, 2e-2)):
            a, b = a.double().cpu().numpy(), b.double().cpu().numpy()
            assert np.all(np.isfinite(a))
            # the oracle: logsumexp and loss are 1-Lipschitz in the logits' max-norm, so the
            # logits bar (2e-2 of their RMS) bounds them by 2e-2 and 4e-2 of that RMS
            assert np.abs(a - o).max() <= bar * z_rms, (call_no, np.abs(a - o).max() / z_rms)
            assert np.linalg.norm(a - o) <= 2e-3 * np.linalg.norm(o)
            # the entry point with caller scratch
            assert np.abs(a - b).max() <= 2e-3 * np.abs(b).max(), (call_no, np.abs(a - b).max())


@pytest.mark.gpu
def test_noalloc_target_out_of_range_gets_nan_not_a_stale_value():
    """A target outside [0, V) has no logit, so its slot in the shared array is not written by
    the product: after a valid call, that row must come out NaN (reported through the status
    word), never the previous call's value, while every other row stays correct."""
    import decoder_only_gpt_tcgen05_b200 as g
    M, D, V = 1000, 128, 3000
    x = torch.from_numpy(synth.normal((M, D), 35)).bfloat16().to(DEV)
    w = torch.from_numpy(synth.normal((V, D), 36, std=0.1)).bfloat16().to(DEV)
    tg_np = synth.zipf_tokens(M, V, seed=37)
    g.ops.lmhead_ce_fwd_noalloc(x, w, torch.from_numpy(tg_np).to(DEV))
    g.model.sync_status(DEV)
    bad = tg_np.copy()
    bad[3], bad[600] = V, -1
    ell, lse = g.ops.lmhead_ce_fwd_noalloc(x, w, torch.from_numpy(bad).to(DEV))
    with pytest.raises(g.GptError) as e:
        g.model.sync_status(DEV)
    assert e.value.code == 1
    ell, lse = ell.double().cpu().numpy(), lse.double().cpu().numpy()
    assert np.isnan(ell[3]) and np.isnan(ell[600])
    z = x.double().cpu().numpy() @ w.double().cpu().numpy().T
    or_ell, or_lse = O.cross_entropy(z, tg_np)
    keep = np.ones(M, bool)
    keep[[3, 600]] = False
    z_rms = float(np.sqrt(np.mean(z ** 2)))
    assert np.abs(ell[keep] - or_ell[keep]).max() <= 4e-2 * z_rms
    assert np.abs(lse - or_lse).max() <= 2e-2 * z_rms


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
