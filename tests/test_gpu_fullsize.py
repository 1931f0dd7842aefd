"""Parity at the full sizes of the measured workloads, on outputs the oracle can
compute, using properties that hold at any size.

- Sequences are independent, so a batch of B copies of one sequence has the mean
  loss, the bits per byte and the gradients of that single sequence: the GPU runs
  the full launch configuration (d20: B=16 x T=2048; GPT-2: B=8 x T=1024) and the
  oracle runs one sequence.
- Causality: the first P rows of a long sequence's attention equal the length-P
  problem (and with the output gradient zeroed past P, so do the gradients).
- Heads are independent: every row of one (sequence, head) of the full-size
  attention launch is checked against the oracle run on that head alone.
- Rows of the lm_head + cross-entropy are independent: sampled rows are checked
  against fp64 dot products."""
import dataclasses
import math

import numpy as np
import pytest
import torch

import oracle as O
import synth
from bf16_floor import logits_floor

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _pkg():
    import decoder_only_gpt_tcgen05_b200 as g
    return g


def _cos_rel(a, b):
    a, b = a.reshape(-1), b.reshape(-1)
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b))), float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.mark.parametrize("name,B,T,bytes_hi", [("d20", 16, 2048, 16), ("gpt2", 8, 1024, 12)])
def test_full_size_replicated_batch_matches_one_sequence(name, B, T, bytes_hi):
    g = _pkg()
    cfg = g.preset(name)
    ocfg = O.Config(**dataclasses.asdict(cfg))
    model = g.GPT(cfg, B, T, device=DEV, seed=0)
    idx1, tgt1 = synth.next_token_batch(1, T, cfg.vocab_size, seed=1)
    tb = synth.byte_table(cfg.vocab_size, 1, bytes_hi, seed=2, n_zero=5)
    idx = torch.from_numpy(np.repeat(idx1, B, axis=0)).to(DEV)
    tgt = torch.from_numpy(np.repeat(tgt1, B, axis=0)).to(DEV)
    loss = model.forward_loss(idx, tgt).item()
    grads = model.backward().clone()
    model.forward_loss(idx, tgt)
    assert torch.equal(model.backward(), grads)          # bitwise deterministic at full size
    sn, sb, bpb = (t.item() for t in model.eval_bpb(idx, tgt, torch.from_numpy(tb).to(DEV)))
    g.model.sync_status(DEV)
    p = model.params.double().cpu().numpy()
    f = O.forward(ocfg, p, idx1, tgt1)
    rs, rb, _, rbpb = O.bits_per_byte(f["ell"], tgt1, tb)
    assert abs(loss - f["loss"]) / f["loss"] <= 2e-3, (loss, f["loss"])
    assert sb == B * rb
    assert abs(bpb - rbpb) / rbpb <= 2e-3
    assert abs(sn - B * rs) / abs(B * rs) <= 2e-3
    # every token's loss and logsumexp: each of the B copies equals the single sequence, within the
    # logits bar of the model suite (the target's 2e-2 of the RMS, or twice the bf16-operand floor)
    ell, lse = (t.double().cpu().numpy().reshape(B, T) for t in model.token_losses())
    z_rms = float(np.sqrt(np.mean(f["cache"]["z"] ** 2)))
    f_max, _ = logits_floor(ocfg, p, idx1, tgt1, f["cache"]["z"])
    bar = max(2e-2 * z_rms, 2.0 * f_max)
    for got, ref, b in ((lse, f["lse"], bar), (ell, f["ell"], 2 * bar)):
        assert np.abs(got - ref[None, :]).max() <= b, (np.abs(got - ref[None, :]).max() / z_rms, f_max / z_rms)
    assert np.linalg.norm(ell[0] - f["ell"]) <= 2e-3 * np.linalg.norm(f["ell"])
    # every parameter gradient of every layer against the oracle's backward of the one sequence
    ref_g = O.backward(ocfg, p, f)
    got = grads.double().cpu().numpy()
    for nm, (off, shape) in O.param_offsets(ocfg).items():
        n = int(np.prod(shape))
        cos, rel = _cos_rel(got[off:off + n], ref_g[off:off + n])
        assert cos >= 0.999 and rel <= 3e-2, (nm, cos, rel)


def test_attention_sweep_prefix_rows_match_oracle():
    from test_gpu_attention import _oracle_attention, check_stages
    g = _pkg()
    H, hd, P = 10, 128, 512
    # numpy fills row-major, so the first P rows of every draw below are the same numbers:
    # one oracle run on the length-P problem serves every T
    qkv_p = torch.from_numpy(synth.normal((P, 3 * H * hd), 3)).bfloat16()
    dout_p = torch.from_numpy(synth.normal((P, H * hd), 4)).bfloat16()
    o_ref, lse_ref, dqkv_ref = _oracle_attention(qkv_p.double().numpy(), 1, P, H, hd, True, True,
                                                 dout_p.double().numpy())
    for T in (512, 1024, 2048, 4096, 8192):
        B = 32768 // T
        qkv = torch.from_numpy(synth.normal((B * T, 3 * H * hd), 3)).bfloat16()
        dout = torch.from_numpy(synth.normal((B * T, H * hd), 4)).bfloat16()
        assert torch.equal(qkv[:P], qkv_p) and torch.equal(dout[:P], dout_p)
        dout.view(B, T, H * hd)[0, P:] = 0
        f = g.ops.attention_fwd(qkv.to(DEV), B, T, H, hd)
        dq = g.ops.attention_bwd(f, dout.to(DEV), B, T, H, hd)
        torch.cuda.synchronize()
        f_p = {"qkv_norm": f["qkv_norm"][:P], "o": f["o"][:P], "lse": f["lse"][:1, :, :P]}
        check_stages(f_p, qkv_p.double().numpy(), 1, P, H, hd, True, True, None, T)
        got = dq[:T].double().cpu().numpy()   # sequence 0
        for i, nm in enumerate("qkv"):
            sl = slice(i * H * hd, (i + 1) * H * hd)
            cos, rel = _cos_rel(got[:P, sl], dqkv_ref[:, sl])
            assert cos >= 0.999 and rel <= 3e-2, (T, nm, cos, rel)
            if T > P:
                assert np.abs(got[P:, sl]).max() == 0.0, (T, nm)


def test_d26_lmhead_ce_full_size_sampled_rows():
    g = _pkg()
    M, D, V = 32768, 1664, 32768
    x = torch.from_numpy(synth.normal((M, D), 41)).bfloat16()
    w = torch.from_numpy(synth.normal((V, D), 42, std=0.05)).bfloat16()
    tg = torch.from_numpy(synth.zipf_tokens(M, V, seed=43))
    ell, lse = g.ops.lmhead_ce_fwd(x.to(DEV), w.to(DEV), tg.to(DEV))
    torch.cuda.synchronize()
    rows = np.random.default_rng(44).choice(M, 64, replace=False)
    z = x[rows].double().numpy() @ w.double().numpy().T
    ref_ell, ref_lse = O.cross_entropy(z, tg.numpy()[rows])
    assert np.allclose(ell.cpu().numpy()[rows], ref_ell, rtol=2e-3, atol=2e-3)
    assert np.allclose(lse.cpu().numpy()[rows], ref_lse, rtol=1e-4, atol=1e-3)
    assert math.isfinite(float(ell.sum().item()))


@pytest.mark.parametrize("T", [2048, 8192])
def test_attention_every_row_of_one_head_matches_oracle(T):
    """The attention sweep's launch at T (B = 32768 / T, 10 heads of 128): all T rows of the
    first and the last (sequence, head) against the oracle run on that head alone, forward
    (o, logsumexp) and backward (dq, dk, dv through QK-norm and RoPE)."""
    from test_gpu_attention import _oracle_attention, check_stages
    g = _pkg()
    H, hd = 10, 128
    B = 32768 // T
    qkv = torch.from_numpy(synth.normal((B * T, 3 * H * hd), 3)).bfloat16()
    dout = torch.from_numpy(synth.normal((B * T, H * hd), 4)).bfloat16()
    f = g.ops.attention_fwd(qkv.to(DEV), B, T, H, hd)
    dq = g.ops.attention_bwd(f, dout.to(DEV), B, T, H, hd)
    torch.cuda.synchronize()
    o_all = f["o"].double().cpu().numpy()
    lse_all = f["lse"].double().cpu().numpy()
    dq_all = dq.double().cpu().numpy()
    qkv_np = qkv.double().numpy()
    dout_np = dout.double().numpy()
    qn_all = f["qkv_norm"].double().cpu().numpy()
    for b, h in ((0, 0), (B - 1, H - 1)):
        rows = slice(b * T, (b + 1) * T)
        cols = [slice(i * H * hd + h * hd, i * H * hd + (h + 1) * hd) for i in range(3)]
        qkv1 = np.concatenate([qkv_np[rows, c] for c in cols], axis=1)
        _, _, dqkv_ref = _oracle_attention(qkv1, 1, T, 1, hd, True, True, dout_np[rows, h * hd:(h + 1) * hd])
        # forward stages on this head: RoPE + QK-norm, then attention on the op's own bf16 q, k, v
        f1 = {"qkv_norm": torch.from_numpy(np.concatenate([qn_all[rows, c] for c in cols], axis=1)),
              "o": torch.from_numpy(o_all[rows, h * hd:(h + 1) * hd]),
              "lse": torch.from_numpy(lse_all[b:b + 1, h:h + 1])}
        check_stages(f1, qkv1, 1, T, 1, hd, True, True, None, (T, b, h))
        for i, nm in enumerate("qkv"):
            cos, rel = _cos_rel(dq_all[rows, cols[i]], dqkv_ref[:, i * hd:(i + 1) * hd])
            assert cos >= 0.999 and rel <= 3e-2, (T, b, h, nm, cos, rel)
