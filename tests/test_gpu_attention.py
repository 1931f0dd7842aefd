"""RoPE + QK-norm + causal flash attention (tcgen05) through the C ABI vs the oracle.

The oracle runs in fp64 on the same bf16-rounded raw q|k|v; the GPU computes
with bf16 operands and fp32 accumulation.  Tolerances follow the parity bar
used for the whole model: outputs within 2e-2 max-abs relative to their RMS,
gradients at cosine >= 0.999 and relative L2 <= 3e-2."""
import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu


def _ops():
    import decoder_only_gpt_tcgen05_b200 as g
    return g.ops


def _oracle_attention(qkv, B, T, H, hd, rope, qk_norm, dout, eps=1e-5):
    """fp64 forward and backward of one attention layer (without projections)."""
    x = qkv.reshape(B, T, 3, H, hd).transpose(2, 0, 3, 1, 4)  # [3, B, H, T, hd]
    q, k, v = x[0], x[1], x[2]
    phi = O.rope_angles(T, hd, 10000.0) if rope else None
    if rope:
        q, k = O.rope(q, phi), O.rope(k, phi)
    if qk_norm:
        qh, rq = O.rmsnorm(q, eps)
        kh, rk = O.rmsnorm(k, eps)
    else:
        qh, kh = q, k
    o, p = O.causal_attention(qh, kh, v)
    s = (qh @ np.swapaxes(kh, -1, -2)) / np.sqrt(hd)
    s = np.where(np.triu(np.ones((T, T), bool), 1), -np.inf, s)
    mx = s.max(-1, keepdims=True)
    lse = (np.log(np.exp(s - mx).sum(-1, keepdims=True)) + mx)[..., 0]
    do = dout.reshape(B, T, H, hd).transpose(0, 2, 1, 3)
    dq, dk, dv = O.causal_attention_bwd(do, qh, kh, v, p)
    if qk_norm:
        dq, dk = O.rmsnorm_bwd(dq, qh, rq), O.rmsnorm_bwd(dk, kh, rk)
    if rope:
        dq, dk = O.rope_bwd(dq, phi), O.rope_bwd(dk, phi)
    dqkv = np.stack([dq, dk, dv]).transpose(1, 3, 0, 2, 4).reshape(B * T, 3 * H * hd)
    return o.transpose(0, 2, 1, 3).reshape(B * T, H * hd), lse, dqkv


def _cos_rel(a, b):
    a, b = a.reshape(-1), b.reshape(-1)
    cos = float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))
    rel = float(np.linalg.norm(a - b) / np.linalg.norm(b))
    return cos, rel


CASES = [
    # (B, T, H, hd, rope, qk_norm)
    (1, 128, 1, 128, True, True),
    (2, 300, 2, 128, True, True),      # ragged T: several tiles and a partial one
    (1, 257, 3, 64, True, True),
    (2, 200, 2, 64, False, False),     # the GPT-2 attention: no RoPE, no QK-norm
    (1, 17, 2, 128, True, True),       # shorter than one tile
]


@pytest.mark.parametrize("case", CASES)
def test_attention_fwd_bwd_matches_oracle(case):
    B, T, H, hd, rope, qk_norm = case
    M = B * T
    qkv = torch.from_numpy(synth.normal((M, 3 * H * hd), 3)).bfloat16()
    dout = torch.from_numpy(synth.normal((M, H * hd), 4)).bfloat16()
    dev = torch.device("cuda:0")
    ops = _ops()
    f = ops.attention_fwd(qkv.to(dev), B, T, H, hd, rope=rope, qk_norm=qk_norm)
    dqkv = ops.attention_bwd(f, dout.to(dev), B, T, H, hd, rope=rope, qk_norm=qk_norm)
    torch.cuda.synchronize()
    o_ref, lse_ref, dqkv_ref = _oracle_attention(qkv.double().numpy(), B, T, H, hd, rope, qk_norm,
                                                 dout.double().numpy())
    o = f["o"].double().cpu().numpy()
    rms = np.sqrt(np.mean(o_ref ** 2))
    assert np.abs(o - o_ref).max() <= 2e-2 * rms, np.abs(o - o_ref).max() / rms
    cos, rel = _cos_rel(o, o_ref)
    assert cos >= 0.9999 and rel <= 1e-2, (cos, rel)
    lse = f["lse"].double().cpu().numpy()
    assert np.abs(lse - lse_ref).max() < 2e-2
    g = dqkv.double().cpu().numpy()
    for i, name in enumerate("qkv"):
        sl = slice(i * H * hd, (i + 1) * H * hd)
        cos, rel = _cos_rel(g[:, sl], dqkv_ref[:, sl])
        assert cos >= 0.999 and rel <= 3e-2, (name, cos, rel)


def test_attention_long_sequence_prefix_is_exact_by_causality():
    """Rows t < 1024 of a T=4096 sequence only see the first 1024 tokens, so
    they equal the T=1024 prefix problem computed by the oracle."""
    B, T, H, hd, P = 1, 4096, 2, 128, 1024
    M = B * T
    qkv = torch.from_numpy(synth.normal((M, 3 * H * hd), 5)).bfloat16()
    dev = torch.device("cuda:0")
    f = _ops().attention_fwd(qkv.to(dev), B, T, H, hd)
    torch.cuda.synchronize()
    o_ref, lse_ref, _ = _oracle_attention(qkv[:P].double().numpy(), 1, P, H, hd, True, True,
                                          np.zeros((P, H * hd)))
    o = f["o"][:P].double().cpu().numpy()
    cos, rel = _cos_rel(o, o_ref)
    assert cos >= 0.9999 and rel <= 1e-2
    assert np.abs(f["lse"][0, :, :P].double().cpu().numpy() - lse_ref[0]).max() < 2e-2
