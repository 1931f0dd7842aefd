"""tcgen05 GEMM through the C ABI vs an fp64 matmul of the same bf16 inputs."""
import math

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _ops():
    import decoder_only_gpt_tcgen05_b200 as g
    return g.ops


# the last two give N-256 tiles to at least one CTA pair per two SMs, so they run on the
# CTA-pair kernel (256-row tiles); the others on the single-CTA kernel
SHAPES = [(128, 128, 64), (300, 200, 136), (256, 512, 1280), (1, 40, 16), (515, 777, 333), (2560, 2048, 256),
          (2500, 2000, 200)]


@pytest.mark.parametrize("a_mn", [0, 1])
@pytest.mark.parametrize("b_mn", [0, 1])
@pytest.mark.parametrize("bn", [128, 256])
@pytest.mark.parametrize("shape", SHAPES)
def test_gemm_fp32_out(a_mn, b_mn, bn, shape):
    M, N, K = shape
    # pitches rounded up to 8 elements (16 bytes) as the ABI requires
    ka = (M if a_mn else K)
    kb = (N if b_mn else K)
    lda, ldb, ldo = -(-ka // 8) * 8, -(-kb // 8) * 8, -(-N // 4) * 4
    A = torch.from_numpy(synth.normal((M, K), 1)).bfloat16()
    B = torch.from_numpy(synth.normal((N, K), 2)).bfloat16()
    ref = A.double().numpy() @ B.double().numpy().T
    a_store = torch.zeros((K, lda) if a_mn else (M, lda), dtype=torch.bfloat16)
    if a_mn:
        a_store[:, :M] = A.T
    else:
        a_store[:, :K] = A
    b_store = torch.zeros((K, ldb) if b_mn else (N, ldb), dtype=torch.bfloat16)
    if b_mn:
        b_store[:, :N] = B.T
    else:
        b_store[:, :K] = B
    dev = torch.device("cuda:0")
    a_d, b_d = a_store.to(dev), b_store.to(dev)
    out = torch.full((M, ldo), float("nan"), dtype=torch.float32, device=dev)
    _ops().gemm(a_d, b_d, out, a_mn=bool(a_mn), b_mn=bool(b_mn), bn=bn, M=M, N=N, K=K)
    torch.cuda.synchronize()
    got = out[:, :N].double().cpu().numpy()
    err = np.abs(got - ref).max() / (np.abs(ref).max() + 1e-30)
    assert err < 1e-5, err


@pytest.mark.parametrize("bn", [128, 256])
def test_gemm_bf16_out_bias_and_accumulate(bn):
    M, N, K = 384, 520, 200
    A = torch.from_numpy(synth.normal((M, K), 3)).bfloat16()
    B = torch.from_numpy(synth.normal((N, K), 4)).bfloat16()
    bias = torch.from_numpy(synth.normal(N, 5))
    ref = A.double().numpy() @ B.double().numpy().T + bias.double().numpy()[None]
    dev = torch.device("cuda:0")
    out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    _ops().gemm(A.to(dev), B.to(dev), out, bias=bias.to(dev), bn=bn)
    torch.cuda.synchronize()
    got = out.double().cpu().numpy()
    assert np.abs(got - ref).max() / np.abs(ref).max() < 8e-3
    acc = torch.from_numpy(synth.normal((M, N), 6)).to(dev)
    base = acc.double().cpu().numpy()
    _ops().gemm(A.to(dev), B.to(dev), acc, accumulate=True, bn=bn)
    torch.cuda.synchronize()
    ref2 = base + A.double().numpy() @ B.double().numpy().T
    assert np.abs(acc.double().cpu().numpy() - ref2).max() / np.abs(ref2).max() < 1e-5


@pytest.mark.parametrize("a_mn", [0, 1])
@pytest.mark.parametrize("b_mn", [0, 1])
def test_gemm_long_k_accumulate_sampled_rows(a_mn, b_mn):
    """K >= 8192 with accumulation takes the deep-ring variant (the weight-gradient shape);
    checked on every 41st row against fp64."""
    M, N, K = 2560, 2048, 8192
    A = torch.from_numpy(synth.normal((M, K), 7)).bfloat16()
    B = torch.from_numpy(synth.normal((N, K), 8)).bfloat16()
    dev = torch.device("cuda:0")
    a_d = (A.T.contiguous() if a_mn else A).to(dev)
    b_d = (B.T.contiguous() if b_mn else B).to(dev)
    base = torch.from_numpy(synth.normal((M, N), 9))
    out = base.to(dev)
    _ops().gemm(a_d, b_d, out, a_mn=bool(a_mn), b_mn=bool(b_mn), accumulate=True, bn=256, M=M, N=N, K=K)
    torch.cuda.synchronize()
    rows = np.arange(0, M, 41)
    ref = base.double().numpy()[rows] + A.double().numpy()[rows] @ B.double().numpy().T
    got = out.double().cpu().numpy()[rows]
    # fp32 accumulation over K terms: rounding error grows like sqrt(K) * 2^-24; 16x margin
    # for partial sums larger than the final value (8.6e-5 relative at K = 8192)
    tol = 16 * 2.0 ** -24 * math.sqrt(K)
    assert np.abs(got - ref).max() / np.abs(ref).max() < tol
