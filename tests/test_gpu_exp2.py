"""The two exponentials of the attention forward's softmax (gpt_op_exp2) against their error bounds.

The kernel sends 3 of every 8 groups of exponentials to a polynomial on the FMA pipe (range
reduction x = n + f with n = rint(x), a degree-4 minimax polynomial for 2^f on [-1/2, 1/2], n added
to the exponent field) and the rest to the MUFU unit's ex2.approx.  Bounds: relative error below
3e-6 for the polynomial (the fit's 2.6e-6 plus the fp32 Horner steps) and below 5e-7 for
ex2.approx, against 2^x in float64, for -125 <= x <= 127; below -125 (and at -inf) both give a
value in [0, 2^-125]."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def _exp2(x, poly):
    import decoder_only_gpt_tcgen05_b200 as g
    xd = torch.from_numpy(x).to(DEV)
    out = torch.empty_like(xd)
    g._lib.call("gpt_op_exp2", xd.data_ptr(), xd.numel(), int(poly), out.data_ptr(),
                torch.cuda.current_stream(DEV).cuda_stream)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("poly,bound", [(1, 3e-6), (0, 5e-7)])
def test_exp2_within_its_error_bound(poly, bound):
    rng = np.random.default_rng(5)
    x = np.concatenate([
        np.linspace(-125.0, 127.0, 1 << 20),
        rng.uniform(-20.0, 8.0, 1 << 20),               # the softmax's range: s * scale - m <= 8
        np.arange(-125, 128, dtype=np.float64),          # integers (f = 0)
        np.arange(-125, 127, dtype=np.float64) + 0.5,    # ties of the rounding to n
        [0.0, -0.0, 0.25, -0.25, 1e-7, -1e-7],
    ]).astype(np.float32)
    x = x[: x.size - (x.size & 1)]
    got = _exp2(x, poly)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() <= bound, (rel.max(), x[np.argmax(rel)])


@pytest.mark.parametrize("poly", [0, 1])
def test_exp2_below_the_range_is_tiny(poly):
    x = np.array([-125.5, -126.0, -126.7, -150.0, -1e30, -np.inf, -200.0, -125.0000001], dtype=np.float32)
    got = _exp2(x, poly)
    assert np.all(got >= 0.0) and np.all(got <= 2.0 ** -125), got
