"""Oracle for the FP8 matrix products of the linear layers: plain fp64 numpy.

TEST INFRASTRUCTURE ONLY, like the model oracle: imported by the test suite alone.  It shares no
code with the CUDA library.

Source: "Train your own ChatGPT", read the source fp8.py: every tensor is rescaled dynamically
before it is cast, scale = FP8_MAX / max(|tensor|); the product runs on the 8-bit values and the
inverse scales are folded back into it; activations and weights use e4m3 (more precision bits),
gradients e5m2 (more range bits).

Readings where the page is silent (the OCP 8-bit floating-point formats the page names):
  - e4m3: sign, 4 exponent bits (bias 7), 3 mantissa bits, largest finite value 448, subnormals
    down to 2^-9, no infinity; e5m2: sign, 5 exponent bits (bias 15), 2 mantissa bits, largest
    finite 57344, subnormals down to 2^-16;
  - the cast rounds to nearest (ties to even) and saturates at the largest finite value;
  - the scale is a per-tensor fp32 number FP8_MAX / amax (1 when amax is 0), and the product is
    out = (Q(a s_a) Q(b s_b)^T) / (s_a s_b).
"""
from __future__ import annotations

import numpy as np

FORMATS = {
    # name: (exponent bits, mantissa bits, bias, largest finite value)
    "e4m3": (4, 3, 7, 448.0),
    "e5m2": (5, 2, 15, 57344.0),
}


def quantize(x, fmt: str) -> np.ndarray:
    """Round every element of x to the nearest value of the format (ties to even), saturating at
    the largest finite value.  Returns the rounded values as float64."""
    _, man, bias, fmax = FORMATS[fmt]
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), fmax)
    # the spacing of representable values around a: 2^(e - man) with e = floor(log2 a), and the
    # subnormal spacing 2^(1 - bias - man) below the smallest normal 2^(1 - bias)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, 1 - bias)
    step = np.exp2(e - man)
    q = np.round(a / step) * step            # np.round rounds half to even
    q = np.minimum(q, fmax)
    return np.sign(x) * q


def scale_of(x, fmt: str) -> float:
    """FP8_MAX / max(|x|), or 1 for an all-zero tensor."""
    amax = float(np.max(np.abs(np.asarray(x, dtype=np.float64)))) if np.size(x) else 0.0
    return FORMATS[fmt][3] / amax if amax > 0 else 1.0


def scaled_matmul(a, b, fmt_a: str = "e4m3", fmt_b: str = "e4m3", s_a: float | None = None,
                  s_b: float | None = None) -> np.ndarray:
    """out[M, N] = Q(a s_a) Q(b s_b)^T / (s_a s_b) for a [M, K], b [N, K] (the per-tensor scales
    from scale_of unless given)."""
    s_a = scale_of(a, fmt_a) if s_a is None else s_a
    s_b = scale_of(b, fmt_b) if s_b is None else s_b
    qa = quantize(np.asarray(a, dtype=np.float64) * s_a, fmt_a)
    qb = quantize(np.asarray(b, dtype=np.float64) * s_b, fmt_b)
    return (qa @ qb.T) / (s_a * s_b)


def quantize_tensor_fp32(x, fmt: str):
    """The cast of a whole tensor as a kernel performs it in fp32 arithmetic: amax = max |x|,
    s = fp32(FP8_MAX) / amax (one correctly rounded fp32 division; 1 when amax == 0), each product
    x s rounded to fp32, then to the format.  Returns (8-bit values as float64, amax, s, 1 / s), the
    last three as fp32 numbers.  (Where fp32 decides an 8-bit code, the oracle takes the decision in
    the kernel's precision.)"""
    x32 = np.asarray(x, dtype=np.float32)
    amax = np.float32(np.max(np.abs(x32))) if x32.size else np.float32(0)
    s = np.float32(FORMATS[fmt][3]) / amax if amax > 0 else np.float32(1)
    q = quantize((x32 * s).astype(np.float32), fmt)
    return q, amax, s, np.float32(1) / s
