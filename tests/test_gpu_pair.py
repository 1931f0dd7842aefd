"""The CTA-pair GEMM (two SMs per 256-row tile, tcgen05.mma.cta_group::2) on every shape.

By default the library picks CTA pairs only for products with enough 256 x 256 tiles, so the
small and ragged cases of the GEMM and model parity suites run on the single-CTA kernel.  Here
those suites run again in a child process with GPT_GEMM_PAIR=1, which sends every N-256 GEMM
(forward, data and weight gradients, the fused epilogues, the lm_head cross-entropy) through the
pair kernel, against the same fp64 references and the oracle."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("suite, select", [
    ("tests/test_gpu_gemm.py", "not long_k"),
    ("tests/test_gpu_model.py", "forward_backward or deterministic"),
])
def test_suite_with_cta_pairs_forced(suite, select):
    env = dict(os.environ, GPT_GEMM_PAIR="1")
    r = subprocess.run([sys.executable, "-m", "pytest", suite, "-m", "gpu", "-q", "-x", "-k", select,
                        "-p", "no:cacheprovider"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
