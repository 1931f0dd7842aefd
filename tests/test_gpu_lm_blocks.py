"""The lm_head backward in row blocks.

The backward forms the cross-entropy gradient of at most 512 MiB of bf16 dlogits at a time, so the
small parity cases fit in one block and never reach the blocked loop that the measured workloads use.
Here the model parity suite runs again in a child process with GPT_LM_CHUNK_ROWS set: 128-row
blocks (several per batch) and a size that leaves a ragged last block."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("rows", ["128", "200"])
def test_model_parity_with_lm_head_row_blocks(rows):
    env = dict(os.environ, GPT_LM_CHUNK_ROWS=rows)
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_gpu_model.py", "-m", "gpu", "-q", "-x", "-k",
                        "forward_backward and (d20 or gpt2)", "-p", "no:cacheprovider"], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
