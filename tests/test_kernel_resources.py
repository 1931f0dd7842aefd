"""Register and spill budgets of every kernel, from ptxas's resource report (no GPU).

Each csrc/*.cu is compiled for sm_100a with the library's own flags plus -Xptxas -v, and every
kernel entry is checked:
  - its registers fit the largest block it is launched with (threads x registers <= 64K, and for
    the warp-specialised kernels the per-scheduler share: a block's warps are spread over the SM's
    four schedulers, each with 16K registers);
  - it does not spill, except the few entries listed in SPILL_ALLOWANCE with their reason.
A change that pushes a hot kernel into local memory, or past its launch size, fails here before
it reaches a GPU."""
import glob
import math
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "decoder_only_gpt_tcgen05_b200", "csrc")

# threads per block of each kernel's largest launch (the __launch_bounds__ where it has one)
BLOCK_THREADS = [
    (r"gemm_kernel", 320),               # TMA warp, MMA warp, 8 epilogue warps (long-K: 4)
    (r"attn_fwd_kernel", 384),           # TMA, MMA and two idle warps; two softmax warpgroups
    (r"attn_bwd_(dkv|dq)_kernel", 576),  # TMA warp, MMA warp, 16 elementwise warps
    (r"offsets_(global_)?kernel", 1024),
    (r"rms_bwd_kernel", 128),
    (r".*", 256),                        # every other kernel: blocks of at most 256 threads
]

# (entry pattern, spill-store bytes allowed, reason)
SPILL_ALLOWANCE = [
    (r"attn_bwd_dq_kernel", 16, "96-register cap of 18 warps on four schedulers"),
    (r"gemm_kernelILi(128|256)ELi5E", 64, "activation-gradient epilogue at the 168-register cap of 10 warps"),
    (r"norm_bwd_kernelILi(16|24|32)E", 4096, "LayerNorm rows wider than 1664 (no preset uses them)"),
    (r"rms_bwd_kernelILi16E", 1024, "RMSNorm rows wider than 3072 (no preset uses them)"),
]


def _entries(src):
    from decoder_only_gpt_tcgen05_b200 import build as B
    cmd = [B.nvcc(), *B.ARCH, *B.NVCC_FLAGS, "-Xptxas", "-v", "-c", src, "-o", os.devnull]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-3000:]
    out, cur = [], None
    for line in r.stderr.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            cur = {"name": m.group(1), "regs": None, "spill": 0}
            out.append(cur)
            continue
        if cur is None:
            continue
        m = re.search(r"(\d+) bytes spill stores", line)
        if m:
            cur["spill"] = int(m.group(1))
        m = re.search(r"Used (\d+) registers", line)
        if m:
            cur["regs"] = int(m.group(1))
    return out


def _threads(name):
    for pat, t in BLOCK_THREADS:
        if re.search(pat, name):
            return t


def _allowed_spill(name):
    for pat, b, _ in SPILL_ALLOWANCE:
        if re.search(pat, name):
            return b
    return 0


@pytest.mark.skipif(shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"),
                    reason="needs nvcc")
@pytest.mark.parametrize("src", sorted(os.path.basename(p) for p in glob.glob(os.path.join(CSRC, "*.cu"))))
def test_kernels_fit_their_launch_and_do_not_spill(src):
    for e in _entries(os.path.join(CSRC, src)):
        name, regs, spill = e["name"], e["regs"], e["spill"]
        assert regs is not None, name
        t = _threads(name)
        assert t * regs <= 65536, (name, regs, t)
        # warps of a block spread over the four schedulers; each holds 16K registers
        # (allocated per warp in units of 8 registers per thread)
        warps_per_scheduler = math.ceil(t / 32 / 4)
        assert warps_per_scheduler * 32 * (math.ceil(regs / 8) * 8) <= 16384, (name, regs, t)
        assert spill <= _allowed_spill(name), (name, spill)
