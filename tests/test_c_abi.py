"""The C ABI from plain C: include/gpt.h and include/gpt_ops.h compile as C99 with -Wall -Wextra
-Werror, and a C program links the in-tree shared library and gets the documented answers from its
host-side calls (tests/c/abi_host.c).  No GPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "decoder_only_gpt_tcgen05_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs a C compiler")
def test_headers_compile_as_c99_and_host_calls_answer(tmp_path):
    import decoder_only_gpt_tcgen05_b200 as g
    g.lib()                                   # the library exists (built in-tree)
    exe = str(tmp_path / "abi_host")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_host.c"), "-o", exe, "-L", PKG, "-lgpt_b200",
           "-Wl,-rpath," + PKG, "-lm"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip().endswith("OK"), r.stdout + r.stderr
