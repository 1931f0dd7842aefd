"""Host-side checks of the C ABI: no GPU needed, no compute launched.

The library must load, export every symbol the headers declare, lay out the
parameters exactly as the oracle does, and reject bad arguments on the host
with the documented status codes."""
import ctypes as C
import dataclasses
import glob
import os
import re

import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def pkg():
    import decoder_only_gpt_tcgen05_b200 as g
    g.lib()
    return g


def _declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        names |= set(re.findall(r"GPT_API\s+[\w\s\*]+?\b(gpt_\w+)\s*\(", open(h).read()))
    return sorted(names)


def test_library_exports_every_declared_symbol(pkg):
    syms = _declared_symbols()
    assert len(syms) >= 14
    L = pkg.lib()
    for s in syms:
        assert hasattr(L, s), s


CONFIGS = ["tiny", "gpt2", "d20", "d26"]


@pytest.mark.parametrize("name", CONFIGS)
def test_presets_match_oracle(pkg, name):
    assert dataclasses.asdict(pkg.PRESETS[name]) == dataclasses.asdict(O.PRESETS[name])


@pytest.mark.parametrize("name,over", [(n, {}) for n in CONFIGS] + [
    ("tiny", {"tie_embed": 0}), ("gpt2", {"n_layer": 2, "linear_bias": 0}), ("gpt2", {"norm": 0})])
def test_param_layout_matches_oracle(pkg, name, over):
    cfg = pkg.preset(name, **over)
    ocfg = O.Config(**dataclasses.asdict(cfg))
    assert pkg.model.param_count(cfg) == O.param_count(ocfg)
    lay = pkg.model.param_tensors(cfg)
    ref = O.param_offsets(ocfg)
    assert [t[0] for t in lay] == list(ref)
    for nm, off, rows, cols in lay:
        o, shape = ref[nm]
        assert off == o and off % 16 == 0
        assert (rows, cols) == (shape if len(shape) == 2 else (shape[0], 1))


def test_workspace_size_grows_with_batch(pkg):
    cfg = pkg.preset("d20")
    a = pkg.model.workspace_size(cfg, 1, 2048)
    b = pkg.model.workspace_size(cfg, 16, 2048)
    assert 0 < a < b < 80 * 2 ** 30


def _status(pkg, fn, *args):
    return getattr(pkg.lib(), fn)(*args)


def test_bad_arguments_are_rejected_on_the_host(pkg):
    L = pkg.lib()
    n = C.c_int64()
    assert L.gpt_param_count(None, C.byref(n)) == 1
    bad = pkg.preset("tiny", n_embd=24, n_head=4).c()
    assert L.gpt_param_count(C.byref(bad), C.byref(n)) == 2
    bad = pkg.preset("d20", n_head=20).c()   # head dim 64 is fine ...
    assert L.gpt_param_count(C.byref(bad), C.byref(n)) == 0
    bad = pkg.preset("d20", n_head=40).c()   # ... head dim 32 with RoPE is not
    assert L.gpt_param_count(C.byref(bad), C.byref(n)) == 2
    assert b"RoPE" in L.gpt_last_error()
    cfg = pkg.preset("gpt2").c()
    sz = C.c_size_t()
    assert L.gpt_workspace_size(C.byref(cfg), 1, 1025, C.byref(sz)) == 1   # T > block_size
    assert L.gpt_workspace_size(C.byref(cfg), 0, 16, C.byref(sz)) == 1
    assert L.gpt_workspace_size(C.byref(cfg), 2, 1024, C.byref(sz)) == 0
    # null pointers and a too-small workspace: caught before any launch
    fake = C.c_void_p(1 << 20)
    assert L.gpt_forward_loss(C.byref(cfg), None, fake, fake, 2, 1024, fake, sz.value, fake, None) == 1
    assert L.gpt_forward_loss(C.byref(cfg), fake, fake, fake, 2, 1024, fake, sz.value - 1, fake, None) == 3
    assert b"workspace" in L.gpt_last_error()
    mis = C.c_void_p((1 << 20) + 16)
    assert L.gpt_forward_loss(C.byref(cfg), fake, fake, fake, 2, 1024, mis, sz.value, fake, None) == 1
    assert L.gpt_backward(C.byref(cfg), fake, 2, 1024, fake, sz.value, None, 0, None) == 1
    assert L.gpt_eval_bpb(C.byref(cfg), fake, fake, fake, None, 2, 1024, fake, sz.value, None, None, None,
                          None) == 1
    assert L.gpt_set_wait_timeout_ns(0) == 1
    assert L.gpt_op_gemm(0, 192, fake, 64, 0, fake, 64, 0, 8, 8, 8, fake, 8, None, 0, None) == 1
    assert L.gpt_op_attention_fwd(fake, 1, 16, 1, 32, 1, 1, -1, C.c_float(1e4), C.c_float(1e-5), fake, fake, fake,
                                  fake, fake, fake, None) == 2
    assert L.gpt_op_attention_fwd(fake, 1, 16, 1, 64, 1, 1, -2, C.c_float(1e4), C.c_float(1e-5), fake, fake, fake,
                                  fake, fake, fake, None) == 1


@pytest.mark.parametrize("name", CONFIGS)
def test_bench_flop_accounting_matches_oracle(pkg, name):
    """bench.py's MFU numerator is its own formula; it must agree with the oracle's pinned count."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    cfg, ocfg = pkg.preset(name), O.preset(name)
    for B, T in ((16, 2048), (8, 1024), (1, 16)):
        assert bench.step_flops(cfg, B, T) == O.step_flops(ocfg, B, T)
        assert bench.step_flops(cfg, B, T, causal=False) == O.step_flops(ocfg, B, T, causal=False)
    # attention alone: forward 2 B H T^2 hd, i.e. T x 83.9 MFLOP at 32768 tokens, 10 heads of 128
    for T in (512, 2048, 8192):
        f, b = bench.attention_flops(32768 // T, T, 10, 128)
        assert f == T * 83_886_080 and b == 2 * f


def test_lr_schedule_matches_oracle(pkg):
    for warm, decay in ((2000, 600_000), (0, 100), (10, 10), (1, 7)):
        for it in sorted({0, 1, warm // 2, warm, warm + 1, (warm + decay) // 2, decay - 1, decay, decay + 5}):
            if it < 0:
                continue
            got = pkg.lr_schedule(it, warm, decay, 6e-4, 6e-5)
            assert got == pytest.approx(O.optim.lr_schedule(it, warm, decay, 6e-4, 6e-5), rel=1e-14, abs=0), (it, warm)


def test_adamw_rejects_bad_arguments_on_the_host(pkg):
    """Every case below is refused before anything is launched (the pointers are never touched)."""
    from decoder_only_gpt_tcgen05_b200._lib import AdamWParams, lib
    L = lib()
    P = 1 << 20                                   # a 16-byte aligned address that is never dereferenced
    ok = dict(lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, grad_scale=1.0, grad_clip=1.0)

    def op(params=P, grads=P + 4096, m=P + 8192, v=P + 12288, n=1000, starts=(0, 10), decay=(1, 0), step=1,
           scratch=P + 16384, **over):
        h = AdamWParams(**{**ok, **over})
        rs = (C.c_int64 * max(1, len(starts)))(*starts)
        rd = (C.c_uint8 * max(1, len(decay)))(*decay)
        return L.gpt_op_adamw(params, grads, m, v, n, rs, rd, len(starts), step, C.byref(h), scratch, None, None)

    assert op(params=None) == 1
    assert op(grads=P + 4) == 1                   # misaligned
    assert op(scratch=None) == 1
    assert op(n=-1) == 1
    assert op(step=0) == 1
    assert op(beta1=1.0) == 1 and op(beta2=-0.1) == 1
    assert op(eps=0.0) == 1 and op(lr=float("nan")) == 1 and op(lr=-1.0) == 1
    assert op(grad_scale=0.0) == 1 and op(grad_clip=-1.0) == 1
    assert op(lr=2.0, weight_decay=1.0) == 1      # lr * weight_decay > 1
    assert op(starts=(1, 10)) == 1                # the first run must start at 0
    assert op(starts=(0, 10, 10), decay=(1, 0, 1)) == 1
    assert op(starts=(0, 1000), decay=(1, 0)) == 1
    assert op(starts=(), decay=()) == 1
    assert "adamw" in L.gpt_last_error().decode()
    c = pkg.preset("tiny").c()
    h = AdamWParams(**ok)
    assert L.gpt_adamw_step(None, P, P + 4096, P + 8192, P + 12288, 1, C.byref(h), P + 16384, None, None) == 1
    assert L.gpt_adamw_step(C.byref(c), P, P + 4096, P + 8192, P + 12288, 1, None, P + 16384, None, None) == 1
    assert L.gpt_adamw_step(C.byref(c), P, P + 4096, P + 8192, P + 12288, 0, C.byref(h), P + 16384, None, None) == 1
    assert L.gpt_adamw_step(C.byref(c), P + 8, P + 4096, P + 8192, P + 12288, 1, C.byref(h), P + 16384, None,
                            None) == 1
    n = C.c_size_t()
    assert L.gpt_adamw_scratch_size(C.byref(n)) == 0 and n.value >= 8 and n.value % 8 == 0


def test_bench_clock_sample_parsing():
    """bench.py's clocks record: median SM clock, max clock, and only the reasons reported Active."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    lines = [
        "0, 1965, 1965, 300.12, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n",
        "0, 1500, 1965, 998.50, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n",
        "0, 1600, 1965, 990.00, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n",
        "garbage line\n",
        "0, [N/A], 1965, 990.00, 0x0, Not Active, Not Active, Not Active, Active\n",
    ]
    out = bench.parse_clock_samples(lines)
    assert out == {"sm_mhz": 1600.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    hot = bench.parse_clock_samples(["0, 1200, 1965, 700, 0x48, Not Active, Active, Active, Not Active\n"])
    assert hot["reasons"] == ["hw_thermal_slowdown", "sw_thermal_slowdown"]
    assert bench.parse_clock_samples([])["reasons"] == ["no samples"]


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """No fallback: with the shared library absent, every call raises instead of computing."""
    import decoder_only_gpt_tcgen05_b200 as g
    from decoder_only_gpt_tcgen05_b200 import _lib
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "libgpt_b200.so"))
    with pytest.raises(ImportError, match="missing"):
        _lib.lib()
    with pytest.raises(ImportError):
        g.lr_schedule(10, 100, 1000, 1e-3, 1e-4)
    n = C.c_int64()
    with pytest.raises(ImportError):
        _lib.call("gpt_param_count", C.byref(g.preset("tiny").c()), C.byref(n))


def _header_declarations():
    """{name: number of parameters} of every GPT_API function in include/*.h."""
    out = {}
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = re.sub(r"/\*.*?\*/", " ", open(h).read(), flags=re.S)
        for m in re.finditer(r"GPT_API\s+[\w\s\*]+?\b(gpt_\w+)\s*\(([^)]*)\)\s*;", text):
            params = m.group(2).strip()
            out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_signatures_match_the_headers():
    """Every ctypes signature in the binding has the header's parameter count; every declared
    function is either in SIGNATURES or given its own restype/argtypes by the loader."""
    from decoder_only_gpt_tcgen05_b200 import _lib
    decl = _header_declarations()
    assert len(decl) >= 25
    for name, args in _lib.SIGNATURES.items():
        assert name in decl, name
        assert len(args) == decl[name], (name, len(args), decl[name])
    special = {"gpt_last_error", "gpt_launch_count", "gpt_op_lmhead_ce_scratch_bytes",
               "gpt_op_lmhead_ce_noalloc_max_scratch_bytes", "gpt_op_adamw_scratch_bytes"}
    assert set(decl) <= set(_lib.SIGNATURES) | special, set(decl) - set(_lib.SIGNATURES) - special
    loader = open(os.path.join(ROOT, "decoder_only_gpt_tcgen05_b200", "_lib.py")).read()
    for name in special:
        assert f"L.{name}.restype" in loader and f"L.{name}.argtypes" in loader, name


def test_d20_workspace_is_the_documented_size(pkg):
    sz = C.c_size_t()
    assert pkg.lib().gpt_workspace_size(C.byref(pkg.preset("d20").c()), 16, 2048, C.byref(sz)) == 0
    assert sz.value / 2**30 == pytest.approx(25.9, abs=0.05)


def test_profile_families_match_the_library(pkg):
    """bench.py reads per-kernel-family times by position: the Python list of families must have
    exactly the library's number of profiling kinds (gpt_profile_stop returns that number)."""
    assert pkg.lib().gpt_profile_stop(0, None, None, None, None) == len(pkg.ops.PROFILE_FAMILIES)
    assert pkg.ops.PROFILE_FAMILIES[0] == "gemm" and pkg.ops.PROFILE_FAMILIES[-2:] == ["optim", "gemm_muon"]
