#!/usr/bin/env python
"""Benchmark of the B200 GPT hot path: nanochat d20 forward + backward
(tokens/s and MFU against the bf16 peak) and val_bpb evaluation (tokens/s).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...      (one rank per GPU)

A step is one gpt_forward_loss + gpt_backward over one batch of B=16
sequences of T=2048 tokens per GPU (synthetic Zipf(1.1) tokens, random-init
d20 weights), plus an optimizer step with --optimizer.  With N > 1 every rank
processes its own batch (weak scaling) and the gradients are averaged over
ranks inside the step, bucket by bucket on a communication stream while the
backward goes on (--grad-sync overlap, the default; --grad-sync blocking: one
all-reduce after the backward; --optimizer zero2: reduce-scatter, sharded
AdamW, all-gather of the weights).  Rank 0 prints one JSON line.

--impl reference times the oracle (plain fp64 CPU model) on a bounded sample
of the same workload on the host cores: the deliberately slow baseline.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "d20 fwd+bwd tokens/s and MFU vs bf16 peak, 1×B200; val_bpb eval tokens/s"
DATASHEET_BF16_TFLOPS = 2250.0   # B200 dense bf16 (NVIDIA datasheet; context for MFU)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

WORKLOADS = {
    # name: (preset, B, T, description)
    "d20": ("d20", 16, 2048, "nanochat d20 fwd+bwd + val_bpb eval, B=16 x T=2048 (32768 tokens per GPU)"),
    "gpt2": ("gpt2", 8, 1024, "GPT-2 124M shape fwd+bwd + val_bpb eval, B=8 x T=1024 (8192 tokens per GPU)"),
    "d26": ("d26", 16, 2048, "nanochat d26 fwd+bwd + val_bpb eval, B=16 x T=2048 (32768 tokens per GPU)"),
}


def metric_name(preset_name: str) -> str:
    return METRIC if preset_name == "d20" else METRIC.replace("d20", preset_name)


def matmul_params(cfg) -> int:
    """Parameters that take part in a matmul for every token: the block matrices (q, k, v, output
    projection, MLP up and down with width 4D) and the lm_head; embedding lookups are gathers."""
    D = cfg.n_embd
    return cfg.n_layer * (4 * D * D + 2 * D * 4 * D) + cfg.vocab_size * D


def step_flops(cfg, B: int, T: int, causal: bool = True) -> float:
    """Forward + backward FLOPs of one step: 6 per matmul parameter per token plus attention
    ("Train your own ChatGPT", gpt.py estimate_flops: 6 FLOPs per parameter per token plus
    attention terms).  causal=True counts only the unmasked half of the score matrix
    (6 L D T per token), causal=False the full 12 L D T."""
    att = (6 if causal else 12) * cfg.n_layer * cfg.n_embd * T
    return float(B * T) * (6.0 * matmul_params(cfg) + att)


def attention_flops(B: int, T: int, H: int, hd: int):
    """Algorithmic FLOPs of causal attention: the forward's two products (q k^T and P v) over the
    unmasked half of the T x T scores, 2 B H T^2 hd; the backward's four (dP, dV, dQ, dK) twice that."""
    fwd = 2.0 * B * H * T * T * hd
    return fwd, 2.0 * fwd


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        with open(self.path) as f:
            out = parse_clock_samples(f)
        os.unlink(self.path)
        return out


def parse_clock_samples(lines):
    """Median SM clock, maximum SM clock and the throttle reasons seen in `nvidia-smi
    --query-gpu=<ClockSampler.FIELDS> --format=csv,noheader,nounits` lines."""
    rows = []
    for line in lines:
        parts = [x.strip() for x in line.split(",")]
        if len(parts) < 9:
            continue
        try:
            rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
        except ValueError:
            continue
    if not rows:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower() == "active"})
    return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
            "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------- oracle (CPU) timing

def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count()


_ORACLE_PARAMS = {}


def oracle_step_seconds(preset_name: str, T: int, seed: int = 1) -> float:
    """One oracle forward+backward of the workload's model on one sequence of T tokens."""
    import oracle as O
    import synth
    cfg = O.preset(preset_name)
    if preset_name not in _ORACLE_PARAMS:
        # N(0, 0.02^2) weights (drawing them is not part of the timed step)
        _ORACLE_PARAMS[preset_name] = synth.normal(O.param_count(cfg), 0, std=0.02).astype("float64")
    p = _ORACLE_PARAMS[preset_name]
    idx, tgt = synth.next_token_batch(1, T, cfg.vocab_size, seed=seed)
    t0 = time.perf_counter()
    O.loss_and_grad(cfg, p, idx, tgt)
    return time.perf_counter() - t0


def cpu_baseline(preset_name: str, budget_s: float = 30.0):
    """Oracle fwd+bwd tokens/s on a bounded sample: one sequence whose length
    is grown (powers of two from 128, at most the workload's T) while the next
    length's step is expected within `budget_s` seconds (d20: T = 2048 on a
    16-core host)."""
    _, _, T_full, _ = WORKLOADS[preset_name]
    T = 128
    t = oracle_step_seconds(preset_name, T)
    while T * 2 <= T_full and t * 2.2 < budget_s:
        T *= 2
        t = oracle_step_seconds(preset_name, T)
    return {"value": T / t, "unit": "tokens/s", "cores": oracle_threads(), "kind": "oracle",
            "sample": f"{preset_name} fwd+bwd of 1 sequence x {T} tokens (fp64 numpy oracle), {t:.1f} s"}


# ---------------------------------------------------------------- reference arm

def run_reference(args, rank, world):
    if rank != 0:
        return
    preset_name = args.workload
    # size each step so that warm-up + timed steps fit in about two minutes
    probe = oracle_step_seconds(preset_name, 64)
    per_step = 110.0 / max(1, args.steps + args.warmup)
    T = 64
    _, _, T_full, desc = WORKLOADS[preset_name]
    while T * 2 <= T_full and probe * (T * 2 / 64) * 1.3 < per_step:
        T *= 2
    for _ in range(args.warmup):
        oracle_step_seconds(preset_name, T)
    times = [oracle_step_seconds(preset_name, T, seed=1 + k) for k in range(args.steps)]
    ms = 1000.0 * sum(times) / len(times)
    value = T / (ms / 1000.0)
    line = {
        "impl": "reference", "metric": metric_name(preset_name), "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": desc, "sample": f"1 sequence x {T} tokens per step", "parallelism": "cpu"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle_threads(), "kind": "oracle",
                         "sample": f"{preset_name} fwd+bwd of 1 sequence x {T} tokens per step (fp64 numpy)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- our arm

# ---------------------------------------------------------------- attention alone

ATTN_SWEEP_T = (512, 1024, 2048, 4096, 8192)


def run_attn_sweep(args):
    """RoPE + QK-norm + causal attention forward and backward through the op-level calls,
    H = 10 heads of 128 (the d20 layer), B = 32768 / T sequences for each T of the sweep.
    Inputs: raw q|k|v N(0, 1) (seed 3) and dL/do N(0, 1) (seed 4), bf16; the same 32768-token
    arrays serve every T.  Each call is timed with CUDA events over `steps` back-to-back calls;
    a second pass under the library's per-launch profiler splits out the attention kernels."""
    import torch
    import decoder_only_gpt_tcgen05_b200 as g
    import synth

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])   # kernels timed alone: burst peak
    H, hd, tokens = 10, 128, 32768
    qkv = torch.from_numpy(synth.normal((tokens, 3 * H * hd), 3)).to(dev).to(torch.bfloat16)
    dout = torch.from_numpy(synth.normal((tokens, H * hd), 4)).to(dev).to(torch.bfloat16)
    dqkv = torch.empty_like(qkv)
    stream = torch.cuda.current_stream(dev)

    def timed(fn, k):
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(k):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / k

    rows = []
    n0 = g.ops.launch_count()
    n_calls = 0
    with ClockSampler(0) as clk:
        for T in ATTN_SWEEP_T:
            B = tokens // T
            fwd = g.ops.attention_fwd(qkv, B, T, H, hd)
            delta = torch.empty((B, H, T), dtype=torch.float32, device=dev)

            def f():
                g.ops.attention_fwd(qkv, B, T, H, hd, out=fwd)

            def bwd():
                g.ops.attention_bwd(fwd, dout, B, T, H, hd, delta=delta, dqkv=dqkv)
            for _ in range(args.warmup):
                f()
                bwd()
            ms_f = timed(f, args.steps)
            ms_b = timed(bwd, args.steps)
            n_calls += 2 * (args.warmup + args.steps)
            g.ops.profile_start()
            for _ in range(args.steps):
                f()
                bwd()
            torch.cuda.synchronize(dev)
            prof = g.ops.profile_stop()
            n_calls += 2 * args.steps
            fl_f, fl_b = attention_flops(B, T, H, hd)
            k_f = prof["attn_fwd"][0] / args.steps
            k_b = (prof["attn_bwd_dkv"][0] + prof["attn_bwd_dq"][0]) / args.steps
            rows.append({
                "T": T, "B": B, "fwd_ms": ms_f, "bwd_ms": ms_b,
                "fwd_tflops": fl_f / ms_f / 1e9, "bwd_tflops": fl_b / ms_b / 1e9,
                "fwd_bwd_tflops": (fl_f + fl_b) / (ms_f + ms_b) / 1e9,
                "kernel_ms": {k: prof[k][0] / args.steps for k in ("attn_fwd", "attn_bwd_dkv", "attn_bwd_dq", "qk",
                                                                    "delta", "misc")},
                "kernel_fwd_tflops": fl_f / k_f / 1e9 if k_f > 0 else None,
                "kernel_bwd_tflops": fl_b / k_b / 1e9 if k_b > 0 else None,
            })
            g.model.sync_status(dev)
    launches = (g.ops.launch_count() - n0) / max(1, n_calls // 2)   # per forward + backward pair
    head = next(r for r in rows if r["T"] == 2048)
    kms = head["kernel_ms"]["attn_fwd"] + head["kernel_ms"]["attn_bwd_dkv"] + head["kernel_ms"]["attn_bwd_dq"]
    ach = sum(attention_flops(head["B"], 2048, H, hd)) / kms / 1e9 if kms > 0 else None
    line = {
        "metric": "causal attention fwd+bwd TFLOP/s (algorithmic), RoPE + QK-norm, 10 heads x 128, 32768 tokens, T=2048",
        "value": head["fwd_bwd_tflops"], "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": head["fwd_ms"] + head["bwd_ms"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "attention sweep: H=10, hd=128, B*T=32768, T in " + ",".join(map(str, ATTN_SWEEP_T)),
                   "l2": "q|k|v, o and dq|dk|dv 250 MB each, above the 126 MB L2; no flush"},
        "roofline": {"kernel": "attn_fwd + attn_bwd_dkv + attn_bwd_dq at T=2048", "bound": "tensor", "achieved": ach,
                     "peak": peak, "unit": "TFLOP/s", "frac": ach / peak if ach else None, "traffic": None,
                     "peak_source": f"{peak_src} bf16 burst"},
        "sweep": rows,
        "gpu_launches": launches,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


def run_lmhead(args):
    """The fused lm_head + cross-entropy forward alone at the d26 shape: 32768 tokens x width
    1664 x vocabulary 32768 (gpt_op_lmhead_ce_fwd: per-row loss and logsumexp, logits never
    stored).  Inputs: x N(0, 1) (seed 5) and W N(0, 0.02^2) (seed 6) in bf16, Zipf(1.1) targets
    (seed 1).  Timed with CUDA events over `steps` back-to-back calls; x and W (232 MB) are above
    the 126 MB L2."""
    import torch
    import decoder_only_gpt_tcgen05_b200 as g
    import synth

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])   # one kernel timed alone: burst peak
    M, D, V = 32768, 1664, 32768
    x = torch.from_numpy(synth.normal((M, D), 5)).to(dev).to(torch.bfloat16)
    w = torch.from_numpy(synth.normal((V, D), 6, std=0.02)).to(dev).to(torch.bfloat16)
    _, tgt = synth.next_token_batch(16, 2048, V, seed=1)
    tgt = torch.from_numpy(tgt.reshape(-1)).to(dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        g.ops.lmhead_ce_fwd(x, w, tgt)
    torch.cuda.synchronize(dev)
    n0 = g.ops.launch_count()
    with ClockSampler(0) as clk:
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            g.ops.lmhead_ce_fwd(x, w, tgt)
        b.record(stream)
        torch.cuda.synchronize(dev)
    ms = a.elapsed_time(b) / args.steps
    g.model.sync_status(dev)
    launches = (g.ops.launch_count() - n0) / args.steps
    g.ops.profile_start()
    for _ in range(args.steps):
        g.ops.lmhead_ce_fwd(x, w, tgt)
    torch.cuda.synchronize(dev)
    prof = g.ops.profile_stop()
    flops = 2.0 * M * D * V
    gemm_ms = prof["gemm"][0] / args.steps
    ach = flops / gemm_ms / 1e9 if gemm_ms > 0 else None
    line = {
        "metric": "d26 fused lm_head + cross-entropy forward TFLOP/s, 32768 tokens x 32768 vocab",
        "value": flops / ms / 1e9, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "lm_head + CE forward: M=32768, D=1664, V=32768 (d26 shape)",
                   "l2": "x 109 MB + W 109 MB, above the 126 MB L2; no flush"},
        "roofline": {"kernel": "gemm (cross-entropy epilogue)", "bound": "tensor", "achieved": ach, "peak": peak,
                     "unit": "TFLOP/s", "frac": ach / peak if ach else None, "traffic": None,
                     "peak_source": f"{peak_src} bf16 burst"},
        "logits_bytes_not_written": 2 * M * V,
        "gpu_launches": launches,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


def run_gemm_shapes(args):
    """The GEMM kernel alone, bf16 (kind::f16) against 8-bit e4m3 (kind::f8f6f4), on the d20
    projection shapes at 32768 tokens (QKV, out-projection, MLP up, MLP down) and a square 8192^3.
    Inputs N(0, 1) (seeds 7, 8), outputs bf16; each product timed with CUDA events over `steps`
    back-to-back calls.  TFLOP/s on 2 M N K; the 8-bit figures against the bf16 burst peak times
    the nominal fp8 / bf16 ratio of 2."""
    import torch
    import decoder_only_gpt_tcgen05_b200 as g
    import synth

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    stream = torch.cuda.current_stream(dev)
    shapes = [("qkv", 32768, 3840, 1280), ("out_proj", 32768, 1280, 1280), ("mlp_up", 32768, 5120, 1280),
              ("mlp_down", 32768, 1280, 5120), ("square", 8192, 8192, 8192)]

    def timed(fn, k):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(k):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / k

    rows = []
    n0 = g.ops.launch_count()
    n_calls = 0
    with ClockSampler(0) as clk:
        for name, M, N, K in shapes:
            A = torch.from_numpy(synth.normal((M, K), 7)).to(dev).to(torch.bfloat16)
            Bw = torch.from_numpy(synth.normal((N, K), 8, std=0.05)).to(dev).to(torch.bfloat16)
            out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            qa, _, ia = g.ops.fp8_quantize(A, g.ops.FP8_E4M3)
            qb, _, ib = g.ops.fp8_quantize(Bw, g.ops.FP8_E4M3)
            ms16 = timed(lambda: g.ops.gemm(A, Bw, out), args.steps)
            ms8 = timed(lambda: g.ops.gemm_fp8(qa, 0, ia, qb, 0, ib, out), args.steps)
            n_calls += 2 * (args.warmup + args.steps)
            fl = 2.0 * M * N * K
            rows.append({"name": name, "M": M, "N": N, "K": K, "bf16_ms": ms16, "fp8_ms": ms8,
                         "bf16_tflops": fl / ms16 / 1e9, "fp8_tflops": fl / ms8 / 1e9,
                         "bf16_frac": fl / ms16 / 1e9 / peak, "fp8_frac": fl / ms8 / 1e9 / (2 * peak)})
            del A, Bw, out, qa, qb
        g.model.sync_status(dev)
    head = next(r for r in rows if r["name"] == "mlp_up")
    line = {
        "metric": "GEMM TFLOP/s, bf16 and e4m3 operands, d20 projection shapes at 32768 tokens (MLP up headline)",
        "value": head["bf16_tflops"], "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": head["bf16_ms"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "gemm shapes: " + ", ".join(f"{r['name']} {r['M']}x{r['N']}x{r['K']}" for r in rows),
                   "l2": "operands and outputs of the d20 shapes above the 126 MB L2; no flush"},
        "roofline": {"kernel": "gemm (bf16, MLP up)", "bound": "tensor", "achieved": head["bf16_tflops"],
                     "peak": peak, "unit": "TFLOP/s", "frac": head["bf16_frac"], "traffic": None,
                     "peak_source": f"{peak_src} bf16 burst"},
        "shapes": rows,
        "gpu_launches": (g.ops.launch_count() - n0) / max(1, n_calls),
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=list(WORKLOADS) + ["attn_sweep", "lmhead_d26", "gemm"], default="d20",
                    help="attn_sweep: the attention kernels alone over T = 512..8192 at 32768 tokens; "
                         "lmhead_d26: the fused lm_head + cross-entropy forward alone at the d26 shape; "
                         "gemm: the GEMM kernel alone, bf16 and e4m3, on the d20 projection shapes")
    ap.add_argument("--profile-steps", type=int, default=2)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--breakdown", action="store_true", help="also print the per-kernel-family table to stderr")
    ap.add_argument("--batch", type=int, default=None, help="override B (sequences per GPU), e.g. for profiling")
    ap.add_argument("--no-eval", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--optimizer", nargs="?", const="adamw", default=None, choices=["adamw", "muon", "zero2"],
                    help="add an optimizer step to every timed step: adamw (nanoGPT's, clip_grad_norm_ at 1.0, "
                         "decay on 2-D tensors), muon (Muon on the block matrices + AdamW), zero2 (AdamW on "
                         "each rank's slice after a reduce-scatter, then an all-gather of the weights)")
    ap.add_argument("--grad-sync", choices=["overlap", "blocking"], default="overlap",
                    help="with N > 1: average the gradient bucket by bucket while the backward runs (overlap), "
                         "or in one all-reduce after it (blocking)")
    ap.add_argument("--fp8", action="store_true",
                    help="the forward's block projections on e4m3 operands with dynamic per-tensor scales")
    ap.add_argument("--graph", action="store_true",
                    help="time replays of one step captured in a CUDA graph (one GPU)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.workload == "attn_sweep":
        if args.impl != "ours" or world != 1:
            ap.error("attn_sweep times this library's attention kernels on one GPU")
        run_attn_sweep(args)
        return
    if args.workload == "gemm":
        if args.impl != "ours" or world != 1:
            ap.error("gemm times this library's GEMM kernel on one GPU")
        run_gemm_shapes(args)
        return
    if args.workload == "lmhead_d26":
        if args.impl != "ours" or world != 1:
            ap.error("lmhead_d26 times this library's fused lm_head + cross-entropy on one GPU")
        run_lmhead(args)
        return
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.graph and world != 1:
        ap.error("--graph times one GPU (the step's all-reduce is not captured)")

    import torch
    import torch.distributed as dist
    import decoder_only_gpt_tcgen05_b200 as g
    import synth

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", device_id=dev, timeout=timedelta(seconds=120))
    peaks, peak_src = load_peaks()

    preset_name, B, T, desc = WORKLOADS[args.workload]
    if args.batch:
        B = args.batch
        desc += f" [batch overridden: B={B}]"
    cfg = g.preset(preset_name, fp8=1 if args.fp8 else 0)
    if args.fp8:
        desc += " [fp8 e4m3 forward projections]"
    model = g.GPT(cfg, B, T, device=dev, seed=0)
    idx, tgt = synth.next_token_batch(B, T, cfg.vocab_size, seed=1 + rank)
    tb = synth.byte_table(cfg.vocab_size, 1, 16 if preset_name != "gpt2" else 12, seed=2)
    idx_d, tgt_d = torch.from_numpy(idx).to(dev), torch.from_numpy(tgt).to(dev)
    tb_d = torch.from_numpy(tb).to(dev)
    stream = torch.cuda.current_stream(dev)

    from decoder_only_gpt_tcgen05_b200 import dist as gdist
    if args.optimizer == "zero2" and world == 1:
        ap.error("--optimizer zero2 shards the optimizer over ranks: it needs N > 1")
    sync = None
    if world > 1 and (args.grad_sync == "overlap" or args.optimizer == "zero2"):
        sync = gdist.OverlappedGradSync(model, "reduce_scatter" if args.optimizer == "zero2" else "allreduce")
    if args.optimizer == "adamw":
        opt = g.AdamW(model, lr=6e-4, betas=(0.9, 0.95), weight_decay=0.1, grad_clip=1.0)
    elif args.optimizer == "muon":
        opt = g.MuonAdamW(model, lr=0.02, momentum=0.95, adam_lr=3e-4, betas=(0.9, 0.95), weight_decay=0.0)
    elif args.optimizer == "zero2":
        opt = gdist.ShardedAdamW(sync, lr=6e-4, betas=(0.9, 0.95), weight_decay=0.1)
    else:
        opt = None

    def step():
        model.forward_loss(idx_d, tgt_d)
        if sync is not None:
            sync.backward()
        else:
            model.backward()
            if world > 1:
                gdist.allreduce_grads_(model.grads)
        if opt is not None:
            opt.step()

    def barrier():
        if world > 1:
            dist.barrier()

    def timed(fn, k):
        barrier()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(k):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        ms = a.elapsed_time(b) / k
        if world > 1:
            t = torch.tensor([ms], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ms = t.item()
        return ms

    # ---- warm-up, then the timed training steps
    for _ in range(args.warmup):
        step()
    g.model.sync_status(dev)
    timed_step = step
    graph_launches = None
    if args.graph:
        # one step captured once; each timed iteration replays it (kernel arguments, tensor maps
        # and buffers are the eager step's, so the replay recomputes the same loss and gradients)
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step()
        stream.wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        n_cap = g.ops.launch_count()
        with torch.cuda.graph(graph):
            step()
        graph_launches = g.ops.launch_count() - n_cap
        timed_step = graph.replay
        for _ in range(args.warmup):
            timed_step()
    n0 = g.ops.launch_count()
    with ClockSampler(local) as clk:
        torch.cuda.nvtx.range_push("timed")
        ms = timed(timed_step, args.steps)
        torch.cuda.nvtx.range_pop()
    launches = (g.ops.launch_count() - n0) // args.steps if graph_launches is None else graph_launches
    clocks = clk.summary()
    g.model.sync_status(dev)

    # ---- eval (val_bpb) throughput
    def evalstep():
        model.eval_bpb(idx_d, tgt_d, tb_d)
    ms_eval = None
    if not args.no_eval:
        for _ in range(args.warmup):
            evalstep()
        ms_eval = timed(evalstep, args.steps)

    # ---- end to end through the public API with host buffers
    idx_h = torch.from_numpy(idx).pin_memory()
    tgt_h = torch.from_numpy(tgt).pin_memory()
    loss_h = torch.empty(1, dtype=torch.float32).pin_memory()

    def e2e_step():
        idx_d.copy_(idx_h, non_blocking=True)
        tgt_d.copy_(tgt_h, non_blocking=True)
        step()
        loss_h.copy_(model.loss, non_blocking=True)
    ms_e2e = None
    if not args.no_e2e:
        for _ in range(2):
            e2e_step()
        ms_e2e = timed(e2e_step, args.steps)
    h2d = idx_h.numel() * 4 + tgt_h.numel() * 4
    d2h = 4

    # ---- per-kernel-family times inside extra profiled steps (CUDA events around each launch)
    g.ops.profile_start()
    for _ in range(args.profile_steps):
        step()
    torch.cuda.synchronize(dev)
    prof = g.ops.profile_stop()
    nprof = max(1, args.profile_steps)
    g.model.sync_status(dev)

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    flops = step_flops(cfg, B, T)                    # per GPU, causal attention count
    flops_nc = step_flops(cfg, B, T, causal=False)
    tokens = B * T * world
    value = tokens / (ms / 1000.0)
    tflops = flops / (ms / 1000.0) / 1e12            # per GPU
    peak_sus = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    total_prof_ms = sum(v[0] for v in prof.values()) or 1.0
    # the dominant kernel: the GEMM kernel (all its roles) when it leads, else the leading family
    fam = dict(prof)
    gemm_roles = [k for k in fam if k.startswith("gemm")]
    fam["gemm"] = tuple(sum(fam[k][i] for k in gemm_roles) for i in range(4))
    for k in gemm_roles:
        if k != "gemm":
            del fam[k]
    dom = max(fam, key=lambda k: fam[k][0])
    prof_dom = fam
    dms, dcnt, dfl, dby = prof_dom[dom]
    if dms <= 0:
        roof = None
    elif dfl > 0:
        ach_exec = dfl / (dms / 1000.0) / 1e12
        if dom == "gemm":
            # algorithmic: the linear layers' 6 N tokens of the step (without the lm_head logits the
            # backward recomputes, and without the Muon products of an optimizer step)
            alg = 6.0 * matmul_params(cfg) * B * T * nprof
            fam_ms = dms - prof.get("gemm_muon", (0.0,))[0]
            ach = alg / (fam_ms / 1000.0) / 1e12
        else:
            ach = ach_exec
        roof = {"kernel": dom, "bound": "tensor", "achieved": ach, "peak": peak_sus, "unit": "TFLOP/s",
                "frac": ach / peak_sus, "achieved_executed": ach_exec, "frac_executed": ach_exec / peak_sus,
                "traffic": None, "launches_per_step": dcnt // nprof,
                "share_of_step": dms / total_prof_ms, "peak_source": f"{peak_src} bf16 sustained"}
    else:
        ach = dby / (dms / 1000.0) / 1e9
        roof = {"kernel": dom, "bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"], "traffic": None, "share_of_step": dms / total_prof_ms,
                "peak_source": f"{peak_src} hbm copy"}
    traffic_file = os.path.join(ROOT, "profiles", "traffic.json")
    if roof is not None and os.path.exists(traffic_file):
        try:
            import hashlib
            t = json.load(open(traffic_file)).get(dom)
            # counters taken on one workload and batch describe that launch mix only, and only while
            # every source file that shapes those launches is unchanged
            if t and t.get("workload") == args.workload and t.get("batch") == B:
                h = hashlib.sha256()
                for f in t["sources"]:
                    h.update(open(os.path.join(ROOT, f), "rb").read())
                if h.hexdigest() == t["sources_sha256"]:
                    roof["traffic"] = t["bytes_per_launch"]
        except Exception:
            pass

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(preset_name)

    breakdown = {k: {"ms_per_step": v[0] / nprof, "launches_per_step": v[1] // nprof,
                     "tflops": (v[2] / (v[0] / 1000) / 1e12) if v[0] > 0 and v[2] > 0 else None,
                     "gbs": (v[3] / (v[0] / 1000) / 1e9) if v[0] > 0 and v[3] > 0 else None}
                 for k, v in prof.items() if v[1] > 0}
    if args.breakdown:
        for k, v in sorted(breakdown.items(), key=lambda kv: -kv[1]["ms_per_step"]):
            print(f"{k:14s} {v['ms_per_step']:9.3f} ms  x{v['launches_per_step']:5d}  "
                  f"{(v['tflops'] or 0):8.1f} TF/s  {(v['gbs'] or 0):8.1f} GB/s", file=sys.stderr)

    # fp32 weights and gradients, and the step's workspace (their bf16 copy, the saved activations)
    working_set_gb = (model.params.numel() * 8 + model.ws_bytes) / 1e9
    line = {
        "metric": metric_name(preset_name), "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16+e4m3" if args.fp8 else "bf16", "data": "synthetic",
        "config": {"workload": desc, "B": B, "T": T, "tokens_per_step": tokens,
                   "parallelism": f"dp{world}" if world > 1 else "single",
                   "launch": "CUDA graph replay of one captured step" if args.graph else "eager stream launches",
                   "optimizer": {None: "none: forward + backward",
                                 "adamw": "AdamW step inside every timed step (clip 1.0, decay on 2-D tensors)",
                                 "muon": "Muon (5 Newton-Schulz steps, bf16 tensor cores) on the block matrices "
                                         "+ AdamW on the rest, inside every timed step",
                                 "zero2": "reduce-scatter + AdamW on each rank's slice + all-gather of the "
                                          "weights, inside every timed step"}[args.optimizer],
                   "grad_sync": (None if world == 1 else
                                 "bucketed on a second stream while the backward runs" if sync is not None
                                 else "one NCCL all-reduce after the backward"),
                   "l2": f"working set ({working_set_gb:.1f} GB of weights, gradients and workspace) far above the "
                         "126 MB L2; no flush"},
        "mfu": {"tflops_per_gpu": tflops, "vs_measured_sustained": tflops / peak_sus,
                "vs_measured_burst": tflops / peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]),
                "vs_datasheet_2250": tflops / DATASHEET_BF16_TFLOPS,
                "flops_per_step": flops, "flops_per_step_noncausal": flops_nc,
                "peak_source": peak_src},
        "eval": ({"metric": "val_bpb eval tokens/s", "value": tokens / (ms_eval / 1000.0), "ms_per_step": ms_eval}
                 if ms_eval else None),
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": ({"value": tokens / (ms_e2e / 1000.0), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                 "d2h_bytes_per_step": d2h} if ms_e2e else None),
        "gpu_launches": int(launches),
        "clocks": clocks,
        "breakdown": breakdown,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
