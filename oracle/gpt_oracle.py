"""Oracle for the decoder-only GPT hot path: a plain, slow, fp64 CPU model.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check and
the benchmark's CPU-baseline leg may import this module.  It shares no code
with the CUDA library: no kernels, headers, helpers or tables.  Every step is
written straight from its definition with numpy (matmul is the only library
primitive used), in float64, with no blocking, fusion or reordering.

Sources (page title, section):
  [GPT2] "nanoGPT - Karpathy's minimal GPT pretraining repo", How it works /
         model.py - the GPT (architecture walkthrough): GPTConfig, Block,
         CausalSelfAttention, MLP, weight tying, scaled residual init;
         train.py - the loop: targets are inputs shifted by 1.
  [CHAT] "Train your own ChatGPT" (lab 03), section 6.2 reading notes:
         gpt.py (init_weights, estimate_flops), loss_eval.py (bits per byte).
  [D20]  "nanochat-d20-chat" model card, Architecture table: 20 layers,
         width 1280, 10 heads, RoPE + QK-norm, 2048 context, separate token
         and output tables.

Readings where the pages are silent (each is one config field, identical on
both sides): norm epsilon (default 1e-5); a final norm before lm_head in every
configuration; RoPE pairs dimension i with i + hd/2 and rotates by angle
t * base^(-2i/hd); RoPE is applied before the per-head QK RMSNorm (the two
commute in exact arithmetic); the attention scale stays 1/sqrt(hd); GELU is the
exact erf form; ReLU^2 is relu(u)^2; the loss is the mean over all B*T
targets; tokens with a byte length of 0 are dropped from both sums of bpb.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
from scipy.special import erf

NORM_RMS, NORM_LN = 0, 1
POS_LEARNED, POS_ROPE = 0, 1
ACT_GELU, ACT_RELU2 = 0, 1


@dataclass(frozen=True)
class Config:
    """Model shape; field meanings follow GPTConfig ([GPT2] model.py)."""
    n_layer: int
    n_embd: int
    n_head: int
    block_size: int
    vocab_size: int
    norm: int = NORM_RMS          # 0: parameter-free RMSNorm, 1: LayerNorm (gain, optional bias)
    pos: int = POS_LEARNED        # 0: learned absolute wpe, 1: RoPE
    act: int = ACT_GELU           # 0: GELU (erf), 1: ReLU^2
    tie_embed: int = 1            # lm_head shares wte ([GPT2] weight tying)
    qk_norm: int = 0              # per-head RMSNorm of q and k ([D20])
    linear_bias: int = 0          # biases on every Linear and on LayerNorm ([GPT2] bias=True)
    scale_resid_init: int = 0     # residual out-projections init std 0.02/sqrt(2*n_layer)
    rope_base: float = 10000.0
    norm_eps: float = 1e-5
    # sliding-window layers ([CHAT] gpt.py: _compute_window_sizes() expands a pattern such as
    # "SSSL" into per-layer (left, right) windows): layer l is a short-window layer when bit
    # (l mod window_period) of window_pattern is set and window_short > 0; its query i then
    # sees the keys i - window_short .. i (right window 0: causal).  Other layers see every
    # earlier key.
    window_short: int = 0
    window_pattern: int = 0
    window_period: int = 1
    # [CHAT] fp8.py: the forward's block projections on e4m3 operands, every activation and
    # weight cast with its own dynamic scale (the lm_head and the backward stay unquantized)
    fp8: int = 0

    @property
    def head_dim(self) -> int:
        return self.n_embd // self.n_head

    @property
    def d_ff(self) -> int:
        return 4 * self.n_embd


# ---------------------------------------------------------------- parameters

def param_shapes(cfg: Config):
    """Ordered (name, shape) list of the flat fp32 parameter buffer.

    Linear weights are [out, in] (nn.Linear convention, [GPT2] model.py)."""
    D, V, F = cfg.n_embd, cfg.vocab_size, cfg.d_ff
    ln = cfg.norm == NORM_LN
    bias = bool(cfg.linear_bias)
    out = [("wte", (V, D))]
    if cfg.pos == POS_LEARNED:
        out.append(("wpe", (cfg.block_size, D)))
    for l in range(cfg.n_layer):
        p = f"h{l}."
        if ln:
            out.append((p + "ln1_g", (D,)))
            if bias:
                out.append((p + "ln1_b", (D,)))
        out.append((p + "w_qkv", (3 * D, D)))
        if bias:
            out.append((p + "b_qkv", (3 * D,)))
        out.append((p + "w_o", (D, D)))
        if bias:
            out.append((p + "b_o", (D,)))
        if ln:
            out.append((p + "ln2_g", (D,)))
            if bias:
                out.append((p + "ln2_b", (D,)))
        out.append((p + "w_up", (F, D)))
        if bias:
            out.append((p + "b_up", (F,)))
        out.append((p + "w_down", (D, F)))
        if bias:
            out.append((p + "b_down", (D,)))
    if ln:
        out.append(("lnf_g", (D,)))
        if bias:
            out.append(("lnf_b", (D,)))
    if not cfg.tie_embed:
        out.append(("lm_head", (V, D)))
    return out


def param_count(cfg: Config) -> int:
    return sum(int(np.prod(s)) for _, s in param_shapes(cfg))


def param_offsets(cfg: Config):
    off, res = 0, {}
    for name, shape in param_shapes(cfg):
        n = int(np.prod(shape))
        res[name] = (off, shape)
        off += n
    return res


def unflatten(cfg: Config, flat: np.ndarray):
    """Dict of named views into the flat parameter (or gradient) vector."""
    return {name: flat[o:o + int(np.prod(s))].reshape(s)
            for name, (o, s) in param_offsets(cfg).items()}


# ------------------------------------------------------------ initialisation

_GAMMA = 0x9E3779B97F4A7C15
_MASK = (1 << 64) - 1


def splitmix64(state: int) -> int:
    """One output of SplitMix64 (Steele, Lea, Flood 2014; Vigna's reference
    splitmix64.c) for the state *after* the increment: the mixing function."""
    z = state & _MASK
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK
    return z ^ (z >> 31)


def splitmix64_stream(seed: int, n: np.ndarray) -> np.ndarray:
    """Outputs number n (0-based) of SplitMix64 seeded with ``seed``: the
    generator's state after n+1 increments of the golden gamma, mixed.
    Vectorised over uint64 ``n``."""
    with np.errstate(over="ignore"):
        z = (np.uint64(seed) + (n.astype(np.uint64) + np.uint64(1)) * np.uint64(_GAMMA))
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        z = z ^ (z >> np.uint64(31))
    return z


def counter_normal(seed: int, index: np.ndarray) -> np.ndarray:
    """Standard normal for each flat element index, by Box-Muller on two
    24-bit uniforms taken from SplitMix64 outputs 2*i and 2*i+1:
    u1 = (hi24(r0) + 1) / 2^24 in (0, 1], u2 = hi24(r1) / 2^24 in [0, 1),
    z = sqrt(-2 ln u1) cos(2 pi u2)."""
    i = index.astype(np.uint64)
    r0 = splitmix64_stream(seed, np.uint64(2) * i)
    r1 = splitmix64_stream(seed, np.uint64(2) * i + np.uint64(1))
    u1 = ((r0 >> np.uint64(40)).astype(np.float64) + 1.0) * 2.0 ** -24
    u2 = (r1 >> np.uint64(40)).astype(np.float64) * 2.0 ** -24
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def init_params(cfg: Config, seed: int) -> np.ndarray:
    """Initial flat parameters ([GPT2] 'Two details': N(0, 0.02^2) for every
    matrix and embedding, residual output projections scaled by
    1/sqrt(2 n_layer) when ``scale_resid_init``; biases 0, LayerNorm gains 1)."""
    n = param_count(cfg)
    out = np.zeros(n, dtype=np.float64)
    for name, (off, shape) in param_offsets(cfg).items():
        size = int(np.prod(shape))
        base = name.split(".")[-1]
        if base in ("ln1_g", "ln2_g") or name == "lnf_g":
            out[off:off + size] = 1.0
        elif base.startswith("b_") or base.endswith("_b"):
            out[off:off + size] = 0.0
        else:
            std = 0.02
            if cfg.scale_resid_init and base in ("w_o", "w_down"):
                std = 0.02 / math.sqrt(2.0 * cfg.n_layer)
            out[off:off + size] = std * counter_normal(seed, np.arange(off, off + size))
    return out


# ------------------------------------------------------------------ pieces

def rmsnorm(x, eps):
    """Parameter-free RMSNorm over the last axis: x / sqrt(mean(x^2) + eps)."""
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return x * r, r


def rmsnorm_bwd(dy, y, r):
    """Reverse of y = x * r, r = (mean(x^2)+eps)^-1/2:  dx = r (dy - y mean(dy*y))."""
    return r * (dy - y * np.mean(dy * y, axis=-1, keepdims=True))


def layernorm(x, g, b, eps):
    """LayerNorm with biased variance ([GPT2] hand-rolled LayerNorm, bias optional)."""
    mu = np.mean(x, axis=-1, keepdims=True)
    xc = x - mu
    r = 1.0 / np.sqrt(np.mean(xc * xc, axis=-1, keepdims=True) + eps)
    xh = xc * r
    y = xh * g
    if b is not None:
        y = y + b
    return y, xh, r


def layernorm_bwd(dy, xh, r, g):
    dxh = dy * g
    dx = r * (dxh - np.mean(dxh, axis=-1, keepdims=True)
              - xh * np.mean(dxh * xh, axis=-1, keepdims=True))
    dg = np.sum(dy * xh, axis=tuple(range(dy.ndim - 1)))
    db = np.sum(dy, axis=tuple(range(dy.ndim - 1)))
    return dx, dg, db


def rope_angles(T, hd, base):
    """phi[t, i] = t * base^(-2i/hd) for i < hd/2."""
    i = np.arange(hd // 2, dtype=np.float64)
    inv = base ** (-2.0 * i / hd)
    return np.arange(T, dtype=np.float64)[:, None] * inv[None, :]


def rope(x, phi):
    """Rotate pairs (x_i, x_{i+hd/2}) by phi; x is [..., T, hd], phi [T, hd/2]."""
    h = x.shape[-1] // 2
    c, s = np.cos(phi), np.sin(phi)
    a, b = x[..., :h], x[..., h:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def rope_bwd(dy, phi):
    """The rotation is orthogonal, so its reverse is the rotation by -phi."""
    return rope(dy, -phi)


def gelu(u):
    return 0.5 * u * (1.0 + erf(u / math.sqrt(2.0)))


def gelu_grad(u):
    return 0.5 * (1.0 + erf(u / math.sqrt(2.0))) + u * np.exp(-0.5 * u * u) / math.sqrt(2.0 * math.pi)


def relu2(u):
    r = np.maximum(u, 0.0)
    return r * r


def relu2_grad(u):
    return 2.0 * np.maximum(u, 0.0)


def pattern_bits(pattern: str) -> int:
    """The window_pattern bits of a pattern string such as "SSSL" (bit i set for an 'S')."""
    return sum(1 << i for i, ch in enumerate(pattern) if ch == "S")


def layer_window(cfg: Config, layer: int):
    """Left window of a layer's attention (keys i - w .. i visible from query i), or None for
    the full causal prefix ([CHAT] gpt.py, _compute_window_sizes: pattern letter
    window_pattern[layer mod period], 'S' short, 'L' long)."""
    if cfg.window_short > 0 and (cfg.window_pattern >> (layer % cfg.window_period)) & 1:
        return int(cfg.window_short)
    return None


def causal_attention(q, k, v, window=None):
    """softmax(q k^T / sqrt(hd) + mask) v with S[i, j] = -inf for j > i
    ([GPT2] CausalSelfAttention, the manual path with the explicit mask), and also for
    j < i - window when a left window is given ([CHAT] gpt.py, per-layer windows).
    q, k, v: [B, H, T, hd].  Returns (o, P)."""
    T, hd = q.shape[-2], q.shape[-1]
    s = (q @ np.swapaxes(k, -1, -2)) / math.sqrt(hd)
    mask = np.triu(np.ones((T, T), dtype=bool), k=1)
    if window is not None:
        mask |= np.tril(np.ones((T, T), dtype=bool), k=-(window + 1))
    s = np.where(mask, -np.inf, s)
    s = s - np.max(s, axis=-1, keepdims=True)
    p = np.exp(s)
    p = p / np.sum(p, axis=-1, keepdims=True)
    return p @ v, p


def causal_attention_bwd(do, q, k, v, p):
    """Reverse of causal_attention given its probabilities p."""
    hd = q.shape[-1]
    dv = np.swapaxes(p, -1, -2) @ do
    dp = do @ np.swapaxes(v, -1, -2)
    ds = p * (dp - np.sum(dp * p, axis=-1, keepdims=True))
    dq = (ds @ k) / math.sqrt(hd)
    dk = (np.swapaxes(ds, -1, -2) @ q) / math.sqrt(hd)
    return dq, dk, dv


def cross_entropy(z, y):
    """Per-row next-token loss l_m = logsumexp(z_m) - z_m[y_m] (nats)."""
    zmax = np.max(z, axis=-1, keepdims=True)
    lse = np.log(np.sum(np.exp(z - zmax), axis=-1)) + zmax[:, 0]
    return lse - z[np.arange(z.shape[0]), y], lse


def bits_per_byte(ell, targets, token_bytes):
    """[CHAT] loss_eval.py: sum the loss in nats over the evaluated targets,
    sum the byte lengths of those targets, divide (with ln 2 for nats->bits).
    Targets whose byte length is 0 (special tokens) are left out of both sums.
    Returns (sum_nats float, sum_bytes int, n_tokens int, bpb float)."""
    y = np.asarray(targets).reshape(-1)
    nb = np.asarray(token_bytes, dtype=np.int64)[y]
    keep = nb > 0
    sum_nats = float(np.sum(np.asarray(ell, dtype=np.float64).reshape(-1)[keep]))
    sum_bytes = int(np.sum(nb))
    bpb = sum_nats / (math.log(2.0) * sum_bytes) if sum_bytes > 0 else float("nan")
    return sum_nats, sum_bytes, int(np.count_nonzero(keep)), bpb


# ------------------------------------------------------------------ model

def _norm(cfg, x, pr, name):
    if cfg.norm == NORM_RMS:
        y, r = rmsnorm(x, cfg.norm_eps)
        return y, ("rms", y, r)
    g = pr[name + "_g"]
    b = pr.get(name + "_b") if cfg.linear_bias else None
    y, xh, r = layernorm(x, g, b, cfg.norm_eps)
    return y, ("ln", xh, r)


def _norm_bwd(cfg, dy, cache, pr, grads, name):
    if cache[0] == "rms":
        return rmsnorm_bwd(dy, cache[1], cache[2])
    dx, dg, db = layernorm_bwd(dy, cache[1], cache[2], pr[name + "_g"])
    grads[name + "_g"] += dg
    if cfg.linear_bias:
        grads[name + "_b"] += db
    return dx


def _linear(x, w, b, fp8=False):
    if fp8:
        from .fp8_oracle import scaled_matmul
        y = scaled_matmul(x, w, "e4m3", "e4m3")
    else:
        y = x @ w.T
    return y + b if b is not None else y


def forward(cfg: Config, params, idx, targets, keep_cache=True, return_logits=False):
    """Loss of one batch ([GPT2] forward: wte (+wpe) -> n_layer Blocks -> final
    norm -> lm_head -> next-token cross-entropy, mean over B*T).

    idx, targets: int [B, T].  Returns a dict with 'loss' (mean nats),
    'ell' (per-token nats, [B*T]), 'lse', optionally 'logits', and 'cache'."""
    p = np.asarray(params, dtype=np.float64)
    pr = unflatten(cfg, p)
    idx = np.asarray(idx)
    targets = np.asarray(targets)
    B, T = idx.shape
    if T > cfg.block_size:
        raise ValueError("T exceeds block_size")
    D, H, hd = cfg.n_embd, cfg.n_head, cfg.head_dim
    M = B * T
    bias = bool(cfg.linear_bias)
    x = pr["wte"][idx.reshape(-1)]
    if cfg.pos == POS_LEARNED:
        x = x + np.tile(pr["wpe"][:T], (B, 1))
    phi = rope_angles(T, hd, cfg.rope_base) if cfg.pos == POS_ROPE else None
    layers = []
    for l in range(cfg.n_layer):
        P = f"h{l}."
        c = {}
        a1, c["n1"] = _norm(cfg, x, pr, P + "ln1")
        q8 = bool(cfg.fp8)
        qkv = _linear(a1, pr[P + "w_qkv"], pr.get(P + "b_qkv") if bias else None, q8)
        q, k, v = (qkv[:, i * D:(i + 1) * D].reshape(B, T, H, hd).transpose(0, 2, 1, 3)
                   for i in range(3))
        if phi is not None:
            q, k = rope(q, phi), rope(k, phi)
        if cfg.qk_norm:
            q_rot, k_rot = q, k
            q, rq = rmsnorm(q_rot, cfg.norm_eps)
            k, rk = rmsnorm(k_rot, cfg.norm_eps)
            c["qn"] = (q, rq, k, rk)
        o, pa = causal_attention(q, k, v, layer_window(cfg, l))
        o2 = o.transpose(0, 2, 1, 3).reshape(M, D)
        c.update(a1=a1, q=q, k=k, v=v, P=pa, o=o2)
        x = x + _linear(o2, pr[P + "w_o"], pr.get(P + "b_o") if bias else None, q8)
        a2, c["n2"] = _norm(cfg, x, pr, P + "ln2")
        u = _linear(a2, pr[P + "w_up"], pr.get(P + "b_up") if bias else None, q8)
        h = relu2(u) if cfg.act == ACT_RELU2 else gelu(u)
        c.update(a2=a2, u=u, h=h)
        x = x + _linear(h, pr[P + "w_down"], pr.get(P + "b_down") if bias else None, q8)
        layers.append(c)
    af, nf = _norm(cfg, x, pr, "lnf")
    w_lm = pr["wte"] if cfg.tie_embed else pr["lm_head"]
    z = af @ w_lm.T
    y = targets.reshape(-1)
    ell, lse = cross_entropy(z, y)
    out = {"loss": float(np.mean(ell)), "ell": ell, "lse": lse}
    if return_logits:
        out["logits"] = z
    if keep_cache:
        out["cache"] = dict(B=B, T=T, idx=idx, y=y, layers=layers, af=af, nf=nf, z=z, phi=phi)
    return out


def backward(cfg: Config, params, fwd):
    """Gradient of the mean loss w.r.t. every parameter, by hand-derived
    reverse mode of ``forward``.  Returns a flat float64 vector laid out like
    the parameters."""
    p = np.asarray(params, dtype=np.float64)
    pr = unflatten(cfg, p)
    g = np.zeros_like(p)
    gr = unflatten(cfg, g)
    c = fwd["cache"]
    B, T, y, z = c["B"], c["T"], c["y"], c["z"]
    D, H, hd = cfg.n_embd, cfg.n_head, cfg.head_dim
    M = B * T
    bias = bool(cfg.linear_bias)
    # d loss / d z = (softmax(z) - onehot(y)) / M
    dz = np.exp(z - fwd["lse"][:, None])
    dz[np.arange(M), y] -= 1.0
    dz /= M
    w_lm = pr["wte"] if cfg.tie_embed else pr["lm_head"]
    dw_lm = dz.T @ c["af"]
    if cfg.tie_embed:
        gr["wte"] += dw_lm
    else:
        gr["lm_head"] += dw_lm
    daf = dz @ w_lm
    dx = _norm_bwd(cfg, daf, c["nf"], pr, gr, "lnf")
    for l in reversed(range(cfg.n_layer)):
        P = f"h{l}."
        L = c["layers"][l]
        # MLP sublayer: x_out = x_mid + act(N(x_mid) W_up^T + b) W_down^T + b
        gr[P + "w_down"] += dx.T @ L["h"]
        if bias:
            gr[P + "b_down"] += dx.sum(0)
        dh = dx @ pr[P + "w_down"]
        du = dh * (relu2_grad(L["u"]) if cfg.act == ACT_RELU2 else gelu_grad(L["u"]))
        gr[P + "w_up"] += du.T @ L["a2"]
        if bias:
            gr[P + "b_up"] += du.sum(0)
        da2 = du @ pr[P + "w_up"]
        dx = dx + _norm_bwd(cfg, da2, L["n2"], pr, gr, P + "ln2")
        # attention sublayer: x_mid = x_in + attn(N(x_in)) W_o^T + b
        gr[P + "w_o"] += dx.T @ L["o"]
        if bias:
            gr[P + "b_o"] += dx.sum(0)
        do = (dx @ pr[P + "w_o"]).reshape(B, T, H, hd).transpose(0, 2, 1, 3)
        dq, dk, dv = causal_attention_bwd(do, L["q"], L["k"], L["v"], L["P"])
        if cfg.qk_norm:
            qh, rq, kh, rk = L["qn"]
            dq = rmsnorm_bwd(dq, qh, rq)
            dk = rmsnorm_bwd(dk, kh, rk)
        if c["phi"] is not None:
            dq, dk = rope_bwd(dq, c["phi"]), rope_bwd(dk, c["phi"])
        dqkv = np.concatenate([t.transpose(0, 2, 1, 3).reshape(M, D) for t in (dq, dk, dv)], axis=1)
        gr[P + "w_qkv"] += dqkv.T @ L["a1"]
        if bias:
            gr[P + "b_qkv"] += dqkv.sum(0)
        da1 = dqkv @ pr[P + "w_qkv"]
        dx = dx + _norm_bwd(cfg, da1, L["n1"], pr, gr, P + "ln1")
    # embeddings: x0[m] = wte[idx[m]] (+ wpe[t])
    np.add.at(gr["wte"], c["idx"].reshape(-1), dx)
    if cfg.pos == POS_LEARNED:
        gr["wpe"][:T] += dx.reshape(B, T, D).sum(0)
    return g


def loss_and_grad(cfg: Config, params, idx, targets):
    f = forward(cfg, params, idx, targets)
    return f["loss"], backward(cfg, params, f)


# ------------------------------------------------------------- accounting

def matmul_params(cfg: Config) -> int:
    """Parameters that take part in a matmul per token: the transformer
    matrices plus the lm_head (embedding lookups are not matmuls)."""
    D, F = cfg.n_embd, cfg.d_ff
    per_layer = 3 * D * D + D * D + 2 * D * F
    return cfg.n_layer * per_layer + cfg.vocab_size * D


def step_flops(cfg: Config, B: int, T: int, causal: bool = True) -> float:
    """Forward+backward FLOPs of one step: 6 per matmul parameter per token
    plus attention ([CHAT] gpt.py estimate_flops: '6 FLOPs per parameter per
    token plus attention terms').  With causal=True the attention term counts
    only the unmasked half: 6 * n_layer * D * T per token; otherwise 12."""
    M = B * T
    att = (6 if causal else 12) * cfg.n_layer * cfg.n_embd * T
    return float(M) * (6.0 * matmul_params(cfg) + att)


def eval_flops(cfg: Config, B: int, T: int) -> float:
    """Forward-only FLOPs (2 per matmul parameter per token + causal attention)."""
    M = B * T
    return float(M) * (2.0 * matmul_params(cfg) + 2.0 * cfg.n_layer * cfg.n_embd * T)
