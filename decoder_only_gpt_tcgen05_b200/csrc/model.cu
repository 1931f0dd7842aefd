// Model-level C ABI (include/gpt.h): parameter layout, workspace planner, and the
// stream-ordered launch sequences of the forward loss, the backward and the bpb
// evaluation.
//
// Forward (per layer): norm -> QKV GEMM (+bias, RoPE, QK-norm in the epilogue) ->
// flash attention -> out-proj GEMM (+bias, residual add in the epilogue) -> norm ->
// MLP-up GEMM (+bias, activation in the epilogue) -> MLP-down GEMM (+bias, residual).
// Then the final norm and the lm_head GEMM whose epilogue keeps an online logsumexp
// per row over each vocab tile, so the logits never reach memory.
//
// Backward: cross-entropy gradient tiles (recomputed logits, softmax - onehot, bf16
// dlogits for a block of rows, at most 512 MiB of them) feed the lm_head data- and
// weight-gradient GEMMs; each layer then runs
// its GEMM gradients (MN-major operands, no transposes), the activation gradient in
// the data-gradient epilogue, the flash-attention backward, the QK-norm/RoPE
// reverse, the norm backward with the residual add, and finally the deterministic
// embedding scatter.
#include <cstdlib>
#include <cmath>
#include <cstring>
#include <string>
#include <vector>

#include "gemm.cuh"
#include "gpt.h"
#include "host.cuh"
#include "kernels.cuh"

namespace gptk {

void set_wait_timeout_ns(unsigned long long ns);
int norm_bwd_max_blocks();

// ------------------------------------------------------------------ parameter layout

struct ParamInfo {
  std::string name;
  long long off, rows, cols;
};

struct LayerOff {
  long long ln1_g = -1, ln1_b = -1, w_qkv = -1, b_qkv = -1, w_o = -1, b_o = -1;
  long long ln2_g = -1, ln2_b = -1, w_up = -1, b_up = -1, w_down = -1, b_down = -1;
};

struct Layout {
  std::vector<ParamInfo> list;
  long long wte = -1, wpe = -1, lnf_g = -1, lnf_b = -1, lm_head = -1;
  std::vector<LayerOff> layer;
  std::vector<long long> layer_begin, layer_end;  // element range of each layer's tensors
  long long total = 0;
};

static long long add_param(Layout& L, const std::string& name, long long rows, long long cols) {
  ParamInfo p{name, L.total, rows, cols};
  L.list.push_back(p);
  L.total += rows * cols;
  return p.off;
}

static Layout make_layout(const gpt_config& c) {
  Layout L;
  const long long D = c.n_embd, V = c.vocab_size, F = 4LL * c.n_embd;
  const bool ln = c.norm == 1, bias = c.linear_bias != 0;
  L.wte = add_param(L, "wte", V, D);
  if (c.pos == 0) L.wpe = add_param(L, "wpe", c.block_size, D);
  for (int l = 0; l < c.n_layer; ++l) {
    LayerOff o;
    L.layer_begin.push_back(L.total);
    const std::string p = "h" + std::to_string(l) + ".";
    if (ln) {
      o.ln1_g = add_param(L, p + "ln1_g", D, 1);
      if (bias) o.ln1_b = add_param(L, p + "ln1_b", D, 1);
    }
    o.w_qkv = add_param(L, p + "w_qkv", 3 * D, D);
    if (bias) o.b_qkv = add_param(L, p + "b_qkv", 3 * D, 1);
    o.w_o = add_param(L, p + "w_o", D, D);
    if (bias) o.b_o = add_param(L, p + "b_o", D, 1);
    if (ln) {
      o.ln2_g = add_param(L, p + "ln2_g", D, 1);
      if (bias) o.ln2_b = add_param(L, p + "ln2_b", D, 1);
    }
    o.w_up = add_param(L, p + "w_up", F, D);
    if (bias) o.b_up = add_param(L, p + "b_up", F, 1);
    o.w_down = add_param(L, p + "w_down", D, F);
    if (bias) o.b_down = add_param(L, p + "b_down", D, 1);
    L.layer.push_back(o);
    L.layer_end.push_back(L.total);
  }
  if (ln) {
    L.lnf_g = add_param(L, "lnf_g", D, 1);
    if (bias) L.lnf_b = add_param(L, "lnf_b", D, 1);
  }
  if (!c.tie_embed) L.lm_head = add_param(L, "lm_head", V, D);
  return L;
}

// Gradient buckets in the order the backward completes them: the final norm and an untied
// lm_head (after the lm_head backward), then the layers in pairs from the top (the weight
// gradients of an odd layer are launched together with those of the even layer below it), then
// the embeddings (and a tied lm_head, whose table they share).  Each is one contiguous range.
struct Bucket {
  long long begin, end;
};
static std::vector<Bucket> grad_buckets(const gpt_config& c, const Layout& L) {
  std::vector<Bucket> b;
  const long long head = L.lnf_g >= 0 ? L.lnf_g : (c.tie_embed ? L.total : L.lm_head);
  b.push_back(Bucket{head, L.total});  // may be empty (tied, no LayerNorm)
  for (int l = c.n_layer - 1; l >= 0; --l)
    if (!((l & 1) && l > 0)) b.push_back(Bucket{L.layer_begin[l], L.layer_end[(l + 1 < c.n_layer && (l + 1) & 1) ? l + 1 : l]});
  b.push_back(Bucket{0, L.layer_begin[0]});
  return b;
}

static int validate(const gpt_config* c) {
  if (!c) return set_error(ST_INVALID_ARG, "null config");
  if (c->n_layer < 1 || c->n_embd < 1 || c->n_head < 1 || c->vocab_size < 1 || c->block_size < 1)
    return set_error(ST_INVALID_ARG, "config: every size must be >= 1");
  if (c->norm < 0 || c->norm > 1 || c->pos < 0 || c->pos > 1 || c->act < 0 || c->act > 1)
    return set_error(ST_INVALID_ARG, "config: norm, pos and act must be 0 or 1");
  if (!(c->norm_eps > 0.f)) return set_error(ST_INVALID_ARG, "config: norm_eps must be > 0");
  if (c->pos == 1 && !(c->rope_base > 1.f)) return set_error(ST_INVALID_ARG, "config: rope_base must be > 1");
  if (c->n_embd % 16) return set_error(ST_UNSUPPORTED, "config: n_embd must be a multiple of 16");
  if (c->n_embd > 4096) return set_error(ST_UNSUPPORTED, "config: n_embd above 4096");
  if (c->n_embd % c->n_head) return set_error(ST_INVALID_ARG, "config: n_embd must be divisible by n_head");
  const int hd = c->n_embd / c->n_head;
  if (hd % 2 || hd > 128) return set_error(ST_UNSUPPORTED, "config: head dim must be even and at most 128");
  if ((c->pos == 1 || c->qk_norm) && hd != 64 && hd != 128)
    return set_error(ST_UNSUPPORTED, "config: RoPE / QK-norm need a head dim of 64 or 128");
  if (c->window_short < 0 || c->window_period < 1 || c->window_period > 32)
    return set_error(ST_INVALID_ARG, "config: window_short must be >= 0 and window_period in 1..32");
  if (c->fp8 != 0 && c->fp8 != 1) return set_error(ST_INVALID_ARG, "config: fp8 must be 0 or 1");
  return ST_OK;
}

// left window of layer l's attention (-1: every earlier key), from the layer pattern
static int layer_window(const gpt_config& c, int l) {
  if (c.window_short > 0 && ((static_cast<unsigned>(c.window_pattern) >> (l % c.window_period)) & 1u))
    return c.window_short;
  return -1;
}

// ------------------------------------------------------------------ workspace plan

static inline size_t al(size_t x) { return (x + 255) & ~size_t(255); }

struct Plan {
  int B, T, M, D, H, hd, hdp, F, L, V, Vp, ntn, Mc;
  int nsplit, ks;  // vocabulary pieces of the lm_head logits-gradient product and their K
  long long P;
  // byte offsets into the workspace
  size_t wbf, rope_cs, idx, tgt, xs, a1, st1, qkv, rq, rk, o, lse, a2, st2, u, h, af, stf;
  size_t ce_part, zy, ell, lse_ce, loss_d, loss_i, loss_f;
  size_t f8w, f8a, f8s;  // 8-bit block weights, one 8-bit activation, (amax, 1/scale) pairs
  size_t dlog, da_parts, da, dres, dres_bf, du, do_pad, delta, dqkv_pad, dqkv, part_a, part_b, embed;
  size_t total;
  long long partN;
};

static Plan make_plan(const gpt_config& c, int B, int T, long long P) {
  Plan p;
  p.B = B;
  p.T = T;
  p.M = B * T;
  p.D = c.n_embd;
  p.H = c.n_head;
  p.hd = c.n_embd / c.n_head;
  p.hdp = p.hd <= 64 ? 64 : 128;
  p.F = 4 * c.n_embd;
  p.L = c.n_layer;
  p.V = c.vocab_size;
  p.Vp = (c.vocab_size + 7) / 8 * 8;
  p.ntn = (c.vocab_size + 255) / 256;
  // lm_head backward row block: the bf16 dlogits of one block of rows stay within 512 MiB (8192
  // rows at V = 32768), so the whole M x V gradient is never held.  The logits-gradient product
  // d af = dlogits W_lm of a block is split along the vocabulary into pieces that run as one
  // grouped launch (a 256-row-tile product over 1280 columns alone would leave most SM pairs
  // idle in its last wave).
  {
    const long long cap = (512LL << 20) / ((long long)p.Vp * 2);
    long long mc = cap / 256 * 256;
    if (mc < 256) mc = 256;
    // GPT_LM_CHUNK_ROWS=<n> forces n-row blocks (tests of the blocked path on small batches)
    static const long long forced = []() {
      const char* e = std::getenv("GPT_LM_CHUNK_ROWS");
      return e ? std::atoll(e) : 0LL;
    }();
    if (forced > 0) mc = forced;
    p.Mc = (int)(mc < p.M ? mc : p.M);
    // vocabulary pieces of d af = dlogits W_lm: about one block's rows of K each, at most 8
    int ns = (p.V + p.Mc - 1) / p.Mc;
    if (ns > kMaxProblems) ns = kMaxProblems;
    if (ns < 1) ns = 1;
    p.ks = ((p.V + ns - 1) / ns + 63) / 64 * 64;
    p.nsplit = (p.V + p.ks - 1) / p.ks;
  }
  p.P = P;
  const size_t M = p.M, D = p.D, F = p.F, L = p.L, H = p.H, hdp = p.hdp;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t r = off;
    off += al(bytes);
    return r;
  };
  p.wbf = take((size_t)P * 2);
  p.rope_cs = take((size_t)T * (p.hd / 2) * 8);
  p.idx = take(M * 4);
  p.tgt = take(M * 4);
  p.xs = take((2 * L + 1) * M * D * 4);
  p.a1 = take(L * M * D * 2);
  p.st1 = take(L * 2 * M * 4);
  p.qkv = take(L * M * 3 * H * hdp * 2);
  p.rq = take(L * M * H * 4);
  p.rk = take(L * M * H * 4);
  p.o = take(L * M * D * 2);
  p.lse = take(L * M * H * 4);
  p.a2 = take(L * M * D * 2);
  p.st2 = take(L * 2 * M * 4);
  p.u = take(c.act == 1 ? 256 : L * M * F * 2);  // pre-activations are kept for GELU only
  p.h = take(L * M * F * 2);
  p.af = take(M * D * 2);
  p.stf = take(2 * M * 4);
  p.ce_part = take(M * p.ntn * 8);
  p.zy = take(M * 4);
  p.ell = take(M * 4);
  p.lse_ce = take(M * 4);
  p.loss_d = take(loss_reduce_blocks() * 2 * 8);
  p.loss_i = take(loss_reduce_blocks() * 2 * 8);
  p.loss_f = take(64);
  if (c.fp8) {
    p.f8w = take((size_t)L * 12 * D * D);               // w_qkv, w_o, w_up, w_down of every layer
    p.f8a = take(M * (F > D ? F : D));
    p.f8s = take((size_t)(8 * L) * 2 * 4);                // (amax, 1/scale): 4L weights, 4L activations
  } else {
    p.f8w = p.f8a = p.f8s = 0;
  }
  p.dlog = take((size_t)p.Mc * p.Vp * 2);
  p.da = take(M * D * 4);
  p.dres = take(M * D * 4);
  // the scratch gradients the weight-gradient GEMMs read have two slots (layer parity): a pair of
  // layers' weight gradients is launched together
  p.dres_bf = take(4 * M * D * 2);  // [slot][sublayer]
  p.du = take(2 * M * F * 2);
  // the lm_head backward's per-piece d af buffers: in du, which is idle until the first layer's
  // backward, when it is large enough
  {
    const size_t need = p.nsplit > 1 ? (size_t)p.nsplit * p.Mc * p.D * 4 : 256;
    p.da_parts = need <= 2 * M * F * 2 ? p.du : take(need);
  }
  p.do_pad = take(M * H * hdp * 2);
  p.delta = take(M * H * 4);
  p.dqkv_pad = take((p.hdp == p.hd ? 2 : 1) * M * 3 * H * hdp * 2);  // [slot] when it is dqkv itself
  p.dqkv = take(2 * M * 3 * D * 2);
  long long maxN = F > 3 * D ? F : 3 * D;
  long long rows = norm_bwd_max_blocks() > colsum_max_chunks() ? norm_bwd_max_blocks() : colsum_max_chunks();
  p.partN = maxN;
  p.part_a = take((size_t)rows * maxN * 4);
  p.part_b = take((size_t)rows * maxN * 4);
  p.embed = take((size_t)embed_bwd_scratch_bytes(p.M, p.V, p.D));
  p.total = off;
  return p;
}

static int check_batch(const gpt_config* c, int B, int T) {
  if (B < 1 || T < 1) return set_error(ST_INVALID_ARG, "B and T must be >= 1");
  if (c->pos == 0 && T > c->block_size) return set_error(ST_INVALID_ARG, "T exceeds block_size");
  if ((long long)B * T > (1LL << 30)) return set_error(ST_UNSUPPORTED, "B*T too large");
  if ((long long)B * c->n_head > 65535) return set_error(ST_UNSUPPORTED, "B * n_head above 65535");
  return ST_OK;
}

template <typename T>
static T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

// ------------------------------------------------------------------ GEMM helper

static GemmParams gp(int M, int N, int K) {
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.M = M;
  p.N = N;
  p.K = K;
  p.hd = p.hdp = 1;
  return p;
}

// tile width: 256 unless that leaves most SMs idle
static int pick_bn(int M, int N) {
  const long long t256 = (long long)((M + 127) / 128) * ((N + 255) / 256);
  return (N <= 128 || t256 < num_sms()) ? 128 : 256;
}

static int gemm(int epi, const Operand& A, const Operand& Bm, GemmParams p, cudaStream_t st, int bn = 0) {
  if (bn == 0) bn = pick_bn(p.M, p.N);
  return run_gemm(epi, bn, A, Bm, p, st);
}

// ------------------------------------------------------------------ forward

static int forward_impl(const gpt_config& c, const Layout& Lo, const Plan& pl, const float* params, const int* idx,
                        const int* targets, const int* token_bytes, void* ws, float* loss, double* sum_nats,
                        long long* sum_bytes, float* bpb, cudaStream_t st) {
  const int M = pl.M, D = pl.D, H = pl.H, hd = pl.hd, hdp = pl.hdp, F = pl.F, T = pl.T, B = pl.B, V = pl.V;
  const int ln = c.norm == 1;
  __nv_bfloat16* wbf = at<__nv_bfloat16>(ws, pl.wbf);
  float2* cs = at<float2>(ws, pl.rope_cs);
  int* idx_ws = at<int>(ws, pl.idx);
  int* tgt_ws = at<int>(ws, pl.tgt);
  GPTK_CUDA(cudaMemcpyAsync(idx_ws, idx, (size_t)M * 4, cudaMemcpyDeviceToDevice, st));
  GPTK_CUDA(cudaMemcpyAsync(tgt_ws, targets, (size_t)M * 4, cudaMemcpyDeviceToDevice, st));
  GPTK_TRY(launch_cast_bf16(params, wbf, pl.P, st));
  if (c.pos == 1) GPTK_TRY(launch_rope_table(cs, T, hd / 2, (double)c.rope_base, st));

  // 8-bit forward projections: every block weight cast once per forward, each with its own scale;
  // the activation operand of each projection is cast just before its product, from the max |x|
  // that its producer (the norm, the attention output, the MLP-up epilogue) folded into the
  // activation's slot (slots 4L + 4l + k, zeroed once per forward)
  uint8_t* f8w = c.fp8 ? at<uint8_t>(ws, pl.f8w) : nullptr;
  uint8_t* f8a = c.fp8 ? at<uint8_t>(ws, pl.f8a) : nullptr;
  float* f8s = c.fp8 ? at<float>(ws, pl.f8s) : nullptr;  // [slot][amax, 1/scale]
  const size_t DD = (size_t)D * D;
  auto f8w_of = [&](int l, int which) {  // which: 0 qkv, 1 o, 2 up, 3 down
    const size_t off[4] = {0, 3 * DD, 4 * DD, 8 * DD};
    return f8w + (size_t)l * 12 * DD + off[which];
  };
  // GPT_FP8_AMAX_PASS=1 (tests): the activations' max |x| from a pass of its own instead of their
  // producers, which must give the same scales bit for bit
  static const bool amax_pass = [] {
    const char* e = std::getenv("GPT_FP8_AMAX_PASS");
    return e != nullptr && std::atoi(e) == 1;
  }();
  auto act_slot = [&](int l, int k) -> float* { return c.fp8 ? f8s + 2 * (4 * pl.L + 4 * l + k) : nullptr; };
  auto fold_slot = [&](int l, int k) -> float* { return amax_pass ? nullptr : act_slot(l, k); };
  if (c.fp8) {
    GPTK_CUDA(cudaMemsetAsync(f8s + 2 * 4 * pl.L, 0, (size_t)4 * pl.L * 2 * sizeof(float), st));
    for (int l = 0; l < pl.L; ++l) {
      const LayerOff& o = Lo.layer[l];
      const long long offs[4] = {o.w_qkv, o.w_o, o.w_up, o.w_down};
      const size_t sizes[4] = {3 * DD, DD, 4 * DD, 4 * DD};
      for (int w = 0; w < 4; ++w)
        GPTK_TRY(launch_fp8_quantize(params + offs[w], 1, (long long)sizes[w], 0, f8w_of(l, w),
                                     f8s + 2 * (4 * l + w), f8s + 2 * (4 * l + w) + 1, st));
    }
  }
  // the 8-bit operands of one projection: the activation act [M, K] cast into f8a with the scale
  // from its slot's max |act|
  auto f8_setup = [&](GemmParams& p, const __nv_bfloat16* act, long long n, int l, int which, int k) -> int {
    float* sa = act_slot(l, k);
    if (amax_pass) GPTK_TRY(launch_fp8_quantize(act, 0, n, 0, f8a, sa, sa + 1, st));
    else GPTK_TRY(launch_fp8_cast(act, 0, n, 0, f8a, sa, sa + 1, st));
    p.f8_fmt_a = p.f8_fmt_b = 0;
    p.f8_inv_a = sa + 1;
    p.f8_inv_b = f8s + 2 * (4 * l + which) + 1;
    return ST_OK;
  };

  float* xs = at<float>(ws, pl.xs);
  const size_t MD = (size_t)M * D;
  GPTK_TRY(launch_embed_fwd(idx_ws, params + Lo.wte, Lo.wpe >= 0 ? params + Lo.wpe : nullptr, xs, M, T, D, V, st));

  for (int l = 0; l < pl.L; ++l) {
    const LayerOff& o = Lo.layer[l];
    float* x_in = xs + (size_t)(2 * l) * MD;
    float* x_mid = xs + (size_t)(2 * l + 1) * MD;
    float* x_out = xs + (size_t)(2 * l + 2) * MD;
    __nv_bfloat16* a1 = at<__nv_bfloat16>(ws, pl.a1) + (size_t)l * MD;
    float* st1 = at<float>(ws, pl.st1) + (size_t)l * 2 * M;
    __nv_bfloat16* qkv = at<__nv_bfloat16>(ws, pl.qkv) + (size_t)l * M * 3 * H * hdp;
    float* rq = at<float>(ws, pl.rq) + (size_t)l * M * H;
    float* rk = at<float>(ws, pl.rk) + (size_t)l * M * H;
    __nv_bfloat16* ob = at<__nv_bfloat16>(ws, pl.o) + (size_t)l * MD;
    float* lse = at<float>(ws, pl.lse) + (size_t)l * M * H;
    __nv_bfloat16* a2 = at<__nv_bfloat16>(ws, pl.a2) + (size_t)l * MD;
    float* st2 = at<float>(ws, pl.st2) + (size_t)l * 2 * M;
    __nv_bfloat16* u = at<__nv_bfloat16>(ws, pl.u) + (size_t)l * M * F;
    __nv_bfloat16* h = at<__nv_bfloat16>(ws, pl.h) + (size_t)l * M * F;

    // attention sublayer
    GPTK_TRY(launch_norm_fwd(x_in, M, D, ln ? params + o.ln1_g : nullptr, o.ln1_b >= 0 ? params + o.ln1_b : nullptr, ln,
                             c.norm_eps, a1, D, st1, st1 + M, st, fold_slot(l, 0)));
    {
      // q|k|v = a1 W_qkv^T (+ b): straight into the attention layout when it is unpadded.
      // With 128-wide heads and no bias, RoPE and QK-norm run in the GEMM epilogue on the fp32
      // accumulator; otherwise they follow as an in-place pass on q and k.
      const bool padded = hdp != hd;
      const bool fused = !padded && hd == 128 && D % 256 == 0 && o.b_qkv < 0 && (c.pos == 1 || c.qk_norm);
      __nv_bfloat16* raw = padded ? at<__nv_bfloat16>(ws, pl.dqkv) : qkv;
      GemmParams p = gp(M, 3 * D, D);
      p.out = raw;
      p.ldo = 3LL * D;
      p.bias = o.b_qkv >= 0 ? params + o.b_qkv : nullptr;
      p.prof_kind = PK_GEMM_QKV;
      Operand qa{a1, D, 0}, qb{wbf + o.w_qkv, D, 0};
      if (c.fp8) {
        GPTK_TRY(f8_setup(p, a1, (long long)MD, l, 0, 0));
        qa = Operand{f8a, D, 0};
        qb = Operand{f8w_of(l, 0), D, 0};
      }
      if (fused) {
        p.rope_cs = cs;
        p.rope_T = T;
        p.qk_D = D;
        p.qk_H = H;
        p.qk_rope = c.pos == 1;
        p.qk_norm = c.qk_norm;
        p.qk_eps = c.norm_eps;
        p.rstd_q = rq;
        p.rstd_k = rk;
        GPTK_TRY(gemm(EPI_QKV, qa, qb, p, st, 256));
      } else {
        GPTK_TRY(gemm(EPI_BF16, qa, qb, p, st));
        if (padded) GPTK_CUDA(cudaMemsetAsync(qkv, 0, (size_t)M * 3 * H * hdp * 2, st));
        if (padded || c.pos == 1 || c.qk_norm)
          GPTK_TRY(launch_qk_fwd(raw, cs, M, T, H, hd, hdp, c.pos == 1, c.qk_norm, c.norm_eps, qkv, rq, rk, st));
      }
    }
    AttnShape as{B, T, H, hd, hdp, 3LL * H * hdp, layer_window(c, l)};
    GPTK_TRY(launch_attn_fwd(qkv, as, ob, D, lse, st, fold_slot(l, 1)));
    {
      GemmParams p = gp(M, D, D);
      p.out = x_mid;
      p.ldo = D;
      p.resid = x_in;
      p.ldr = D;
      p.bias = o.b_o >= 0 ? params + o.b_o : nullptr;
      p.prof_kind = PK_GEMM_O;
      if (c.fp8) {
        GPTK_TRY(f8_setup(p, ob, (long long)MD, l, 1, 1));
        GPTK_TRY(gemm(EPI_RESID, Operand{f8a, D, 0}, Operand{f8w_of(l, 1), D, 0}, p, st));
      } else {
        GPTK_TRY(gemm(EPI_RESID, Operand{ob, D, 0}, Operand{wbf + o.w_o, D, 0}, p, st));
      }
    }
    // MLP sublayer
    GPTK_TRY(launch_norm_fwd(x_mid, M, D, ln ? params + o.ln2_g : nullptr, o.ln2_b >= 0 ? params + o.ln2_b : nullptr,
                             ln, c.norm_eps, a2, D, st2, st2 + M, st, fold_slot(l, 2)));
    {
      GemmParams p = gp(M, F, D);
      p.out = c.act == 1 ? nullptr : u;  // ReLU^2 keeps only h: the backward uses 2 relu(u) = 2 sqrt(h)
      p.out2 = h;
      p.ldo = F;
      p.act = c.act;
      p.bias = o.b_up >= 0 ? params + o.b_up : nullptr;
      p.prof_kind = PK_GEMM_UP;
      if (c.fp8) {
        GPTK_TRY(f8_setup(p, a2, (long long)MD, l, 2, 2));
        p.amax_h = reinterpret_cast<unsigned int*>(fold_slot(l, 3));
        GPTK_TRY(gemm(EPI_UP, Operand{f8a, D, 0}, Operand{f8w_of(l, 2), D, 0}, p, st));
      } else {
        GPTK_TRY(gemm(EPI_UP, Operand{a2, D, 0}, Operand{wbf + o.w_up, D, 0}, p, st));
      }
    }
    {
      GemmParams p = gp(M, D, F);
      p.out = x_out;
      p.ldo = D;
      p.resid = x_mid;
      p.ldr = D;
      p.bias = o.b_down >= 0 ? params + o.b_down : nullptr;
      p.prof_kind = PK_GEMM_DOWN;
      if (c.fp8) {
        GPTK_TRY(f8_setup(p, h, (long long)M * F, l, 3, 3));
        GPTK_TRY(gemm(EPI_RESID, Operand{f8a, F, 0}, Operand{f8w_of(l, 3), F, 0}, p, st));
      } else {
        GPTK_TRY(gemm(EPI_RESID, Operand{h, F, 0}, Operand{wbf + o.w_down, F, 0}, p, st));
      }
    }
  }
  // final norm + lm_head + cross-entropy
  __nv_bfloat16* af = at<__nv_bfloat16>(ws, pl.af);
  float* stf = at<float>(ws, pl.stf);
  GPTK_TRY(launch_norm_fwd(xs + (size_t)(2 * pl.L) * MD, M, D, ln ? params + Lo.lnf_g : nullptr,
                           Lo.lnf_b >= 0 ? params + Lo.lnf_b : nullptr, ln, c.norm_eps, af, D, stf, stf + M, st));
  const long long wlm = c.tie_embed ? Lo.wte : Lo.lm_head;
  float2* part = at<float2>(ws, pl.ce_part);
  float* zy = at<float>(ws, pl.zy);
  {
    GemmParams p = gp(M, V, D);
    p.targets = tgt_ws;
    p.ce_part = part;
    p.ce_zy = zy;
    p.prof_kind = PK_GEMM_LM_FWD;
      GPTK_TRY(gemm(EPI_CE_FWD, Operand{af, D, 0}, Operand{wbf + wlm, D, 0}, p, st, 256));
  }
  float* ell = at<float>(ws, pl.ell);
  float* lse_ce = at<float>(ws, pl.lse_ce);
  GPTK_TRY(launch_ce_combine(part, pl.ntn, zy, tgt_ws, V, M, ell, lse_ce, st));
  GPTK_TRY(launch_loss_reduce(ell, tgt_ws, token_bytes, V, M, at<double>(ws, pl.loss_d), at<long long>(ws, pl.loss_i),
                              loss ? loss : at<float>(ws, pl.loss_f), sum_nats, sum_bytes, bpb, st));
  return ST_OK;
}

// ------------------------------------------------------------------ backward

static int bias_grad_f32(const float* a, int M, int N, float* part, float* dst, cudaStream_t st) {
  int R = 0;
  GPTK_TRY(launch_colsum_f32(a, N, M, N, part, &R, st));
  return launch_colreduce(part, R, N, dst, 1, st);
}

static int bias_grad_bf16(const __nv_bfloat16* a, int M, int N, float* part, float* dst, cudaStream_t st) {
  int R = 0;
  GPTK_TRY(launch_colsum_bf16(a, N, M, N, part, &R, st));
  return launch_colreduce(part, R, N, dst, 1, st);
}

// dy: fp32, or bf16 when dy_bf16 (RMSNorm only); y: the saved bf16 output of the forward norm
static int norm_backward(const gpt_config& c, const Plan& pl, const void* dy, int dy_bf16, const float* x,
                         const __nv_bfloat16* y, const float* stats, const float* params, long long g_off,
                         long long b_off, float* grads, float* dres, int dres_init, __nv_bfloat16* dres_bf, float* pa,
                         float* pb, cudaStream_t st) {
  const int ln = c.norm == 1;
  const int M = pl.M, D = pl.D;
  // RMSNorm (no gain): the backward needs only the bf16 output and rstd, not the fp32 input
  if (!ln) return launch_rms_bwd(dy, dy_bf16, y, stats + M, M, D, dres, dres_init, dres_bf, st);
  if (dy_bf16) return set_error(ST_INVALID_ARG, "LayerNorm backward takes an fp32 dy");
  int nblk = 0;
  GPTK_TRY(launch_norm_bwd(static_cast<const float*>(dy), x, stats, stats + M, params + g_off, ln, M, D, dres,
                           dres_init, dres_bf, pa, pb, &nblk, st));
  if (ln) {
    GPTK_TRY(launch_colreduce(pa, nblk, D, grads + g_off, 1, st));
    if (b_off >= 0) GPTK_TRY(launch_colreduce(pb, nblk, D, grads + b_off, 1, st));
  }
  return ST_OK;
}

static int backward_impl(const gpt_config& c, const Layout& Lo, const Plan& pl, const float* params, void* ws,
                         float* grads, int accumulate, cudaStream_t st, void* const* events = nullptr) {
  int bucket = 0;  // next gradient bucket to complete (events[bucket] is recorded when it is final)
  auto done = [&]() -> int {
    if (events) GPTK_CUDA(cudaEventRecord(static_cast<cudaEvent_t>(events[bucket]), st));
    ++bucket;
    return ST_OK;
  };
  const int M = pl.M, D = pl.D, H = pl.H, hd = pl.hd, hdp = pl.hdp, F = pl.F, T = pl.T, B = pl.B, V = pl.V;
  const size_t MD = (size_t)M * D;
  const int rms = c.norm == 0;  // RMSNorm: the norm backward reads bf16 data gradients
  __nv_bfloat16* wbf = at<__nv_bfloat16>(ws, pl.wbf);
  const float2* cs = at<float2>(ws, pl.rope_cs);
  const int* idx_ws = at<int>(ws, pl.idx);
  const int* tgt_ws = at<int>(ws, pl.tgt);
  float* xs = at<float>(ws, pl.xs);
  __nv_bfloat16* af = at<__nv_bfloat16>(ws, pl.af);
  float* stf = at<float>(ws, pl.stf);
  float* lse_ce = at<float>(ws, pl.lse_ce);
  float* da = at<float>(ws, pl.da);
  float* dres = at<float>(ws, pl.dres);
  __nv_bfloat16* do_pad = at<__nv_bfloat16>(ws, pl.do_pad);
  float* delta = at<float>(ws, pl.delta);
  float* pa = at<float>(ws, pl.part_a);
  float* pb = at<float>(ws, pl.part_b);
  __nv_bfloat16* dlog = at<__nv_bfloat16>(ws, pl.dlog);
  // Scratch gradients read by the weight-gradient GEMMs, in two slots by layer parity: the
  // weight gradients of an odd layer wait and run in one grouped launch with those of the even
  // layer below it (eight products: better-filled waves than four), so an odd layer's bf16
  // residual gradients (one per sublayer), du and dqkv must outlive the next layer's backward.
  auto dres_bf_mlp_of = [&](int l) { return at<__nv_bfloat16>(ws, pl.dres_bf) + (size_t)(2 * (l & 1)) * MD; };
  auto dres_bf_att_of = [&](int l) { return at<__nv_bfloat16>(ws, pl.dres_bf) + (size_t)(2 * (l & 1) + 1) * MD; };
  auto du_of = [&](int l) { return at<__nv_bfloat16>(ws, pl.du) + (size_t)(l & 1) * M * F; };
  auto dqkv_pad_of = [&](int l) {
    return at<__nv_bfloat16>(ws, pl.dqkv_pad) + (hdp == hd ? (size_t)(l & 1) * M * 3 * H * hdp : 0);
  };
  auto dqkv_of = [&](int l) {
    return hdp == hd ? dqkv_pad_of(l) : at<__nv_bfloat16>(ws, pl.dqkv) + (size_t)(l & 1) * M * 3 * D;
  };
  GroupProblem pending[4];  // an odd layer's weight-gradient products, waiting for the next layer
  int n_pending = 0;

  if (!accumulate) GPTK_CUDA(cudaMemsetAsync(grads, 0, (size_t)pl.P * 4, st));

  // ---- lm_head + cross-entropy backward, one block of pl.Mc rows at a time: the block's bf16
  //      dlogits (recomputed logits, softmax - onehot) feed the weight gradient and the
  //      logits-gradient product, then the next block reuses the buffer
  const long long wlm = c.tie_embed ? Lo.wte : Lo.lm_head;
  const int nsplit = pl.nsplit, ks = pl.ks;
  for (int r0 = 0; r0 < M; r0 += pl.Mc) {
    const int mc = (M - r0) < pl.Mc ? (M - r0) : pl.Mc;
    {
      GemmParams p = gp(mc, V, D);
      p.out = dlog;
      p.ldo = pl.Vp;
      p.targets = tgt_ws + r0;
      p.ce_lse = lse_ce + r0;
      p.ce_scale = 1.f / (float)M;
      p.prof_kind = PK_GEMM_LM_BWD;
      GPTK_TRY(gemm(EPI_CE_BWD, Operand{af + (size_t)r0 * D, D, 0}, Operand{wbf + wlm, D, 0}, p, st, 256));
    }
    {  // d W_lm += dlogits^T af
      GemmParams p = gp(V, D, mc);
      p.out = grads + wlm;
      p.ldo = D;
      p.accumulate = 1;
      p.prof_kind = PK_GEMM_WGRAD;
      GPTK_TRY(gemm(EPI_F32, Operand{dlog, pl.Vp, 1}, Operand{af + (size_t)r0 * D, D, 1}, p, st));
    }
    if (nsplit == 1) {  // d af = dlogits W_lm
      GemmParams p = gp(mc, D, V);
      p.out = da + (size_t)r0 * D;
      p.ldo = D;
      p.prof_kind = PK_GEMM_LM_BWD;
      GPTK_TRY(gemm(EPI_F32, Operand{dlog, pl.Vp, 0}, Operand{wbf + wlm, D, 1}, p, st));
    } else {
      // d af = sum over vocabulary pieces j of dlogits[:, piece j] W_lm[piece j, :]: each piece to
      // its own fp32 buffer (stored, not accumulated, so no two tiles add into the same element),
      // then one pass adds them in piece order: deterministic
      float* parts = at<float>(ws, pl.da_parts);
      GroupProblem pieces[kMaxProblems];
      for (int j = 0; j < nsplit; ++j) {
        const int k0 = j * ks;
        const int kext = (V - k0) < ks ? (V - k0) : ks;
        pieces[j] = GroupProblem{dlog + k0, pl.Vp, wbf + wlm + (size_t)k0 * D, D, mc, D,
                                 parts + (size_t)j * pl.Mc * D, D, kext};
      }
      GPTK_TRY(run_gemm_group(nsplit, pieces, ks, 0, 1, 256, PK_GEMM_LM_BWD, st, EPI_F32, 0));
      GPTK_TRY(launch_sum_parts(parts, nsplit, (size_t)pl.Mc * D, (size_t)mc * D, da + (size_t)r0 * D, st));
    }
  }
  GPTK_TRY(norm_backward(c, pl, da, 0, xs + (size_t)(2 * pl.L) * MD, af, stf, params, Lo.lnf_g, Lo.lnf_b, grads, dres, 1,
                         dres_bf_mlp_of(pl.L - 1), pa, pb, st));
  GPTK_TRY(done());  // final norm (+ untied lm_head)

  for (int l = pl.L - 1; l >= 0; --l) {
    const LayerOff& o = Lo.layer[l];
    __nv_bfloat16* dres_bf_mlp = dres_bf_mlp_of(l);
    __nv_bfloat16* dres_bf_att = dres_bf_att_of(l);
    __nv_bfloat16* du = du_of(l);
    __nv_bfloat16* dqkv_pad = dqkv_pad_of(l);
    __nv_bfloat16* dqkv = dqkv_of(l);
    const float* x_in = xs + (size_t)(2 * l) * MD;
    const float* x_mid = xs + (size_t)(2 * l + 1) * MD;
    const __nv_bfloat16* a1 = at<__nv_bfloat16>(ws, pl.a1) + (size_t)l * MD;
    const float* st1 = at<float>(ws, pl.st1) + (size_t)l * 2 * M;
    const __nv_bfloat16* qkv = at<__nv_bfloat16>(ws, pl.qkv) + (size_t)l * M * 3 * H * hdp;
    const float* rq = at<float>(ws, pl.rq) + (size_t)l * M * H;
    const float* rk = at<float>(ws, pl.rk) + (size_t)l * M * H;
    const __nv_bfloat16* ob = at<__nv_bfloat16>(ws, pl.o) + (size_t)l * MD;
    const float* lse = at<float>(ws, pl.lse) + (size_t)l * M * H;
    const __nv_bfloat16* a2 = at<__nv_bfloat16>(ws, pl.a2) + (size_t)l * MD;
    const float* st2 = at<float>(ws, pl.st2) + (size_t)l * 2 * M;
    const __nv_bfloat16* u = at<__nv_bfloat16>(ws, pl.u) + (c.act == 1 ? 0 : (size_t)l * M * F);
    const __nv_bfloat16* h = at<__nv_bfloat16>(ws, pl.h) + (size_t)l * M * F;

    // ---- MLP: x_out = x_mid + act(N(x_mid) W_up^T + b_up) W_down^T + b_down
    {  // du = (dres W_down) * act'(u)
      GemmParams p = gp(M, F, D);
      p.out = du;
      p.ldo = F;
      p.aux = c.act == 1 ? h : u;
      p.ld_aux = F;
      p.act = c.act == 1 ? 2 : c.act;
      p.prof_kind = PK_GEMM_DGRAD;
      GPTK_TRY(gemm(EPI_ACTBWD, Operand{dres_bf_mlp, D, 0}, Operand{wbf + o.w_down, F, 1}, p, st));
    }
    if (o.b_down >= 0) GPTK_TRY(bias_grad_f32(dres, M, D, pa, grads + o.b_down, st));
    {  // da = du W_up (bf16 for RMSNorm, whose backward reads a bf16 dy)
      GemmParams p = gp(M, D, F);
      p.out = da;
      p.ldo = D;
      p.prof_kind = PK_GEMM_DGRAD;
      GPTK_TRY(gemm(rms ? EPI_BF16 : EPI_F32, Operand{du, F, 0}, Operand{wbf + o.w_up, D, 1}, p, st));
    }
    if (o.b_up >= 0) GPTK_TRY(bias_grad_bf16(du, M, F, pa, grads + o.b_up, st));
    GPTK_TRY(norm_backward(c, pl, da, rms, x_mid, a2, st2, params, o.ln2_g, o.ln2_b, grads, dres, 0, dres_bf_att, pa,
                           pb, st));

    // ---- attention: x_mid = x_in + attn(N(x_in)) W_o^T + b_o
    if (hdp != hd) GPTK_CUDA(cudaMemsetAsync(do_pad, 0, (size_t)M * H * hdp * 2, st));
    {  // do = dres W_o  (written in the head-padded layout the attention kernels read)
      GemmParams p = gp(M, D, D);
      p.out = do_pad;
      p.ldo = (long long)H * hdp;
      p.hd = hd;
      p.hdp = hdp;
      p.prof_kind = PK_GEMM_DGRAD;
      GPTK_TRY(gemm(EPI_BF16, Operand{dres_bf_att, D, 0}, Operand{wbf + o.w_o, D, 1}, p, st));
    }
    if (o.b_o >= 0) GPTK_TRY(bias_grad_f32(dres, M, D, pa, grads + o.b_o, st));
    GPTK_TRY(launch_attn_delta(ob, do_pad, B, T, H, hd, hdp, delta, st));
    AttnShape as{B, T, H, hd, hdp, 3LL * H * hdp, layer_window(c, l)};
    GPTK_TRY(launch_attn_bwd(qkv, do_pad, lse, delta, as, dqkv_pad, st));
    GPTK_TRY(launch_qk_bwd(dqkv_pad, qkv, rq, rk, cs, M, T, H, hd, hdp, c.pos == 1, c.qk_norm, dqkv, st));
    {  // da = dqkv W_qkv (bf16 for RMSNorm)
      GemmParams p = gp(M, D, 3 * D);
      p.out = da;
      p.ldo = D;
      p.prof_kind = PK_GEMM_DGRAD;
      GPTK_TRY(gemm(rms ? EPI_BF16 : EPI_F32, Operand{dqkv, 3LL * D, 0}, Operand{wbf + o.w_qkv, D, 1}, p, st));
    }
    if (o.b_qkv >= 0) GPTK_TRY(bias_grad_bf16(dqkv, M, 3 * D, pa, grads + o.b_qkv, st));
    {  // the layer's four weight gradients W += dY^T X over all tokens, launched together with the
       // pending four of the layer above (odd layers wait for the even one below them)
      const GroupProblem probs[4] = {
          {dres_bf_mlp, D, h, F, D, F, grads + o.w_down, F},
          {du, F, a2, D, F, D, grads + o.w_up, D},
          {dres_bf_att, D, ob, D, D, D, grads + o.w_o, D},
          {dqkv, 3LL * D, a1, D, 3 * D, D, grads + o.w_qkv, D},
      };
      if ((l & 1) && l > 0) {
        for (int q = 0; q < 4; ++q) pending[q] = probs[q];
        n_pending = 4;
      } else {
        GroupProblem all[8];
        for (int q = 0; q < n_pending; ++q) all[q] = pending[q];
        for (int q = 0; q < 4; ++q) all[n_pending + q] = probs[q];
        GPTK_TRY(run_gemm_group(n_pending + 4, all, M, 1, 1, 256, PK_GEMM_WGRAD, st));
        n_pending = 0;
      }
    }
    // the residual gradient of the layer below goes to that layer's slot
    GPTK_TRY(norm_backward(c, pl, da, rms, x_in, a1, st1, params, o.ln1_g, o.ln1_b, grads, dres, 0,
                           l > 0 ? dres_bf_mlp_of(l - 1) : dres_bf_mlp_of(0), pa, pb, st));
    if (!((l & 1) && l > 0)) GPTK_TRY(done());  // this layer (and the odd one above it)
  }
  // ---- embeddings
  GPTK_TRY(launch_embed_bwd(idx_ws, dres, M, D, V, grads + Lo.wte, at<void>(ws, pl.embed), st));
  if (Lo.wpe >= 0) GPTK_TRY(launch_pos_bwd(dres, B, T, D, grads + Lo.wpe, 1, st));
  return done();  // embeddings
}

// ------------------------------------------------------------------ init

static int init_impl(const gpt_config& c, const Layout& Lo, unsigned long long seed, float* params, cudaStream_t st) {
  for (const ParamInfo& p : Lo.list) {
    const std::string& n = p.name;
    const long long size = p.rows * p.cols;
    const std::string base = n.substr(n.find('.') == std::string::npos ? 0 : n.find('.') + 1);
    if (base == "ln1_g" || base == "ln2_g" || base == "lnf_g") {
      GPTK_TRY(launch_fill(params + p.off, size, 1.f, st));
    } else if (base.rfind("b_", 0) == 0 || base == "ln1_b" || base == "ln2_b" || base == "lnf_b") {
      GPTK_TRY(launch_fill(params + p.off, size, 0.f, st));
    } else {
      float stdv = 0.02f;
      if (c.scale_resid_init && (base == "w_o" || base == "w_down"))
        stdv = (float)(0.02 / std::sqrt(2.0 * c.n_layer));
      GPTK_TRY(launch_init_normal(params, p.off, size, seed, stdv, st));
    }
  }
  return ST_OK;
}

}  // namespace gptk

using namespace gptk;

// ====================================================================== C ABI

extern "C" {

GPT_API int gpt_param_count(const gpt_config* cfg, int64_t* n_out) {
  set_error(ST_OK, "");
  GPTK_TRY(validate(cfg));
  if (!n_out) return set_error(ST_INVALID_ARG, "null output");
  *n_out = make_layout(*cfg).total;
  return ST_OK;
}

GPT_API int gpt_param_tensor_count(const gpt_config* cfg, int32_t* n_out) {
  set_error(ST_OK, "");
  GPTK_TRY(validate(cfg));
  if (!n_out) return set_error(ST_INVALID_ARG, "null output");
  *n_out = (int32_t)make_layout(*cfg).list.size();
  return ST_OK;
}

GPT_API int gpt_param_tensor(const gpt_config* cfg, int32_t i, char* name, int32_t name_len, int64_t* offset,
                             int64_t* rows, int64_t* cols) {
  set_error(ST_OK, "");
  GPTK_TRY(validate(cfg));
  Layout L = make_layout(*cfg);
  if (i < 0 || i >= (int32_t)L.list.size()) return set_error(ST_INVALID_ARG, "tensor index out of range");
  const ParamInfo& p = L.list[i];
  if (name && name_len > 0) {
    std::strncpy(name, p.name.c_str(), (size_t)name_len - 1);
    name[name_len - 1] = '\0';
  }
  if (offset) *offset = p.off;
  if (rows) *rows = p.rows;
  if (cols) *cols = p.cols;
  return ST_OK;
}

GPT_API int gpt_adamw_step(const gpt_config* cfg, float* params, const float* grads, float* m, float* v,
                           int64_t step, const gpt_adamw* h, void* scratch, double* grad_norm, void* stream) {
  set_error(ST_OK, "");
  GPTK_TRY(validate(cfg));
  if (!h) return set_error(ST_INVALID_ARG, "gpt_adamw_step: null hyperparameters");
  // weight decay on the 2-D tensors (vectors are stored with cols == 1); adjacent tensors with
  // the same flag merge into one run
  Layout L = make_layout(*cfg);
  std::vector<long long> start;
  std::vector<unsigned char> decay;
  for (const ParamInfo& p : L.list) {
    const unsigned char d = p.cols > 1 ? 1 : 0;
    if (decay.empty() || decay.back() != d) {
      start.push_back(p.off);
      decay.push_back(d);
    }
  }
  return launch_adamw(params, grads, m, v, L.total, start.data(), decay.data(), (int)start.size(), step, *h, scratch,
                      grad_norm, static_cast<cudaStream_t>(stream));
}

// The Muon matrices of a layout (block Linear weights) and the runs of every other tensor
static void muon_split(const Layout& L, std::vector<long long>& offs, std::vector<int>& rows,
                       std::vector<int>& cols, std::vector<std::vector<const ParamInfo*>>& adam_ranges) {
  std::vector<const ParamInfo*> cur;
  for (const ParamInfo& p : L.list) {
    const std::string base = p.name.substr(p.name.find('.') == std::string::npos ? 0 : p.name.find('.') + 1);
    const bool muon = base == "w_qkv" || base == "w_o" || base == "w_up" || base == "w_down";
    if (muon) {
      offs.push_back(p.off);
      rows.push_back((int)p.rows);
      cols.push_back((int)p.cols);
      if (!cur.empty()) adam_ranges.push_back(cur);
      cur.clear();
    } else {
      cur.push_back(&p);
    }
  }
  if (!cur.empty()) adam_ranges.push_back(cur);
}

GPT_API int gpt_muon_scratch_size(const gpt_config* cfg, size_t* bytes) {
  set_error(ST_OK, "");
  GPTK_TRY(validate(cfg));
  if (!bytes) return set_error(ST_INVALID_ARG, "null output");
  Layout L = make_layout(*cfg);
  std::vector<long long> offs;
  std::vector<int> rows, cols;
  std::vector<std::vector<const ParamInfo*>> ranges;
  muon_split(L, offs, rows, cols, ranges);
  *bytes = muon_scratch_bytes(offs, rows, cols);
  return ST_OK;
}

GPT_API int gpt_muon_step(const gpt_config* cfg, float* params, const float* grads, float* mom, float* v,
                          int64_t step, const gpt_muon* h, void* scratch, void* stream) {
  set_error(ST_OK, "");
  GPTK_TRY(validate(cfg));
  if (!h) return set_error(ST_INVALID_ARG, "gpt_muon_step: null hyperparameters");
  if (!params || !grads || !mom || !v || !scratch) return set_error(ST_INVALID_ARG, "gpt_muon_step: null pointer");
  if (reinterpret_cast<uintptr_t>(scratch) & 255) return set_error(ST_INVALID_ARG, "gpt_muon_step: scratch alignment");
  for (const void* q : {(const void*)params, (const void*)grads, (const void*)mom, (const void*)v})
    if (reinterpret_cast<uintptr_t>(q) & 15) return set_error(ST_INVALID_ARG, "gpt_muon_step: 16-byte alignment");
  if (step < 1) return set_error(ST_INVALID_ARG, "gpt_muon_step: step must be >= 1");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Layout L = make_layout(*cfg);
  std::vector<long long> offs;
  std::vector<int> rows, cols;
  std::vector<std::vector<const ParamInfo*>> ranges;
  muon_split(L, offs, rows, cols, ranges);
  // AdamW on every other tensor, one launch pair per contiguous range (decay on 2-D tensors);
  // the AdamW scratch is the start of the Muon scratch
  gpt_adamw ah;
  ah.lr = h->adam_lr;
  ah.beta1 = h->beta1;
  ah.beta2 = h->beta2;
  ah.eps = h->eps;
  ah.weight_decay = h->weight_decay;
  ah.grad_scale = 1.f;
  ah.grad_clip = 0.f;
  for (const auto& rg : ranges) {
    const long long r0 = rg.front()->off;
    const long long n = rg.back()->off + rg.back()->rows * rg.back()->cols - r0;
    std::vector<long long> start;
    std::vector<unsigned char> decay;
    for (const ParamInfo* p : rg) {
      const unsigned char d = p->cols > 1 ? 1 : 0;
      if (decay.empty() || decay.back() != d) {
        start.push_back(p->off - r0);
        decay.push_back(d);
      }
    }
    GPTK_TRY(launch_adamw(params + r0, grads + r0, mom + r0, v + r0, n, start.data(), decay.data(), (int)start.size(),
                          step, ah, scratch, nullptr, st));
  }
  return launch_muon(params, grads, mom, offs, rows, cols, *h, scratch, st);
}

GPT_API int gpt_workspace_size(const gpt_config* cfg, int32_t B, int32_t T, size_t* bytes) {
  set_error(ST_OK, "");
  GPTK_TRY(validate(cfg));
  GPTK_TRY(check_batch(cfg, B, T));
  if (!bytes) return set_error(ST_INVALID_ARG, "null output");
  Layout L = make_layout(*cfg);
  *bytes = make_plan(*cfg, B, T, L.total).total;
  return ST_OK;
}

GPT_API int gpt_init_weights(const gpt_config* cfg, uint64_t seed, float* params, void* stream) {
  set_error(ST_OK, "");
  GPTK_TRY(validate(cfg));
  if (!params) return set_error(ST_INVALID_ARG, "null params");
  return init_impl(*cfg, make_layout(*cfg), seed, params, static_cast<cudaStream_t>(stream));
}

static int check_ws(void* ws, size_t have, size_t need) {
  if (!ws) return set_error(ST_INVALID_ARG, "null workspace");
  if (reinterpret_cast<uintptr_t>(ws) & 255) return set_error(ST_INVALID_ARG, "workspace must be 256-byte aligned");
  if (have < need)
    return set_error(ST_WORKSPACE_TOO_SMALL,
                     "workspace has " + std::to_string(have) + " bytes, needs " + std::to_string(need));
  return ST_OK;
}

GPT_API int gpt_forward_loss(const gpt_config* cfg, const float* params, const int32_t* idx, const int32_t* targets,
                             int32_t B, int32_t T, void* workspace, size_t workspace_bytes, float* loss,
                             void* stream) {
  set_error(ST_OK, "");
  GPTK_TRY(validate(cfg));
  GPTK_TRY(check_batch(cfg, B, T));
  if (!params || !idx || !targets || !loss) return set_error(ST_INVALID_ARG, "null pointer");
  Layout L = make_layout(*cfg);
  Plan pl = make_plan(*cfg, B, T, L.total);
  GPTK_TRY(check_ws(workspace, workspace_bytes, pl.total));
  return forward_impl(*cfg, L, pl, params, idx, targets, nullptr, workspace, loss, nullptr, nullptr, nullptr,
                      static_cast<cudaStream_t>(stream));
}

GPT_API int gpt_backward(const gpt_config* cfg, const float* params, int32_t B, int32_t T, void* workspace,
                         size_t workspace_bytes, float* grads, int32_t accumulate, void* stream) {
  set_error(ST_OK, "");
  GPTK_TRY(validate(cfg));
  GPTK_TRY(check_batch(cfg, B, T));
  if (!params || !grads) return set_error(ST_INVALID_ARG, "null pointer");
  Layout L = make_layout(*cfg);
  Plan pl = make_plan(*cfg, B, T, L.total);
  GPTK_TRY(check_ws(workspace, workspace_bytes, pl.total));
  return backward_impl(*cfg, L, pl, params, workspace, grads, accumulate, static_cast<cudaStream_t>(stream));
}

GPT_API int gpt_grad_buckets(const gpt_config* cfg, int32_t max_buckets, int32_t* n_out, int64_t* begin,
                             int64_t* end) {
  set_error(ST_OK, "");
  GPTK_TRY(validate(cfg));
  if (!n_out) return set_error(ST_INVALID_ARG, "null output");
  const std::vector<Bucket> b = grad_buckets(*cfg, make_layout(*cfg));
  *n_out = (int32_t)b.size();
  if (max_buckets < (int32_t)b.size() && (begin || end))
    return set_error(ST_INVALID_ARG, "gpt_grad_buckets: room for " + std::to_string(max_buckets) + " buckets, " +
                                         std::to_string(b.size()) + " needed");
  for (size_t k = 0; k < b.size(); ++k) {
    if (begin) begin[k] = b[k].begin;
    if (end) end[k] = b[k].end;
  }
  return ST_OK;
}

GPT_API int gpt_backward_bucketed(const gpt_config* cfg, const float* params, int32_t B, int32_t T, void* workspace,
                                  size_t workspace_bytes, float* grads, int32_t accumulate, void* const* events,
                                  int32_t n_events, void* stream) {
  set_error(ST_OK, "");
  GPTK_TRY(validate(cfg));
  GPTK_TRY(check_batch(cfg, B, T));
  if (!params || !grads || !events) return set_error(ST_INVALID_ARG, "null pointer");
  Layout L = make_layout(*cfg);
  if (n_events != (int32_t)grad_buckets(*cfg, L).size())
    return set_error(ST_INVALID_ARG, "gpt_backward_bucketed: one event per gradient bucket (gpt_grad_buckets)");
  for (int32_t k = 0; k < n_events; ++k)
    if (!events[k]) return set_error(ST_INVALID_ARG, "gpt_backward_bucketed: null event");
  Plan pl = make_plan(*cfg, B, T, L.total);
  GPTK_TRY(check_ws(workspace, workspace_bytes, pl.total));
  return backward_impl(*cfg, L, pl, params, workspace, grads, accumulate, static_cast<cudaStream_t>(stream), events);
}

GPT_API int gpt_eval_bpb(const gpt_config* cfg, const float* params, const int32_t* idx, const int32_t* targets,
                         const int32_t* token_bytes, int32_t B, int32_t T, void* workspace, size_t workspace_bytes,
                         double* sum_nats, int64_t* sum_bytes, float* bpb, void* stream) {
  set_error(ST_OK, "");
  GPTK_TRY(validate(cfg));
  GPTK_TRY(check_batch(cfg, B, T));
  if (!params || !idx || !targets || !token_bytes) return set_error(ST_INVALID_ARG, "null pointer");
  Layout L = make_layout(*cfg);
  Plan pl = make_plan(*cfg, B, T, L.total);
  GPTK_TRY(check_ws(workspace, workspace_bytes, pl.total));
  return forward_impl(*cfg, L, pl, params, idx, targets, token_bytes, workspace, nullptr, sum_nats,
                      reinterpret_cast<long long*>(sum_bytes), bpb, static_cast<cudaStream_t>(stream));
}

GPT_API int gpt_token_losses(const gpt_config* cfg, int32_t B, int32_t T, const void* workspace,
                             size_t workspace_bytes, float* ell, float* lse, void* stream) {
  set_error(ST_OK, "");
  GPTK_TRY(validate(cfg));
  GPTK_TRY(check_batch(cfg, B, T));
  Layout L = make_layout(*cfg);
  Plan pl = make_plan(*cfg, B, T, L.total);
  GPTK_TRY(check_ws(const_cast<void*>(workspace), workspace_bytes, pl.total));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (ell) GPTK_CUDA(cudaMemcpyAsync(ell, at<float>(const_cast<void*>(workspace), pl.ell), (size_t)pl.M * 4,
                                     cudaMemcpyDeviceToDevice, st));
  if (lse) GPTK_CUDA(cudaMemcpyAsync(lse, at<float>(const_cast<void*>(workspace), pl.lse_ce), (size_t)pl.M * 4,
                                     cudaMemcpyDeviceToDevice, st));
  return ST_OK;
}

GPT_API int gpt_debug_logits(const gpt_config* cfg, int32_t B, int32_t T, void* workspace, size_t workspace_bytes,
                             float* logits, void* stream) {
  set_error(ST_OK, "");
  GPTK_TRY(validate(cfg));
  GPTK_TRY(check_batch(cfg, B, T));
  if (!logits) return set_error(ST_INVALID_ARG, "null logits");
  Layout L = make_layout(*cfg);
  Plan pl = make_plan(*cfg, B, T, L.total);
  GPTK_TRY(check_ws(workspace, workspace_bytes, pl.total));
  // the lm_head product of the fused cross-entropy, on the same operands (the saved final-norm
  // output and the bf16 weight mirror), with its fp32 tiles stored instead of folded
  const long long wlm = cfg->tie_embed ? L.wte : L.lm_head;
  GemmParams p = gp(pl.M, pl.V, pl.D);
  p.out = logits;
  p.ldo = pl.V;
  return gemm(EPI_F32, Operand{at<__nv_bfloat16>(workspace, pl.af), pl.D, 0},
              Operand{at<__nv_bfloat16>(workspace, pl.wbf) + wlm, pl.D, 0}, p, static_cast<cudaStream_t>(stream), 256);
}

GPT_API int gpt_sync_status(void* stream) {
  set_error(ST_OK, "");
  GPTK_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  DevCtl c = device_ctl();
  if (!c.status) return set_error(ST_CUDA, "device status word unavailable");
  unsigned int v = 0;
  GPTK_CUDA(cudaMemcpy(&v, c.status, sizeof(v), cudaMemcpyDeviceToHost));
  if (v == 0) return ST_OK;
  const unsigned int zero = 0;
  GPTK_CUDA(cudaMemcpy(c.status, &zero, sizeof(zero), cudaMemcpyHostToDevice));
  const unsigned int code = v >> 24, site = (v >> 16) & 0xff, blk = v & 0xffff;
  if (code == DEV_ERR_TIMEOUT)
    return set_error(ST_DEVICE_TIMEOUT, "a kernel gave up a bounded wait (site " + std::to_string(site) + ", block " +
                                            std::to_string(blk) + ")");
  if (code == DEV_ERR_BAD_TOKEN) return set_error(ST_INVALID_ARG, "a token id was outside [0, vocab_size)");
  return set_error(ST_CUDA, "device status word " + std::to_string(v));
}

GPT_API int gpt_set_wait_timeout_ns(uint64_t ns) {
  set_error(ST_OK, "");
  if (ns == 0) return set_error(ST_INVALID_ARG, "timeout must be > 0");
  set_wait_timeout_ns(ns);
  return ST_OK;
}

}  // extern "C"
