/* Op-level entry points of the B200 GPT library: the individual steps of the
 * hot path, callable one at a time for unit tests and for the attention-only
 * and lm_head-only measurements.  The model-level calls are in gpt.h.
 *
 * Conventions (shared with gpt.h):
 *   - every pointer argument is DEVICE memory owned by the caller, unless a
 *     comment says otherwise; the library allocates nothing and frees nothing;
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream); every call only enqueues work and returns;
 *   - bf16 tensors are passed as `const void*` holding IEEE bfloat16 values;
 *   - matrices are row-major with an explicit pitch `ld*` in elements, which
 *     must make every row start on a 16-byte boundary (ld multiple of 8 for
 *     bf16, of 4 for fp32); base pointers must be 16-byte aligned;
 *   - return value: 0 (GPT_OK) or a gpt_status code from gpt.h, with a
 *     message in gpt_last_error(); argument errors are detected on the host
 *     before anything is launched.
 */
#ifndef GPT_OPS_H
#define GPT_OPS_H

#include "gpt.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Epilogues of gpt_op_gemm. */
#define GPT_GEMM_OUT_BF16 0 /* out (bf16) = A B^T (+ bias)                          */
#define GPT_GEMM_OUT_F32 1  /* out (fp32) = A B^T (+ bias), or out += A B^T          */

/* The tensor-core matrix product used by every linear layer of the model
 * ("nanoGPT" wiki page, model.py walkthrough: c_attn, c_proj, c_fc and
 * lm_head are nn.Linear layers, y = x W^T + b):
 *
 *   out[M,N] = A[M,K] * B[N,K]^T
 *
 * A is given K-major (a_mn = 0: element (m,k) at a[m*lda + k]) or MN-major
 * (a_mn = 1: element (m,k) at a[k*lda + m]); likewise B (b_mn = 0: (n,k) at
 * b[n*ldb + k]; b_mn = 1: (n,k) at b[k*ldb + n]).  A and B are bf16; the
 * product accumulates in fp32.  `bias` (fp32 [N], may be NULL) is added to
 * every row.  With GPT_GEMM_OUT_F32 and accumulate != 0 the product is added
 * to the existing contents of `out`.  bn selects the tile width (128 or 256).
 * Any M, N, K >= 1 is accepted; ragged edges are handled in the kernel. */
GPT_API int gpt_op_gemm(int epilogue, int bn, const void* a, long long lda, int a_mn, const void* b,
                        long long ldb, int b_mn, int M, int N, int K, void* out, long long ldo,
                        const float* bias, int accumulate, void* stream);

/* 8-bit cast with a dynamic per-tensor scale ("Train your own ChatGPT", read
 * the source fp8.py: each tensor is rescaled before the cast, scale =
 * FP8_MAX / max(|tensor|); e4m3 for activations and weights, e5m2 for
 * gradients):
 *   amax = max |x|;  s = FP8_MAX / amax (1 when amax == 0);  out = cast(x s)
 *   inv_scale = 1 / s
 * with FP8_MAX = 448 (fmt 0, e4m3) or 57344 (fmt 1, e5m2) and a cast that
 * rounds to nearest (ties to even) and saturates at FP8_MAX.
 *   x          n values, bf16 (x_fp32 == 0) or fp32 (x_fp32 != 0)
 *   out        n bytes (8-bit floats); amax, inv_scale: fp32 [1], device
 * n >= 1. */
GPT_API int gpt_op_fp8_quantize(const void* x, int x_fp32, long long n, int fmt, void* out, float* amax,
                                float* inv_scale, void* stream);

/* The product of two 8-bit tensors with their inverse scales folded back in
 * (same page: the matmul runs on the 8-bit values, as torch._scaled_mm does):
 *   out[M,N] = (A[M,K] B[N,K]^T) * inv_a * inv_b   (+ bias, or += with accumulate)
 * on the tensor cores (tcgen05 kind::f8f6f4, fp32 accumulation).  A and B are
 * K-major 8-bit floats of formats fmt_a, fmt_b (0 e4m3, 1 e5m2; the two may
 * differ) with row pitches lda, ldb in elements, multiples of 16; inv_a and
 * inv_b are device fp32 scalars (gpt_op_fp8_quantize's inv_scale).  The
 * epilogue, bias, accumulate, bn and out are as for gpt_op_gemm. */
GPT_API int gpt_op_gemm_fp8(int epilogue, int bn, const void* a, long long lda, int fmt_a, const void* b,
                            long long ldb, int fmt_b, int M, int N, int K, const float* inv_a, const float* inv_b,
                            void* out, long long ldo, const float* bias, int accumulate, void* stream);

/* Causal self-attention of one layer with RoPE and QK-norm, forward
 * ("nanoGPT" wiki page, CausalSelfAttention: q, k, v split from one fused
 * projection, reshaped to (B, n_head, T, head_dim), causal mask;
 * "nanochat-d20-chat" card, Architecture: RoPE + QK-norm; "Train your own
 * ChatGPT", read the source gpt.py: per-layer (left, right) windows).
 *
 *   window   -1: query i sees keys 0 .. i; >= 0: only keys i - window .. i
 *            (a sliding-window layer; the right window is 0, causal)
 *   qkv      in  bf16 [B*T, 3*H*hd]  raw q|k|v rows (token-major; head h of q
 *                 at columns h*hd .. h*hd+hd-1, k after all q heads, v after k)
 *   qkv_norm out bf16 [B*T, 3*H*hd]  q, k after RoPE (if rope) and per-head
 *                 RMSNorm (if qk_norm); v copied
 *   rstd_q, rstd_k out fp32 [B*T, H]  per-head 1/rms of q and k (qk_norm only;
 *                 may be NULL otherwise)
 *   rope_cs  out fp32 [T, hd/2, 2]   (cos, sin) of t * base^(-2i/hd) (rope
 *                 only; may be NULL otherwise); kept for the backward
 *   o        out bf16 [B*T, H*hd]    softmax(q k^T / sqrt(hd) + mask) v
 *   lse      out fp32 [B, H, T]      natural-log logsumexp of each score row
 * hd must be 64 or 128.  RoPE rotates the pairs (i, i + hd/2). */
GPT_API int gpt_op_attention_fwd(const void* qkv, int B, int T, int H, int hd, int rope, int qk_norm, int window,
                                 float rope_base, float eps, void* qkv_norm, float* rstd_q, float* rstd_k,
                                 float* rope_cs, void* o, float* lse, void* stream);

/* Backward of gpt_op_attention_fwd: given dout = dL/do (bf16 [B*T, H*hd]) and
 * the forward's outputs, writes dqkv = dL/dqkv (bf16 [B*T, 3*H*hd], the
 * gradient w.r.t. the RAW projection output, through QK-norm and RoPE), with
 * the forward's window.  delta is caller scratch, fp32 [B, H, T].
 * Deterministic. */
GPT_API int gpt_op_attention_bwd(const void* qkv_norm, const float* rstd_q, const float* rstd_k,
                                 const float* rope_cs, const void* o, const float* lse, const void* dout, int B,
                                 int T, int H, int hd, int rope, int qk_norm, int window, float* delta, void* dqkv,
                                 void* stream);

/* Fused lm_head + cross-entropy, forward ("nanoGPT" wiki page, model.py
 * walkthrough: final norm -> lm_head linear to vocab logits; next-token loss
 * l_m = logsumexp(z_m) - z_m[y_m]).  z = x W^T is produced tile by tile on
 * the tensor cores and folded into a per-row online logsumexp over each
 * 256-wide vocab tile; the M x V logits are never written.
 *   x        bf16 [M, D] (normalised final hidden states), w bf16 [V, D]
 *   targets  int32 [M]; ell, lse out fp32 [M] (loss and logsumexp per row); a
 *            target outside [0, V) gives its row a NaN loss and is reported
 *            by gpt_sync_status (GPT_ERR_INVALID_ARG)
 *   scratch  caller memory of gpt_op_lmhead_ce_scratch_bytes(M, V) bytes
 *            (per-row partials of each vocab tile), 256-byte aligned
 * D must be a multiple of 8. */
GPT_API size_t gpt_op_lmhead_ce_scratch_bytes(int M, int V);
GPT_API int gpt_op_lmhead_ce_fwd(const void* x, const void* w, const int32_t* targets, int M, int D, int V,
                                 float* ell, float* lse, void* scratch, void* stream);

/* The same lm_head + cross-entropy forward for callers that cannot allocate
 * device memory (the pages have no counterpart: this is a deployment
 * variant).  A serving or training loop whose device memory is all reserved
 * up front by its own pool cannot hand out scratch, and a cudaMalloc there
 * would fail or fragment the pool (and may synchronise the device mid-step).
 * This entry point takes no scratch argument: it uses a fixed file-scope
 * device array of gpt_op_lmhead_ce_noalloc_max_scratch_bytes() bytes
 * (16 MiB) that every GPU loading the library holds until exit, and it calls
 * no allocator.  It needs gpt_op_lmhead_ce_scratch_bytes(M, V) <= that size
 * (else GPT_ERR_INVALID_ARG, nothing launched).  The first call on a device
 * looks up the array's device address (cudaGetSymbolAddress) and caches it
 * once the lookup has succeeded (a failed lookup is tried again by the next
 * call); make that first call before any stream capture.  All calls share the one
 * array, which keeps the last call's contents (the call clears what must
 * start at zero); calls that overlap on the GPU race on it, so order them on
 * one stream or with events.  Arguments as gpt_op_lmhead_ce_fwd. */
GPT_API size_t gpt_op_lmhead_ce_noalloc_max_scratch_bytes(void);
GPT_API int gpt_op_lmhead_ce_fwd_noalloc(const void* x, const void* w, const int32_t* targets, int M, int D,
                                         int V, float* ell, float* lse, void* stream);

/* Failure-detection probe (no counterpart on the pages): launches one kernel
 * that waits on an mbarrier nothing ever arrives at, through the same bounded
 * wait every pipeline kernel uses.  After timeout_ns (at most 10 s) the kernel
 * records a timeout in the device status word and returns, so the next
 * gpt_sync_status() reports GPT_ERR_DEVICE_TIMEOUT and the context stays
 * usable.  Nothing faults, traps or hangs. */
GPT_API int gpt_op_wait_probe(unsigned long long timeout_ns, void* stream);

/* The attention softmax's exponential and an FMA-pipe alternative to it, for
 * testing them against their error bounds (no counterpart on the pages):
 * out[i] = 2^x[i] for the n (even) fp32 values at x, with poly = 0 the MUFU
 * approximation the attention kernels use (ex2.approx.ftz) and poly = 1 the
 * FMA-pipe polynomial (range reduction to
 * [-1/2, 1/2], degree-4 minimax polynomial, relative error below 3e-6 for
 * -125 <= x <= 127; x below -125, -inf included, gives a value in
 * [0, 2^-125]).  x and out: device, 8-byte aligned, fp32.  Invalid n or
 * alignment: GPT_ERR_INVALID_ARG. */
GPT_API int gpt_op_exp2(const float* x, long long n, int poly, float* out, void* stream);

/* Measurement hooks (no counterpart on the pages).
 * gpt_launch_count: kernels this process has launched through the library.
 * gpt_profile_start: from now on, bracket every launch with CUDA events on its
 *   stream (adds a few microseconds per launch).
 * gpt_profile_stop: synchronise those events and add up, per kernel family
 *   k < max_kinds, the elapsed milliseconds, launches, algorithmic FLOPs and
 *   algorithmic bytes (host arrays of max_kinds entries, any may be NULL).
 *   Returns the number of families, or GPT_ERR_CUDA (with gpt_last_error) if
 *   an event could not be read.  Families, in order: gemm, attn_fwd,
 *   attn_bwd_dkv, attn_bwd_dq, norm_fwd, norm_bwd, embed_fwd, embed_bwd,
 *   cast, ce_combine, loss, qk, delta, colsum, misc, then the model's GEMMs by
 *   role: gemm_qkv, gemm_o, gemm_up, gemm_down, gemm_lm_fwd, gemm_lm_bwd,
 *   gemm_dgrad, gemm_wgrad (op-level GEMMs count as gemm), then optim (the
 *   optimizers' elementwise steps) and gemm_muon (the Muon step's products). */
GPT_API unsigned long long gpt_launch_count(void);
GPT_API int gpt_profile_start(void);
GPT_API int gpt_profile_stop(int max_kinds, double* ms, long long* count, double* flops, double* bytes);

/* The optimizer step of gpt_adamw_step on any fp32 buffer of n elements, with
 * an explicit weight-decay table in HOST memory: run r covers elements
 * [run_start[r], run_start[r + 1]) (the last run up to n) and is decayed when
 * run_decay[r] != 0.  run_start[0] == 0 and the starts increase strictly and
 * stay below n.  scratch: gpt_op_adamw_scratch_bytes() bytes of device memory,
 * 8-byte aligned.  n == 0 writes a zero grad_norm and launches nothing else. */
GPT_API size_t gpt_op_adamw_scratch_bytes(void);
GPT_API int gpt_op_adamw(float* params, const float* grads, float* m, float* v, int64_t n,
                         const int64_t* run_start, const uint8_t* run_decay, int32_t n_runs, int64_t step,
                         const gpt_adamw* h, void* scratch, double* grad_norm, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GPT_OPS_H */
