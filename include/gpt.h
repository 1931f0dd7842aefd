/* B200 (sm_100a) library for the training hot path of a decoder-only GPT:
 * forward and backward of next-token cross-entropy, plus the bits-per-byte
 * evaluation.
 *
 * The model is the GPT-2 / nanoGPT block ("nanoGPT - Karpathy's minimal GPT
 * pretraining repo", How it works, model.py walkthrough: token (+ learned
 * position) embedding, n_layer pre-norm blocks x += attn(norm(x)),
 * x += mlp(norm(x)), final norm, lm_head) with the nanochat refinements of
 * the d20 card ("nanochat-d20-chat", Architecture: RoPE + QK-norm, untied
 * token embedding and lm_head, parameter-free RMSNorm, ReLU^2 MLP).  The
 * metric is bits per byte ("Train your own ChatGPT", read the source
 * loss_eval.py): summed nats over ln 2 times summed target-token bytes.
 *
 * Conventions:
 *   - every pointer argument is DEVICE memory owned by the caller unless a
 *     comment says otherwise; the library allocates nothing and frees nothing;
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream); calls enqueue work and return without synchronising;
 *   - argument errors are found on the host before any launch; the return
 *     value is a gpt_status and gpt_last_error() has the message.
 */
#ifndef GPT_H
#define GPT_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GPT_API __attribute__((visibility("default")))
#else
#define GPT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gpt_status {
  GPT_OK = 0,
  GPT_ERR_INVALID_ARG = 1,          /* null pointer, bad shape, T > block_size, ...            */
  GPT_ERR_UNSUPPORTED = 2,          /* a shape the kernels do not handle (see gpt_config)      */
  GPT_ERR_WORKSPACE_TOO_SMALL = 3,  /* workspace smaller than gpt_workspace_size()             */
  GPT_ERR_CUDA = 4,                 /* a CUDA runtime call or launch failed                    */
  GPT_ERR_DEVICE_TIMEOUT = 5        /* a kernel gave up a bounded wait (see gpt_sync_status)   */
} gpt_status;

/* Model shape (GPTConfig of the "nanoGPT" wiki page, model.py walkthrough,
 * plus the nanochat switches of the d20 card).
 *
 * Supported shapes (else GPT_ERR_UNSUPPORTED): n_embd a multiple of 16 and at
 * most 4096; n_embd divisible by n_head with an even head dim of at most 128;
 * with RoPE or QK-norm the head dim must be 64 or 128. */
typedef struct gpt_config {
  int32_t n_layer;          /* number of blocks                                         */
  int32_t n_embd;           /* width D                                                  */
  int32_t n_head;           /* heads H; head dim hd = D / H                             */
  int32_t block_size;       /* maximum context (rows of the learned position table)     */
  int32_t vocab_size;       /* V                                                        */
  int32_t norm;             /* 0: parameter-free RMSNorm, 1: LayerNorm (gain, + bias if linear_bias) */
  int32_t pos;              /* 0: learned absolute position embedding, 1: RoPE          */
  int32_t act;              /* MLP activation: 0 GELU (erf form), 1 ReLU^2              */
  int32_t tie_embed;        /* 1: lm_head shares the token embedding ("weight tying")   */
  int32_t qk_norm;          /* 1: per-head RMSNorm of q and k after RoPE                */
  int32_t linear_bias;      /* 1: biases on every Linear and LayerNorm (GPT-2 shape)    */
  int32_t scale_resid_init; /* 1: init std of attn/MLP output projections 0.02/sqrt(2 n_layer) */
  float rope_base;          /* RoPE base (10000)                                        */
  float norm_eps;           /* epsilon of every norm (1e-5)                             */
  /* Sliding-window layers ("Train your own ChatGPT", read the source gpt.py:
   * _compute_window_sizes() expands a pattern such as "SSSL" into per-layer
   * (left, right) windows).  Layer l is a short-window layer when
   * window_short > 0 and bit (l mod window_period) of window_pattern is set
   * ("SSSL" = 0x7 with period 4); its query i then sees only the keys
   * i - window_short .. i.  Every other layer sees all earlier keys.
   * window_short = 0 turns windows off; window_period is 1..32. */
  int32_t window_short;
  int32_t window_pattern;
  int32_t window_period;
  /* 1: the forward's block projections (q|k|v, attention output, MLP up and
   * down) run on 8-bit e4m3 operands, each activation and weight cast with
   * its own dynamic scale FP8_MAX / max|tensor| ("Train your own ChatGPT",
   * read the source fp8.py); the lm_head and the backward stay bf16.  0: bf16. */
  int32_t fp8;
} gpt_config;

/* Parameters: ONE flat fp32 buffer, tensors back to back in this order:
 *   wte [V, D]; wpe [block_size, D] (pos == 0); then per layer l:
 *   ln1_g [D], ln1_b [D] (LayerNorm; _b only with linear_bias),
 *   w_qkv [3D, D], b_qkv [3D], w_o [D, D], b_o [D], ln2_g, ln2_b,
 *   w_up [4D, D], b_up [4D], w_down [D, 4D], b_down [D]   (b_* only with linear_bias);
 *   then lnf_g, lnf_b (LayerNorm); lm_head [V, D] (untied only).
 * Linear weights are [out, in] row-major (y = x W^T + b).  Gradients use the
 * same layout.  Every tensor starts at a multiple of 16 elements. */
GPT_API int gpt_param_count(const gpt_config* cfg, int64_t* n_out);
GPT_API int gpt_param_tensor_count(const gpt_config* cfg, int32_t* n_out);
/* Name (NUL-terminated, truncated to name_len), element offset and shape of
 * tensor i (cols = 1 for vectors). */
GPT_API int gpt_param_tensor(const gpt_config* cfg, int32_t i, char* name, int32_t name_len, int64_t* offset,
                             int64_t* rows, int64_t* cols);

/* Bytes of device workspace that gpt_forward_loss / gpt_backward /
 * gpt_eval_bpb need for a batch of B sequences of T tokens.  The workspace
 * holds the bf16 weight copies, the activations the backward reuses, and the
 * scratch of every kernel.  It must be 256-byte aligned. */
GPT_API int gpt_workspace_size(const gpt_config* cfg, int32_t B, int32_t T, size_t* bytes);

/* Initial weights into `params` (fp32 [gpt_param_count]): every matrix and
 * embedding N(0, 0.02^2) (0.02/sqrt(2 n_layer) for w_o and w_down when
 * scale_resid_init), biases 0, LayerNorm gains 1.  Element i draws
 * SplitMix64 outputs 2i and 2i+1 of the stream seeded with `seed` and turns
 * them into one normal by Box-Muller, so the result does not depend on the
 * launch configuration. */
GPT_API int gpt_init_weights(const gpt_config* cfg, uint64_t seed, float* params, void* stream);

/* Forward pass and mean next-token cross-entropy of one batch.
 *   params   fp32 [gpt_param_count]
 *   idx      int32 [B, T] input token ids in [0, V)
 *   targets  int32 [B, T] next-token ids (the inputs shifted by one)
 *   loss     fp32 [1] out: mean over the B*T targets of logsumexp(z) - z[y]
 * The logits are never written to memory: the lm_head product streams vocab
 * tiles through an online logsumexp.  The activations the backward needs
 * stay in `workspace` (copies of idx and targets included).  T <= block_size
 * when pos == 0.  An input id or a target outside [0, V) is reported by
 * gpt_sync_status (a bad target also makes that token's loss NaN). */
GPT_API int gpt_forward_loss(const gpt_config* cfg, const float* params, const int32_t* idx, const int32_t* targets,
                             int32_t B, int32_t T, void* workspace, size_t workspace_bytes, float* loss,
                             void* stream);

/* Gradient of that mean loss w.r.t. every parameter, into `grads` (fp32,
 * parameter layout): written when accumulate == 0, added when != 0.
 * Requires that the last call on this workspace was gpt_forward_loss with the
 * same cfg, params, B and T (the parameters must not have changed since).
 * Deterministic: the same inputs give bitwise the same gradients. */
GPT_API int gpt_backward(const gpt_config* cfg, const float* params, int32_t B, int32_t T, void* workspace,
                         size_t workspace_bytes, float* grads, int32_t accumulate, void* stream);

/* Gradient buckets for data-parallel training ("nanoGPT" wiki page, DDP:
 * gradients averaged over ranks; "Train your own ChatGPT", read the source
 * optim.py: DistMuonAdamW launches every gradient reduce_scatter at once so
 * that communication overlaps compute).  Bucket k is the flat range
 * [begin[k], end[k]) of the gradient buffer; buckets are listed in the order
 * the backward completes them (final norm and an untied lm_head; the layers
 * in pairs from the top; the embeddings last), they do not overlap and
 * together cover every parameter.  *n_out is the count; begin and end (host
 * arrays of max_buckets entries) may be NULL to query only the count. */
GPT_API int gpt_grad_buckets(const gpt_config* cfg, int32_t max_buckets, int32_t* n_out, int64_t* begin,
                             int64_t* end);

/* gpt_backward that also records events[k] (a cudaEvent_t passed as void*,
 * created by the caller) on `stream` as soon as bucket k of gpt_grad_buckets
 * holds its final gradient, so that the caller can start reducing it on
 * another stream while the backward goes on.  n_events must equal the bucket
 * count.  The first bucket may be empty; its event is recorded all the same. */
GPT_API int gpt_backward_bucketed(const gpt_config* cfg, const float* params, int32_t B, int32_t T, void* workspace,
                                  size_t workspace_bytes, float* grads, int32_t accumulate, void* const* events,
                                  int32_t n_events, void* stream);

/* Bits per byte of one batch ("Train your own ChatGPT", read the source
 * loss_eval.py): sum_nats = sum of the per-token loss over targets whose
 * byte length token_bytes[y] > 0; sum_bytes = sum of token_bytes[y] over all
 * targets; bpb = sum_nats / (ln 2 * sum_bytes) (NaN when sum_bytes == 0).
 *   token_bytes int32 [V]; sum_nats fp64 [1]; sum_bytes int64 [1]; bpb fp32 [1]
 *   (any of the three outputs may be NULL).
 * The sums are reduced in a fixed order (bitwise reproducible). */
GPT_API int gpt_eval_bpb(const gpt_config* cfg, const float* params, const int32_t* idx, const int32_t* targets,
                         const int32_t* token_bytes, int32_t B, int32_t T, void* workspace, size_t workspace_bytes,
                         double* sum_nats, int64_t* sum_bytes, float* bpb, void* stream);

/* Hyperparameters of one optimizer step ("nanoGPT - Karpathy's minimal GPT
 * pretraining repo", How it works: configure_optimizers builds AdamW; train.py
 * clips the gradient with clip_grad_norm_ and divides the loss by the number
 * of accumulated micro-steps). */
typedef struct gpt_adamw {
  float lr;            /* learning rate of this step (see gpt_lr_schedule), >= 0                */
  float beta1, beta2;  /* decay rates of the first and second moments, in [0, 1)                */
  float eps;           /* > 0, added to the root of the bias-corrected second moment            */
  float weight_decay;  /* >= 0: p <- p (1 - lr weight_decay) on decayed tensors; lr wd <= 1      */
  float grad_scale;    /* > 0: multiplies the gradient first (1 / micro-steps, 1 / ranks)       */
  float grad_clip;     /* >= 0: clip the scaled gradient to this global L2 norm; 0 = no clipping */
} gpt_adamw;

/* Bytes of device scratch (8-byte aligned) that gpt_adamw_step needs: the
 * partial sums of the gradient-norm reduction.  Independent of the model. */
GPT_API int gpt_adamw_scratch_size(size_t* bytes);

/* One optimizer step of nanoGPT's training loop on the flat parameter buffer:
 * global L2 norm of grad_scale * grads, clip_grad_norm_'s factor
 * min(1, grad_clip / (norm + 1e-6)), then AdamW with decoupled weight decay:
 *   g = grads * grad_scale * factor
 *   m <- beta1 m + (1 - beta1) g;   v <- beta2 v + (1 - beta2) g^2
 *   p <- p (1 - lr weight_decay)    (2-D tensors only: wte, wpe, lm_head and
 *                                    the Linear weights; biases and LayerNorm
 *                                    gains are not decayed)
 *   p <- p - lr / (1 - beta1^step) * m / (sqrt(v) / sqrt(1 - beta2^step) + eps)
 *   params    fp32 [gpt_param_count], updated in place
 *   grads     fp32 [gpt_param_count], read only
 *   m, v      fp32 [gpt_param_count]: the moments (zero before step 1), updated
 *   step      1-based step number
 *   scratch   gpt_adamw_scratch_size bytes
 *   grad_norm fp64 [1] out: the norm before clipping (may be NULL)
 * params, grads, m and v are distinct, 16-byte aligned buffers.  The norm is
 * reduced over a fixed partition, so results are bitwise reproducible. */
GPT_API int gpt_adamw_step(const gpt_config* cfg, float* params, const float* grads, float* m, float* v,
                           int64_t step, const gpt_adamw* h, void* scratch, double* grad_norm, void* stream);

/* Learning rate at iteration `it` (host arithmetic, nothing launched): linear
 * warmup from 0 at it = 0 to learning_rate at it = warmup_iters, then cosine
 * decay, lr = min_lr + 0.5 (1 + cos(pi r)) (learning_rate - min_lr) with
 * r = (it - warmup_iters) / (lr_decay_iters - warmup_iters), and min_lr after
 * lr_decay_iters ("nanoGPT" wiki page, train.py: LR schedule).  Needs
 * 0 <= warmup_iters <= lr_decay_iters and it >= 0. */
GPT_API int gpt_lr_schedule(int64_t it, int64_t warmup_iters, int64_t lr_decay_iters, double learning_rate,
                            double min_lr, double* lr_out);

/* Per-token results of the last gpt_forward_loss or gpt_eval_bpb on this
 * workspace (same cfg, B and T): ell fp32 [B*T], the loss logsumexp(z) - z[y]
 * of each target (the next-token cross-entropy of the "nanoGPT" wiki page,
 * model.py walkthrough, before its mean), and lse fp32 [B*T], the logsumexp
 * of its logits row, in token order.  Device-to-device copies out of the workspace, enqueued on
 * `stream`; either output may be NULL. */
GPT_API int gpt_token_losses(const gpt_config* cfg, int32_t B, int32_t T, const void* workspace,
                             size_t workspace_bytes, float* ell, float* lse, void* stream);

/* Debug view of the logits of the last forward on this workspace (the
 * lm_head output of the "nanoGPT" wiki page, model.py walkthrough), fp32
 * [B*T, V] row-major, written to the caller's buffer (B*T*V*4 bytes; meant
 * for small batches).  The training and evaluation calls never form this
 * matrix: their lm_head product folds each vocab tile into the cross-entropy
 * in registers.  This call runs the same product (the same kernel on the same
 * operands: the saved final-norm output and the bf16 weight copy) and stores
 * its fp32 tiles instead, so tests can compare logits with a reference. */
GPT_API int gpt_debug_logits(const gpt_config* cfg, int32_t B, int32_t T, void* workspace, size_t workspace_bytes,
                             float* logits, void* stream);

/* Hyperparameters of the split optimizer step ("Train your own ChatGPT", read
 * the source optim.py -- Muon + AdamW: the transformer's 2-D weight matrices go
 * to Muon, which orthogonalizes each update, making all its singular values
 * equal; embeddings, the lm_head and the other tensors go to AdamW). */
typedef struct gpt_muon {
  float lr;            /* Muon learning rate, >= 0                                             */
  float momentum;      /* mu in [0, 1): buf <- mu buf + (1 - mu) g                             */
  int32_t nesterov;    /* 1: orthogonalize (1 - mu) g + mu buf; 0: buf                         */
  int32_t ns_steps;    /* Newton-Schulz steps, 1..32 (5)                                       */
  float adam_lr;       /* AdamW on every other tensor: learning rate                           */
  float beta1, beta2, eps;
  float weight_decay;  /* AdamW decay, on the 2-D tensors among them (embeddings, lm_head)     */
} gpt_muon;

/* Bytes of device scratch (256-byte aligned) that gpt_muon_step needs. */
GPT_API int gpt_muon_scratch_size(const gpt_config* cfg, size_t* bytes);

/* One step of the split optimizer on the flat parameter buffer.  Every block
 * matrix (w_qkv, w_o, w_up, w_down of every layer) takes a Muon step, read as
 * its authors published it (K. Jordan et al., 2024): momentum
 * buf <- mu buf + (1 - mu) g; u = (1 - mu) g + mu buf (Nesterov) or buf;
 * X = u / (||u||_F + 1e-7) on the wide orientation; ns_steps of the quintic
 * Newton-Schulz iteration X <- a X + (b A + c A^2) X, A = X X^T,
 * (a, b, c) = (3.4445, -4.7750, 2.0315), in bf16 on the tensor cores;
 * p <- p - lr sqrt(max(1, rows / cols)) X.  Every other tensor takes
 * gpt_adamw_step's AdamW (no clipping, grad_scale 1) with adam_lr.
 *   params  fp32 [gpt_param_count], updated in place
 *   grads   fp32 [gpt_param_count], read only
 *   mom     fp32 [gpt_param_count]: the Muon momentum of the block matrices and
 *           the AdamW first moment of the rest (zero before step 1), updated
 *   v       fp32 [gpt_param_count]: the AdamW second moment (unused entries of
 *           the block matrices stay untouched), updated
 *   step    1-based step number (AdamW bias correction)
 *   scratch gpt_muon_scratch_size bytes
 * All buffers are distinct and 16-byte aligned. */
GPT_API int gpt_muon_step(const gpt_config* cfg, float* params, const float* grads, float* mom, float* v,
                          int64_t step, const gpt_muon* h, void* scratch, void* stream);

/* Synchronises `stream`, then reads and clears the device status word that
 * kernels set when a bounded wait runs out (GPT_ERR_DEVICE_TIMEOUT) or an
 * input id is out of range (GPT_ERR_INVALID_ARG). */
GPT_API int gpt_sync_status(void* stream);

/* Wall-time limit of every bounded wait inside the kernels, in nanoseconds
 * (default 2e9).  For tests of the timeout path. */
GPT_API int gpt_set_wait_timeout_ns(uint64_t ns);

/* Last error message of the calling thread ("" after success). */
GPT_API const char* gpt_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* GPT_H */
