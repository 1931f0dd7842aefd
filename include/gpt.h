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

/* Last error message of the calling thread ("" after success). */
GPT_API const char* gpt_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* GPT_H */
