/* A plain C99 client of the library's host-side calls: it compiles against
 * include/gpt.h and include/gpt_ops.h with warnings as errors and links the
 * shared library.  Nothing here launches work or touches a GPU: parameter
 * layout, workspace sizing, argument checks and the learning-rate schedule
 * are all answered on the host. */
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "gpt_ops.h"

static int fails = 0;
#define CHECK(cond)                                                   \
  do {                                                                \
    if (!(cond)) {                                                    \
      printf("FAIL line %d: %s (%s)\n", __LINE__, #cond, gpt_last_error()); \
      ++fails;                                                        \
    }                                                                 \
  } while (0)

int main(void) {
  /* nanochat d20: RMSNorm, RoPE, ReLU^2, untied, QK-norm, no biases */
  const gpt_config d20 = {20, 1280, 10, 2048, 32768, 0, 1, 1, 0, 1, 0, 0, 10000.f, 1e-5f, 0, 0, 1, 0};
  /* GPT-2 124M: LayerNorm + biases, learned positions, GELU, tied, scaled residual init */
  const gpt_config gpt2 = {12, 768, 12, 1024, 50304, 1, 0, 0, 1, 0, 1, 1, 10000.f, 1e-5f, 0, 0, 1, 0};
  int64_t n = 0, off = -1, rows = 0, cols = 0;
  int32_t nt = 0;
  char name[32];
  size_t bytes = 0, bytes2 = 0;
  double lr = -1.0;
  gpt_config bad = d20;
  const gpt_adamw h = {1e-3f, 0.9f, 0.95f, 1e-8f, 0.1f, 1.f, 1.f};

  CHECK(gpt_param_count(&d20, &n) == GPT_OK && n == 477102080LL);   /* 12 L D^2 + 2 V D */
  CHECK(gpt_param_count(&gpt2, &n) == GPT_OK && n == 124475904LL);
  CHECK(gpt_param_tensor_count(&gpt2, &nt) == GPT_OK && nt == 2 + 12 * 12 + 2);
  CHECK(gpt_param_tensor(&gpt2, 0, name, (int32_t)sizeof name, &off, &rows, &cols) == GPT_OK);
  CHECK(strcmp(name, "wte") == 0 && off == 0 && rows == 50304 && cols == 768);
  CHECK(gpt_param_tensor(&gpt2, nt - 1, name, (int32_t)sizeof name, &off, &rows, &cols) == GPT_OK);
  CHECK(strcmp(name, "lnf_b") == 0 && off + rows * cols == 124475904LL && cols == 1);
  CHECK(gpt_param_tensor(&gpt2, nt, name, (int32_t)sizeof name, &off, &rows, &cols) == GPT_ERR_INVALID_ARG);

  CHECK(gpt_workspace_size(&d20, 16, 2048, &bytes) == GPT_OK && bytes > 0 && bytes % 256 == 0);
  CHECK(gpt_workspace_size(&d20, 32, 2048, &bytes2) == GPT_OK && bytes2 > bytes);
  CHECK(gpt_workspace_size(&gpt2, 1, 2048, &bytes) == GPT_ERR_INVALID_ARG);   /* T > block_size */
  bad.n_embd = 1000;
  CHECK(gpt_param_count(&bad, &n) == GPT_ERR_UNSUPPORTED && strlen(gpt_last_error()) > 0);
  CHECK(gpt_param_count(NULL, &n) == GPT_ERR_INVALID_ARG);

  CHECK(gpt_lr_schedule(1000, 2000, 600000, 6e-4, 6e-5, &lr) == GPT_OK && fabs(lr - 3e-4) < 1e-18);
  CHECK(gpt_lr_schedule(600001, 2000, 600000, 6e-4, 6e-5, &lr) == GPT_OK && lr == 6e-5);
  CHECK(gpt_lr_schedule(5, 10, 3, 6e-4, 6e-5, &lr) == GPT_ERR_INVALID_ARG);

  CHECK(gpt_adamw_scratch_size(&bytes) == GPT_OK && bytes == gpt_op_adamw_scratch_bytes());
  CHECK(gpt_adamw_step(&d20, NULL, NULL, NULL, NULL, 0, &h, NULL, NULL, NULL) == GPT_ERR_INVALID_ARG);
  CHECK(gpt_forward_loss(&d20, NULL, NULL, NULL, 16, 2048, NULL, 0, NULL, NULL) == GPT_ERR_INVALID_ARG);
  CHECK(gpt_op_lmhead_ce_scratch_bytes(4096, 32768) > 0);

  printf(fails ? "FAILED (%d)\n" : "OK\n", fails);
  return fails != 0;
}
