"""Named model shapes (oracle side).  Sizes follow the pages: the GPT-2 124M
GPTConfig defaults ("nanoGPT - Karpathy's minimal GPT pretraining repo",
model.py walkthrough), the nanochat d20 card ("nanochat-d20-chat",
Architecture), and the 27-token microGPT alphabet ("Train your own ChatGPT",
introduction).  d26 keeps the d20 block with width 64 * 26.

TEST INFRASTRUCTURE ONLY (see the package docstring)."""
from .gpt_oracle import (Config, NORM_RMS, NORM_LN, POS_LEARNED, POS_ROPE,
                         ACT_GELU, ACT_RELU2)

PRESETS = {
    "tiny": Config(n_layer=1, n_embd=16, n_head=4, block_size=16, vocab_size=27,
                   norm=NORM_RMS, pos=POS_LEARNED, act=ACT_GELU, tie_embed=1),
    "gpt2": Config(n_layer=12, n_embd=768, n_head=12, block_size=1024, vocab_size=50304,
                   norm=NORM_LN, pos=POS_LEARNED, act=ACT_GELU, tie_embed=1,
                   linear_bias=1, scale_resid_init=1),
    "d20": Config(n_layer=20, n_embd=1280, n_head=10, block_size=2048, vocab_size=32768,
                  norm=NORM_RMS, pos=POS_ROPE, act=ACT_RELU2, tie_embed=0, qk_norm=1),
    "d26": Config(n_layer=26, n_embd=1664, n_head=13, block_size=2048, vocab_size=32768,
                  norm=NORM_RMS, pos=POS_ROPE, act=ACT_RELU2, tie_embed=0, qk_norm=1),
}


def preset(name: str, **over) -> Config:
    import dataclasses
    return dataclasses.replace(PRESETS[name], **over)
