"""Failure detection on the GPU without a GPU fault.

Every wait inside the kernels is bounded in wall time; when one runs out the
kernel records the event in a device status word and returns.  The probe
entry point waits on a barrier that nothing ever arrives at, so the bounded
wait must run out, the host must read GPT_ERR_DEVICE_TIMEOUT, and the context
must stay usable.  An out-of-range token id is reported the same way."""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def test_bounded_wait_times_out_and_context_survives():
    import decoder_only_gpt_tcgen05_b200 as g
    from decoder_only_gpt_tcgen05_b200._lib import GptError
    g.model.sync_status(DEV)
    g._lib.call("gpt_op_wait_probe", 20_000_000, torch.cuda.current_stream(DEV).cuda_stream)
    with pytest.raises(GptError) as e:
        g.model.sync_status(DEV)
    assert e.value.code == 5
    assert "bounded wait" in str(e.value)
    # the status word is cleared and the context still runs kernels
    g.model.sync_status(DEV)
    a = torch.ones(256, 128, dtype=torch.bfloat16, device=DEV)
    out = torch.empty(256, 256, dtype=torch.float32, device=DEV)
    g.ops.gemm(a, a, out)
    g.model.sync_status(DEV)
    assert torch.all(out == 128.0)


def test_out_of_range_token_is_reported():
    import decoder_only_gpt_tcgen05_b200 as g
    from decoder_only_gpt_tcgen05_b200._lib import GptError
    cfg = g.preset("tiny")
    m = g.GPT(cfg, 1, 16, device=DEV)
    idx, tgt = synth.next_token_batch(1, 16, cfg.vocab_size, dist="uniform", seed=1)
    idx[0, 3] = cfg.vocab_size + 5
    m.forward_loss(torch.from_numpy(idx).to(DEV), torch.from_numpy(tgt).to(DEV))
    with pytest.raises(GptError) as e:
        g.model.sync_status(DEV)
    assert e.value.code == 1 and "token id" in str(e.value)
    g.model.sync_status(DEV)
