"""Failure detection on the GPU without a fault: a kernel's bounded wait runs
out, the kernel gives up cleanly and the host reads the status.

The context's wait limit is shortened to 1 ns, so the first wait of the
LM-head kernel that does not complete at once runs out (its epilogue waits
for a whole vocabulary tile's mainloop): every CTA that gives up records
FDL_ETIMEOUT, waits with the fixed 2 s limit for the TMA loads and the MMA
commits it has already started, frees its TMEM and returns. The host sees
FDL_ETIMEOUT from fdl_get_device_status, destroys the context, and a new
context on the same device computes the same call correctly."""
import numpy as np
import pytest
import torch

import oracle as O
from block_kv_cache_b200 import synth

pytestmark = pytest.mark.gpu

CONF_TOL = 1e-5


def test_wait_runs_out_reports_timeout_and_a_new_context_works():
    from block_kv_cache_b200 import fdllm
    c = synth.lmhead_case(rows=32, hidden=4096, vocab=32768, dtype="bf16", seed=5, w_seed=5,
                          mask_id=32767)
    h = torch.from_numpy(c.h).to(torch.bfloat16).cuda()
    w = torch.from_numpy(c.w).to(torch.bfloat16).cuda()
    bt = torch.from_numpy(c.bias_tok).cuda()
    bv = torch.from_numpy(c.bias_val).cuda()

    ctx = fdllm.Context(0)
    with pytest.raises(fdllm.FdlError) as e:
        ctx.set_wait_timeout(0)                       # outside [1, 60e9]
    assert e.value.code == fdllm.FDL_EINVAL
    ctx.set_wait_timeout(1)
    ctx.lmhead_confidence(h, w, bt, bv)
    with pytest.raises(fdllm.FdlError) as e:
        ctx.device_status()
    assert e.value.code == fdllm.FDL_ETIMEOUT
    ctx.close()

    torch.cuda.synchronize()                          # the device is still usable
    ctx = fdllm.Context(0)
    for _ in range(2):
        conf, tok = ctx.lmhead_confidence(h, w, bt, bv)
        ctx.device_status()
        ref = O.lmhead_confidence(c.h, c.w, c.bias_tok, c.bias_val)
        assert np.abs(conf.cpu().numpy() - ref.conf).max() <= CONF_TOL
        sure = ref.gap > 1e-3
        assert np.array_equal(tok.cpu().numpy()[sure], ref.tok[sure])
    ctx.close()
