"""fdl_lmhead_confidence_noalloc: the LM-head confidence call for callers that
cannot supply scratch memory (C hosts owning only their inputs and outputs,
engines whose device memory is all held by their own pool). It must give the
workspace entry point's results, call after call, although every call reuses
the one scratch array built into the library. This file is named so that
pytest collects it last."""
import numpy as np
import pytest
import torch

from block_kv_cache_b200 import synth

pytestmark = pytest.mark.gpu

CONF_TOL = 1e-5


@pytest.fixture(scope="module")
def ctx():
    from block_kv_cache_b200 import fdllm
    c = fdllm.Context(0)
    yield c
    c.close()


def _case(dtype, rows, hidden, vocab, seed):
    c = synth.lmhead_case(rows=rows, hidden=hidden, vocab=vocab, dtype=dtype, seed=seed,
                          bias_hi=12.0)
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    return (torch.from_numpy(c.h).to(td).cuda(), torch.from_numpy(c.w).to(td).cuda(),
            torch.from_numpy(c.bias_tok).cuda(), torch.from_numpy(c.bias_val).cuda())


@pytest.mark.parametrize("dtype,rows,hidden,vocab", [
    ("bf16", 32, 4096, 126464),      # one block of the LLaDA-8B-shaped LM head
    ("bf16", 300, 512, 20000),
    ("f32", 40, 256, 1024),
])
def test_noalloc_matches_workspace_call_twice(ctx, dtype, rows, hidden, vocab):
    first = _case(dtype, rows, hidden, vocab, seed=1)
    second = _case(dtype, rows, hidden, vocab, seed=2)
    for h, w, bt, bv in (first, second):       # two calls in a row on the shared scratch
        ref_conf, ref_tok = ctx.lmhead_confidence(h, w, bt, bv)
        conf, tok = ctx.lmhead_confidence_noalloc(h, w, bt, bv)
        torch.cuda.synchronize()
        assert np.abs(conf.cpu().numpy() - ref_conf.cpu().numpy()).max() <= CONF_TOL
        assert np.array_equal(tok.cpu().numpy(), ref_tok.cpu().numpy())
    ctx.device_status()


def test_noalloc_rejects_shapes_beyond_its_scratch(ctx):
    from block_kv_cache_b200 import fdllm
    # 1024 rows x 988 tiles x 12 bytes > 8 MiB: refused before anything runs
    h = torch.zeros((1024, 64), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((126464, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fdllm.FdlError) as e:
        ctx.lmhead_confidence_noalloc(h, w)
    assert e.value.code == fdllm.FDL_EINVAL
    assert "scratch" in str(e.value)
