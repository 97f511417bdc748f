"""Parity of the CUDA path (through the C-ABI) with the CPU oracle.

Tolerances: attention max|gpu - ref| / max|ref| <= 1e-4 (f32) and 2e-2 (bf16);
confidences |gpu - ref| <= 1e-5; unmask decisions and token ids bit-exact
when the oracle decides on the GPU's confidences. Token ids from the LM head
are compared exactly where the oracle's top-2 logit gap exceeds 1e-3; where
it does not (several ids are within rounding of the max), the GPU's id must
be one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from block_kv_cache_b200 import synth

pytestmark = pytest.mark.gpu

ATT_TOL = {"f32": 1e-4, "bf16": 2e-2}
CONF_TOL = 1e-5
GAP = 1e-3


@pytest.fixture(scope="module")
def ctx():
    from block_kv_cache_b200 import fdllm
    c = fdllm.Context(0)
    yield c
    c.close()


def dev(a, dtype):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)          # values are exact in bf16 by construction
    return t.cuda()


def rel_err(gpu, ref):
    return float(np.abs(gpu - ref).max() / max(np.abs(ref).max(), 1e-30))


def check_tokens(tok_gpu, ref: O.Confidence, z=None):
    exact = ref.gap > GAP
    assert np.array_equal(tok_gpu[exact], ref.tok[exact])
    if z is not None:
        for r in np.nonzero(~exact)[0]:
            assert z[r, tok_gpu[r]] >= ref.zmax[r] - GAP


# ----------------------------------------------------------------- attention
def run_attention(ctx, a: synth.AttnCase, want_lse=True):
    q = dev(a.q, a.dtype)
    kc = dev(a.k_cache, a.dtype)
    vc = dev(a.v_cache, a.dtype)
    kb = dev(a.k_blk, a.dtype)
    vb = dev(a.v_blk, a.dtype)
    ctx.kv_store(kb, vb, kc, vc, a.block_start)
    out, lse = ctx.dualcache_attention(q, kc, vc, a.block_start, want_lse=True)
    torch.cuda.synchronize()
    ctx.device_status()
    return out.float().cpu().numpy(), lse.cpu().numpy(), kc, vc


def oracle_attention(a: synth.AttnCase):
    kc = a.k_cache.astype(np.float64)
    vc = a.v_cache.astype(np.float64)
    O.kv_store(kc, vc, a.k_blk, a.v_blk, a.block_start)
    o, lse = O.dualcache_attention(a.q, kc, vc)
    return o, lse, kc, vc


def check_attention(ctx, a):
    o_g, lse_g, kc_g, vc_g = run_attention(ctx, a)
    o_r, lse_r, kc_r, vc_r = oracle_attention(a)
    # the store is a copy: bit-exact
    assert np.array_equal(kc_g.float().cpu().numpy(), kc_r.astype(np.float32))
    assert np.array_equal(vc_g.float().cpu().numpy(), vc_r.astype(np.float32))
    assert rel_err(o_g, o_r) <= ATT_TOL[a.dtype], rel_err(o_g, o_r)
    np.testing.assert_allclose(lse_g, lse_r, rtol=0, atol=1e-4 if a.dtype == "f32" else 2e-3)
    # softmax rows sum to one under the GPU's LSE
    scale = 1.0 / math.sqrt(a.head_dim)
    grp = a.n_q_heads // a.n_kv_heads
    for b in range(a.batch):
        for h in range(0, a.n_q_heads, max(1, a.n_q_heads // 4)):
            s = (a.q[b, :, h, :].astype(np.float64) @ kc_r[b, h // grp].T) * scale
            tot = np.exp(s - lse_g[b, h][:, None].astype(np.float64)).sum(1)
            np.testing.assert_allclose(tot, 1.0, atol=1e-6 if a.dtype == "f32" else 2e-3)


@pytest.mark.parametrize("seed", range(20))
def test_attention_f32_tiny_step(ctx, seed):
    # batch 1, 4 heads, d 64, prefix 64 + block 32 + suffix 32
    check_attention(ctx, synth.attn_case(seed=seed, dtype="f32"))


@pytest.mark.parametrize("blk", range(8))
def test_attention_bf16_llada_layer(ctx, blk):
    # 32 heads MHA, d 128, prompt 512 + gen 256, block 32 at 512 + 32 blk
    a = synth.attn_case(batch=1, n_q_heads=32, head_dim=128, prefix=512 + 32 * blk, block=32,
                        suffix=256 - 32 * (blk + 1), dtype="bf16", seed=100 + blk)
    check_attention(ctx, a)


@pytest.mark.parametrize("kw", [
    dict(batch=2, n_q_heads=28, n_kv_heads=4, head_dim=128, prefix=512, block=32, suffix=480),
    dict(batch=3, n_q_heads=8, n_kv_heads=2, head_dim=64, prefix=37, block=5, suffix=11),
    dict(batch=1, n_q_heads=2, head_dim=128, prefix=0, block=1, suffix=0),
    dict(batch=1, n_q_heads=3, head_dim=64, prefix=0, block=128, suffix=1),
    dict(batch=2, n_q_heads=4, head_dim=128, prefix=1000, block=17, suffix=3),
])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_attention_shapes_and_edges(ctx, kw, dtype):
    check_attention(ctx, synth.attn_case(dtype=dtype, seed=7, **kw))


def test_attention_rejects_bad_arguments(ctx):
    from block_kv_cache_b200 import fdllm
    a = synth.attn_case(dtype="f32", seed=0)
    q, kc, vc = dev(a.q, "f32"), dev(a.k_cache, "f32"), dev(a.v_cache, "f32")
    with pytest.raises(fdllm.FdlError) as e:
        ctx.dualcache_attention(q, kc, vc, a.seq_len)          # block past the end
    assert e.value.code == fdllm.FDL_EINVAL
    with pytest.raises(fdllm.FdlError) as e:
        ctx.dualcache_attention(q, kc, vc, 0, ws=torch.empty(16, dtype=torch.uint8,
                                                                device="cuda"))
    assert e.value.code == fdllm.FDL_EWORKSPACE
    q96 = torch.zeros((1, 32, 4, 96), device="cuda")
    k96 = torch.zeros((1, 4, 128, 96), device="cuda")
    with pytest.raises(fdllm.FdlError) as e:
        ctx.dualcache_attention(q96, k96, k96, 0)
    assert e.value.code == fdllm.FDL_EUNSUPPORTED


# ----------------------------------------------------------------- LM head
def run_lmhead(ctx, c: synth.LMHeadCase, rows=None):
    h = dev(c.h, c.dtype)
    w = dev(c.w, c.dtype)
    bt = torch.from_numpy(c.bias_tok).cuda()
    bv = torch.from_numpy(c.bias_val).cuda()
    conf, tok = ctx.lmhead_confidence(h, w, bt, bv)
    torch.cuda.synchronize()
    return conf.cpu().numpy(), tok.cpu().numpy()


def test_lmhead_f32_tiny(ctx):
    for seed in range(20):
        s = synth.step_case(seed)
        # the tiny step's LM-head input: the block's attention output, heads concatenated
        o_r, _, _, _ = oracle_attention(s.attn)
        h = o_r[0].reshape(32, -1).astype(np.float32)
        c = synth.LMHeadCase("f32", 32, 256, 1024, 1023, h, s.w, s.bias_tok, s.bias_val)
        conf, tok = run_lmhead(ctx, c)
        ref = O.lmhead_confidence(h, s.w, s.bias_tok, s.bias_val)
        assert np.abs(conf - ref.conf).max() <= CONF_TOL
        z = O.lm_logits(h, s.w, s.bias_tok, s.bias_val)
        check_tokens(tok, ref, z)


_W_CACHE = {}


def llada_lmhead_case(rows):
    """hidden 4096, vocab 126464, mask id 126336, one shared weight matrix."""
    if "w" not in _W_CACHE:
        _W_CACHE["w"] = synth.lmhead_case(rows=1, seed=0, w_seed=0, mask_id=126336).w
    full = synth.lmhead_case(rows=rows, hidden=4096, vocab=2, seed=rows)
    w = _W_CACHE["w"]
    g = synth.rng(50_000 + rows)
    bt = g.integers(0, w.shape[0] - 1, rows).astype(np.int32)
    bt[bt >= 126336] += 1
    bv = g.uniform(0.0, 16.0, rows).astype(np.float32)
    return synth.LMHeadCase("bf16", rows, 4096, w.shape[0], 126336, full.h, w, bt, bv)


@pytest.mark.parametrize("rows", [32, 256, 1024])
def test_lmhead_bf16_llada_vocab(ctx, rows):
    # hidden 4096, vocab 126464, mask id 126336; batch = rows / 32
    c = llada_lmhead_case(rows)
    conf, tok = run_lmhead(ctx, c)
    # every row up to 64; beyond, the first and last row of every 128-row tile
    # (the MMA's M) plus random rows, 64 in all
    if rows <= 64:
        sample = np.arange(rows)
    else:
        edges = np.unique(np.concatenate([np.arange(0, rows, 128),
                                          np.minimum(np.arange(127, rows + 127, 128), rows - 1)]))
        rest = np.setdiff1d(np.arange(rows), edges)
        extra = synth.rng(rows).choice(rest, 64 - len(edges), replace=False)
        sample = np.sort(np.concatenate([edges, extra]))
    ref = O.lmhead_confidence(c.h[sample], c.w, c.bias_tok[sample], c.bias_val[sample])
    err = np.abs(conf[sample] - ref.conf).max()
    assert err <= CONF_TOL, err
    z = O.lm_logits(c.h[sample], c.w, c.bias_tok[sample], c.bias_val[sample])
    check_tokens(tok[sample], ref, z)
    assert np.all((conf > 0) & (conf <= 1))
    assert np.all((tok >= 0) & (tok < c.vocab))


@pytest.mark.parametrize("shape", [(1, 64, 2), (5, 128, 1000), (130, 192, 333), (33, 4096, 5000)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_lmhead_ragged_shapes(ctx, shape, dtype):
    M, D, V = shape
    c = synth.lmhead_case(rows=M, hidden=D, vocab=V, dtype=dtype, seed=M + V, bias_hi=8.0)
    conf, tok = run_lmhead(ctx, c)
    ref = O.lmhead_confidence(c.h, c.w, c.bias_tok, c.bias_val)
    assert np.abs(conf - ref.conf).max() <= CONF_TOL
    check_tokens(tok, ref, O.lm_logits(c.h, c.w, c.bias_tok, c.bias_val))


def test_lmhead_closed_form_zero_weight(ctx):
    # W = 0 and one planted bias b per row: conf = e^b / (e^b + V - 1), tok = planted
    M, D, V = 64, 256, 3000
    c = synth.lmhead_case(rows=M, hidden=D, vocab=V, dtype="bf16", seed=3, bias_hi=12.0)
    c.w[:] = 0
    c.bias_val[0] = 0.0          # all logits equal: conf = 1/V, tok = 0
    conf, tok = run_lmhead(ctx, c)
    e = np.exp(c.bias_val.astype(np.float64))
    np.testing.assert_allclose(conf, e / (e + V - 1), atol=CONF_TOL, rtol=0)
    assert tok[0] == 0
    np.testing.assert_array_equal(tok[1:], c.bias_tok[1:])


# ----------------------------------------------------------------- unmask
def run_unmask(ctx, u: synth.UnmaskCase, tau, conf=None, tok=None):
    conf = u.conf if conf is None else conf
    tok = u.tok if tok is None else tok
    x = torch.from_numpy(u.x).cuda()
    m = torch.from_numpy(u.masked).cuda()
    nd = torch.empty(u.batch, dtype=torch.int32, device="cuda")
    rem = ctx.threshold_unmask(torch.from_numpy(conf).cuda(), torch.from_numpy(tok).cuda(), x, m,
                               u.block_start, tau, n_decoded=nd)
    torch.cuda.synchronize()
    return x.cpu().numpy(), m.cpu().numpy(), rem.cpu().numpy(), nd.cpu().numpy()


@pytest.mark.parametrize("tau", [0.0, 0.5, 0.7, 0.9, 1.0])
@pytest.mark.parametrize("B", [1, 7, 32, 33, 100, 1024])
def test_unmask_bit_exact(ctx, tau, B):
    for seed in range(3):
        u = synth.unmask_case(batch=5, seq_len=B + 40, block_start=20, block_len=B,
                              seed=seed * 31 + B)
        xg, mg, rg, ng = run_unmask(ctx, u, tau)
        xr, mr, rr, nr = O.threshold_unmask(u.x, u.masked, u.conf, u.tok, 20, B, tau)
        assert np.array_equal(xg, xr)
        assert np.array_equal(mg, mr)
        assert np.array_equal(rg, rr) and np.array_equal(ng, nr)
        ctx.device_status()


def test_unmask_no_candidates_and_all_nan(ctx):
    from block_kv_cache_b200 import fdllm
    u = synth.unmask_case(batch=2, seq_len=64, block_start=16, block_len=32, seed=1)
    u.masked[0, 16:48] = 0                     # sequence 0: block already complete
    u.x[0, 16:48] = 5
    u.conf[1, :] = np.nan                      # sequence 1: every confidence NaN
    xg, mg, rg, ng = run_unmask(ctx, u, 0.9)
    assert ng[0] == 0 and rg[0] == 0 and np.array_equal(xg[0], u.x[0])
    assert ng[1] == 0 and rg[1] == int(u.masked[1, 16:48].sum())
    with pytest.raises(fdllm.FdlError) as e:
        ctx.device_status()
    assert e.value.code == fdllm.FDL_EDEVICE
    ctx.device_status()                        # cleared


# ----------------------------------------------------------------- the tiny block step
@pytest.mark.parametrize("seed", range(20))
def test_tiny_block_step_end_to_end(ctx, seed):
    """attention (f32) -> LM head on the block rows -> threshold unmask, each
    stage fed with the GPU's own previous output; decisions bit-exact against
    the oracle given the GPU's confidences, confidences within 1e-5 of the
    oracle's on the GPU's hidden states."""
    s = synth.step_case(seed)
    a = s.attn
    o_g, _, _, _ = run_attention(ctx, a)
    h = o_g[0].reshape(a.block_len, -1).astype(np.float32)
    c = synth.LMHeadCase("f32", a.block_len, h.shape[1], s.w.shape[0], s.w.shape[0] - 1, h,
                         s.w, s.bias_tok, s.bias_val)
    conf, tok = run_lmhead(ctx, c)
    ref = O.lmhead_confidence(h, s.w, s.bias_tok, s.bias_val)
    assert np.abs(conf - ref.conf).max() <= CONF_TOL
    u = s.unmask
    xg, mg, rg, ng = run_unmask(ctx, u, s.tau, conf[None, :], tok[None, :])
    xr, mr, rr, nr = O.threshold_unmask(u.x, u.masked, conf[None, :], tok[None, :],
                                        u.block_start, u.block_len, s.tau)
    assert np.array_equal(xg, xr) and np.array_equal(mg, mr)
    assert np.array_equal(rg, rr) and np.array_equal(ng, nr)
    assert ng[0] >= 1
