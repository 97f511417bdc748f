"""Parity of the transformer scaffold and of whole DualCache decodes with the
CPU oracle, through the C-ABI.

Per-op tolerances: bf16 outputs max|gpu - ref| / max|ref| <= 2e-2 (one bf16
rounding, 2^-9 relative, plus f32 accumulation); f32 outputs (the residual
stream) <= 1e-4 relative; copies and gathers bit-exact.

Whole decodes are checked step by step with the oracle replaying the GPU's
own trajectory (same tokens before every step, caches refreshed at the same
points): confidences agree within CONF_MODEL_TOL, which allows for the bf16
rounding of activations between kernels that the float64 oracle does not
have; token ids agree wherever the oracle's top-2 logit gap exceeds 0.05;
the unmask decisions are bit-exact given the GPU's confidences.
"""
import numpy as np
import pytest
import torch

import oracle as O
from block_kv_cache_b200 import synth

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2
CONF_MODEL_TOL = 2e-2
TOK_GAP = 0.05
CONF_TOL = 1e-5


@pytest.fixture(scope="module")
def ctx():
    from block_kv_cache_b200 import fdllm
    c = fdllm.Context(0)
    yield c
    c.close()


def bf(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).cuda()


def f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def rel(g, r):
    return float(np.abs(g - r).max() / max(np.abs(r).max(), 1e-30))


def bf_vals(a):
    return synth.bf16_value(synth.bf16_bits(np.asarray(a, np.float32)))


# ------------------------------------------------------------------ single ops
def test_rmsnorm_with_row_map(ctx):
    g = synth.rng(1)
    h = (g.standard_normal((300, 1024)) * 3).astype(np.float32)
    w = g.uniform(0.5, 1.5, 1024).astype(np.float32)
    rm = g.integers(0, 300, 77).astype(np.int32)
    out = ctx.rmsnorm(f32(h), f32(w), 1e-5, row_map=torch.from_numpy(rm).cuda())
    ref = O.rms_norm(h[rm], w, 1e-5)
    assert rel(out.float().cpu().numpy(), ref) <= BF16_TOL


def test_embed_gather_exact(ctx):
    g = synth.rng(2)
    table = bf_vals(g.standard_normal((500, 256)))
    ids = g.integers(0, 500, (3, 40)).astype(np.int32)
    rm = np.array([0, 5, 39, 40, 119, 7], np.int32)
    out = ctx.embed(torch.from_numpy(ids).cuda(), bf(table), row_map=torch.from_numpy(rm).cuda())
    assert np.array_equal(out.cpu().numpy(), table[ids.reshape(-1)[rm]])


@pytest.mark.parametrize("M,N,K", [(32, 4096, 4096), (300, 512, 256), (1, 64, 64), (129, 320, 192),
                                   (32, 4096, 12288), (200, 1024, 512), (1, 128, 64),
                                   (64, 12288, 4096),
                                   (300, 3584, 256), (1000, 3584, 512),    # Dream widths
                                   # the 128-row GEMM at the refresh's and the Dream-shape
                                   # cached step's sizes, and ragged rows
                                   (1024, 3584, 3584), (2048, 4096, 4096), (1000, 1024, 1280)])
def test_linear_residual(ctx, M, N, K):
    g = synth.rng(M + N)
    x = bf_vals(g.standard_normal((M, K)))
    w = bf_vals(g.standard_normal((N, K)) * 0.02)
    h0 = g.standard_normal((M, N)).astype(np.float32)
    h = f32(h0)
    ctx.linear_residual(bf(x), bf(w), h)
    ref = h0.astype(np.float64) + x.astype(np.float64) @ w.astype(np.float64).T
    assert rel(h.cpu().numpy(), ref) <= 1e-4


@pytest.mark.parametrize("M,F,K", [(32, 1024, 512), (257, 96, 128), (32, 12288, 4096),
                                   (100, 256, 256)])
def test_linear_swiglu(ctx, M, F, K):
    g = synth.rng(M + F)
    x = bf_vals(g.standard_normal((M, K)))
    wg = bf_vals(g.standard_normal((F, K)) * 0.05)
    wu = bf_vals(g.standard_normal((F, K)) * 0.05)
    wgu = np.empty((2 * F, K), np.float32)
    wgu[0::2], wgu[1::2] = wg, wu
    out = ctx.linear_swiglu(bf(x), bf(wgu))
    x64 = x.astype(np.float64)
    ref = O.silu(x64 @ wg.T) * (x64 @ wu.T)
    assert rel(out.float().cpu().numpy(), ref) <= BF16_TOL


@pytest.mark.parametrize("M,D,F,norm", [(32, 4096, 12288, True), (32, 4096, 12288, False),
                                        (32, 512, 1024, True), (7, 256, 640, True),
                                        (64, 1024, 4096, True), (300, 256, 192, True),
                                        (1, 128, 128, False)])
def test_ffn_block(ctx, M, D, F, norm):
    """h += SwiGLU(RMSNorm(h) or x) Wd^T in one call; for few rows the norm runs
    in the gate/up kernel and the SwiGLU of the split-K sums in the down
    projection's kernel, each behind a grid barrier. Called twice so that
    the context's scratch (zeroed sums, barrier words) is checked to be
    reusable."""
    g = synth.rng(M * 7 + F + norm)
    wg = bf_vals(g.standard_normal((F, D)) * 0.05)
    wu = bf_vals(g.standard_normal((F, D)) * 0.05)
    wd = bf_vals(g.standard_normal((D, F)) * 0.03)
    wgu = np.empty((2 * F, D), np.float32)
    wgu[0::2], wgu[1::2] = wg, wu
    h0 = (g.standard_normal((M, D)) * 2).astype(np.float32)
    wn = g.uniform(0.5, 1.5, D).astype(np.float32)
    x_in = bf_vals(g.standard_normal((M, D)))
    x_ref = O.rms_norm(h0, wn, 1e-5) if norm else x_in.astype(np.float64)
    wgug, wdg = bf(wgu), bf(wd)
    for rep in range(2):
        h = f32(h0)
        x = torch.empty((M, D), dtype=torch.bfloat16, device="cuda") if norm else bf(x_in)
        f = ctx.ffn(x, wgug, wdg, h, norm_w=f32(wn) if norm else None, eps=1e-5)
        if norm:
            assert rel(x.float().cpu().numpy(), x_ref) <= BF16_TOL, rep
        xg64 = x.float().cpu().numpy().astype(np.float64)   # the operand the GEMMs consumed
        f_ref = O.silu(xg64 @ wg.T) * (xg64 @ wu.T)
        assert rel(f.float().cpu().numpy(), f_ref) <= BF16_TOL, rep
        ref = h0.astype(np.float64) + f.float().cpu().numpy().astype(np.float64) @ wd.astype(np.float64).T
        assert rel(h.cpu().numpy(), ref) <= 1e-4, rep
    ctx.device_status()


@pytest.mark.parametrize("batch,Hq,Hkv,bias,B,pos0,L,D,norm", [
    (1, 32, 32, False, 32, 1024, 2048, 4096, True),   # LLaDA-8B layer: fused path
    (1, 32, 32, False, 32, 1024, 2048, 4096, False),
    (1, 8, 8, False, 32, 96, 256, 1024, True),        # fused, several splits per head
    (2, 28, 4, True, 32, 512, 1024, 3584, True),      # GQA 7:1 with bias (Dream / Qwen2.5)
    (2, 4, 2, True, 32, 64, 160, 256, True),          # no K split: separate calls
    (1, 8, 8, False, 32, 48, 256, 1024, False),       # block slot across two splits
    (1, 8, 4, True, 16, 192, 224, 1024, True),        # block in the ragged last tile
    (1, 32, 2, False, 32, 64, 256, 1024, False),      # GQA 16:1, two query chunks: separate calls
])
def test_qkv_attention(ctx, batch, Hq, Hkv, bias, B, pos0, L, D, norm):
    """Norm + block-slot projection + DualCache attention in one call equals
    the oracle's norm, projection, RoPE, cache store and attention."""
    g = synth.rng(Hq * 3 + L + D + norm)
    d = 128
    M = batch * B
    N = (Hq + 2 * Hkv) * d
    h0 = (g.standard_normal((M, D)) * 2).astype(np.float32)
    wn = g.uniform(0.5, 1.5, D).astype(np.float32)
    x_in = bf_vals(g.standard_normal((M, D)))
    w = bf_vals(g.standard_normal((N, D)) * (1.0 / np.sqrt(D)))
    bvec = (g.standard_normal(N) * 0.1).astype(np.float32) if bias else None
    k0 = bf_vals(g.standard_normal((batch, Hkv, L, d)))
    v0 = bf_vals(g.standard_normal((batch, Hkv, L, d)))
    from block_kv_cache_b200 import fdllm
    rope = torch.from_numpy(fdllm.rope_table(10000.0, L, d)).cuda()
    kc, vc = bf(k0), bf(v0)
    q = torch.empty((M, Hq, d), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((batch, B, Hq, d), dtype=torch.bfloat16, device="cuda")
    wg = bf(w)
    bg = None if bvec is None else f32(bvec)
    hg, wng = f32(h0), f32(wn)
    for rep in range(2):                       # scratch and barrier words are reusable
        xg = torch.empty((M, D), dtype=torch.bfloat16, device="cuda") if norm else bf(x_in)
        ctx.qkv_attention(xg, wg, rope, q, kc, vc, out, n_q_heads=Hq, rows_per_seq=B,
                          pos0=pos0, bias=bg, h=hg if norm else None,
                          norm_w=wng if norm else None, eps=1e-5)
        ctx.device_status()
        x = xg.float().cpu().numpy()            # the operand the projection consumed
        if norm:
            assert rel(x, O.rms_norm(h0, wn, 1e-5)) <= BF16_TOL
        y = x.astype(np.float64) @ w.astype(np.float64).T
        if bvec is not None:
            y = y + bvec
        pos = pos0 + np.arange(M) % B
        qr = O.apply_rope(y[:, :Hq * d].reshape(M, Hq, d), pos)
        kr = O.apply_rope(y[:, Hq * d:(Hq + Hkv) * d].reshape(M, Hkv, d), pos)
        vr = y[:, (Hq + Hkv) * d:].reshape(M, Hkv, d)
        assert rel(q.float().cpu().numpy(), qr) <= BF16_TOL
        kg, vg = kc.float().cpu().numpy(), vc.float().cpu().numpy()
        og = out.float().cpu().numpy()
        for sq in range(batch):
            rows = slice(sq * B, (sq + 1) * B)
            kref = k0[sq].astype(np.float64).copy()
            vref = v0[sq].astype(np.float64).copy()
            kref[:, pos0:pos0 + B] = kr[rows].transpose(1, 0, 2)
            vref[:, pos0:pos0 + B] = vr[rows].transpose(1, 0, 2)
            assert rel(kg[sq], kref) <= BF16_TOL and rel(vg[sq], vref) <= BF16_TOL
            keep = np.ones(L, bool)
            keep[pos0:pos0 + B] = False
            assert np.array_equal(kg[sq][:, keep], k0[sq][:, keep])
            o_ref, _ = O.attention(qr[rows], kref, vref)
            assert rel(og[sq], o_ref) <= BF16_TOL, (rep, sq)


@pytest.mark.parametrize("b,Hq,Hkv,L", [(1, 32, 32, 256), (2, 28, 4, 128), (2, 8, 2, 96),
                                        (1, 32, 32, 2048),     # LLaDA-8B refresh: 8 query blocks
                                        (2, 28, 4, 1024)])     # Dream-7B refresh, two sequences
def test_full_attention(ctx, b, Hq, Hkv, L):
    """Bidirectional attention of every position (the refresh), against the
    oracle for every query row; the L = 2048 MHA case runs the 256-row query
    blocks (eight per head) of the LLaDA-8B refresh."""
    g = synth.rng(b * Hq + L)
    d = 128
    q = bf_vals(g.standard_normal((b, L, Hq, d)))
    k = bf_vals(g.standard_normal((b, Hkv, L, d)))
    v = bf_vals(g.standard_normal((b, Hkv, L, d)))
    out = ctx.full_attention(bf(q), bf(k), bf(v)).float().cpu().numpy()
    for s in range(b):
        o, _ = O.attention(q[s], k[s], v[s])
        assert rel(out[s], o) <= BF16_TOL


# ------------------------------------------------------------------ whole decodes
def _small_params(seed, n_layers=2, hq=2, hkv=2, bias=False):
    return synth.model_params(vocab=512, hidden=256, n_layers=n_layers, n_q_heads=hq,
                              n_kv_heads=hkv, head_dim=128, ffn=512, seed=seed, dtype="bf16",
                              qkv_bias=bias, w_std=0.06, lm_std=0.15)


def _replay_check(P, rec, x_final, B, tau, tok_gap=TOK_GAP, bias=None):
    """Oracle replay of a recorded GPU decode (see module docstring), step kind
    by step kind: a refresh is the full forward (and rebuilds the oracle's
    caches), a DualCache step the block forward, a PrefixCache step the
    forward of the block and suffix over the cached prefix. At every step
    also the LM-head boundary on its own: the oracle's confidences of the
    GPU's final-norm rows (the exact LM-head input) within CONF_TOL of the
    GPU's, token ids exact where the oracle's top-2 logit gap exceeds 1e-3.
    bias = (bias_tok, bias_val, prompt_len): the planted bias [b, gen] of the
    generated positions, added by the LM head."""
    b = rec[0][2].shape[0]
    caches = [None] * b
    max_err = 0.0
    for n, (kind, s, xb, mb, conf, tok, xn) in enumerate(rec):
        conf = conf.reshape(b, B)
        tok = tok.reshape(b, B)
        xn = xn.reshape(b, B, -1)
        for i in range(b):
            if kind == "refresh":
                hf, kv = O.full_hidden(P, xb[i])
                caches[i] = [(k.copy(), v.copy()) for k, v in kv]
                hb = hf[s:s + B]
            elif kind == "cached":
                hb = O.block_hidden(P, xb[i, s:s + B], s, caches[i])
            else:
                assert kind == "prefix"
                hb = O.prefix_hidden(P, xb[i, s:], s, caches[i])[:B]
            bt = bv = None
            if bias is not None:
                bt = bias[0][i, s - bias[2]:s - bias[2] + B]
                bv = bias[1][i, s - bias[2]:s - bias[2] + B]
            c = O.lmhead_confidence(hb, P.lm_head, bt, bv)
            max_err = max(max_err, float(np.abs(conf[i] - c.conf).max()))
            sure = c.gap > tok_gap
            assert np.array_equal(tok[i][sure], c.tok[sure]), (n, i)
            cb = O.lmhead_confidence(xn[i], P.lm_head, bt, bv)
            assert np.abs(conf[i] - cb.conf).max() <= CONF_TOL, (n, i)
            sure = cb.gap > 1e-3
            assert np.array_equal(tok[i][sure], cb.tok[sure]), (n, i)
    # decisions on the GPU's confidences, bit-exact
        xa, ma, _, nd = O.threshold_unmask(xb, mb, conf, tok, s, B, tau)
        x_next = rec[n + 1][2] if n + 1 < len(rec) else x_final
        m_next = rec[n + 1][3] if n + 1 < len(rec) else None
        assert np.array_equal(xa, x_next), n
        if m_next is not None:
            assert np.array_equal(ma, m_next), n
    assert max_err <= CONF_MODEL_TOL, max_err
    return max_err


@pytest.mark.parametrize("seed,tau,hq,hkv,bias", [(0, 0.9, 2, 2, False), (1, 0.5, 4, 2, True),
                                                  (2, 1.0, 2, 1, False)])
def test_decode_matches_oracle_step_by_step(ctx, seed, tau, hq, hkv, bias):
    from block_kv_cache_b200.model import BlockDecoder, DeviceWeights
    P = _small_params(seed, hq=hq, hkv=hkv, bias=bias)
    w = DeviceWeights.from_params(P)
    b, Lp, gen, B = 2, 64, 64, 32
    dec = BlockDecoder(ctx, w, b, Lp + gen, B)
    prompt = synth.prompt_ids(seed, b, Lp, P.mask_id)
    rec = []
    x, steps = dec.generate(prompt, gen, tau=tau, record=rec)
    ctx.device_status()
    xf = x.cpu().numpy()
    assert steps == len(rec)
    if tau == 1.0:
        assert steps == gen                              # one token per step
    _replay_check(P, rec, xf, B, tau)


@pytest.mark.parametrize("cache,seed,tau,hq,hkv,bias", [("prefix", 3, 0.9, 2, 2, False),
                                                        ("prefix", 4, 0.5, 4, 2, True),
                                                        ("none", 5, 0.7, 2, 1, False)])
def test_cache_modes_match_oracle_step_by_step(ctx, cache, seed, tau, hq, hkv, bias):
    """PrefixCache (block and suffix recomputed over the cached prefix) and
    no-cache decoding (a full forward every step), replayed by the oracle on
    the GPU's own trajectory like the DualCache decode."""
    from block_kv_cache_b200.model import BlockDecoder, DeviceWeights
    P = _small_params(seed, hq=hq, hkv=hkv, bias=bias)
    w = DeviceWeights.from_params(P)
    b, Lp, gen, B = 2, 64, 64, 32
    dec = BlockDecoder(ctx, w, b, Lp + gen, B, cache=cache)
    prompt = synth.prompt_ids(seed, b, Lp, P.mask_id)
    rec = []
    x, steps = dec.generate(prompt, gen, tau=tau, record=rec)
    ctx.device_status()
    kinds = {r[0] for r in rec}
    assert kinds == ({"refresh", "prefix"} if cache == "prefix" else {"refresh"})
    _replay_check(P, rec, x.cpu().numpy(), B, tau)


def test_planted_bias_decode_matches_oracle(ctx):
    """With a planted logit bias on one token per generated position (the
    synthetic way to make the threshold rule fire with random weights), the
    DualCache decode decodes several positions per step and the oracle's
    replay (with the same bias in its LM head) agrees at every step."""
    from block_kv_cache_b200.model import BlockDecoder, DeviceWeights
    P = _small_params(6, hq=4, hkv=2, bias=True)
    w = DeviceWeights.from_params(P)
    b, Lp, gen, B, tau = 2, 64, 64, 32, 0.9
    g = synth.rng(66)
    bt = g.integers(0, P.mask_id, (b, gen)).astype(np.int32)
    bv = g.uniform(0.0, 16.0, (b, gen)).astype(np.float32)
    dec = BlockDecoder(ctx, w, b, Lp + gen, B, bias_tok=torch.from_numpy(bt).cuda(),
                       bias_val=torch.from_numpy(bv).cuda())
    prompt = synth.prompt_ids(6, b, Lp, P.mask_id)
    rec = []
    x, steps = dec.generate(prompt, gen, tau=tau, record=rec)
    ctx.device_status()
    assert steps < gen                               # the rule fires: some steps decode several
    _replay_check(P, rec, x.cpu().numpy(), B, tau, bias=(bt, bv, Lp))


@pytest.mark.parametrize("cache", ["prefix", "none"])
def test_native_generate_cache_modes_equal_the_python_decoder(ctx, cache):
    """fdl_generate in the PrefixCache and no-cache modes, with a planted bias,
    takes the same steps and decodes the same tokens as the Python decoder of
    the same mode (the same kernels in the same order)."""
    from block_kv_cache_b200.model import BlockDecoder, DeviceWeights
    P = _small_params(7, hq=4, hkv=2, bias=True)
    w = DeviceWeights.from_params(P)
    b, Lp, gen, B, tau = 2, 64, 64, 32, 0.9
    g = synth.rng(67)
    bt = torch.from_numpy(g.integers(0, P.mask_id, (b, gen)).astype(np.int32)).cuda()
    bv = torch.from_numpy(g.uniform(0.0, 16.0, (b, gen)).astype(np.float32)).cuda()
    prompt = synth.prompt_ids(7, b, Lp, P.mask_id)
    dec = BlockDecoder(ctx, w, b, Lp + gen, B, cache=cache, bias_tok=bt, bias_val=bv)
    x_py, steps_py = dec.generate(prompt, gen, tau=tau)
    x_nat, steps_nat = ctx.generate(w.native(), torch.from_numpy(prompt), gen, block=B, tau=tau,
                                    cache=cache, bias_tok=bt, bias_val=bv)
    ctx.device_status()
    assert not x_nat.is_cuda                         # host prompt in, host sequence out
    assert steps_nat == steps_py
    assert np.array_equal(x_nat.numpy(), x_py.cpu().numpy())


# Two layers at the full widths of the two model families, so that a decode the
# oracle replays runs the fused split-K calls (RMSNorm prologue, per-CTA query
# tiles of the q/k/v epilogue, SwiGLU prologue behind grid barriers) and the
# whole-vocabulary LM head. The LM head has the LM-head workload's weight
# distribution (W ~ N(0, 0.02)) and one planted logit bias ~ U(0, 24) per
# generated position, so that confidences spread over (0, 1) and steps decode
# several positions.
# Logits carry an error of a few hundredths from the bf16 activations of two
# layers (the 2e-2 confidence bound at confidence ~0.5 allows ~0.04), so token
# ids are compared where the oracle's top-2 gap exceeds 0.2, five times that.
WIDE_TOK_GAP = 0.2
WIDE_MODELS = {
    # LLaDA-8B widths: MHA 32 x 128, FFN 12288, vocab 126464, mask id 126336
    "llada": dict(vocab=126464, hidden=4096, n_q_heads=32, n_kv_heads=32, ffn=12288,
                  qkv_bias=False, mask_id=126336, batch=1),
    # Dream-7B (Qwen2.5-7B) widths: GQA 28/4 with q/k/v bias, FFN 18944, vocab 152064
    "dream": dict(vocab=152064, hidden=3584, n_q_heads=28, n_kv_heads=4, ffn=18944,
                  qkv_bias=True, mask_id=152063, batch=2),
}


@pytest.mark.parametrize("name", sorted(WIDE_MODELS))
def test_two_layer_full_width_decode_matches_oracle(ctx, name):
    """A 2-layer model at the full widths, prompt 32 + gen 64, block 32, tau
    0.9: every step replayed by the oracle on the GPU's own trajectory
    (confidences within 2e-2, decisions bit-exact given the GPU's
    confidences) and, at every step, the LM-head boundary within 1e-5 on the
    GPU's own final-norm rows."""
    from block_kv_cache_b200.model import BlockDecoder, DeviceWeights
    m = WIDE_MODELS[name]
    D = m["hidden"]
    P = synth.model_params(vocab=m["vocab"], hidden=D, n_layers=2, n_q_heads=m["n_q_heads"],
                           n_kv_heads=m["n_kv_heads"], head_dim=128, ffn=m["ffn"], seed=71,
                           dtype="bf16", qkv_bias=m["qkv_bias"], lm_std=0.02)
    P.mask_id = m["mask_id"]
    w = DeviceWeights.from_params(P)
    # the oracle widens its operands to float64 at every use; widen the layer
    # and LM-head weights once here instead (the same values)
    for Lw in P.layers:
        for k in list(Lw):
            Lw[k] = Lw[k].astype(np.float64)
    P.lm_head = P.lm_head.astype(np.float64)
    b, Lp, gen, B, tau = m["batch"], 32, 64, 32, 0.9
    g = synth.rng(73)
    bt = g.integers(0, P.mask_id, (b, gen)).astype(np.int32)
    bv = g.uniform(0.0, 24.0, (b, gen)).astype(np.float32)
    dec = BlockDecoder(ctx, w, b, Lp + gen, B, bias_tok=torch.from_numpy(bt).cuda(),
                       bias_val=torch.from_numpy(bv).cuda())
    prompt = synth.prompt_ids(72, b, Lp, P.mask_id)
    rec = []
    x, steps = dec.generate(prompt, gen, tau=tau, record=rec)
    ctx.device_status()
    assert steps == len(rec) and steps < gen          # some steps decoded several positions
    _replay_check(P, rec, x.cpu().numpy(), B, tau, tok_gap=WIDE_TOK_GAP, bias=(bt, bv, Lp))


@pytest.mark.parametrize("seed,tau,hq,hkv,bias", [(0, 0.9, 2, 2, False), (1, 0.5, 4, 2, True),
                                                  (2, 1.0, 2, 1, False)])
def test_native_generate_equals_the_python_decoder(ctx, seed, tau, hq, hkv, bias):
    """fdl_generate (the decode loop in the library) takes the same steps and
    decodes the same tokens as the Python decoder above, whose trajectory the
    oracle replays (same kernels in the same order; at these shapes no
    projection splits K, so both runs are bit-identical)."""
    from block_kv_cache_b200.model import BlockDecoder, DeviceWeights
    P = _small_params(seed, hq=hq, hkv=hkv, bias=bias)
    w = DeviceWeights.from_params(P)
    b, Lp, gen, B = 2, 64, 64, 32
    prompt = synth.prompt_ids(seed, b, Lp, P.mask_id)
    dec = BlockDecoder(ctx, w, b, Lp + gen, B)
    x_py, steps_py = dec.generate(prompt, gen, tau=tau)
    x_nat, steps_nat = ctx.generate(w.native(), torch.from_numpy(prompt).cuda(), gen, block=B,
                                    tau=tau)
    ctx.device_status()
    assert steps_nat == steps_py
    assert np.array_equal(x_nat.cpu().numpy(), x_py.cpu().numpy())


@pytest.mark.parametrize("cache,bias", [("dual", False), ("dual", True), ("prefix", True),
                                        ("none", False)])
def test_native_device_loop_equals_host_loop(ctx, cache, bias):
    """fdl_generate with the device loop (the whole decode as one CUDA graph,
    a conditional WHILE node per block around its cached steps) takes the
    same steps and decodes the same tokens as the host loop; a second call
    launches the graph kept in the context, a call with another tau captures
    a new one."""
    from block_kv_cache_b200.model import DeviceWeights
    P = _small_params(8, hq=4, hkv=2, bias=True)
    w = DeviceWeights.from_params(P)
    m = w.native()
    b, Lp, gen, B = 2, 64, 64, 32
    kw = dict(block=B, cache=cache)
    if bias:
        g = synth.rng(68)
        kw["bias_tok"] = torch.from_numpy(g.integers(0, P.mask_id, (b, gen)).astype(np.int32)).cuda()
        kw["bias_val"] = torch.from_numpy(g.uniform(0.0, 16.0, (b, gen)).astype(np.float32)).cuda()
    prompt = torch.from_numpy(synth.prompt_ids(8, b, Lp, P.mask_id)).cuda()
    for tau in (0.9, 0.9, 0.5):
        x_h, s_h = ctx.generate(m, prompt, gen, tau=tau, **kw)
        x_d, s_d = ctx.generate(m, prompt, gen, tau=tau, device_loop=True, **kw)
        ctx.device_status()
        assert s_d == s_h
        assert np.array_equal(x_d.cpu().numpy(), x_h.cpu().numpy())


def _spread_bias(mask_id, b, gen, seed):
    """Planted bias whose strength differs by sequence (sequence i gets
    U(0, hi_i) with hi_i from 0 to 16), so that at tau < 1 the sequences of a
    batch finish a block after different numbers of steps."""
    g = synth.rng(seed)
    hi = np.linspace(16.0, 0.0, b)[:, None]
    tok = g.integers(0, mask_id, (b, gen)).astype(np.int32)
    val = (g.uniform(0.0, 1.0, (b, gen)) * hi).astype(np.float32)
    return torch.from_numpy(tok).cuda(), torch.from_numpy(val).cuda()


@pytest.mark.parametrize("tau", [0.9, 0.5])
def test_native_generate_compact_equals_lockstep(ctx, tau):
    """fdl_generate with compaction (each cached step only on the sequences
    that still have masked positions in the block) decodes the same tokens in
    the same steps as the lockstep decode, on a batch whose sequences finish
    their blocks after different numbers of steps (planted bias of a
    different strength per sequence). At these shapes no projection splits K,
    so both decodes are deterministic and the comparison is exact."""
    from block_kv_cache_b200.model import DeviceWeights
    P = _small_params(11, hq=4, hkv=2, bias=True)
    w = DeviceWeights.from_params(P)
    m = w.native()
    b, Lp, gen, B = 5, 64, 96, 32
    bias_tok, bias_val = _spread_bias(P.mask_id, b, gen, 71)
    prompt = torch.from_numpy(synth.prompt_ids(12, b, Lp, P.mask_id)).cuda()
    kw = dict(block=B, tau=tau, bias_tok=bias_tok, bias_val=bias_val)
    x_l, s_l = ctx.generate(m, prompt, gen, **kw)
    x_c, s_c = ctx.generate(m, prompt, gen, batching="compact", **kw)
    ctx.device_status()
    assert s_c == s_l
    assert np.array_equal(x_c.cpu().numpy(), x_l.cpu().numpy())
    # the sequences did not finish in lockstep: compaction had work to skip
    per_seq = [ctx.generate(m, prompt[i:i + 1].contiguous(), gen, block=B, tau=tau,
                            bias_tok=bias_tok[i:i + 1].contiguous(),
                            bias_val=bias_val[i:i + 1].contiguous())[1] for i in (0, b - 1)]
    assert per_seq[0] < s_l and per_seq[1] <= s_l
    # a single sequence decodes alone exactly as it does inside the batch
    x_1, _ = ctx.generate(m, prompt[:1].contiguous(), gen, block=B, tau=tau,
                          bias_tok=bias_tok[:1].contiguous(), bias_val=bias_val[:1].contiguous())
    assert np.array_equal(x_1.cpu().numpy()[0], x_c.cpu().numpy()[0])


@pytest.mark.parametrize("tau", [0.9, 0.5])
def test_native_generate_per_sequence_blocks(ctx, tau):
    """fdl_generate with every sequence moving to its next block as soon as
    its own block is decoded (a step refreshes the sequences that have just
    moved on, each at its own positions, and takes a DualCache step of the
    others at their own blocks): bit for bit the tokens of the lockstep decode
    (the attention plans its splits for the whole batch, so a sequence's sums
    do not depend on which others share a launch), in no more steps; one
    sequence alone decodes exactly as the lockstep decode of it alone."""
    from block_kv_cache_b200.model import DeviceWeights
    P = _small_params(11, hq=4, hkv=2, bias=True)
    w = DeviceWeights.from_params(P)
    m = w.native()
    b, Lp, gen, B = 5, 64, 96, 32
    bias_tok, bias_val = _spread_bias(P.mask_id, b, gen, 71)
    prompt = torch.from_numpy(synth.prompt_ids(12, b, Lp, P.mask_id)).cuda()
    kw = dict(block=B, tau=tau, bias_tok=bias_tok, bias_val=bias_val)
    x_l, s_l = ctx.generate(m, prompt, gen, **kw)
    x_p, s_p = ctx.generate(m, prompt, gen, batching="per_sequence", **kw)
    ctx.device_status()
    assert np.array_equal(x_p.cpu().numpy(), x_l.cpu().numpy())
    assert s_p <= s_l
    one = dict(block=B, tau=tau, bias_tok=bias_tok[:1].contiguous(),
               bias_val=bias_val[:1].contiguous())
    x_a, s_a = ctx.generate(m, prompt[:1].contiguous(), gen, **one)
    x_1, s_1 = ctx.generate(m, prompt[:1].contiguous(), gen, batching="per_sequence", **one)
    assert s_1 == s_a
    assert np.array_equal(x_1.cpu().numpy(), x_a.cpu().numpy())
    # no bias: every sequence decodes one position per step, in lockstep anyway
    x_n, s_n = ctx.generate(m, prompt, gen, block=B, tau=1.0, batching="per_sequence")
    assert s_n == gen
    assert np.array_equal(x_n.cpu().numpy(), ctx.generate(m, prompt, gen, block=B, tau=1.0)[0]
                          .cpu().numpy())


@pytest.mark.parametrize("B,Lp,gen,tau", [(16, 48, 112, 0.9), (64, 64, 128, 0.7), (32, 32, 96, 0.0)])
def test_native_generate_batchings_other_blocks(ctx, B, Lp, gen, tau):
    """The three batchings on other block sizes and lengths (blocks of 16 and
    64, whose attention takes the unfused calls; L = 160 ends in a partial key
    tile; tau = 0 decodes a whole block per step): the same tokens bit for bit,
    and with tau = 0 one step per block. A total length that is not a
    multiple of 32 is refused before any work."""
    from block_kv_cache_b200.model import DeviceWeights
    P = _small_params(17, hq=2, hkv=2, bias=False)
    w = DeviceWeights.from_params(P)
    m = w.native()
    b = 4
    bias_tok, bias_val = _spread_bias(P.mask_id, b, gen, 73)
    prompt = torch.from_numpy(synth.prompt_ids(18, b, Lp, P.mask_id)).cuda()
    kw = dict(block=B, tau=tau, bias_tok=bias_tok, bias_val=bias_val)
    x_l, s_l = ctx.generate(m, prompt, gen, **kw)
    for batching in ("compact", "per_sequence"):
        x_b, s_b = ctx.generate(m, prompt, gen, batching=batching, **kw)
        ctx.device_status()
        assert np.array_equal(x_b.cpu().numpy(), x_l.cpu().numpy()), batching
        assert s_b <= s_l
        if tau == 0.0:
            assert s_b == s_l == gen // B
    if B == 16:   # 48 + 112 - 16 = 144: not a multiple of 32
        from block_kv_cache_b200 import fdllm
        with pytest.raises(fdllm.FdlError):
            ctx.generate(m, prompt, gen - B, block=B, tau=tau)


def test_native_generate_compact_fused_shapes(ctx):
    """Compaction and per-sequence blocks on shapes that take the fused
    split-K calls (hidden 1024, GQA 8/2 with bias; the sequence map and the
    per-sequence block starts reach the split-K q/k/v sums, the attention's
    block-slot writes and its cache reads, and the refresh of a subset): the
    prompts are kept, every position is decoded, and the tokens agree with the
    lockstep decode (exactly, unless the order of split-K atomic additions
    tips a decision; at least 90 % of positions). Compaction is refused with
    the device loop and outside the DualCache mode."""
    from block_kv_cache_b200 import fdllm
    from block_kv_cache_b200.model import DeviceWeights, ModelShape
    sh = ModelShape(4096, 1024, 2, 8, 2, 1024, 4095, 128, qkv_bias=True)
    w = DeviceWeights.random(sh, seed=6)
    b, Lp, gen, B = 6, 64, 64, 32
    prompt = torch.from_numpy(synth.prompt_ids(13, b, Lp, sh.mask_id)).cuda()
    bias_tok, bias_val = _spread_bias(sh.mask_id, b, gen, 72)
    bias_val = bias_val * 2.0
    m = w.native()
    kw = dict(block=B, tau=0.9, bias_tok=bias_tok, bias_val=bias_val)
    x_l, s_l = ctx.generate(m, prompt, gen, **kw)
    for batching in ("compact", "per_sequence"):
        x_c, s_c = ctx.generate(m, prompt, gen, batching=batching, **kw)
        ctx.device_status()
        xc, xl = x_c.cpu().numpy(), x_l.cpu().numpy()
        assert np.array_equal(xc[:, :Lp], prompt.cpu().numpy())
        assert (xc[:, Lp:] != sh.mask_id).all() and xc.min() >= 0 and xc.max() < sh.vocab
        assert (xc[:, Lp:] == xl[:, Lp:]).mean() >= 0.9
        assert s_c <= gen and s_l <= gen
    for bad in (dict(batching="compact", device_loop=True), dict(batching="compact", cache="prefix"),
                dict(batching="per_sequence", device_loop=True),
                dict(batching="per_sequence", cache="none")):
        with pytest.raises(fdllm.FdlError):
            ctx.generate(m, prompt, gen, **kw, **bad)


def test_native_generate_fused_shapes(ctx):
    """fdl_generate on shapes that take the fused split-K calls (hidden 1024,
    GQA 8/2 with bias): the prompt is kept, every position is decoded, tau = 1
    decodes exactly one position per step, and bad arguments are rejected."""
    from block_kv_cache_b200 import fdllm
    from block_kv_cache_b200.model import DeviceWeights, ModelShape
    sh = ModelShape(4096, 1024, 2, 8, 2, 1024, 4095, 128, qkv_bias=True)
    w = DeviceWeights.random(sh, seed=5)
    b, Lp, gen, B = 3, 96, 64, 32
    prompt = torch.from_numpy(synth.prompt_ids(9, b, Lp, sh.mask_id)).cuda()
    m = w.native()
    x, steps = ctx.generate(m, prompt, gen, block=B, tau=1.0)
    ctx.device_status()
    assert steps == gen                                         # one position per step
    xd, steps_d = ctx.generate(m, prompt, gen, block=B, tau=1.0, device_loop=True)
    ctx.device_status()
    assert steps_d == gen
    assert np.array_equal(xd.cpu().numpy()[:, :Lp], prompt.cpu().numpy())
    xh = x.cpu().numpy()
    assert np.array_equal(xh[:, :Lp], prompt.cpu().numpy())
    assert xh.min() >= 0 and xh.max() < sh.vocab
    with pytest.raises(fdllm.FdlError):
        ctx.generate(m, prompt, 48, block=B)                    # gen not a multiple of block
    with pytest.raises(fdllm.FdlError):
        ctx.generate(m, prompt[:, :Lp - 8].contiguous(), gen, block=B)   # prompt not either


def test_tau_one_single_layer_gpu_equals_sequential(ctx):
    """tau = 1 and one layer: the GPU's DualCache decode equals sequential
    greedy decoding of the oracle wherever the oracle's choices are not
    near-ties (checked token by token along the GPU's own trajectory)."""
    from block_kv_cache_b200.model import BlockDecoder, DeviceWeights
    P = _small_params(5, n_layers=1)
    w = DeviceWeights.from_params(P)
    dec = BlockDecoder(ctx, w, 1, 96, 32)
    prompt = synth.prompt_ids(5, 1, 32, P.mask_id)
    rec = []
    x, steps = dec.generate(prompt, 64, tau=1.0, record=rec)
    assert steps == 64
    # each step decodes exactly the position the sequential rule picks
    for kind, s, xb, mb, conf, tok, _ in rec:
        logits, _ = O.full_forward(P, xb[0])
        c = O.confidence_from_logits(logits[s:s + 32])
        cand = mb[0, s:s + 32] != 0
        order = np.argsort(-np.where(cand, c.conf, -1.0), kind="stable")
        top, second = order[0], order[1] if cand.sum() > 1 else None
        if second is not None and c.conf[top] - c.conf[second] < 2 * CONF_MODEL_TOL:
            continue                                   # near tie: either choice is correct
        gpu_pick = int(np.argmax(np.where(cand, conf, -1.0)))
        assert gpu_pick == top


def test_dream_shape_full_decode(ctx):
    """The Dream-7B-shaped configuration at full size: random-init 28 layers,
    hidden 3584, GQA 28/4 with q/k/v bias, FFN 18944, vocab 152064, bf16,
    batch 32, prompt 512 + gen 512, block 32, tau 0.9. The whole decode:
    every step's unmask decisions bit-exact against the oracle given the GPU's
    confidences; each sequence with masked positions in the block decodes at
    least one per step; nothing outside the block changes; everything is
    decoded at the end and the prompt is untouched. Then the LM-head
    confidences of sampled rows of the last step against the oracle on the
    GPU's own final hidden states (within 1e-5)."""
    from block_kv_cache_b200.model import BlockDecoder, DeviceWeights, ModelShape
    sh = ModelShape(152064, 3584, 28, 28, 4, 18944, 152063, 128, qkv_bias=True)
    w = DeviceWeights.random(sh, seed=77)
    b, Lp, gen, B, tau = 32, 512, 512, 32, 0.9
    dec = BlockDecoder(ctx, w, b, Lp + gen, B)
    prompt = synth.prompt_ids(3, b, Lp, sh.mask_id)
    rec = []
    x, steps = dec.generate(prompt, gen, tau=tau, record=rec)
    ctx.device_status()
    xf = x.cpu().numpy()
    assert steps == len(rec) and gen // B <= steps <= gen
    total = np.zeros(b, np.int64)
    for n, (kind, s, xb, mb, conf, tok, _) in enumerate(rec):
        conf, tok = conf.reshape(b, B), tok.reshape(b, B)
        xa, ma, _, nd = O.threshold_unmask(xb, mb, conf, tok, s, B, tau)
        x_next = rec[n + 1][2] if n + 1 < len(rec) else xf
        assert np.array_equal(xa, x_next), n
        if n + 1 < len(rec):
            assert np.array_equal(ma, rec[n + 1][3]), n
        assert not np.any(ma.astype(bool) & ~mb.astype(bool)), n   # never re-masked
        had = mb[:, s:s + B].any(axis=1)
        dec_now = (mb[:, s:s + B].astype(bool) & ~ma[:, s:s + B].astype(bool)).sum(axis=1)
        assert np.all(dec_now[had] >= 1), n                         # progress every step
        total += dec_now
        out = np.ones(Lp + gen, bool)
        out[s:s + B] = False
        assert np.array_equal(x_next[:, out], xb[:, out]), n
    assert np.all(total == gen)                                     # everything decoded
    assert np.array_equal(xf[:, :Lp], np.asarray(prompt))
    assert xf.min() >= 0 and xf.max() < sh.vocab
    # LM head of the last step on the GPU's final hidden states
    rows = np.array([0, 31, 517, 1023])
    h = dec.xn[torch.from_numpy(rows).cuda()].float().cpu().numpy()
    lm = w.lm_head.float().cpu().numpy()
    r = O.lmhead_confidence(h, lm)
    conf_g = dec.conf.cpu().numpy().reshape(-1)[rows]
    tok_g = dec.tok.cpu().numpy().reshape(-1)[rows]
    assert np.abs(conf_g - r.conf).max() <= 1e-5
    sure = r.gap > 1e-3
    assert np.array_equal(tok_g[sure], r.tok[sure])
