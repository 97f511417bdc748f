"""Pins for the CPU oracle: closed forms, library routines, invariants and
hand-worked cases, each chosen so that a plausible slip in the oracle (a
dropped term, a wrong sign or index, a transposed operand, a wrong GQA group,
a non-strict comparison, a wrong tie rule) fails at least one of them.
No GPU, no CUDA library."""
import json
import math
import os

import numpy as np
import pytest
import scipy.special as sps
import torch
import torch.nn.functional as F

import oracle
from oracle import fastdllm as O
from block_kv_cache_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- attention
def _sdpa(q, k, v):
    """torch's scaled_dot_product_attention (float64, CPU, no mask) on the
    oracle's layouts: q [Bq, Hq, d], k/v [Hkv, L, d]."""
    qt = torch.from_numpy(np.ascontiguousarray(np.transpose(q, (1, 0, 2))))[None]
    kt = torch.from_numpy(np.ascontiguousarray(k))[None]
    vt = torch.from_numpy(np.ascontiguousarray(v))[None]
    o = F.scaled_dot_product_attention(qt, kt, vt, enable_gqa=True)
    return np.transpose(o[0].numpy(), (1, 0, 2))


@pytest.mark.parametrize("Hq,Hkv,d,L,Bq", [(4, 4, 64, 128, 32), (8, 2, 16, 37, 5),
                                           (7, 1, 8, 9, 3), (28, 4, 32, 40, 32)])
def test_attention_matches_sdpa(Hq, Hkv, d, L, Bq):
    g = synth.rng(Hq * 1000 + L)
    q = g.standard_normal((Bq, Hq, d))
    k = g.standard_normal((Hkv, L, d))
    v = g.standard_normal((Hkv, L, d))
    o, _ = O.attention(q, k, v)
    np.testing.assert_allclose(o, _sdpa(q, k, v), rtol=1e-12, atol=1e-12)


def test_attention_single_key_returns_value():
    g = synth.rng(1)
    q = g.standard_normal((5, 3, 8))
    k = g.standard_normal((3, 1, 8))
    v = g.standard_normal((3, 1, 8))
    o, lse = O.attention(q, k, v)
    for h in range(3):
        np.testing.assert_allclose(o[:, h, :], np.broadcast_to(v[h, 0], (5, 8)), atol=1e-15)
        np.testing.assert_allclose(lse[h], (q[:, h, :] @ k[h, 0]) / math.sqrt(8), atol=1e-13)


def test_attention_zero_keys_mean_of_values():
    g = synth.rng(2)
    L = 50
    q = g.standard_normal((4, 2, 16))
    k = np.zeros((2, L, 16))
    v = g.standard_normal((2, L, 16))
    o, lse = O.attention(q, k, v)
    for h in range(2):
        np.testing.assert_allclose(o[:, h, :], np.broadcast_to(v[h].mean(0), (4, 16)), atol=1e-14)
    np.testing.assert_allclose(lse, math.log(L), atol=1e-14)


def test_attention_two_keys_closed_form():
    # q = a e0, k0 = e0, k1 = 0: scores (a/sqrt(d), 0) -> o = sigmoid(a/sqrt d) v0 + (1 - .) v1
    d, a = 4, 3.0
    q = np.zeros((1, 1, d)); q[0, 0, 0] = a
    k = np.zeros((1, 2, d)); k[0, 0, 0] = 1.0
    v = np.array([[[1.0, 2.0, 3.0, 4.0], [-1.0, 0.5, 0.0, 2.0]]])
    o, lse = O.attention(q, k, v)
    s = a / math.sqrt(d)
    p0 = 1.0 / (1.0 + math.exp(-s))
    np.testing.assert_allclose(o[0, 0], p0 * v[0, 0] + (1 - p0) * v[0, 1], atol=1e-15)
    assert abs(lse[0, 0] - math.log(math.exp(s) + 1.0)) < 1e-14


def test_attention_key_permutation_invariance_and_value_linearity():
    g = synth.rng(3)
    q = g.standard_normal((6, 4, 8))
    k = g.standard_normal((2, 20, 8))
    v = g.standard_normal((2, 20, 8))
    o, lse = O.attention(q, k, v)
    perm = g.permutation(20)
    o2, lse2 = O.attention(q, k[:, perm], v[:, perm])
    np.testing.assert_allclose(o, o2, atol=1e-13)
    np.testing.assert_allclose(lse, lse2, atol=1e-13)
    o3, _ = O.attention(q, k, 2.5 * v + 1.0)
    np.testing.assert_allclose(o3, 2.5 * o + 1.0, atol=1e-12)


def test_attention_lse_normalises_rows():
    # rows of exp(s - lse) sum to one; s formed through torch (a library matmul)
    g = synth.rng(4)
    q = g.standard_normal((5, 2, 16))
    k = g.standard_normal((2, 33, 16))
    v = g.standard_normal((2, 33, 16))
    _, lse = O.attention(q, k, v)
    for h in range(2):
        s = torch.from_numpy(q[:, h, :]) @ torch.from_numpy(k[h]).T / 4.0
        tot = torch.exp(s - torch.from_numpy(lse[h])[:, None]).sum(1).numpy()
        np.testing.assert_allclose(tot, 1.0, atol=1e-13)


def test_dualcache_batch_and_kv_store_layout():
    a = synth.attn_case(batch=2, n_q_heads=4, n_kv_heads=2, head_dim=8,
                        prefix=5, block=4, suffix=3, seed=9)
    kc, vc = a.k_cache.astype(np.float64), a.v_cache.astype(np.float64)
    O.kv_store(kc, vc, a.k_blk, a.v_blk, a.block_start)
    for b in range(2):
        for t in range(a.block_len):
            for h in range(2):
                assert np.array_equal(kc[b, h, a.block_start + t], a.k_blk[b, t, h])
                assert np.array_equal(vc[b, h, a.block_start + t], a.v_blk[b, t, h])
    # rows outside the slot untouched
    assert np.array_equal(kc[:, :, :a.block_start], a.k_cache[:, :, :a.block_start])
    assert np.array_equal(vc[:, :, a.block_start + 4:], a.v_cache[:, :, a.block_start + 4:])
    o, lse = O.dualcache_attention(a.q, kc, vc)
    assert o.shape == (2, 4, 4, 8) and lse.shape == (2, 4, 4)
    for b in range(2):
        np.testing.assert_allclose(o[b], _sdpa(a.q[b].astype(np.float64), kc[b], vc[b]), atol=1e-12)


# ---------------------------------------------------------------- transformer pieces
def test_rope_complex_form_and_relative_property():
    g = synth.rng(5)
    d, n = 16, 7
    x = g.standard_normal((n, 3, d))
    pos = g.integers(0, 500, n)
    y = O.apply_rope(x, pos, 10000.0)
    # complex form: (x_i + i x_{i+d/2}) * exp(i pos theta^(-2i/d))
    z = x[..., : d // 2] + 1j * x[..., d // 2:]
    w = np.exp(1j * np.outer(pos, 10000.0 ** (-np.arange(d // 2) * 2.0 / d)))[:, None, :]
    zr = z * w
    np.testing.assert_allclose(y[..., : d // 2], zr.real, atol=1e-12)
    np.testing.assert_allclose(y[..., d // 2:], zr.imag, atol=1e-12)
    # position 0 is the identity; norms are preserved
    np.testing.assert_allclose(O.apply_rope(x, np.zeros(n, int)), x, atol=0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-12)
    # <R(m) q, R(n) k> depends only on m - n
    q, k = g.standard_normal((1, 1, d)), g.standard_normal((1, 1, d))
    dots = [np.sum(O.apply_rope(q, [m]) * O.apply_rope(k, [m - 5])) for m in (5, 17, 301)]
    np.testing.assert_allclose(dots, dots[0], rtol=1e-11)


def test_rmsnorm_and_silu_match_torch():
    g = synth.rng(6)
    x = g.standard_normal((5, 32)) * 3
    w = g.standard_normal(32)
    ref = F.rms_norm(torch.from_numpy(x), (32,), torch.from_numpy(w), eps=1e-5).numpy()
    np.testing.assert_allclose(O.rms_norm(x, w, 1e-5), ref, rtol=1e-13)
    np.testing.assert_allclose(O.silu(x), F.silu(torch.from_numpy(x)).numpy(), rtol=1e-13)


# ---------------------------------------------------------------- LM head / confidence
def test_confidence_closed_form_single_planted_bias():
    V, D, M = 1000, 16, 6
    h = synth.rng(7).standard_normal((M, D))
    w = np.zeros((V, D))
    bt = np.array([3, 999, 0, 500, 17, 998])
    bv = np.array([0.0, 1.0, 5.0, 12.0, 16.0, 0.25])
    c = O.lmhead_confidence(h, w, bt, bv)
    expect = np.exp(bv) / (np.exp(bv) + V - 1)
    np.testing.assert_allclose(c.conf, expect, rtol=1e-13)
    # b = 0: all logits equal -> conf = 1/V and the lowest id wins
    assert c.tok[0] == 0
    np.testing.assert_array_equal(c.tok[1:], bt[1:])
    assert abs(c.conf[0] - 1.0 / V) < 1e-16


def test_confidence_ties_lowest_id():
    g = synth.rng(8)
    w = g.standard_normal((50, 8))
    w[31] = w[12]                      # duplicated row: exact tie between 12 and 31
    h = g.standard_normal((40, 8))
    c = O.lmhead_confidence(h, w)
    z = h @ w.T
    for r in range(40):
        if z[r].argmax() in (12, 31):
            assert c.tok[r] == 12
    # a row whose max is one of the duplicated pair exists
    h2 = w[12][None, :] * 10
    assert O.lmhead_confidence(h2, w).tok[0] == 12


def test_confidence_matches_scipy_softmax_and_chunking():
    g = synth.rng(9)
    M, D, V = 37, 24, 1003
    h = g.standard_normal((M, D))
    w = g.standard_normal((V, D)) * 0.3
    bt = g.integers(0, V, M)
    bv = g.uniform(0, 8, M)
    z = (torch.from_numpy(h) @ torch.from_numpy(w).T).numpy()
    z[np.arange(M), bt] += bv
    ref_conf = sps.softmax(z, axis=1).max(axis=1)
    ref_lse = sps.logsumexp(z, axis=1)
    for vc, rc in [(16384, 256), (100, 5), (7, 1)]:
        c = O.confidence_from_logits(O.lm_logits(h, w, bt, bv, vocab_chunk=vc))
        np.testing.assert_allclose(c.conf, ref_conf, rtol=1e-12)
        np.testing.assert_allclose(c.lse, ref_lse, rtol=1e-13)
        c2 = O.lmhead_confidence(h, w, bt, bv, row_chunk=rc)
        np.testing.assert_allclose(c2.conf, ref_conf, rtol=1e-12)
        np.testing.assert_array_equal(c2.tok, z.argmax(1))
    # shift invariance
    c3 = O.confidence_from_logits(z + 123.0)
    np.testing.assert_allclose(c3.conf, ref_conf, rtol=1e-10)


# ---------------------------------------------------------------- select / scatter
def _golden_cases():
    with open(os.path.join(GOLD, "threshold_select.json")) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_select_golden(case):
    conf = np.array([float(c) for c in case["conf"]], np.float32)
    sel = O.select_positions(conf, np.array(case["candidate"], bool), case["tau"])
    assert sorted(np.nonzero(sel)[0].tolist()) == case["expected"]


def _select_by_sorting(conf, cand, tau):
    """Same rule, second formulation: order the candidates by (confidence
    descending, position ascending) with np.lexsort; take the leading run that
    exceeds tau, or the first one if that run is empty."""
    t = float(np.float32(tau))
    idx = np.nonzero(cand & ~np.isnan(conf))[0]
    if len(idx) == 0:
        return set()
    order = idx[np.lexsort((idx, -conf[idx].astype(np.float64)))]
    above = [i for i in order if conf[i] > t]
    return set(above) if above else {order[0]}


def test_select_brute_force_random():
    g = synth.rng(10)
    for trial in range(3000):
        B = int(g.integers(1, 9))
        conf = g.choice(np.array([0.1, 0.5, 0.7, 0.9, 0.95, 1.0, 0.3], np.float32), B)
        if trial % 3 == 0:
            conf = g.uniform(0, 1, B).astype(np.float32)
        if trial % 17 == 0:
            conf[g.integers(0, B)] = np.nan
        cand = g.uniform(size=B) < 0.7
        tau = float(g.choice([0.0, 0.5, 0.7, 0.9, 1.0]))
        sel = O.select_positions(conf, cand, tau)
        assert set(np.nonzero(sel)[0].tolist()) == _select_by_sorting(conf, cand, tau)
        if cand.any() and not np.isnan(conf[cand]).all():
            assert sel.sum() >= 1
        assert not (sel & ~cand).any()
        if tau == 1.0:
            assert sel.sum() == (1 if (cand & ~np.isnan(conf)).any() else 0)


def test_threshold_unmask_invariants_over_a_block():
    for seed in range(20):
        u = synth.unmask_case(batch=3, seq_len=96, block_start=32, block_len=32, seed=seed)
        x, m = u.x.copy(), u.masked.copy()
        g = synth.rng(seed + 500)
        steps = 0
        tau = [0.0, 0.7, 0.9, 1.0][seed % 4]
        while (m[:, 32:64] != 0).any():
            conf = g.uniform(0, 1, (3, 32)).astype(np.float32)
            tok = g.integers(0, u.mask_id, (3, 32)).astype(np.int32)
            x2, m2, rem, nd = O.threshold_unmask(x, m, conf, tok, 32, 32, tau)
            for b in range(3):
                before = int(m[b, 32:64].sum())
                if before:
                    assert nd[b] >= 1
                    if tau == 1.0:
                        assert nd[b] == 1
                    if tau == 0.0:
                        assert nd[b] == before
                assert rem[b] == before - nd[b] == int(m2[b, 32:64].sum())
            # decoded positions never re-masked, their tokens never change
            assert not ((m == 0) & (m2 != 0)).any()
            assert np.array_equal(x2[m == 0], x[m == 0])
            # only the current block changes
            assert np.array_equal(x2[:, :32], x[:, :32]) and np.array_equal(x2[:, 64:], x[:, 64:])
            # newly decoded positions hold the step's tokens
            newly = (m != 0) & (m2 == 0)
            bi, pi = np.nonzero(newly)
            assert np.array_equal(x2[bi, pi], tok[bi, pi - 32])
            x, m = x2, m2
            steps += 1
            assert steps <= 32


# ---------------------------------------------------------------- decode loops
def _tiny_model(n_layers, seed, **kw):
    return synth.model_params(vocab=64, hidden=32, n_layers=n_layers, n_q_heads=4,
                              head_dim=8, ffn=48, seed=seed, **kw)


def test_dualcache_block_step_equals_full_forward_when_cache_current():
    """With the cache holding the K/V of the current sequence, the DualCache
    block step reproduces the full bidirectional forward on the block rows,
    for any depth (each layer's block inputs are then the same)."""
    for n_layers, kvh, bias in [(1, 4, False), (3, 2, True)]:
        P = synth.model_params(vocab=64, hidden=32, n_layers=n_layers, n_q_heads=4,
                               n_kv_heads=kvh, head_dim=8, ffn=48, seed=n_layers,
                               qkv_bias=bias)
        x = synth.rng(11).integers(0, 63, 40)
        x[20:] = P.mask_id
        x[25] = 5
        logits, kv = O.full_forward(P, x)
        caches = [(k.copy(), v.copy()) for k, v in kv]
        lb = O.block_forward(P, x[16:24], 16, caches)
        np.testing.assert_allclose(lb, logits[16:24], rtol=1e-10, atol=1e-10)
        for (k, v), (kc, vc) in zip(kv, caches):
            np.testing.assert_allclose(kc, k, atol=1e-12)
            np.testing.assert_allclose(vc, v, atol=1e-12)


def test_block_step_uses_the_suffix_cache():
    """Perturbing the cached suffix K/V changes the block's logits (the
    suffix is attended, not dropped); perturbing a row the block overwrites
    does not."""
    P = _tiny_model(2, 3)
    x = synth.rng(12).integers(0, 63, 40)
    x[16:] = P.mask_id
    _, kv = O.full_forward(P, x)
    base = O.block_forward(P, x[16:24], 16, [(k.copy(), v.copy()) for k, v in kv])
    c1 = [(k.copy(), v.copy()) for k, v in kv]
    c1[0][1][:, 30, :] += 1.0
    assert np.abs(O.block_forward(P, x[16:24], 16, c1) - base).max() > 1e-6
    c2 = [(k.copy(), v.copy()) for k, v in kv]
    c2[1][0][:, 18, :] += 5.0
    np.testing.assert_allclose(O.block_forward(P, x[16:24], 16, c2), base, atol=1e-12)


@pytest.mark.parametrize("seed", range(4))
def test_tau_one_single_layer_equals_sequential(seed):
    """tau = 1.0: exactly one token per step, and DualCache decoding of a
    one-layer model (where cached K/V depend only on each token's own
    embedding and position) gives the sequential greedy result."""
    P = _tiny_model(1, seed)
    prompt = synth.prompt_ids(seed, 1, 12, P.mask_id)[0]
    a = O.generate_dualcache(P, prompt, 32, block=8, tau=1.0)
    s = O.generate_sequential(P, prompt, 32, block=8)
    assert all(len(d) == 1 for _, d in a.per_step)
    assert a.steps == 32 and a.refreshes == 4
    assert [d for _, d in a.per_step] == [d for _, d in s.per_step]
    np.testing.assert_array_equal(a.x, s.x)


@pytest.mark.parametrize("seed", range(3))
def test_refresh_every_step_equals_no_cache(seed):
    P = _tiny_model(3, 10 + seed)
    prompt = synth.prompt_ids(seed, 1, 10, P.mask_id)[0]
    for tau in (1.0, 0.5):
        a = O.generate_dualcache(P, prompt, 24, block=8, tau=tau, refresh_every_step=True)
        n = O.generate_nocache(P, prompt, 24, block=8, tau=tau)
        assert [d for _, d in a.per_step] == [d for _, d in n.per_step]
        np.testing.assert_array_equal(a.x, n.x)
        if tau == 1.0:
            s = O.generate_sequential(P, prompt, 24, block=8)
            np.testing.assert_array_equal(a.x, s.x)


def test_parallel_decode_progress_and_blocks_left_to_right():
    P = _tiny_model(2, 21)
    prompt = synth.prompt_ids(21, 1, 8, P.mask_id)[0]
    tr = O.generate_dualcache(P, prompt, 32, block=8, tau=0.5)
    seen = set()
    last_blk = 0
    per_blk = {}
    for blk, dec in tr.per_step:
        assert len(dec) >= 1
        assert blk >= last_blk
        last_blk = blk
        for p in dec:
            assert 8 + 8 * blk <= p < 16 + 8 * blk
            assert p not in seen
            seen.add(p)
        per_blk[blk] = per_blk.get(blk, 0) + 1
    assert seen == set(range(8, 40))
    assert all(v <= 8 for v in per_blk.values())
    assert tr.refreshes == 4
    assert tr.steps < 32          # some steps decoded more than one token


# ---------------------------------------------------------------- PrefixCache
def test_prefix_step_equals_full_forward_when_cache_current():
    """With the cache holding the K/V of the current sequence, the PrefixCache
    step (block and suffix recomputed over the cached prefix) reproduces the
    full bidirectional forward on every row from the block start on, for any
    depth, and leaves the cache as the full forward computed it."""
    for n_layers, kvh, bias in [(1, 4, False), (3, 2, True)]:
        P = synth.model_params(vocab=64, hidden=32, n_layers=n_layers, n_q_heads=4,
                               n_kv_heads=kvh, head_dim=8, ffn=48, seed=20 + n_layers,
                               qkv_bias=bias)
        x = synth.rng(13).integers(0, 63, 40)
        x[20:] = P.mask_id
        x[27] = 9
        logits, kv = O.full_forward(P, x)
        caches = [(k.copy(), v.copy()) for k, v in kv]
        lp = O.prefix_forward(P, x[16:], 16, caches)
        assert lp.shape == (24, 64)
        np.testing.assert_allclose(lp, logits[16:], rtol=1e-10, atol=1e-10)
        for (k, v), (kc, vc) in zip(kv, caches):
            np.testing.assert_allclose(kc, k, atol=1e-12)
            np.testing.assert_allclose(vc, v, atol=1e-12)


def test_prefix_step_reads_only_the_prefix_cache():
    """The PrefixCache step attends over the cached prefix (perturbing a
    prefix row changes the block's logits) and recomputes everything from the
    block start on (perturbing a cached block or suffix row changes nothing),
    unlike the DualCache step, which reads the cached suffix."""
    P = _tiny_model(2, 4)
    x = synth.rng(14).integers(0, 63, 40)
    x[16:] = P.mask_id
    _, kv = O.full_forward(P, x)
    fresh = lambda: [(k.copy(), v.copy()) for k, v in kv]
    base = O.prefix_forward(P, x[16:], 16, fresh())
    c1 = fresh()
    c1[0][0][:, 5, :] += 1.0                       # prefix row
    assert np.abs(O.prefix_forward(P, x[16:], 16, c1) - base).max() > 1e-6
    c2 = fresh()
    c2[1][1][:, 30, :] += 5.0                      # suffix row: recomputed
    c2[0][0][:, 18, :] -= 3.0                      # block row: recomputed
    np.testing.assert_allclose(O.prefix_forward(P, x[16:], 16, c2), base, atol=1e-12)


@pytest.mark.parametrize("seed", range(3))
def test_prefix_cache_single_layer_equals_no_cache(seed):
    """One layer: the cached prefix K/V depend only on the prefix tokens and
    positions, which do not change inside a block, so PrefixCache decoding
    equals decoding without a cache, step for step, for any threshold; at
    tau = 1 both equal the sequential greedy decode."""
    P = _tiny_model(1, 30 + seed)
    prompt = synth.prompt_ids(40 + seed, 1, 12, P.mask_id)[0]
    for tau in (1.0, 0.5, 0.05):
        a = O.generate_prefixcache(P, prompt, 24, block=8, tau=tau)
        n = O.generate_nocache(P, prompt, 24, block=8, tau=tau)
        assert [d for _, d in a.per_step] == [d for _, d in n.per_step]
        np.testing.assert_array_equal(a.x, n.x)
        assert a.refreshes == 3
        if tau == 1.0:
            s = O.generate_sequential(P, prompt, 24, block=8)
            np.testing.assert_array_equal(a.x, s.x)
