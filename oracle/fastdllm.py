"""CPU oracle for the Fast-dLLM block-decoding step.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports, calls, links or
executes this module: only the tests, the smoke check in __graft_entry__ and
the CPU-baseline leg of bench.py do. It shares no code with the CUDA library
(block_kv_cache_b200/csrc) and does not import the package's binding.

Everything here is plain NumPy in float64, written to be read against the
pages one step at a time: loops over sequences, heads and rows, a library
matrix product as the only building block, no blocking, fusion or
reordering. Inputs that the GPU sees as bf16 or fp32 arrive here as the same
numbers widened to float64.

Sources (titles of the pages this follows; sections named per function):
  [abstract]  "Fast-dLLM: Training-free Acceleration of Diffusion LLM by
              Enabling KV Cache and Parallel Decoding" (arXiv 2505.22618v3),
              original English abstract.
  [reviews]   ICLR review page for the same paper (submission 2543).
  [news]      aibase news item on Fast-dLLM, "Innovations in the Fast-dLLM
              Framework", items 1 and 2.
  [readme]    Fast-DLLM README mirror (gittoolsai), "Key techniques" 1-3 and
              the usage flags (--block_size, --use_cache,
              --if_cache_position, --threshold).

Where the pages leave a step open the function says which reading it takes;
the list of readings is kept with the design notes.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

F64 = np.float64


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=F64)


def tau_as_single(tau: float) -> float:
    """The threshold is carried as an IEEE single, as the C-ABI takes it."""
    return float(np.float32(tau))


# ---------------------------------------------------------------------------
# transformer pieces of the LLaDA / Dream family (scaffold, not the method)
# ---------------------------------------------------------------------------
def rms_norm(x, g, eps=1e-5):
    """y = x / sqrt(mean(x^2) + eps) * g over the last axis."""
    x = _f64(x)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * _f64(g)


def rope_angles(positions, head_dim, theta=10000.0):
    """Angle pos * theta^(-2i/d) for i in [0, d/2): [n, d/2]."""
    i = np.arange(head_dim // 2, dtype=F64)
    inv = theta ** (-2.0 * i / head_dim)
    return np.outer(_f64(positions), inv)


def apply_rope(x, positions, theta=10000.0):
    """Rotary embedding, rotate-half convention: the pair (x_i, x_{i+d/2}) is
    rotated by angle pos * theta^(-2i/d). x: [n, H, d] with row r at
    positions[r]."""
    x = _f64(x)
    d = x.shape[-1]
    ang = rope_angles(positions, d, theta)[:, None, :]       # [n, 1, d/2]
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., : d // 2], x[..., d // 2:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def silu(x):
    x = _f64(x)
    return x / (1.0 + np.exp(-x))


# ---------------------------------------------------------------------------
# (a2) DualCache block attention
# ---------------------------------------------------------------------------
def attention(q, k, v, scale=None):
    """Bidirectional (unmasked) attention of one sequence.

    q: [Bq, Hq, d] query rows (token-major); k, v: [Hkv, L, d].
    Head h reads kv head h // (Hq / Hkv) (contiguous GQA groups).
    Returns o [Bq, Hq, d] and lse [Hq, Bq] (natural log of the softmax
    denominator, scores included).

    Masked diffusion LLMs attend bidirectionally ([abstract]; [news],
    "Challenges": every position sees every other), so there is no mask.
    Scale 1/sqrt(d) is the standard choice (not stated on the pages).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    Bq, Hq, d = q.shape
    Hkv = k.shape[0]
    assert Hq % Hkv == 0
    grp = Hq // Hkv
    scale = 1.0 / math.sqrt(d) if not scale else float(scale)
    o = np.zeros((Bq, Hq, d))
    lse = np.zeros((Hq, Bq))
    for h in range(Hq):
        kh, vh = k[h // grp], v[h // grp]
        s = (q[:, h, :] @ kh.T) * scale                        # [Bq, L]
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        den = p.sum(axis=1, keepdims=True)
        o[:, h, :] = (p / den) @ vh
        lse[h] = m[:, 0] + np.log(den[:, 0])
    return o, lse


def kv_store(k_cache, v_cache, k_new, v_new, start):
    """Write fresh K/V rows into the cache in place.

    k_cache, v_cache: [b, Hkv, L, d]; k_new, v_new: [b, n, Hkv, d]
    (token-major, as a projection produces them); rows [start, start+n).
    Used for the block slot at every step and, with n = L, for the refresh
    after a block completes ([reviews], review 4 question 2: all K/V are
    recomputed once a block is done)."""
    n = k_new.shape[1]
    k_cache[:, :, start:start + n, :] = np.transpose(k_new, (0, 2, 1, 3))
    v_cache[:, :, start:start + n, :] = np.transpose(v_new, (0, 2, 1, 3))


def dualcache_attention(q, k_cache, v_cache, scale=None):
    """DualCache block step ([news], Innovations 1; [readme], Key techniques 1):
    the block's queries attend over [cached prefix | block | cached masked
    suffix], i.e. over the whole cache whose block slot holds the block's
    fresh K/V (written by kv_store beforehand).

    q: [b, B, Hq, d]; caches: [b, Hkv, L, d].
    Returns o [b, B, Hq, d] and lse [b, Hq, B]."""
    b = q.shape[0]
    outs, lses = [], []
    for i in range(b):
        o, lse = attention(q[i], k_cache[i], v_cache[i], scale)
        outs.append(o)
        lses.append(lse)
    return np.stack(outs), np.stack(lses)


# ---------------------------------------------------------------------------
# (a4) LM head + confidence
# ---------------------------------------------------------------------------
@dataclass
class Confidence:
    conf: np.ndarray      # [M] max softmax probability
    tok: np.ndarray       # [M] lowest id among the maximal logits
    zmax: np.ndarray      # [M] maximal logit
    lse: np.ndarray       # [M] log-sum-exp of the logits
    gap: np.ndarray       # [M] maximal logit minus the second largest logit


def confidence_from_logits(z) -> Confidence:
    """Per row: confidence = the largest softmax probability,
    exp(max z - LSE(z)) = 1 / sum_v exp(z_v - max z); token = argmax z,
    lowest id on ties.

    The pages decode "tokens exceeding a confidence threshold" ([abstract];
    [readme], Key techniques 2) without defining confidence; the plainest
    reading of a per-token scalar compared with a threshold in (0, 1] is the
    probability of the predicted token."""
    z = _f64(z)
    zmax = z.max(axis=1)
    tok = np.argmax(z, axis=1)            # first (lowest) index of the max
    den = np.exp(z - zmax[:, None]).sum(axis=1)
    conf = 1.0 / den
    lse = zmax + np.log(den)
    srt = np.sort(z, axis=1)
    gap = srt[:, -1] - srt[:, -2] if z.shape[1] > 1 else np.full(len(z), np.inf)
    return Confidence(conf, tok.astype(np.int64), zmax, lse, gap)


def lm_logits(h, w, bias_tok=None, bias_val=None, vocab_chunk=16384):
    """z = h W^T (+ one planted bias per row at bias_tok[r]) in float64.
    The product is formed vocab-chunk by vocab-chunk only to bound host
    memory; each logit is the same dot product either way."""
    h = _f64(h)
    V = w.shape[0]
    z = np.empty((h.shape[0], V))
    for v0 in range(0, V, vocab_chunk):
        z[:, v0:v0 + vocab_chunk] = h @ _f64(w[v0:v0 + vocab_chunk]).T
    if bias_tok is not None:
        r = np.arange(h.shape[0])
        z[r, np.asarray(bias_tok)] += _f64(bias_val)
    return z


def lmhead_confidence(h, w, bias_tok=None, bias_val=None, row_chunk=256) -> Confidence:
    """Fused stage (b) of the step, unfused here: logits for the block's
    masked rows, then max / LSE / argmax over the vocabulary. Rows are
    independent, so they are processed in groups to bound host memory."""
    parts = []
    M = h.shape[0]
    for r0 in range(0, M, row_chunk):
        sl = slice(r0, r0 + row_chunk)
        bt = None if bias_tok is None else np.asarray(bias_tok)[sl]
        bv = None if bias_val is None else np.asarray(bias_val)[sl]
        parts.append(confidence_from_logits(lm_logits(h[sl], w, bt, bv)))
    cat = lambda n: np.concatenate([getattr(p, n) for p in parts])
    return Confidence(cat("conf"), cat("tok"), cat("zmax"), cat("lse"), cat("gap"))


# ---------------------------------------------------------------------------
# (a5) confidence-aware parallel unmask: threshold select + scatter
# ---------------------------------------------------------------------------
def select_positions(conf, candidate, tau):
    """Which block positions to decode this step.

    conf: [B] confidences, candidate: [B] bool (masked positions of the
    current block). Rule ([abstract]; [readme], Key techniques 2; [news],
    Innovations 2): decode every candidate whose confidence exceeds tau
    (strictly greater); the others stay masked for later steps. If no
    candidate exceeds tau, decode the single most confident candidate, the
    lowest position on ties, so that every step makes progress. A NaN
    confidence is never selected. Returns a [B] bool array."""
    conf = _f64(conf)
    cand = np.asarray(candidate, bool)
    t = tau_as_single(tau)
    sel = np.zeros(len(conf), bool)
    for i in range(len(conf)):
        if cand[i] and conf[i] > t:
            sel[i] = True
    if sel.any() or not cand.any():
        return sel
    best = -1
    for i in range(len(conf)):
        if cand[i] and not np.isnan(conf[i]):
            if best < 0 or conf[i] > conf[best]:
                best = i
    if best >= 0:
        sel[best] = True
    return sel


def threshold_unmask(x, masked, conf, tok, block_start, block_len, tau):
    """Apply one unmask step to a batch, returning new arrays.

    x: [b, L] token ids, masked: [b, L] 0/1, conf/tok: [b, B] with slot i
    describing position block_start + i (slots of unmasked positions are
    ignored). Selected positions receive their token and leave the mask;
    decoded positions are never re-masked. Returns (x, masked, remaining,
    n_decoded) with remaining = masked positions left in the block."""
    x = np.array(x, copy=True)
    masked = np.array(masked, copy=True)
    b = x.shape[0]
    s, B = block_start, block_len
    remaining = np.zeros(b, np.int64)
    ndec = np.zeros(b, np.int64)
    for i in range(b):
        cand = masked[i, s:s + B] != 0
        sel = select_positions(conf[i, :B], cand, tau)
        for j in range(B):
            if sel[j]:
                x[i, s + j] = tok[i, j]
                masked[i, s + j] = 0
        ndec[i] = sel.sum()
        remaining[i] = int((masked[i, s:s + B] != 0).sum())
    return x, masked, remaining, ndec


# ---------------------------------------------------------------------------
# the model forward: full (no cache / refresh) and cached block step
# ---------------------------------------------------------------------------
def _layer_qkv(P, Lw, hn, positions):
    """q [n, Hq, d], k/v [n, Hkv, d] for normalised hidden rows hn [n, D]."""
    n = hn.shape[0]
    q = hn @ _f64(Lw["wq"]).T
    k = hn @ _f64(Lw["wk"]).T
    v = hn @ _f64(Lw["wv"]).T
    if P.qkv_bias:
        q = q + _f64(Lw["bq"])
        k = k + _f64(Lw["bk"])
        v = v + _f64(Lw["bv"])
    q = q.reshape(n, P.n_q_heads, P.head_dim)
    k = k.reshape(n, P.n_kv_heads, P.head_dim)
    v = v.reshape(n, P.n_kv_heads, P.head_dim)
    q = apply_rope(q, positions, P.rope_theta)
    k = apply_rope(k, positions, P.rope_theta)
    return q, k, v


def _layer_rest(P, Lw, h, o):
    """Output projection + residual, then the SwiGLU FFN + residual."""
    n = h.shape[0]
    h = h + o.reshape(n, -1) @ _f64(Lw["wo"]).T
    f = rms_norm(h, Lw["ffn_norm"], P.rms_eps)
    g = f @ _f64(Lw["wg"]).T
    u = f @ _f64(Lw["wu"]).T
    return h + (silu(g) * u) @ _f64(Lw["wd"]).T


def _embed_rows(P, ids):
    """f64 embedding rows of `ids` (the rows are picked before widening: the
    values are the same, the table is not copied)."""
    return _f64(np.asarray(P.embed)[np.asarray(ids)])


def full_hidden(P, ids):
    """No-cache forward of one sequence ids [L]: every position attends to
    every position ([news], "Challenges": without a cache all attention
    states are recomputed at every step).
    Returns the final-norm hidden rows [L, D] and per-layer (k, v) as
    [Hkv, L, d]."""
    L = len(ids)
    pos = np.arange(L)
    h = _embed_rows(P, ids)
    kv = []
    for Lw in P.layers:
        hn = rms_norm(h, Lw["attn_norm"], P.rms_eps)
        q, k, v = _layer_qkv(P, Lw, hn, pos)
        kt, vt = np.transpose(k, (1, 0, 2)), np.transpose(v, (1, 0, 2))
        kv.append((kt.copy(), vt.copy()))
        o, _ = attention(q, kt, vt)
        h = _layer_rest(P, Lw, h, o)
    return rms_norm(h, P.final_norm, P.rms_eps), kv


def full_forward(P, ids):
    """full_hidden followed by the LM head: logits [L, V] and the per-layer
    (k, v)."""
    hf, kv = full_hidden(P, ids)
    return lm_logits(hf, P.lm_head), kv


def block_hidden(P, blk_ids, block_start, caches):
    """DualCache step of one sequence: only the block's tokens go through the
    layers; at each layer their fresh K/V overwrite the cache's block slot and
    the block attends over the whole cache ([news], Innovations 1: prefix and
    suffix K/V are reused from the cache; [readme], Key techniques 1).
    caches: list of (k, v) [Hkv, L, d] per layer, updated in place.
    Returns the final-norm hidden rows [B, D] of the block."""
    B = len(blk_ids)
    pos = np.arange(block_start, block_start + B)
    h = _embed_rows(P, blk_ids)
    for Lw, (kc, vc) in zip(P.layers, caches):
        hn = rms_norm(h, Lw["attn_norm"], P.rms_eps)
        q, k, v = _layer_qkv(P, Lw, hn, pos)
        kc[:, block_start:block_start + B, :] = np.transpose(k, (1, 0, 2))
        vc[:, block_start:block_start + B, :] = np.transpose(v, (1, 0, 2))
        o, _ = attention(q, kc, vc)
        h = _layer_rest(P, Lw, h, o)
    return rms_norm(h, P.final_norm, P.rms_eps)


def block_forward(P, blk_ids, block_start, caches):
    """block_hidden followed by the LM head: logits [B, V] of the block rows."""
    return lm_logits(block_hidden(P, blk_ids, block_start, caches), P.lm_head)


def prefix_hidden(P, tail_ids, start, caches):
    """PrefixCache step of one sequence (the cache without the DualCache
    extension: [readme], usage flags --use_cache without
    --if_cache_position; [news], Innovations 1 describes DualCache as the
    version that also caches the suffix). Only the prefix [0, start) is
    taken from the cache: every position from the block start to the end
    (the block and the masked suffix, tail_ids [L - start]) goes through the
    layers, its fresh K/V overwrite cache rows [start, L), and those rows
    attend over the whole cache [cached prefix | fresh block and suffix].
    caches: list of (k, v) [Hkv, L, d] per layer, updated in place.
    Returns the final-norm hidden rows [L - start, D]; the block's are the
    first B of them."""
    n = len(tail_ids)
    pos = np.arange(start, start + n)
    h = _embed_rows(P, tail_ids)
    for Lw, (kc, vc) in zip(P.layers, caches):
        assert kc.shape[1] == start + n
        hn = rms_norm(h, Lw["attn_norm"], P.rms_eps)
        q, k, v = _layer_qkv(P, Lw, hn, pos)
        kc[:, start:, :] = np.transpose(k, (1, 0, 2))
        vc[:, start:, :] = np.transpose(v, (1, 0, 2))
        o, _ = attention(q, kc, vc)
        h = _layer_rest(P, Lw, h, o)
    return rms_norm(h, P.final_norm, P.rms_eps)


def prefix_forward(P, tail_ids, start, caches):
    """prefix_hidden followed by the LM head: logits [L - start, V]."""
    return lm_logits(prefix_hidden(P, tail_ids, start, caches), P.lm_head)


# ---------------------------------------------------------------------------
# decode loops
# ---------------------------------------------------------------------------
@dataclass
class DecodeTrace:
    x: np.ndarray                      # final ids [L]
    steps: int = 0                     # forward passes that produced logits
    refreshes: int = 0                 # full forwards that rewrote the caches
    per_step: list = field(default_factory=list)   # (block, positions decoded)


def _step_select(x, masked, logits_blk, s, B, tau):
    c = confidence_from_logits(logits_blk)
    cand = masked[s:s + B] != 0
    sel = select_positions(c.conf, cand, tau)
    dec = []
    for j in range(B):
        if sel[j]:
            x[s + j] = int(c.tok[j])
            masked[s + j] = 0
            dec.append(s + j)
    return dec


def generate_dualcache(P, prompt, gen_len, block=32, tau=0.9,
                       refresh_every_step=False, cache="dual") -> DecodeTrace:
    """Fast-dLLM block decoding of one sequence with a block-wise K/V cache
    and the confidence-aware threshold rule.

    The generated region (gen_len mask tokens after the prompt) is split into
    blocks of `block` positions, decoded left to right ([news], Innovations 1;
    [readme], --block_size). For each block: one full forward computes every
    position's K/V (the refresh) and also gives the logits of the block's
    first step; then cached block steps run until the block has no masked
    position; after the block completes the next block's refresh rewrites all
    K/V ([reviews], review 4 question 2). No refresh follows the last block.
    cache="dual": a cached step recomputes only the block and reuses the
    cached prefix and masked-suffix K/V (DualCache, block_forward);
    cache="prefix": it recomputes the block and the suffix and reuses the
    cached prefix only (prefix_forward).
    With refresh_every_step the cache is rebuilt before every step."""
    assert gen_len % block == 0 and cache in ("dual", "prefix")
    Lp = len(prompt)
    x = np.concatenate([np.asarray(prompt), np.full(gen_len, P.mask_id)]).astype(np.int64)
    masked = np.zeros(len(x), np.int8)
    masked[Lp:] = 1
    tr = DecodeTrace(x)
    for blk in range(gen_len // block):
        s = Lp + blk * block
        logits, kv = full_forward(P, x)
        tr.refreshes += 1
        caches = [(k.copy(), v.copy()) for k, v in kv]
        dec = _step_select(x, masked, logits[s:s + block], s, block, tau)
        tr.steps += 1
        tr.per_step.append((blk, dec))
        while (masked[s:s + block] != 0).any():
            if refresh_every_step:
                logits, kv = full_forward(P, x)
                tr.refreshes += 1
                lg = logits[s:s + block]
            elif cache == "dual":
                lg = block_forward(P, x[s:s + block], s, caches)
            else:
                lg = prefix_forward(P, x[s:], s, caches)[:block]
            dec = _step_select(x, masked, lg, s, block, tau)
            assert len(dec) >= 1
            tr.steps += 1
            tr.per_step.append((blk, dec))
    tr.x = x
    return tr


def generate_prefixcache(P, prompt, gen_len, block=32, tau=0.9) -> DecodeTrace:
    """Block decoding with the PrefixCache: generate_dualcache(cache="prefix")."""
    return generate_dualcache(P, prompt, gen_len, block, tau, cache="prefix")


def generate_nocache(P, prompt, gen_len, block=32, tau=0.9) -> DecodeTrace:
    """Parallel decoding without any cache: a full forward at every step,
    threshold rule on the current block (the "+parallel" variant of the
    README's evaluation table)."""
    Lp = len(prompt)
    x = np.concatenate([np.asarray(prompt), np.full(gen_len, P.mask_id)]).astype(np.int64)
    masked = np.zeros(len(x), np.int8)
    masked[Lp:] = 1
    tr = DecodeTrace(x)
    for blk in range(gen_len // block):
        s = Lp + blk * block
        while (masked[s:s + block] != 0).any():
            logits, _ = full_forward(P, x)
            dec = _step_select(x, masked, logits[s:s + block], s, block, tau)
            tr.steps += 1
            tr.per_step.append((blk, dec))
    tr.x = x
    return tr


def generate_sequential(P, prompt, gen_len, block=32) -> DecodeTrace:
    """Sequential greedy decoding: no cache, a full forward per step, and
    exactly one token per step, the most confident masked position of the
    current block (lowest position on ties), decoded with its argmax token.
    This is the one-token-per-step baseline the equivalence result of the
    paper compares greedy parallel decoding against ([reviews], reviews 1
    and 2, Theorem 1)."""
    Lp = len(prompt)
    x = np.concatenate([np.asarray(prompt), np.full(gen_len, P.mask_id)]).astype(np.int64)
    masked = np.zeros(len(x), np.int8)
    masked[Lp:] = 1
    tr = DecodeTrace(x)
    for blk in range(gen_len // block):
        s = Lp + blk * block
        for _ in range(block):
            logits, _ = full_forward(P, x)
            c = confidence_from_logits(logits[s:s + block])
            best = -1
            for j in range(block):
                if masked[s + j] and (best < 0 or c.conf[j] > c.conf[best]):
                    best = j
            x[s + best] = int(c.tok[best])
            masked[s + best] = 0
            tr.steps += 1
            tr.per_step.append((blk, [s + best]))
    tr.x = x
    return tr
