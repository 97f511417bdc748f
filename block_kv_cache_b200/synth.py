"""Seeded synthetic inputs for the Fast-dLLM block-decoding step.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests. It holds random draws and the host-side bf16 rounding of those
draws only: none of the method's arithmetic (attention, softmax, confidence,
threshold selection) lives here, so it cannot make the two sides agree by
construction.

Every generator takes a seed and uses NumPy's PCG64, so a case is reproduced
bit for bit on any host. bf16 tensors are produced by round-to-nearest-even
of a float32 draw on the host; the GPU receives the 16-bit patterns and the
oracle receives the same values widened to float64, so both sides start from
identical numbers.

Shapes and distributions follow the workloads the Fast-dLLM pages evaluate
(LLaDA-8B / Dream-7B shapes, block size 32, threshold 0.9): the pages' own
datasets (GSM8K, HumanEval, ...) and trained weights are not available, so
these seeded draws stand in for them.
"""
from __future__ import annotations

import os
from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "rng", "bf16_bits", "bf16_value", "AttnCase", "attn_case", "LMHeadCase",
    "lmhead_case", "UnmaskCase", "unmask_case", "StepCase", "step_case",
    "ModelParams", "model_params", "prompt_ids",
]


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest, ties to even.
    Inputs are finite (the draws here never produce NaN)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_value(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> the float32 numbers they encode (exact)."""
    u = bits.astype(np.uint32) << 16
    return u.view(np.float32)


_CHUNK = 1 << 22


def _fill(seed, n, std, dtype):
    a = rng(int(seed)).standard_normal(n, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    if dtype == "bf16":
        a = bf16_value(bf16_bits(a))
    return a


def _draw(g: np.random.Generator, shape, std: float, dtype: str) -> np.ndarray:
    """Gaussian draw N(0, std^2) as float32 values exactly representable in
    `dtype` ("f32" or "bf16"). Large draws are split into fixed 4 Mi-element
    chunks, each from its own PCG64 stream seeded by `g`, and filled on a
    thread pool; the result depends only on `g`'s state and the shape."""
    n = int(np.prod(shape))
    nch = max(1, (n + _CHUNK - 1) // _CHUNK)
    seeds = g.integers(0, 2**63 - 1, nch)
    if nch == 1:
        return _fill(seeds[0], n, std, dtype).reshape(shape)
    from concurrent.futures import ThreadPoolExecutor
    sizes = [min(_CHUNK, n - i * _CHUNK) for i in range(nch)]
    with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
        parts = list(ex.map(lambda i: _fill(seeds[i], sizes[i], std, dtype), range(nch)))
    return np.concatenate(parts).reshape(shape)


# ---------------------------------------------------------------------------
# attention (one layer, one block step)
# ---------------------------------------------------------------------------
@dataclass
class AttnCase:
    dtype: str                 # "f32" | "bf16"
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    seq_len: int
    block_start: int
    block_len: int
    q: np.ndarray              # [b, B, Hq, d] float32 (values exact in dtype)
    k_cache: np.ndarray        # [b, Hkv, L, d]
    v_cache: np.ndarray        # [b, Hkv, L, d]
    k_blk: np.ndarray          # [b, B, Hkv, d]  fresh block keys (token-major)
    v_blk: np.ndarray          # [b, B, Hkv, d]


def attn_case(*, batch=1, n_q_heads=4, n_kv_heads=None, head_dim=64,
              prefix=64, block=32, suffix=32, dtype="f32", seed=0,
              std=None) -> AttnCase:
    """One DualCache attention step: a cache of length prefix+block+suffix whose
    block slot holds stale values, plus fresh block K/V to be stored there."""
    n_kv_heads = n_kv_heads or n_q_heads
    if std is None:
        std = 1.0 / 8.0 if dtype == "f32" else 1.0
    g = rng(seed)
    L = prefix + block + suffix
    q = _draw(g, (batch, block, n_q_heads, head_dim), std, dtype)
    k = _draw(g, (batch, n_kv_heads, L, head_dim), std, dtype)
    v = _draw(g, (batch, n_kv_heads, L, head_dim), std, dtype)
    kb = _draw(g, (batch, block, n_kv_heads, head_dim), std, dtype)
    vb = _draw(g, (batch, block, n_kv_heads, head_dim), std, dtype)
    return AttnCase(dtype, batch, n_q_heads, n_kv_heads, head_dim, L, prefix,
                    block, q, k, v, kb, vb)


# ---------------------------------------------------------------------------
# LM head + confidence
# ---------------------------------------------------------------------------
@dataclass
class LMHeadCase:
    dtype: str
    rows: int
    hidden: int
    vocab: int
    mask_id: int
    h: np.ndarray              # [M, D]
    w: np.ndarray              # [V, D]
    bias_tok: np.ndarray       # [M] int32, planted token per row (never mask_id)
    bias_val: np.ndarray       # [M] float32


def lmhead_case(*, rows=32, hidden=4096, vocab=126464, dtype="bf16", seed=0,
                h_std=1.0, w_std=0.02, bias_hi=16.0, mask_id=None,
                w_seed=None) -> LMHeadCase:
    """Rows of hidden states against a vocab projection, with one planted logit
    bias per row so that confidences spread across (0, 1).

    `w_seed` lets several cases share one weight matrix (the weight is drawn
    from its own stream)."""
    mask_id = vocab - 1 if mask_id is None else mask_id
    g = rng(seed)
    gw = rng(seed if w_seed is None else w_seed + 7919)
    h = _draw(g, (rows, hidden), h_std, dtype)
    w = _draw(gw, (vocab, hidden), w_std, dtype)
    tok = g.integers(0, vocab - 1, rows).astype(np.int32)
    tok[tok >= mask_id] += 1            # skip the mask id: range [0, V) \ {mask}
    val = g.uniform(0.0, bias_hi, rows).astype(np.float32)
    return LMHeadCase(dtype, rows, hidden, vocab, mask_id, h, w, tok, val)


# ---------------------------------------------------------------------------
# threshold select + scatter
# ---------------------------------------------------------------------------
@dataclass
class UnmaskCase:
    batch: int
    seq_len: int
    block_start: int
    block_len: int
    mask_id: int
    x: np.ndarray              # [b, L] int32
    masked: np.ndarray         # [b, L] uint8
    conf: np.ndarray           # [b, B] float32 (one slot per block position)
    tok: np.ndarray            # [b, B] int32


def unmask_case(*, batch=1, seq_len=128, block_start=64, block_len=32,
                vocab=1024, mask_id=None, seed=0, p_masked=0.75,
                ties=True) -> UnmaskCase:
    """Sequences whose suffix from `block_start` is fully masked and whose
    current block is partly decoded; random confidences with planted ties and
    values on common thresholds."""
    mask_id = vocab - 1 if mask_id is None else mask_id
    g = rng(seed)
    L, s, B = seq_len, block_start, block_len
    x = g.integers(0, mask_id, (batch, L)).astype(np.int32)
    masked = np.zeros((batch, L), np.uint8)
    masked[:, s:] = 1
    blk = (g.uniform(size=(batch, B)) < p_masked).astype(np.uint8)
    for b in range(batch):
        if blk[b].sum() == 0:
            blk[b, g.integers(0, B)] = 1
    masked[:, s:s + B] = blk
    x[masked == 1] = mask_id
    conf = g.uniform(0.0, 1.0, (batch, B)).astype(np.float32)
    if ties:
        special = np.array([0.9, 0.7, 1.0, 0.5], np.float32)
        pick = g.uniform(size=(batch, B)) < 0.15
        conf[pick] = special[g.integers(0, 4, pick.sum())]
        # duplicate the row maximum somewhere else to create argmax ties
        for b in range(batch):
            if g.uniform() < 0.5:
                j = g.integers(0, B)
                conf[b, j] = conf[b].max()
    tok = g.integers(0, mask_id, (batch, B)).astype(np.int32)
    return UnmaskCase(batch, L, s, B, mask_id, x, masked, conf, tok)


# ---------------------------------------------------------------------------
# tiny end-to-end block step: attention -> LM head -> select
# ---------------------------------------------------------------------------
@dataclass
class StepCase:
    attn: AttnCase
    w: np.ndarray              # [V, Hq*d]
    bias_tok: np.ndarray       # [B] per block position
    bias_val: np.ndarray
    unmask: UnmaskCase
    tau: float


def step_case(seed: int, *, dtype="f32", n_heads=4, head_dim=64, prefix=64,
              block=32, suffix=32, vocab=1024, tau=0.9, bias_hi=12.0) -> StepCase:
    """The tiny single-block-step workload: batch 1, one layer, H heads of
    dim d, hidden H*d, cache = prefix + block + suffix, Q/K/V ~ N(0,1)/8,
    an LM head hidden->vocab with W ~ N(0, 0.02) and one planted logit bias
    ~ U(0, bias_hi) per row. The LM-head input is the block's attention output
    with the heads concatenated."""
    a = attn_case(batch=1, n_q_heads=n_heads, head_dim=head_dim, prefix=prefix,
                  block=block, suffix=suffix, dtype=dtype, seed=seed)
    g = rng(10_000 + seed)
    w = _draw(g, (vocab, n_heads * head_dim), 0.02, dtype)
    mask_id = vocab - 1
    bt = g.integers(0, mask_id, block).astype(np.int32)
    bv = g.uniform(0.0, bias_hi, block).astype(np.float32)
    u = unmask_case(batch=1, seq_len=a.seq_len, block_start=prefix,
                    block_len=block, vocab=vocab, mask_id=mask_id,
                    seed=20_000 + seed, ties=False)
    return StepCase(a, w, bt, bv, u, tau)


# ---------------------------------------------------------------------------
# small bidirectional transformer (for decode-loop tests)
# ---------------------------------------------------------------------------
@dataclass
class ModelParams:
    vocab: int
    hidden: int
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    mask_id: int
    rope_theta: float = 10000.0
    rms_eps: float = 1e-5
    qkv_bias: bool = False
    embed: np.ndarray = None             # [V, D]
    layers: list = field(default_factory=list)   # dicts of arrays
    final_norm: np.ndarray = None        # [D]
    lm_head: np.ndarray = None           # [V, D]


def model_params(*, vocab=64, hidden=32, n_layers=1, n_q_heads=4,
                 n_kv_heads=None, head_dim=8, ffn=64, seed=0, dtype="f32",
                 qkv_bias=False, w_std=None, embed_std=1.0,
                 lm_std=None) -> ModelParams:
    """Random-init weights for a pre-norm bidirectional transformer of the
    LLaDA / Dream family. The mask id is vocab - 1. Linear weights are stored
    [out, in] (K-major for the GEMM that consumes them)."""
    n_kv_heads = n_kv_heads or n_q_heads
    g = rng(seed)
    std = w_std if w_std is not None else 1.0 / np.sqrt(hidden)
    P = ModelParams(vocab, hidden, n_layers, n_q_heads, n_kv_heads, head_dim,
                    ffn, vocab - 1, qkv_bias=qkv_bias)
    P.embed = _draw(g, (vocab, hidden), embed_std, dtype)
    for _ in range(n_layers):
        L = dict(
            attn_norm=np.ones(hidden, np.float32),
            wq=_draw(g, (n_q_heads * head_dim, hidden), std, dtype),
            wk=_draw(g, (n_kv_heads * head_dim, hidden), std, dtype),
            wv=_draw(g, (n_kv_heads * head_dim, hidden), std, dtype),
            wo=_draw(g, (hidden, n_q_heads * head_dim), std, dtype),
            ffn_norm=np.ones(hidden, np.float32),
            wg=_draw(g, (ffn, hidden), std, dtype),
            wu=_draw(g, (ffn, hidden), std, dtype),
            wd=_draw(g, (hidden, ffn), 1.0 / np.sqrt(ffn), dtype),
        )
        if qkv_bias:
            L["bq"] = _draw(g, (n_q_heads * head_dim,), 0.1, dtype)
            L["bk"] = _draw(g, (n_kv_heads * head_dim,), 0.1, dtype)
            L["bv"] = _draw(g, (n_kv_heads * head_dim,), 0.1, dtype)
        P.layers.append(L)
    P.final_norm = np.ones(hidden, np.float32)
    P.lm_head = _draw(g, (vocab, hidden),
                      lm_std if lm_std is not None else 1.0, dtype)
    return P


def prompt_ids(seed: int, batch: int, prompt_len: int, mask_id: int) -> np.ndarray:
    """Uniform random prompt ids, never equal to the mask id."""
    g = rng(seed)
    return g.integers(0, mask_id, (batch, prompt_len)).astype(np.int32)
