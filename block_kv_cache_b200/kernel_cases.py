"""Run one library call repeatedly on seeded synthetic input and time it.

    python -m block_kv_cache_b200.kernel_cases lmhead --rows 32 [--iters 20]
    python -m block_kv_cache_b200.kernel_cases attention --heads 32 --kv-heads 32 \
        --prefix 512 --block 32 --suffix 224 [--layers 32]
    python -m block_kv_cache_b200.kernel_cases swiglu|resid|qkv --rows 32 --n 24576 --k 4096

Used to profile a single kernel (e.g. under ncu with -k/-c) and to time it
with CUDA events. With --graph the timed calls are captured once in a CUDA
graph and replayed, so host-side launch cost is excluded. Prints one JSON
line: mean µs per call and the achieved algorithmic bandwidth / throughput.
"""
from __future__ import annotations

import argparse
import json

import numpy as np
import torch

from block_kv_cache_b200 import fdllm, synth


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).cuda()


def _timed(a, call):
    """Mean µs per call of call(i) over a.iters calls (graph-replayed with --graph)."""
    for i in range(a.warmup):
        call(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if a.graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(a.iters):
                call(i)
        g.replay()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(a.reps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) * 1e3 / (a.iters * a.reps)
    e0.record()
    for i in range(a.iters):
        call(i)
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e3 / a.iters


def run_lmhead(a, ctx):
    c = synth.lmhead_case(rows=a.rows, hidden=a.hidden, vocab=a.vocab, seed=1, w_seed=0,
                          mask_id=min(126336, a.vocab - 1))
    h, w = _bf16(c.h), _bf16(c.w)
    bt, bv = torch.from_numpy(c.bias_tok).cuda(), torch.from_numpy(c.bias_val).cuda()
    conf, tok = ctx.lmhead_confidence(h, w, bt, bv)
    us = _timed(a, lambda i: ctx.lmhead_confidence(h, w, bt, bv, conf=conf, tok=tok))
    ctx.device_status()
    nbytes = a.vocab * a.hidden * 2 + a.rows * a.hidden * 2 + a.rows * 16
    flops = 2.0 * a.rows * a.hidden * a.vocab
    return {"op": "lmhead_confidence", "rows": a.rows, "hidden": a.hidden, "vocab": a.vocab,
            "graph": a.graph, "us": us, "GBps": nbytes / us / 1e3, "TFLOPs": flops / us / 1e6}


def run_attention(a, ctx):
    cases = [synth.attn_case(batch=a.batch, n_q_heads=a.heads, n_kv_heads=a.kv_heads,
                             head_dim=a.head_dim, prefix=a.prefix, block=a.block,
                             suffix=a.suffix, dtype="bf16", seed=l) for l in range(a.layers)]
    q = [_bf16(c.q) for c in cases]
    kc = [_bf16(c.k_cache) for c in cases]
    vc = [_bf16(c.v_cache) for c in cases]
    out = torch.empty_like(q[0])
    s = a.prefix
    us = _timed(a, lambda i: ctx.dualcache_attention(q[i % a.layers], kc[i % a.layers],
                                                     vc[i % a.layers], s, out=out))
    ctx.device_status()
    L = a.prefix + a.block + a.suffix
    nbytes = (2 * a.batch * a.kv_heads * L * a.head_dim * 2
              + 2 * a.batch * a.block * a.heads * a.head_dim * 2)
    flops = 4.0 * a.batch * a.heads * a.block * L * a.head_dim
    return {"op": "dualcache_attention", "heads": a.heads, "kv_heads": a.kv_heads, "L": L,
            "block": a.block, "batch": a.batch, "graph": a.graph, "us": us, "GBps": nbytes / us / 1e3,
            "TFLOPs": flops / us / 1e6}


def run_full(a, ctx):
    """Full bidirectional attention of every position (the refresh forward):
    q [b, L, Hq, d], caches [b, Hkv, L, d], `layers` distinct caches cycled."""
    L = a.prefix + a.block + a.suffix
    g = torch.Generator(device="cuda")
    g.manual_seed(0)
    qs = [torch.randn(a.batch, L, a.heads, a.head_dim, generator=g, device="cuda").to(
        torch.bfloat16) for _ in range(a.layers)]
    ks = [torch.randn(a.batch, a.kv_heads, L, a.head_dim, generator=g, device="cuda").to(
        torch.bfloat16) for _ in range(a.layers)]
    vs = [torch.randn_like(k) for k in ks]
    out = torch.empty_like(qs[0])
    us = _timed(a, lambda i: ctx.full_attention(qs[i % a.layers], ks[i % a.layers],
                                                vs[i % a.layers], out=out))
    ctx.device_status()
    flops = 4.0 * a.batch * a.heads * L * L * a.head_dim
    nbytes = 2 * a.batch * a.kv_heads * L * a.head_dim * 2 + 2 * a.batch * L * a.heads * a.head_dim * 2
    return {"op": "full_attention", "heads": a.heads, "kv_heads": a.kv_heads, "L": L,
            "batch": a.batch, "graph": a.graph, "us": us, "GBps": nbytes / us / 1e3,
            "TFLOPs": flops / us / 1e6}


def run_qkv_attention(a, ctx):
    """The attention half of a cached step: RMSNorm + block-slot projection +
    DualCache attention (`layers` distinct weights and caches cycled)."""
    from block_kv_cache_b200 import fdllm as F
    L = a.prefix + a.block + a.suffix
    Hq, Hkv, d, D = a.heads, a.kv_heads, a.head_dim, a.hidden
    N = (Hq + 2 * Hkv) * d
    rows = a.batch * a.block
    g = torch.Generator(device="cuda")
    g.manual_seed(0)
    ws = [(torch.randn(N, D, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
          for _ in range(a.layers)]
    kc = [torch.randn(a.batch, Hkv, L, d, generator=g, device="cuda").to(torch.bfloat16)
          for _ in range(a.layers)]
    vc = [torch.randn_like(k) for k in kc]
    h = torch.randn(rows, D, generator=g, device="cuda")
    nw = torch.ones(D, device="cuda")
    x = torch.empty((rows, D), dtype=torch.bfloat16, device="cuda")
    q = torch.empty((rows, Hq, d), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((a.batch, a.block, Hq, d), dtype=torch.bfloat16, device="cuda")
    rope = torch.from_numpy(F.rope_table(10000.0, L, d)).cuda()
    us = _timed(a, lambda i: ctx.qkv_attention(x, ws[i % a.layers], rope, q, kc[i % a.layers],
                                               vc[i % a.layers], out, n_q_heads=Hq,
                                               rows_per_seq=a.block, pos0=a.prefix, h=h,
                                               norm_w=nw))
    ctx.device_status()
    nbytes = N * D * 2 + 2 * a.batch * Hkv * L * d * 2 + rows * D * 6 + 2 * rows * Hq * d * 2
    return {"op": "qkv_attention", "rows": rows, "hidden": D, "heads": Hq, "kv_heads": Hkv,
            "L": L, "graph": a.graph, "us": us, "GBps": nbytes / us / 1e3}


def run_linear(a, ctx):
    """One projection of the transformer at (rows, n, k); `layers` distinct weight
    matrices are cycled so the weight stream comes from HBM, not L2."""
    g = torch.Generator(device="cuda")
    g.manual_seed(0)
    ws = [(torch.randn(a.n, a.k, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
          for _ in range(a.layers)]
    x = torch.randn(a.rows, a.k, generator=g, device="cuda").to(torch.bfloat16)
    if a.op == "swiglu":
        out = torch.empty((a.rows, a.n // 2), dtype=torch.bfloat16, device="cuda")
        call = lambda i: ctx.linear_swiglu(x, ws[i % a.layers], out=out)
    elif a.op == "resid":
        h = torch.zeros((a.rows, a.n), dtype=torch.float32, device="cuda")
        call = lambda i: ctx.linear_residual(x, ws[i % a.layers], h)
    else:
        from block_kv_cache_b200 import fdllm as F
        nq = a.heads
        nkv = (a.n // 128 - nq) // 2
        L = 2048
        rope = torch.from_numpy(F.rope_table(10000.0, L, 128)).cuda()
        q = torch.empty((a.rows, nq, 128), dtype=torch.bfloat16, device="cuda")
        kc = torch.zeros((1, nkv, L, 128), dtype=torch.bfloat16, device="cuda")
        vc = torch.zeros_like(kc)
        call = lambda i: ctx.qkv_rope_store(x, ws[i % a.layers], rope, q, kc, vc, n_q_heads=nq,
                                            rows_per_seq=a.rows, pos0=a.prefix)
    us = _timed(a, call)
    ctx.device_status()
    nbytes = a.n * a.k * 2 + a.rows * a.k * 2
    return {"op": a.op, "rows": a.rows, "n": a.n, "k": a.k, "graph": a.graph, "us": us,
            "GBps": nbytes / us / 1e3, "TFLOPs": 2.0 * a.rows * a.n * a.k / us / 1e6}


def run_ffn(a, ctx):
    """The feed-forward call at (rows, hidden = k, ffn = n): gate/up [2n, k] and
    down [k, n] weights, `layers` distinct sets cycled."""
    g = torch.Generator(device="cuda")
    g.manual_seed(0)
    wgu = [(torch.randn(2 * a.n, a.k, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
           for _ in range(a.layers)]
    wd = [(torch.randn(a.k, a.n, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
          for _ in range(a.layers)]
    x = torch.empty((a.rows, a.k), dtype=torch.bfloat16, device="cuda")
    h = torch.randn(a.rows, a.k, generator=g, device="cuda")
    nw = torch.ones(a.k, device="cuda")
    f = torch.empty((a.rows, a.n), dtype=torch.bfloat16, device="cuda")
    # as in a decoder layer: x = RMSNorm(h), h += down(SwiGLU(x))
    us = _timed(a, lambda i: ctx.ffn(x, wgu[i % a.layers], wd[i % a.layers], h, f=f, norm_w=nw))
    ctx.device_status()
    nbytes = 3 * a.n * a.k * 2 + a.rows * a.k * 2 + 2 * a.rows * a.n * 2 + 2 * a.rows * a.k * 4
    return {"op": "ffn", "rows": a.rows, "hidden": a.k, "ffn": a.n, "graph": a.graph, "us": us,
            "GBps": nbytes / us / 1e3, "TFLOPs": 6.0 * a.rows * a.n * a.k / us / 1e6}


TL_EVENTS = {
    "attention": ["entry", "after dependency wait + prologue", "first S MMA issued",
                  "last PV committed", "first P tile written", "epilogue start",
                  "split merge done", "exit"],
    "skinny": ["entry", "after dependency wait", "after prologue barrier", "first MMA issued",
               "last MMA issued", "last epilogue chunk", "-", "exit"],
}
TL_KINDS = {
    "attention": ["DualCache (no prologue)", "DualCache with the q/k/v prologue",
                  "full attention (two 128-row tiles)"],
    "skinny": ["split-K sums with the RMSNorm prologue (q/k/v, gate/up)",
               "down projection with the SwiGLU prologue", "residual (O projection)",
               "split-K sums", "SwiGLU epilogue", "other"],
}


def timeline_summary():
    """Per-CTA event clocks of the last launch of each kernel kind, read from
    the instrumented library (FDLLM_LIB=.../libfdllm_timeline.so): for every
    event, the median / min / max over CTAs of its time after the earliest
    CTA entry of that launch (µs)."""
    import ctypes
    L = fdllm.load()
    K, C, E = 8, 512, 8
    out = {}
    for name in ("attention", "skinny"):
        fn = getattr(L, f"fdl_timeline_{name}", None)
        if fn is None:
            raise RuntimeError("not an instrumented library: set FDLLM_LIB to "
                               "libfdllm_timeline.so")
        buf = (ctypes.c_ulonglong * (K * C * E))()
        if fn(buf) != 0:
            raise RuntimeError("timeline read failed")
        a = np.frombuffer(buf, dtype=np.uint64).reshape(K, C, E).astype(np.int64)
        for k in range(K):
            ctas = np.nonzero(a[k, :, 0])[0]
            if len(ctas) == 0:
                continue
            t0 = a[k, ctas, 0].min()
            ev = {}
            for e in range(E):
                v = a[k, ctas, e]
                v = v[v > 0]
                if len(v):
                    d = (v - t0) / 1e3
                    ev[TL_EVENTS[name][e]] = {"median": round(float(np.median(d)), 2),
                                              "min": round(float(d.min()), 2),
                                              "max": round(float(d.max()), 2), "ctas": int(len(v))}
            kind = TL_KINDS[name][k] if k < len(TL_KINDS[name]) else str(k)
            out[f"{name}: {kind}"] = ev
    return out


def main():
    p = argparse.ArgumentParser()
    p.add_argument("op", choices=["lmhead", "attention", "full", "qkvattn", "swiglu", "resid",
                                  "qkv", "ffn"])
    p.add_argument("--n", type=int, default=24576)
    p.add_argument("--k", type=int, default=4096)
    p.add_argument("--rows", type=int, default=32)
    p.add_argument("--hidden", type=int, default=4096)
    p.add_argument("--vocab", type=int, default=126464)
    p.add_argument("--batch", type=int, default=1)
    p.add_argument("--heads", type=int, default=32)
    p.add_argument("--kv-heads", type=int, default=32)
    p.add_argument("--head-dim", type=int, default=128)
    p.add_argument("--prefix", type=int, default=512)
    p.add_argument("--block", type=int, default=32)
    p.add_argument("--suffix", type=int, default=224)
    p.add_argument("--layers", type=int, default=32)
    p.add_argument("--iters", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--graph", action="store_true", help="replay the timed calls as a CUDA graph")
    p.add_argument("--reps", type=int, default=5, help="graph replays timed (with --graph)")
    p.add_argument("--timeline", action="store_true",
                   help="also print the per-CTA event clocks of the last launch of each "
                        "kernel kind (needs FDLLM_LIB=.../libfdllm_timeline.so)")
    a = p.parse_args()
    ctx = fdllm.Context(0)
    if a.op == "lmhead":
        r = run_lmhead(a, ctx)
    elif a.op == "attention":
        r = run_attention(a, ctx)
    elif a.op == "ffn":
        r = run_ffn(a, ctx)
    elif a.op == "full":
        r = run_full(a, ctx)
    elif a.op == "qkvattn":
        r = run_qkv_attention(a, ctx)
    else:
        r = run_linear(a, ctx)
    print(json.dumps(r), flush=True)
    if a.timeline:
        print(json.dumps({"timeline_us": timeline_summary()}), flush=True)
    ctx.close()


if __name__ == "__main__":
    main()
