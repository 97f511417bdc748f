"""Fast-dLLM block decoding of a LLaDA / Dream-shaped bidirectional
transformer on the GPU, driven through the C-ABI library.

Every arithmetic step runs in libfdllm.so kernels; this module only holds the
device buffers (torch allocations) and issues the calls in order:

  refresh (a full forward over all L positions; Fast-dLLM recomputes every
  position's K/V once a block completes - ICLR reviews, review 4 question 2):
      embed -> per layer [RMSNorm -> QKV + RoPE written into the K/V caches
      (every row) -> full attention -> O proj + residual -> RMSNorm -> SwiGLU
      -> down proj + residual] -> final RMSNorm of the current block's rows
      -> LM head confidence -> threshold unmask
  cached block step (DualCache; aibase news "Innovations" 1):
      the same per layer, but only the block's B rows go through the layers:
      their K/V overwrite the cache slot and the block attends over the whole
      cache [prefix | block | masked suffix]

Layouts: weights are stored [out, in] (K-major); the gate and up projections
are interleaved by rows (row 2f = gate f, 2f+1 = up f) so the SwiGLU
epilogue finds both halves of a feature in one tile.
"""
from __future__ import annotations

import contextlib
import ctypes
import time
from dataclasses import dataclass

import numpy as np
import torch

from . import fdllm


@dataclass
class ModelShape:
    vocab: int
    hidden: int
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    ffn: int
    mask_id: int
    head_dim: int = 128
    rope_theta: float = 10000.0
    rms_eps: float = 1e-5
    qkv_bias: bool = False


def graph_kernel_count(g: "torch.cuda.CUDAGraph") -> int:
    """Kernel nodes of a captured CUDA graph (kept with keep_graph=True): the
    kernels one replay launches, read through the CUDA driver API."""
    cu = ctypes.CDLL("libcuda.so.1")
    cu.cuGraphGetNodes.argtypes = [ctypes.c_void_p, ctypes.c_void_p,
                                   ctypes.POINTER(ctypes.c_size_t)]
    cu.cuGraphNodeGetType.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_int)]
    h = ctypes.c_void_p(g.raw_cuda_graph())
    n = ctypes.c_size_t(0)
    if cu.cuGraphGetNodes(h, None, ctypes.byref(n)) != 0:
        raise RuntimeError("cuGraphGetNodes failed")
    nodes = (ctypes.c_void_p * n.value)()
    if cu.cuGraphGetNodes(h, nodes, ctypes.byref(n)) != 0:
        raise RuntimeError("cuGraphGetNodes failed")
    kind = ctypes.c_int(-1)
    count = 0
    for nd in nodes:
        if cu.cuGraphNodeGetType(ctypes.c_void_p(nd), ctypes.byref(kind)) != 0:
            raise RuntimeError("cuGraphNodeGetType failed")
        count += kind.value == 0                  # CU_GRAPH_NODE_TYPE_KERNEL
    return count


def _bf16(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).to(dev)


def _f32(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev)


class DeviceWeights:
    """bf16 weights (f32 norms and biases) on one device."""

    def __init__(self, shape: ModelShape, layers, embed, final_norm, lm_head):
        self.shape = shape
        self.layers = layers
        self.embed = embed
        self.final_norm = final_norm
        self.lm_head = lm_head

    @staticmethod
    def from_params(P, device="cuda") -> "DeviceWeights":
        """From synth.ModelParams (host float32 values exact in bf16)."""
        sh = ModelShape(P.vocab, P.hidden, P.n_layers, P.n_q_heads, P.n_kv_heads, P.ffn,
                        P.mask_id, P.head_dim, P.rope_theta, P.rms_eps, P.qkv_bias)
        layers = []
        for Lw in P.layers:
            wgu = np.empty((2 * P.ffn, P.hidden), np.float32)
            wgu[0::2] = Lw["wg"]
            wgu[1::2] = Lw["wu"]
            d = dict(attn_norm=_f32(Lw["attn_norm"], device),
                     w_qkv=_bf16(np.concatenate([Lw["wq"], Lw["wk"], Lw["wv"]]), device),
                     wo=_bf16(Lw["wo"], device), ffn_norm=_f32(Lw["ffn_norm"], device),
                     w_gu=_bf16(wgu, device), wd=_bf16(Lw["wd"], device), bias=None)
            if P.qkv_bias:
                d["bias"] = _f32(np.concatenate([Lw["bq"], Lw["bk"], Lw["bv"]]), device)
            layers.append(d)
        return DeviceWeights(sh, layers, _bf16(P.embed, device), _f32(P.final_norm, device),
                             _bf16(P.lm_head, device))

    @staticmethod
    def random(shape: ModelShape, seed=0, device="cuda", w_std=0.02) -> "DeviceWeights":
        """Seeded random-init weights drawn on the device (for full-size runs whose
        weights would take minutes to draw on the host). Norm weights are 1."""
        g = torch.Generator(device=device)
        g.manual_seed(seed)
        D, F, d = shape.hidden, shape.ffn, shape.head_dim
        nqkv = (shape.n_q_heads + 2 * shape.n_kv_heads) * d

        def rnd(*sz):
            return (torch.randn(*sz, generator=g, device=device, dtype=torch.float32)
                    * w_std).to(torch.bfloat16)

        layers = []
        for _ in range(shape.n_layers):
            layers.append(dict(
                attn_norm=torch.ones(D, device=device), w_qkv=rnd(nqkv, D),
                wo=rnd(D, shape.n_q_heads * d), ffn_norm=torch.ones(D, device=device),
                w_gu=rnd(2 * F, D), wd=rnd(D, F),
                bias=(torch.randn(nqkv, generator=g, device=device) * w_std)
                if shape.qkv_bias else None))
        embed = (torch.randn(shape.vocab, D, generator=g, device=device)).to(torch.bfloat16)
        return DeviceWeights(shape, layers, embed, torch.ones(D, device=device),
                             rnd(shape.vocab, D))

    def native(self) -> "fdllm.Model":
        """These weights recorded in the library, for Context.generate (the
        whole decode loop in native code)."""
        sh = self.shape
        return fdllm.Model(vocab=sh.vocab, hidden=sh.hidden, n_q_heads=sh.n_q_heads,
                           n_kv_heads=sh.n_kv_heads, ffn=sh.ffn, mask_id=sh.mask_id,
                           embed=self.embed, final_norm=self.final_norm, lm_head=self.lm_head,
                           layers=self.layers, head_dim=sh.head_dim, rope_theta=sh.rope_theta,
                           rms_eps=sh.rms_eps)

    def nbytes(self) -> int:
        n = self.embed.numel() * 2 + self.lm_head.numel() * 2
        for L in self.layers:
            n += sum(t.numel() * t.element_size() for t in L.values() if t is not None)
        return n


CACHE_MODES = ("dual", "prefix", "none")


class BlockDecoder:
    """Block decoding with the threshold rule of `batch` sequences of length
    seq_len, with one of three cache modes (Fast-dLLM README usage flags and
    evaluation table):
      "dual"   (--use_cache --if_cache_position): DualCache; a cached step runs
               only the block's rows over [cached prefix | block | cached suffix];
      "prefix" (--use_cache): PrefixCache; a cached step runs the block and the
               masked suffix (rows [s, L)) over [cached prefix | fresh rows];
      "none"   (no cache): every step is a full forward over all positions.
    In every mode a block's first step is the full forward (the refresh).

    With bias_tok / bias_val ([b, gen] int32 / f32 on the device), the LM head
    adds bias_val to the logit of token bias_tok at each generated position
    (a synthetic planted-token bias, so that confidences can exceed the
    threshold with random weights)."""

    def __init__(self, ctx: fdllm.Context, w: DeviceWeights, batch: int, seq_len: int,
                 block: int = 32, device="cuda", cache: str = "dual", bias_tok=None,
                 bias_val=None):
        assert cache in CACHE_MODES
        sh = w.shape
        self.ctx, self.w, self.sh = ctx, w, sh
        self.b, self.L, self.B = batch, seq_len, block
        self.cache = cache
        dev = device
        D, d = sh.hidden, sh.head_dim
        self.rope = torch.from_numpy(fdllm.rope_table(sh.rope_theta, seq_len, d)).to(dev)
        self.kc = [torch.zeros((batch, sh.n_kv_heads, seq_len, d), dtype=torch.bfloat16,
                               device=dev) for _ in range(sh.n_layers)]
        self.vc = [torch.zeros_like(k) for k in self.kc]
        rows_full = batch * seq_len
        self.h_full = torch.empty((rows_full, D), dtype=torch.float32, device=dev)
        self.x_full = torch.empty((rows_full, D), dtype=torch.bfloat16, device=dev)
        self.q_full = torch.empty((rows_full, sh.n_q_heads, d), dtype=torch.bfloat16, device=dev)
        self.o_full = torch.empty_like(self.q_full)
        self.f_full = torch.empty((rows_full, sh.ffn), dtype=torch.bfloat16, device=dev)
        rb = batch * block
        self.h_blk = torch.empty((rb, D), dtype=torch.float32, device=dev)
        self.x_blk = torch.empty((rb, D), dtype=torch.bfloat16, device=dev)
        self.q_blk = torch.empty((rb, sh.n_q_heads, d), dtype=torch.bfloat16, device=dev)
        self.o_blk = torch.empty_like(self.q_blk)
        self.f_blk = torch.empty((rb, sh.ffn), dtype=torch.bfloat16, device=dev)
        self.xn = torch.empty((rb, D), dtype=torch.bfloat16, device=dev)
        self.conf = torch.empty(rb, dtype=torch.float32, device=dev)
        self.tok = torch.empty(rb, dtype=torch.int32, device=dev)
        # per-step counters (remaining masked in the block, decoded this step),
        # read back by the host after every step
        self.counts = torch.zeros((2, batch), dtype=torch.int32, device=dev)
        self.remaining, self.n_decoded = self.counts[0], self.counts[1]
        self.counts_host = torch.zeros((2, batch), dtype=torch.int32).pin_memory()
        # decode state (device-resident for the whole decode)
        self.x = torch.empty((batch, seq_len), dtype=torch.int32, device=dev)
        self.masked = torch.empty((batch, seq_len), dtype=torch.uint8, device=dev)
        self.graphs = {}
        self.graph_timers = {}          # graph key -> {call: [(event, event)]} of layer 0
        self.call_us = {}               # (step kind, call) -> µs of each replay (step())
        self._launches = {}             # graph key -> kernels per replay
        self._timers = None
        nblk = (seq_len + block - 1) // block
        i = np.arange(block)
        bi = np.arange(batch)[:, None]
        # rows of block k of every sequence in the flattened [b * L] token rows
        maps = np.stack([(bi * seq_len + k * block + i[None, :]).reshape(-1)
                         for k in range(nblk)]).astype(np.int32)
        self.row_maps = torch.from_numpy(np.minimum(maps, batch * seq_len - 1)).to(dev)
        # PrefixCache: rows [s, L) of every sequence in the [b * L] token rows
        # (tail_maps[k]), and the block's rows within those b * (L - s) rows
        self.tail_maps, self.tail_blk = [], []
        if cache == "prefix":
            for k in range(nblk):
                n = seq_len - k * block
                j = np.arange(n)
                self.tail_maps.append(torch.from_numpy(
                    (bi * seq_len + k * block + j[None, :]).reshape(-1).astype(np.int32)).to(dev))
                self.tail_blk.append(torch.from_numpy(
                    (bi * n + i[None, :]).reshape(-1).astype(np.int32)).to(dev))
        # planted bias per generated position, sliced per block ([nblk, b * B])
        self.bias = None
        if bias_tok is not None:
            gen = bias_tok.shape[1]
            P0 = seq_len - gen
            assert gen % block == 0 and P0 % block == 0
            bt = bias_tok.view(batch, gen // block, block).transpose(0, 1).contiguous()
            bv = bias_val.view(batch, gen // block, block).transpose(0, 1).contiguous()
            self.bias = (P0 // block, bt.view(gen // block, rb), bv.view(gen // block, rb))
        lmd = fdllm.LMHeadDesc(rb, D, sh.vocab, fdllm.FDL_BF16)
        self.ws_lm = torch.empty(max(ctx.lmhead_workspace_bytes(lmd), 16), dtype=torch.uint8,
                                 device=dev)

    # ------------------------------------------------------------------ layers
    @contextlib.contextmanager
    def _timed(self, name, on):
        """CUDA events around one call (layer 0 only: events in a graph cut the
        overlap of neighbouring kernels)."""
        if not on:
            yield
            return
        e0 = torch.cuda.Event(enable_timing=True, external=True)
        e1 = torch.cuda.Event(enable_timing=True, external=True)
        e0.record()
        yield
        e1.record()
        self._timers.setdefault(name, []).append((e0, e1))

    def _layers(self, h, x, q, o, f, rows, rows_per_seq, pos0, full):
        """The layers over `rows` = b * rows_per_seq token rows at positions
        pos0 + [0, rows_per_seq) of every sequence. full: those rows' K/V are
        written into the caches and the rows attend over the whole cache
        (refresh: pos0 = 0; PrefixCache step: pos0 = s); otherwise the fused
        DualCache step of the block rows."""
        ctx, sh = self.ctx, self.sh
        for li, Lw in enumerate(self.w.layers):
            timed = self._timers is not None and li == 0
            if full:
                ctx.rmsnorm(h, Lw["attn_norm"], sh.rms_eps, out=x, rows=rows)
                ctx.qkv_rope_store(x[:rows], Lw["w_qkv"], self.rope, q, self.kc[li], self.vc[li],
                                   n_q_heads=sh.n_q_heads, rows_per_seq=rows_per_seq, pos0=pos0,
                                   bias=Lw["bias"])
                with self._timed("full_attention", timed):
                    ctx.full_attention(
                        q[:rows].view(self.b, rows_per_seq, sh.n_q_heads, sh.head_dim),
                        self.kc[li], self.vc[li], q_start=pos0,
                        out=o[:rows].view(self.b, rows_per_seq, sh.n_q_heads, sh.head_dim))
            else:
                # norm + block-slot projection + DualCache attention of the block rows
                with self._timed("qkv_attention", timed):
                    ctx.qkv_attention(x, Lw["w_qkv"], self.rope, q, self.kc[li], self.vc[li],
                                      o.view(self.b, self.B, sh.n_q_heads, sh.head_dim),
                                      n_q_heads=sh.n_q_heads, rows_per_seq=rows_per_seq,
                                      pos0=pos0, bias=Lw["bias"], h=h, norm_w=Lw["attn_norm"],
                                      eps=sh.rms_eps)
            ctx.linear_residual(o[:rows].view(rows, -1), Lw["wo"], h[:rows])
            with self._timed("ffn", timed):
                ctx.ffn(x[:rows], Lw["w_gu"], Lw["wd"], h[:rows], f=f[:rows],
                        norm_w=Lw["ffn_norm"], eps=sh.rms_eps)

    def refresh(self, x_ids, s):
        """Full forward over all positions of x_ids [b, L] (int32, device): rewrites
        every layer's K/V cache and leaves conf/tok for the rows of block [s, s+B)."""
        rows = self.b * self.L
        self.ctx.embed(x_ids.view(-1), self.w.embed, out=self.h_full)
        self._layers(self.h_full, self.x_full, self.q_full, self.o_full, self.f_full, rows,
                     self.L, 0, True)
        self.ctx.rmsnorm(self.h_full, self.w.final_norm, self.sh.rms_eps, out=self.xn,
                         row_map=self._row_map(s))
        self._confidence(s)

    def block_step(self, x_ids, s):
        """Cached DualCache step for block [s, s+B) of x_ids [b, L]."""
        rows = self.b * self.B
        self.ctx.embed(x_ids, self.w.embed, out=self.h_blk, row_map=self._row_map(s))
        self._layers(self.h_blk, self.x_blk, self.q_blk, self.o_blk, self.f_blk, rows, self.B,
                     s, False)
        self.ctx.rmsnorm(self.h_blk, self.w.final_norm, self.sh.rms_eps, out=self.xn)
        self._confidence(s)

    def prefix_step(self, x_ids, s):
        """Cached PrefixCache step for block [s, s+B): rows [s, L) of every
        sequence go through the layers over the cached prefix."""
        k = s // self.B
        n = self.L - s
        rows = self.b * n
        self.ctx.embed(x_ids, self.w.embed, out=self.h_full, row_map=self.tail_maps[k])
        self._layers(self.h_full, self.x_full, self.q_full, self.o_full, self.f_full, rows, n,
                     s, True)
        self.ctx.rmsnorm(self.h_full, self.w.final_norm, self.sh.rms_eps, out=self.xn,
                         row_map=self.tail_blk[k])
        self._confidence(s)

    def _row_map(self, s):
        assert s % self.B == 0, "blocks start at multiples of the block size"
        return self.row_maps[s // self.B]

    def _confidence(self, s):
        bt = bv = None
        if self.bias is not None:
            k = s // self.B - self.bias[0]
            bt, bv = self.bias[1][k], self.bias[2][k]
        self.ctx.lmhead_confidence(self.xn, self.w.lm_head, bt, bv, conf=self.conf, tok=self.tok,
                                   ws=self.ws_lm)

    def unmask(self, x_ids, masked, s, tau):
        self.ctx.threshold_unmask(self.conf.view(self.b, self.B), self.tok.view(self.b, self.B),
                                  x_ids, masked, s, tau, remaining=self.remaining,
                                  n_decoded=self.n_decoded)

    def _forward(self, kind, x_ids, s):
        if kind == "refresh":
            self.refresh(x_ids, s)
        elif kind == "prefix":
            self.prefix_step(x_ids, s)
        else:
            self.block_step(x_ids, s)

    def cached_kind(self):
        """The kind of a block's steps after its first: the cache mode's step."""
        return {"dual": "cached", "prefix": "prefix", "none": "refresh"}[self.cache]

    # ------------------------------------------------------------------ decode
    def generate(self, prompt, gen_len, tau=0.9, record=None):
        """Decode gen_len tokens after prompt [b, P] (host or device int32) with
        the decoder's cache mode and the threshold rule. Returns (x [b, L] int32
        device, steps). If `record` is a list, each step appends (kind, s,
        x_before, masked_before, conf, tok, xn) as host arrays (for step-wise
        checks; xn holds the final-norm rows the LM head consumed, as float32)."""
        b, P = prompt.shape
        assert P + gen_len == self.L and gen_len % self.B == 0
        dev = self.h_full.device
        x = torch.full((b, self.L), self.sh.mask_id, dtype=torch.int32, device=dev)
        x[:, :P] = torch.as_tensor(prompt, dtype=torch.int32, device=dev)
        masked = torch.zeros((b, self.L), dtype=torch.uint8, device=dev)
        masked[:, P:] = 1
        steps = 0
        host_rem = torch.empty(b, dtype=torch.int32).pin_memory()
        for blk in range(gen_len // self.B):
            s = P + blk * self.B
            kind = "refresh"
            while True:
                if record is not None:
                    xb, mb = x.cpu().numpy(), masked.cpu().numpy()
                self._forward(kind, x, s)
                if record is not None:
                    record.append((kind, s, xb, mb, self.conf.cpu().numpy().copy(),
                                   self.tok.cpu().numpy().copy(),
                                   self.xn.float().cpu().numpy()))
                self.unmask(x, masked, s, tau)
                steps += 1
                host_rem.copy_(self.remaining, non_blocking=True)
                torch.cuda.current_stream().synchronize()
                if int(host_rem.max()) == 0:
                    break
                kind = self.cached_kind()
        return x, steps

    # ------------------------------------------------------- graph-replayed decode
    def _step_calls(self, kind, s, tau):
        self._forward(kind, self.x, s)
        self.unmask(self.x, self.masked, s, tau)
        self.counts_host.copy_(self.counts, non_blocking=True)

    def capture(self, kind, s, tau, time_calls=False):
        """CUDA graph of one decode step (forward, unmask, counter read-back) for
        block start s; kernels read and write the decoder's own x / masked. With
        time_calls, timing events bracket layer 0's attention and FFN calls."""
        key = (kind, s, float(tau))
        if key not in self.graphs:
            g = torch.cuda.CUDAGraph(keep_graph=True)   # the graph stays readable
            self._timers = {} if time_calls else None
            with torch.cuda.graph(g):
                self._step_calls(kind, s, tau)
            g.instantiate()
            self.graph_timers[key] = self._timers or {}
            self._timers = None
            self.graphs[key] = g
        return self.graphs[key]

    def kernel_launches(self, kind, s, tau):
        """Kernels one replay of the step graph (kind, s, tau) launches."""
        key = (kind, s, float(tau))
        if key not in self._launches:
            self._launches[key] = graph_kernel_count(self.capture(kind, s, tau))
        return self._launches[key]

    def last_timers(self):
        """{call: [(event, event)]} of the graph replayed by the last step()."""
        return self.graph_timers.get(self._last_key, {})

    def capture_all(self, prompt_len, gen_len, tau, time_calls=False):
        for blk in range(gen_len // self.B):
            s = prompt_len + blk * self.B
            self.capture("refresh", s, tau, time_calls)
            if self.cache != "none":
                self.capture(self.cached_kind(), s, tau, time_calls)
        torch.cuda.synchronize()

    def begin(self, prompt, tau):
        """Start a decode of prompt [b, P] (host or device int32)."""
        b, P = prompt.shape
        self.P, self.tau = P, float(tau)
        self.x.fill_(self.sh.mask_id)
        self.x[:, :P].copy_(torch.as_tensor(prompt, dtype=torch.int32), non_blocking=True)
        self.masked.zero_()
        self.masked[:, P:] = 1
        self.blk, self.kind, self.done = 0, "refresh", False
        self.steps = 0

    def step(self):
        """One decode step (graph replay). Returns tokens decoded by this step."""
        s = self.P + self.blk * self.B
        self._last_key = (self.kind, s, self.tau)
        self.last_kind = self.kind
        self.capture(self.kind, s, self.tau).replay()
        torch.cuda.current_stream().synchronize()
        for name, pairs in self.graph_timers.get(self._last_key, {}).items():
            us = self.call_us.setdefault((self.kind, name), [])
            us.extend(a.elapsed_time(b) * 1e3 for a, b in pairs)
        rem = int(self.counts_host[0].max())
        nd = int(self.counts_host[1].sum())
        self.steps += 1
        if rem == 0:
            self.blk += 1
            self.kind = "refresh"
            if self.P + self.blk * self.B >= self.L:
                self.done = True
        else:
            self.kind = self.cached_kind()
        return nd

    def block(self):
        """Decode the current block to its end (one refresh, then the cache
        mode's steps until no position of the block is masked). Returns
        (tokens decoded, [(kind, block start, host ms)] per step)."""
        toks, steps = 0, []
        blk = self.blk
        while not self.done and self.blk == blk:
            s = self.P + self.blk * self.B
            t0 = time.perf_counter()
            toks += self.step()
            steps.append((self.last_kind, s, (time.perf_counter() - t0) * 1e3))
        return toks, steps

    # ------------------------------------------------------------------ profiling
    def profile_step(self, kind, s, tau, reps=5):
        """Per-call GPU time of one decode step: the step is captured in a CUDA
        graph with timing events around every library call and replayed (the
        events serialise neighbouring kernels, so this shows where a step's time
        goes rather than the overlapped total). Returns {call: mean us per step}."""
        ctx = self.ctx
        pairs = []
        orig = {}

        def wrap(name):
            fn = getattr(ctx, name)
            orig[name] = fn

            def timed(*a, **k):
                e0 = torch.cuda.Event(enable_timing=True, external=True)
                e1 = torch.cuda.Event(enable_timing=True, external=True)
                e0.record()
                r = fn(*a, **k)
                e1.record()
                pairs.append((name, e0, e1))
                return r
            setattr(ctx, name, timed)

        calls = ["rmsnorm", "embed", "qkv_rope_store", "full_attention", "qkv_attention",
                 "linear_residual", "ffn", "lmhead_confidence", "threshold_unmask"]
        for n in calls:
            wrap(n)
        g = torch.cuda.CUDAGraph()
        try:
            with torch.cuda.graph(g):
                self._step_calls(kind, s, tau)
        finally:
            for n, fn in orig.items():
                setattr(ctx, n, fn)
        tot = {}
        for _ in range(reps):
            g.replay()
            torch.cuda.synchronize()
            for name, a, b in pairs:
                tot[name] = tot.get(name, 0.0) + a.elapsed_time(b) * 1e3
        del g
        return {n: v / reps for n, v in tot.items()}
