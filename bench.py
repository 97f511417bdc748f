#!/usr/bin/env python3
"""Benchmark of the Fast-dLLM block-decoding hot path on B200.

Workload (LLaDA-8B shapes, batch 1, prompt 512 + gen 256, block 32, tau 0.9):
one step is one DualCache block step of the hot path:
  for each of 32 layers: store the block's fresh K/V into the cache slot,
                         DualCache attention of the 32 block queries over the
                         768-row cache (32 heads x 128, bf16);
  LM head over the block's 32 rows (hidden 4096 -> vocab 126464, bf16,
  planted per-row logit bias) fused with the confidence reduction;
  threshold select + scatter into the sequence.
When a block has no masked position left, the caches of all 32 layers are
rewritten (the refresh's cache writes) and the next block starts; after the
8th block the sequence is reset. Tokens/s counts the positions decoded.
The QKV/O projections, norms and FFN of the model are not part of this
workload (they are the transformer scaffold around the method's hot path).

Inputs are seeded synthetic draws, larger than L2 in total (32 layer caches,
403 MB, and the 1.04 GB LM head are read every step), so no flush is needed.

Prints one JSON line (rank 0). `--impl reference` times the CPU oracle on
the same workload instead (host cores, bounded sample per step).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

CFG = dict(layers=32, heads=32, head_dim=128, prompt=512, gen=256, block=32, hidden=4096,
           vocab=126464, tau=0.9, mask_id=126336, batch=1)
WORKLOAD = ("LLaDA-8B-shaped DualCache block step: 32 layers x (block-slot K/V store + "
            "attention, 32 heads x 128, L=768) + LM head 4096->126464 + threshold unmask")
METRIC = "generated tokens/s per B200"
N_POOL = 16          # distinct LM-head inputs rotated across steps


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=60)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--e2e-steps", type=int, default=20)
    p.add_argument("--no-cpu-baseline", action="store_true")
    return p.parse_args()


# ----------------------------------------------------------------------------- inputs
def make_inputs(seed=0):
    """Host (numpy) inputs: per-layer caches, fresh block K/V, queries,
    refresh rows; LM-head weight and a pool of (h, planted bias)."""
    from block_kv_cache_b200 import synth
    c = CFG
    L = c["prompt"] + c["gen"]
    layers = []
    for l in range(c["layers"]):
        a = synth.attn_case(batch=1, n_q_heads=c["heads"], head_dim=c["head_dim"],
                            prefix=c["prompt"], block=c["block"],
                            suffix=c["gen"] - c["block"], dtype="bf16", seed=1000 + l)
        layers.append(a)
    lm = synth.lmhead_case(rows=c["block"] * N_POOL, hidden=c["hidden"], vocab=c["vocab"],
                           seed=7, w_seed=0, mask_id=c["mask_id"])
    prompt = synth.prompt_ids(3, 1, c["prompt"], c["mask_id"])
    return layers, lm, prompt, L


def bf16_dev(a, torch):
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).cuda()


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.25)
        except FileNotFoundError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 7:
                continue
            try:
                sm.append(float(f[0]))
                mx = float(f[1])
            except ValueError:
                continue
            for n, v in zip(names, f[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- GPU arm
class GpuStep:
    def __init__(self, torch, ctx, layers, lm, prompt, L):
        from block_kv_cache_b200 import fdllm
        self.torch, self.ctx, self.L = torch, ctx, L
        c = CFG
        self.kc = [bf16_dev(a.k_cache, torch) for a in layers]
        self.vc = [bf16_dev(a.v_cache, torch) for a in layers]
        self.kb = [bf16_dev(a.k_blk, torch) for a in layers]
        self.vb = [bf16_dev(a.v_blk, torch) for a in layers]
        self.q = [bf16_dev(a.q, torch) for a in layers]
        # refresh rows: the cache contents as a token-major [1, L, H, d] tensor
        self.kfull = [t.permute(0, 2, 1, 3).contiguous() for t in self.kc]
        self.vfull = [t.permute(0, 2, 1, 3).contiguous() for t in self.vc]
        self.o = torch.empty_like(self.q[0])
        self.w = bf16_dev(lm.w, torch)
        self.h = bf16_dev(lm.h, torch).view(N_POOL, c["block"], c["hidden"])
        self.bt = torch.from_numpy(lm.bias_tok).cuda().view(N_POOL, c["block"])
        self.bv = torch.from_numpy(lm.bias_val).cuda().view(N_POOL, c["block"])
        self.conf = torch.empty(c["block"], dtype=torch.float32, device="cuda")
        self.tok = torch.empty(c["block"], dtype=torch.int32, device="cuda")
        ad = ctx.attn_desc(self.q[0], self.kc[0], c["prompt"])
        self.ws_att = torch.empty(ctx.attention_workspace_bytes(ad), dtype=torch.uint8,
                                  device="cuda")
        lmd = fdllm.LMHeadDesc(c["block"], c["hidden"], c["vocab"], fdllm.FDL_BF16)
        self.ws_lm = torch.empty(ctx.lmhead_workspace_bytes(lmd), dtype=torch.uint8,
                                 device="cuda")
        x0 = np.concatenate([prompt[0], np.full(c["gen"], c["mask_id"])]).astype(np.int32)
        m0 = np.zeros(L, np.uint8)
        m0[c["prompt"]:] = 1
        self.x0 = torch.from_numpy(x0[None]).cuda()
        self.m0 = torch.from_numpy(m0[None]).cuda()
        self.x = self.x0.clone()
        self.m = self.m0.clone()
        self.rem = torch.empty(1, dtype=torch.int32, device="cuda")
        self.nd = torch.empty(1, dtype=torch.int32, device="cuda")
        self.host = torch.empty(2, dtype=torch.int32).pin_memory()
        self.blk = 0
        self.i = 0
        self.lm_events = []
        self.launches = 0

    def reset(self):
        self.x.copy_(self.x0)
        self.m.copy_(self.m0)
        self.blk = 0

    def step(self, time_lm=False):
        torch, ctx, c = self.torch, self.ctx, CFG
        s = c["prompt"] + self.blk * c["block"]
        for l in range(c["layers"]):
            ctx.kv_store(self.kb[l], self.vb[l], self.kc[l], self.vc[l], s)
            ctx.dualcache_attention(self.q[l], self.kc[l], self.vc[l], s, out=self.o,
                                    ws=self.ws_att)
        p = self.i % N_POOL
        if time_lm:
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
        ctx.lmhead_confidence(self.h[p], self.w, self.bt[p], self.bv[p], conf=self.conf,
                              tok=self.tok, ws=self.ws_lm)
        if time_lm:
            e1.record()
            self.lm_events.append((e0, e1))
        ctx.threshold_unmask(self.conf.view(1, -1), self.tok.view(1, -1), self.x, self.m, s,
                             c["tau"], remaining=self.rem, n_decoded=self.nd)
        self.host[0:1].copy_(self.rem, non_blocking=True)
        self.host[1:2].copy_(self.nd, non_blocking=True)
        torch.cuda.current_stream().synchronize()
        rem, nd = int(self.host[0]), int(self.host[1])
        self.launches += c["layers"] * 3 + 2 + 1
        if rem == 0:
            self.blk += 1
            if self.blk == c["gen"] // c["block"]:
                self.reset()
            for l in range(c["layers"]):
                ctx.kv_store(self.kfull[l], self.vfull[l], self.kc[l], self.vc[l], 0)
            self.launches += c["layers"]
        self.i += 1
        return nd

    def lm_avg_ms(self):
        ts = [a.elapsed_time(b) for a, b in self.lm_events]
        return sum(ts) / len(ts)


def lm_bytes():
    c = CFG
    return (c["vocab"] * c["hidden"] * 2 + c["block"] * c["hidden"] * 2 + c["block"] * 16)


def run_gpu(args):
    import torch
    import torch.distributed as dist
    from block_kv_cache_b200 import fdllm

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))

    def barrier():
        if world > 1:
            dist.barrier()

    ctx = fdllm.Context(local)
    layers, lm, prompt, L = make_inputs()
    st = GpuStep(torch, ctx, layers, lm, prompt, L)
    for _ in range(max(args.warmup, 3)):
        st.step()
    ctx.device_status()
    st.reset()
    st.launches = 0

    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    toks = 0
    with ClockSampler(local) as clk:
        ev0.record()
        for _ in range(args.steps):
            toks += st.step(time_lm=True)
        ev1.record()
        torch.cuda.synchronize()
    barrier()
    ms = ev0.elapsed_time(ev1)
    ctx.device_status()
    launches = st.launches
    lm_ms = st.lm_avg_ms()

    # max time over ranks, total tokens over ranks
    t = torch.tensor([ms, float(toks)], dtype=torch.float64, device="cuda")
    if world > 1:
        tm = t[0:1].clone()
        dist.all_reduce(tm, op=dist.ReduceOp.MAX)
        tt = t[1:2].clone()
        dist.all_reduce(tt, op=dist.ReduceOp.SUM)
        ms_max, toks_all = float(tm), float(tt)
    else:
        ms_max, toks_all = ms, float(toks)

    # e2e: the same step through the public API with pinned host inputs every step
    e2e = run_e2e(torch, ctx, st, layers, lm, args.e2e_steps)
    if world > 1:
        te = torch.tensor([e2e["ms"], float(e2e["toks"])], dtype=torch.float64, device="cuda")
        a = te[0:1].clone()
        dist.all_reduce(a, op=dist.ReduceOp.MAX)
        b = te[1:2].clone()
        dist.all_reduce(b, op=dist.ReduceOp.SUM)
        e2e_val = float(b) / (float(a) / 1e3)
    else:
        e2e_val = e2e["toks"] / (e2e["ms"] / 1e3)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(layers, lm, prompt, L, budget_s=15.0)

    if rank == 0:
        peaks = read_peaks()
        ach = lm_bytes() / (lm_ms / 1e3) / 1e9
        peak = peaks.get("hbm_gbs")
        out = {
            "metric": METRIC, "value": toks_all / (ms_max / 1e3), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD, "batch": CFG["batch"], "prompt": CFG["prompt"],
                       "gen": CFG["gen"], "block": CFG["block"], "tau": CFG["tau"],
                       "layers": CFG["layers"], "parallelism": f"replicas x{world}",
                       "tokens_decoded": toks, "l2": "inputs larger than L2 (403 MB of caches "
                       "+ 1.04 GB LM head read per step); no flush"},
            "gpu_launches": launches,
            "roofline": {"kernel": "lmhead_confidence (M=32, V=126464, D=4096)", "bound": "hbm",
                         "achieved": ach, "peak": peak, "unit": "GB/s",
                         "frac": (ach / peak) if peak else None, "traffic": None,
                         "peak_source": "MEASURED_PEAKS.json hbm_gbs (measured)" if peak else
                         "fallback 6650 GB/s",
                         "avg_launch_us": lm_ms * 1e3},
            "e2e": {"value": e2e_val, "unit": "tokens/s",
                    "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"]},
            "clocks": clk.summary(),
        }
        if peak is None:
            out["roofline"]["peak"] = 6650.0
            out["roofline"]["frac"] = ach / 6650.0
        out["cpu_baseline"] = cpu
        print(json.dumps(out), flush=True)
    ctx.close()
    if world > 1:
        dist.destroy_process_group()


def run_e2e(torch, ctx, st, layers, lm, steps):
    """Each step: copy the step's inputs (per-layer q and block K/V, the LM-head
    rows and bias) from pinned host memory, run the step, read back x, masked
    and the counters."""
    c = CFG
    hq = [torch.from_numpy(np.ascontiguousarray(a.q)).to(torch.bfloat16).pin_memory()
          for a in layers]
    hk = [torch.from_numpy(np.ascontiguousarray(a.k_blk)).to(torch.bfloat16).pin_memory()
          for a in layers]
    hv = [torch.from_numpy(np.ascontiguousarray(a.v_blk)).to(torch.bfloat16).pin_memory()
          for a in layers]
    hh = torch.from_numpy(lm.h).to(torch.bfloat16).view(N_POOL, c["block"], -1).pin_memory()
    hbt = torch.from_numpy(lm.bias_tok).view(N_POOL, -1).pin_memory()
    hbv = torch.from_numpy(lm.bias_val).view(N_POOL, -1).pin_memory()
    out_x = torch.empty_like(st.x, device="cpu").pin_memory()
    out_m = torch.empty_like(st.m, device="cpu").pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in hq + hk + hv) + \
        hh[0].numel() * 2 + hbt[0].numel() * 4 + hbv[0].numel() * 4
    d2h = out_x.numel() * 4 + out_m.numel() + 8
    st.reset()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    toks = 0
    e0.record()
    for _ in range(steps):
        p = st.i % N_POOL
        for l in range(c["layers"]):
            st.q[l].copy_(hq[l], non_blocking=True)
            st.kb[l].copy_(hk[l], non_blocking=True)
            st.vb[l].copy_(hv[l], non_blocking=True)
        st.h[p].copy_(hh[p], non_blocking=True)
        st.bt[p].copy_(hbt[p], non_blocking=True)
        st.bv[p].copy_(hbv[p], non_blocking=True)
        toks += st.step()
        out_x.copy_(st.x, non_blocking=True)
        out_m.copy_(st.m, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    return {"ms": e0.elapsed_time(e1), "toks": toks, "h2d": h2d, "d2h": d2h}


def read_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except Exception:
        return {}


# ----------------------------------------------------------------------------- CPU oracle
class OracleStep:
    """The same block step computed by the CPU oracle (float64 NumPy)."""

    def __init__(self, layers, lm, prompt, L):
        import oracle as O
        self.O = O
        c = CFG
        self.layers = layers
        self.kc = [a.k_cache.astype(np.float64) for a in layers]
        self.vc = [a.v_cache.astype(np.float64) for a in layers]
        self.lm = lm
        x0 = np.concatenate([prompt[0], np.full(c["gen"], c["mask_id"])]).astype(np.int32)
        self.x = x0[None].copy()
        self.m = np.zeros((1, L), np.uint8)
        self.m[0, c["prompt"]:] = 1
        self.blk = 0
        self.i = 0

    def step(self, layer_sample=None):
        O, c = self.O, CFG
        s = c["prompt"] + self.blk * c["block"]
        nl = c["layers"] if layer_sample is None else layer_sample
        for l in range(nl):
            a = self.layers[l]
            O.kv_store(self.kc[l], self.vc[l], a.k_blk, a.v_blk, s)
            O.dualcache_attention(a.q, self.kc[l], self.vc[l])
        p = self.i % N_POOL
        sl = slice(p * c["block"], (p + 1) * c["block"])
        r = O.lmhead_confidence(self.lm.h[sl], self.lm.w, self.lm.bias_tok[sl],
                                self.lm.bias_val[sl])
        self.x, self.m, rem, nd = O.threshold_unmask(
            self.x, self.m, r.conf[None].astype(np.float32), r.tok[None].astype(np.int32), s,
            c["block"], c["tau"])
        if rem[0] == 0:
            self.blk = (self.blk + 1) % (c["gen"] // c["block"])
        self.i += 1
        return int(nd[0])


def _threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        return os.cpu_count()


def cpu_baseline(layers, lm, prompt, L, budget_s=15.0):
    os_ = OracleStep(layers, lm, prompt, L)
    t0 = time.perf_counter()
    toks, n = 0, 0
    while time.perf_counter() - t0 < budget_s or n == 0:
        toks += os_.step()
        n += 1
    dt = time.perf_counter() - t0
    return {"value": toks / dt, "unit": "tokens/s", "cores": _threads(), "kind": "oracle",
            "host_cpus": os.cpu_count(),
            "sample": f"{n} full block steps of the same workload (all 32 layers, full vocab) "
                      f"in {dt:.1f} s, float64 NumPy"}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    layers, lm, prompt, L = make_inputs()
    os_ = OracleStep(layers, lm, prompt, L)
    for _ in range(args.warmup):
        os_.step()
    t0 = time.perf_counter()
    toks = 0
    for _ in range(args.steps):
        toks += os_.step()
    dt = time.perf_counter() - t0
    val = toks / dt
    out = {"impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": WORKLOAD, "batch": CFG["batch"], "prompt": CFG["prompt"],
                      "gen": CFG["gen"], "block": CFG["block"], "tau": CFG["tau"],
                      "layers": CFG["layers"], "parallelism": "cpu oracle"},
           "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": _threads(),
                            "kind": "oracle", "host_cpus": os.cpu_count(),
                            "sample": f"{args.steps} full block steps after {args.warmup} "
                                      "warm-up steps"},
           "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
