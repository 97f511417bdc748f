#!/usr/bin/env python3
"""Benchmark: Fast-dLLM block decoding of a random-init LLaDA-8B-shaped model
on B200.

Workload: bidirectional transformer of the LLaDA-8B shape (32 layers, hidden
4096, 32 heads x 128, SwiGLU FFN 12288, RMSNorm, RoPE, vocab 126464), bf16,
batch 1, prompt 1024 uniform random ids, gen 1024, block 32, DualCache,
threshold 0.9. One bench step = one whole block of the decode, the unit in
which the method's work repeats:
  * the block's first decode step is the refresh: a full forward over all
    2048 positions rewriting every layer's K/V cache, then the block's logits;
  * the others are cached DualCache steps: only the block's 32 rows go
    through the 32 layers (projection + RoPE + cache-slot write, attention
    over [prefix | block | masked suffix], O proj, SwiGLU FFN), until no
    position of the block is masked;
  every decode step ends with the fused LM-head confidence reduction and the
  threshold select/scatter; the host reads back 8 bytes (remaining and
  decoded counts) to decide refresh vs cached for the next step.
The timed steps start at the first block of a fresh decode (a decode that
reaches its end starts again). Each (step kind, block) is a CUDA graph
captured before timing. Weights are seeded random draws on the device (16 GB,
larger than L2, streamed every step), so no L2 flush is needed. With random
weights no confidence reaches 0.9, so every decode step decodes one position
(the fallback rule); --planted-bias adds a logit bias per position so that
the threshold rule fires. --cache prefix|none selects the PrefixCache or no
cache instead of DualCache (the README's table columns).

The line also carries `kernels`: the DualCache attention on the LLaDA-8B
attention layer (L = 768) and the LM head + unmask at 32 and 1024 rows, each
timed alone, and the fused attention call and full attention as timed inside
the decode; `e2e` is one whole decode through the library's decode loop
(fdl_generate) from a host prompt to a host copy of the sequence.

Prints one JSON line on rank 0. `--impl reference` times the CPU oracle on
the same workload instead (bounded sample per block, extrapolated).
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

CONFIGS = {
    # the headline workload: LLaDA-8B-shaped, batch 1
    "llada": dict(layers=32, hidden=4096, heads=32, kv_heads=32, head_dim=128, ffn=12288,
                  vocab=126464, mask_id=126336, batch=1, prompt=1024, gen=1024, block=32,
                  tau=0.9, qkv_bias=False,
                  workload="LLaDA-8B-shaped random-init model, bf16, batch 1, prompt 1024 + "
                           "gen 1024, block 32, DualCache, tau 0.9: Fast-dLLM block decoding "
                           "steps"),
    # Dream-7B-shaped (Qwen2.5-7B layout: GQA 28/4, q/k/v bias), batch 32; the mask
    # id is not given for it: vocab - 1
    "dream": dict(layers=28, hidden=3584, heads=28, kv_heads=4, head_dim=128, ffn=18944,
                  vocab=152064, mask_id=152063, batch=32, prompt=512, gen=512, block=32,
                  tau=0.9, qkv_bias=True,
                  workload="Dream-7B-shaped random-init model, bf16, batch 32, prompt 512 + "
                           "gen 512, block 32, DualCache, tau 0.9: Fast-dLLM block decoding "
                           "steps"),
}
CFG = dict(CONFIGS["llada"])
WORKLOAD = CFG["workload"]
METRIC = "generated tokens/s per B200"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=32,
                   help="timed steps; a step is one whole block (its refresh, then its "
                        "cached steps)")
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--cache", choices=["dual", "prefix", "none"], default="dual",
                   help="K/V reuse after a block's first step (default: DualCache)")
    p.add_argument("--planted-bias", action="store_true",
                   help="a planted logit bias per generated position, so that the "
                        "threshold rule decodes several positions per step")
    p.add_argument("--bias-hi", type=float, default=16.0,
                   help="upper end of the planted bias U(0, hi) (default 16)")
    p.add_argument("--block", type=int, default=None, help="block size (default 32)")
    p.add_argument("--gen", type=int, default=None, help="generated length (default 1024)")
    p.add_argument("--tau", type=float, default=None, help="threshold (default 0.9)")
    p.add_argument("--no-kernels", dest="kernels", action="store_false",
                   help="skip the per-kernel roofline cases")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--e2e-loop", choices=["device", "host"], default="device",
                   help="fdl_generate's loop for the e2e decode")
    p.add_argument("--batching", choices=["lockstep", "compact", "per_sequence"],
                   default="lockstep",
                   help="how the e2e decode moves a batch through its blocks (compact and "
                        "per_sequence use the host loop): compacted cached steps, or every "
                        "sequence at its own block")
    p.add_argument("--sweep", action="store_true",
                   help="instead of the bench line: the block / tau / gen / cache-mode grid "
                        "with the planted bias, one JSON line per point")
    p.add_argument("--profile-steps", action="store_true",
                   help="also print the per-call time of a cached step and of a refresh")
    p.add_argument("--config", choices=sorted(CONFIGS), default="llada",
                   help="workload: the LLaDA-8B-shaped batch-1 decode (default) or the "
                        "Dream-7B-shaped batch-32 decode")
    return p.parse_args()


def shape():
    from block_kv_cache_b200.model import ModelShape
    c = CFG
    return ModelShape(c["vocab"], c["hidden"], c["layers"], c["heads"], c["kv_heads"], c["ffn"],
                      c["mask_id"], c["head_dim"], qkv_bias=c["qkv_bias"])


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index, self.proc, self.lines = index, None, []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
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


def read_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except Exception:
        return {}




def combine_ranks(dist, world, ms, toks, device):
    """Whole-job figures of a replicated run: the slowest rank's time and the
    tokens of all ranks (every rank decodes its own sequences, so the work per
    GPU is fixed as the rank count grows). Every rank makes the same two
    collective calls."""
    import torch
    if world == 1:
        return float(ms), float(toks)
    t_ms = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    t_tok = torch.tensor([float(toks)], dtype=torch.float64, device=device)
    dist.all_reduce(t_ms, op=dist.ReduceOp.MAX)
    dist.all_reduce(t_tok, op=dist.ReduceOp.SUM)
    return float(t_ms.item()), float(t_tok.item())


# ----------------------------------------------------------------------------- GPU arm
def _peak(peaks, key, fallback):
    v = peaks.get(key)
    return (v, f"MEASURED_PEAKS.json {key} (measured)") if v else (fallback,
                                                                   f"fallback {fallback}")


def _graph_time_us(torch, calls, reps):
    """Mean µs per call of `calls` (a list of callables) captured once in a CUDA
    graph and replayed `reps` times, timed with CUDA events on the current
    stream after one untimed replay."""
    for c in calls[:2]:
        c()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for c in calls:
            c()
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / (reps * len(calls))
    del g
    return us


def kernel_rooflines(torch, ctx, w, peaks):
    """The two kernels the method's targets name, each timed alone (CUDA events
    around graph replays), as fractions of the measured peaks:
      * DualCache block attention on the LLaDA-8B attention layer (32 heads x
        128, prompt 512 + gen 256, block 32 at position 512): 32 distinct layer
        caches (403 MB, > L2) cycled; algorithmic bytes = K and V once + q + out;
      * the LM head fused with the confidence reduction, followed by the
        threshold unmask of the block, at 32 rows (batch 1: HBM-bound, the
        weight stream) and 1024 rows (batch 32: tensor-bound), on the model's
        126464 x 4096 head."""
    from block_kv_cache_b200 import fdllm
    hbm, hbm_src = _peak(peaks, "hbm_gbs", 6650.0)
    tf, tf_src = _peak(peaks, "bf16_tflops", 1590.0)
    out = {}
    dev = "cuda"
    g = torch.Generator(device=dev)
    g.manual_seed(2024)
    # ---- C2: DualCache attention, LLaDA-8B layer, L = 768
    H, d, P, B, S, layers = 32, 128, 512, 32, 224, 32
    L = P + B + S
    qs = [torch.randn(1, B, H, d, generator=g, device=dev).to(torch.bfloat16)
          for _ in range(layers)]
    ks = [torch.randn(1, H, L, d, generator=g, device=dev).to(torch.bfloat16)
          for _ in range(layers)]
    vs = [torch.randn(1, H, L, d, generator=g, device=dev).to(torch.bfloat16)
          for _ in range(layers)]
    o = torch.empty_like(qs[0])
    ws = ctx.workspace(ctx.attention_workspace_bytes(ctx.attn_desc(qs[0], ks[0], P)))
    calls = [(lambda i=i: ctx.dualcache_attention(qs[i], ks[i], vs[i], P, out=o, ws=ws))
             for i in range(layers)]
    us = _graph_time_us(torch, calls, reps=20)
    nbytes = 2 * H * L * d * 2 + 2 * B * H * d * 2
    ach = nbytes / us / 1e3
    out["dualcache_attention"] = {
        "case": "LLaDA-8B attention layer: 32 heads x 128 (MHA), L = 768 (prompt 512 + gen 256), "
                "block 32 at 512, bf16; 32 distinct layer caches cycled",
        "bytes_per_call": nbytes, "us_per_call": us, "bound": "hbm", "achieved": ach,
        "peak": hbm, "unit": "GB/s", "frac": ach / hbm, "peak_source": hbm_src}
    del qs, ks, vs, o, calls
    # ---- LM head + threshold unmask, 32 and 1024 rows of the 126464 x 4096 head
    V, D = w.lm_head.shape
    for b in (1, 32):
        M = 32 * b
        h = torch.randn(M, D, generator=g, device=dev).to(torch.bfloat16)
        conf = torch.empty(M, dtype=torch.float32, device=dev)
        tok = torch.empty(M, dtype=torch.int32, device=dev)
        lws = torch.empty(max(ctx.lmhead_workspace_bytes(
            fdllm.LMHeadDesc(M, D, V, fdllm.FDL_BF16)), 16), dtype=torch.uint8, device=dev)
        x = torch.zeros((b, 2048), dtype=torch.int32, device=dev)
        msk = torch.zeros((b, 2048), dtype=torch.uint8, device=dev)
        msk[:, 1024:] = 1
        rem = torch.empty(b, dtype=torch.int32, device=dev)

        def unit():
            ctx.lmhead_confidence(h, w.lm_head, conf=conf, tok=tok, ws=lws)
            ctx.threshold_unmask(conf.view(b, 32), tok.view(b, 32), x, msk, 1024, 0.9,
                                 remaining=rem)
        us = _graph_time_us(torch, [unit] * 8, reps=5)
        nbytes = V * D * 2 + M * D * 2 + M * 16
        flops = 2.0 * M * D * V
        key = f"lmhead_unmask_m{M}"
        if M <= 256:
            ach = nbytes / us / 1e3
            out[key] = {"case": f"LM head {V} x {D} + confidence reduction + threshold unmask, "
                                f"{M} rows (batch {b} x block 32), bf16",
                        "bytes_per_call": nbytes, "flops_per_call": flops, "us_per_call": us,
                        "bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s",
                        "frac": ach / hbm, "peak_source": hbm_src}
        else:
            ach = flops / us / 1e6
            out[key] = {"case": f"LM head {V} x {D} + confidence reduction + threshold unmask, "
                                f"{M} rows (batch {b} x block 32), bf16",
                        "bytes_per_call": nbytes, "flops_per_call": flops, "us_per_call": us,
                        "bound": "tensor", "achieved": ach, "peak": tf, "unit": "TFLOP/s",
                        "frac": ach / tf, "peak_source": tf_src + " (burst: timed alone)"}
    ctx.device_status()
    return out


def run_gpu(args):
    import torch
    import torch.distributed as dist
    from block_kv_cache_b200 import fdllm, synth
    from block_kv_cache_b200.model import BlockDecoder, DeviceWeights

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))

    def barrier():
        if world > 1:
            dist.barrier()

    c = CFG
    ctx = fdllm.Context(local)
    w = DeviceWeights.random(shape(), seed=1234)
    L = c["prompt"] + c["gen"]
    bias = planted_bias(torch, c, rank, args.bias_hi) if args.planted_bias else (None, None)
    dec = BlockDecoder(ctx, w, c["batch"], L, c["block"], cache=args.cache, bias_tok=bias[0],
                       bias_val=bias[1])
    prompt = torch.from_numpy(synth.prompt_ids(7 + rank, c["batch"], c["prompt"],
                                               c["mask_id"])).cuda()
    t0 = time.perf_counter()
    dec.capture_all(c["prompt"], c["gen"], c["tau"], time_calls=True)
    capture_s = time.perf_counter() - t0
    # kernels each step graph launches (kernel nodes of the captured graphs)
    for key in list(dec.graphs):
        dec.kernel_launches(*key)
    nblk = c["gen"] // c["block"]

    # warm-up: W whole blocks
    dec.begin(prompt, c["tau"])
    for _ in range(max(args.warmup, 3)):
        dec.block()
        if dec.done:
            dec.begin(prompt, c["tau"])
    ctx.device_status()

    # timed: K whole blocks from the first block of a fresh decode (a block =
    # its refresh forward, then cached steps until it is decoded); a decode
    # that reaches its end starts again
    dec.begin(prompt, c["tau"])
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    toks, kinds, launches = 0, {}, 0
    step_ms = {}
    replayed = []
    dec.call_us.clear()
    with ClockSampler(local) as clk:
        ev0.record()
        for _ in range(args.steps):
            n, steps = dec.block()
            toks += n
            for kind, s, ms in steps:
                kinds[kind] = kinds.get(kind, 0) + 1
                step_ms.setdefault(kind, []).append(ms)
                replayed.append((kind, s))
            if dec.done:
                dec.begin(prompt, c["tau"])
        ev1.record()
        torch.cuda.synchronize()
    barrier()
    ms = ev0.elapsed_time(ev1)
    ctx.device_status()
    # kernels launched in the timed region: the kernel nodes of every step
    # graph replayed (counted from the captured graphs)
    launches = sum(dec.kernel_launches(k, s, c["tau"]) for k, s in replayed)

    ms_max, toks_all = combine_ranks(dist, world, ms, toks, "cuda")
    e2e = run_e2e(torch, ctx, w, c, args, rank)
    e2e_ms, e2e_toks = combine_ranks(dist, world, e2e["ms"], e2e["toks"], "cuda")
    e2e_val = e2e_toks / (e2e_ms / 1e3)
    kernels = kernel_rooflines(torch, ctx, w, read_peaks()) if rank == 0 and args.kernels else None

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(budget_s=20.0)

    if rank == 0:
        print(json.dumps(result_line(args, c, world, w, dec, toks, toks_all, kinds, step_ms, ms_max,
                                     capture_s, e2e, e2e_val, kernels, clk, cpu, launches)),
              flush=True)
    if args.profile_steps and rank == 0:
        s0 = c["prompt"]
        prof = {k: dec.profile_step(k, s0, c["tau"]) for k in ("refresh", dec.cached_kind())}
        print(json.dumps({"profile_us_per_step": prof}), flush=True)
    dec.graphs.clear()
    ctx.close()
    if world > 1:
        dist.destroy_process_group()


def planted_bias(torch, c, rank, hi=16.0):
    """A planted logit bias per generated position (token drawn != mask id, value
    ~ U(0, hi); 16 is the LM-head workload's): with random weights no confidence
    reaches tau, and this makes the threshold rule fire, as a trained model's
    confident positions would."""
    from block_kv_cache_b200 import synth
    g = synth.rng(4242 + rank)
    bt = g.integers(0, c["mask_id"], (c["batch"], c["gen"])).astype(np.int32)
    bv = g.uniform(0.0, hi, (c["batch"], c["gen"])).astype(np.float32)
    return torch.from_numpy(bt).cuda(), torch.from_numpy(bv).cuda()


def result_line(args, c, world, w, dec, toks, toks_all, kinds, step_ms, ms_max, capture_s, e2e,
                e2e_val, kernels, clk, cpu, launches):
    peaks = read_peaks()
    M = c["batch"] * c["block"]
    D, F = c["hidden"], c["ffn"]
    # algorithmic bytes of one FFN call: both weights once, the f32 residual
    # rows read for the norm and read + written by the down projection, x and
    # f each written and read back
    ffn_bytes = 3 * F * D * 2 + 2 * M * D * 2 + 2 * M * F * 2 + 3 * M * D * 4
    ffn_flops = 6.0 * M * D * F
    cached = dec.cached_kind()
    ffn_us = dec.call_us.get((cached, "ffn"), [])
    att_us = dec.call_us.get((cached, "qkv_attention"), [])
    full_us = dec.call_us.get(("refresh", "full_attention"), [])
    ffn_avg = statistics.fmean(ffn_us) if ffn_us else None
    roof = None
    if ffn_avg and cached == "cached":
        if M <= 256:
            # few rows: the call streams its weights (HBM-bound)
            kpeak, src = _peak(peaks, "hbm_gbs", 6650.0)
            ach, bound, unit = ffn_bytes / ffn_avg / 1e3, "hbm", "GB/s"
        else:
            # a batch of blocks: two dense GEMMs (tensor-bound) timed inside a
            # long step, so against the sustained bf16 peak
            kpeak, src = _peak(peaks, "bf16_tflops_sustained", 1400.0)
            ach, bound, unit = ffn_flops / ffn_avg / 1e6, "tensor", "TFLOP/s"
        # DRAM bytes read + written by the two kernels of one such call, from an
        # ncu capture of the same kernels at the LLaDA-8B shape (kernel_cases ffn
        # --rows 32 --n 12288 --k 4096): 205.08 + 3.57 + 104.40 + 1.63 MB
        traffic = (205_078_016 + 3_570_944 + 104_399_872 + 1_632_000
                   if (M, D, F) == (32, 4096, 12288) else None)
        roof = {"kernel": f"ffn call of layer 0 of a cached step (M={M}): RMSNorm, gate/up GEMM "
                          f"{2 * F}x{D}, SwiGLU, down GEMM {D}x{F} (with M <= 256 the RMSNorm "
                          f"and the SwiGLU run in the GEMM kernels' prologues)",
                "bytes_per_call": ffn_bytes, "flops_per_call": ffn_flops, "bound": bound,
                "achieved": ach, "peak": kpeak, "unit": unit, "frac": ach / kpeak,
                "traffic": traffic,
                "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum of the two "
                                  "kernels of one call" if traffic else "no capture at this shape",
                "peak_source": src, "avg_launch_us": ffn_avg, "launches_timed": len(ffn_us)}
    if kernels is not None and att_us:
        Hq, Hkv, d = c["heads"], c["kv_heads"], c["head_dim"]
        N = (Hq + 2 * Hkv) * d
        L = c["prompt"] + c["gen"]
        nbytes = (N * D * 2 + 2 * c["batch"] * Hkv * L * d * 2 + M * D * (4 + 2)
                  + 2 * M * Hq * d * 2)
        hbm, src = _peak(peaks, "hbm_gbs", 6650.0)
        a_us = statistics.fmean(att_us)
        kernels["qkv_attention_in_decode"] = {
            "case": f"layer 0 of every cached step: RMSNorm + q/k/v projection {N}x{D} (split-K "
                    f"weight stream) + RoPE + block-slot K/V store + DualCache attention over "
                    f"L = {L} (graph-replayed, events around the call)",
            "bytes_per_call": nbytes, "us_per_call": a_us, "bound": "hbm",
            "achieved": nbytes / a_us / 1e3, "peak": hbm, "unit": "GB/s",
            "frac": nbytes / a_us / 1e3 / hbm, "peak_source": src, "calls_timed": len(att_us)}
    if kernels is not None and full_us:
        Hq, d, L, b = c["heads"], c["head_dim"], c["prompt"] + c["gen"], c["batch"]
        flops = 4.0 * b * Hq * L * L * d
        tfp, src = _peak(peaks, "bf16_tflops_sustained", 1400.0)
        f_us = statistics.fmean(full_us)
        kernels["full_attention_in_refresh"] = {
            "case": f"layer 0 of every refresh: bidirectional attention of all {L} positions "
                    f"({Hq} q heads / {c['kv_heads']} kv heads x {d}, batch {b}; graph-replayed, "
                    f"events around the call)",
            "flops_per_call": flops, "us_per_call": f_us, "bound": "tensor",
            "achieved": flops / f_us / 1e6, "peak": tfp, "unit": "TFLOP/s",
            "frac": flops / f_us / 1e6 / tfp, "peak_source": src + " (inside a long step)",
            "calls_timed": len(full_us)}
    nsteps = sum(kinds.values())
    blocks = args.steps
    wl = WORKLOAD
    if args.cache != "dual" or args.planted_bias:
        wl += f" [cache={args.cache}{', planted bias' if args.planted_bias else ''}]"
    return {
        "metric": METRIC, "value": toks_all / (ms_max / 1e3), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded random init)",
        "config": {"workload": wl, "step": "one block: its refresh forward, then "
                                           f"{cached} steps until no position of the block "
                                           "is masked",
                   "batch": c["batch"], "prompt": c["prompt"], "gen": c["gen"],
                   "block": c["block"], "tau": c["tau"], "cache": args.cache,
                   "planted_bias": bool(args.planted_bias),
                   **({"planted_bias_hi": args.bias_hi} if args.planted_bias else {}),
                   **({"batching": args.batching} if args.batching != "lockstep" else {}),
                   "layers": c["layers"], "hidden": c["hidden"], "vocab": c["vocab"],
                   "parallelism": f"replicas x{world}",
                   "blocks_timed": blocks, "decode_steps_timed": nsteps,
                   "steps_by_kind": kinds, "tokens_decoded": toks,
                   "tokens_per_decode_step": toks / max(nsteps, 1),
                   "host_ms_per_step": {k: statistics.median(v) for k, v in step_ms.items()},
                   "host_ms_per_step_mean": {k: statistics.fmean(v) for k, v in step_ms.items()},
                   "weights_gb": round(w.nbytes() / 1e9, 2),
                   "graph_capture_s": round(capture_s, 2),
                   "l2": f"no flush: {w.nbytes() / 1e9:.0f} GB of weights (> 126 MB L2) are "
                         f"streamed every step"},
        "gpu_launches": launches,
        "roofline": roof,
        "kernels": kernels,
        "e2e": {"value": e2e_val, "unit": "tokens/s", "h2d_bytes_per_step": e2e["h2d"],
                "d2h_bytes_per_step": e2e["d2h"], "path": e2e["path"]},
        "clocks": clk.summary(),
        "cpu_baseline": cpu,
    }


def run_e2e(torch, ctx, w, c, args, rank):
    """Whole decodes through the library's decode entry point (fdl_generate)
    from a pinned host prompt to a host copy of the sequence: the binding copies
    the prompt in, the library runs every block, the binding copies the sequence
    out; CUDA events around the whole call. With the device loop (default) the
    decode is one CUDA graph (each block's cached steps in a conditional WHILE
    node) that the context keeps: one untimed call captures it, as a server
    would once per shape, then one call is timed. The bytes per step are per
    block (the bench's step)."""
    from block_kv_cache_b200 import synth
    hp = torch.from_numpy(synth.prompt_ids(7 + rank, c["batch"], c["prompt"],
                                           c["mask_id"])).pin_memory()
    bias = planted_bias(torch, c, rank, args.bias_hi) if args.planted_bias else (None, None)
    m = w.native()
    device_loop = args.e2e_loop == "device" and args.batching == "lockstep"
    kw = dict(block=c["block"], tau=c["tau"], cache=args.cache, bias_tok=bias[0],
              bias_val=bias[1], device_loop=device_loop, batching=args.batching)
    if device_loop:
        ctx.generate(m, hp, c["gen"], **kw)           # captures and keeps the decode graph
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    x, steps = ctx.generate(m, hp, c["gen"], **kw)
    e1.record()
    torch.cuda.synchronize()
    ctx.device_status()
    m.close()
    blocks = c["gen"] // c["block"]
    d2h = x.numel() * 4 + (4 if device_loop else steps * c["batch"] * 4)
    return {"ms": e0.elapsed_time(e1), "toks": c["batch"] * c["gen"],
            "h2d": hp.numel() * 4 / blocks, "d2h": d2h / blocks,
            "path": f"fdl_generate (the library's decode loop, "
                    f"{'device loop: one CUDA graph per decode' if device_loop else 'host loop'}"
                    f"{'' if args.batching == 'lockstep' else ', batching ' + args.batching}"
                    f") on a host prompt: {steps} decode steps, one whole decode of {blocks} "
                    f"blocks"}


# ----------------------------------------------------------------------------- CPU oracle
class OracleSample:
    """A bounded sample of one block of the decode computed by the CPU oracle
    (float64 NumPy), for one sequence (the rows of a batch are independent, so
    a batch's tokens per second equal one sequence's):
      * a cached step: one transformer layer of the block's rows over the
        sequence's cache, then the full LM-head confidence of the block and the
        select; extrapolated as layers x layer + LM head;
      * the refresh: one layer of the full forward on a slice of REFRESH_ROWS
        query rows (their projections, attention over all L positions, FFN),
        whose cost is linear in the rows, extrapolated as layers x L / rows x
        slice + LM head.
    A block of the random-init workload decodes one position per step: one
    refresh and block - 1 cached steps."""
    REFRESH_ROWS = 128

    def __init__(self, seed=0):
        from oracle import fastdllm as O
        from block_kv_cache_b200 import synth
        self.O = O
        c = CFG
        P = synth.model_params(vocab=8, hidden=c["hidden"], n_layers=1, n_q_heads=c["heads"],
                               n_kv_heads=c["kv_heads"], head_dim=c["head_dim"], ffn=c["ffn"],
                               seed=seed, w_std=0.02, dtype="bf16", qkv_bias=c["qkv_bias"])
        self.P = P
        g = synth.rng(seed + 1)
        L = c["prompt"] + c["gen"]
        self.k = g.standard_normal((c["kv_heads"], L, c["head_dim"]))
        self.v = g.standard_normal((c["kv_heads"], L, c["head_dim"]))
        self.h = g.standard_normal((c["block"], c["hidden"]))
        self.hr = g.standard_normal((self.REFRESH_ROWS, c["hidden"]))
        self.lm = synth.lmhead_case(rows=c["block"], hidden=c["hidden"], vocab=c["vocab"],
                                    seed=seed, w_seed=0, mask_id=c["mask_id"])

    def _layer(self, h, pos):
        O, P = self.O, self.P
        Lw = P.layers[0]
        hn = O.rms_norm(h, Lw["attn_norm"], P.rms_eps)
        q, k, v = O._layer_qkv(P, Lw, hn, pos)
        self.k[:, pos] = np.transpose(k, (1, 0, 2))
        self.v[:, pos] = np.transpose(v, (1, 0, 2))
        o, _ = O.attention(q, self.k, self.v)
        O._layer_rest(P, Lw, h, o)

    def _head(self):
        O, c = self.O, CFG
        r = O.lmhead_confidence(self.lm.h, self.lm.w, self.lm.bias_tok, self.lm.bias_val)
        O.select_positions(r.conf[:c["block"]], np.ones(c["block"], bool), c["tau"])

    def block_seconds(self):
        """(block s, cached step s, refresh s, layer of a cached step s, refresh
        slice s, LM head s)."""
        c = CFG
        L = c["prompt"] + c["gen"]
        s = c["prompt"]
        t0 = time.perf_counter()
        self._layer(self.h, np.arange(s, s + c["block"]))
        t_layer = time.perf_counter() - t0
        t0 = time.perf_counter()
        self._head()
        t_head = time.perf_counter() - t0
        t0 = time.perf_counter()
        self._layer(self.hr, np.arange(0, self.REFRESH_ROWS))
        t_slice = time.perf_counter() - t0
        cached = c["layers"] * t_layer + t_head
        refresh = c["layers"] * t_slice * (L / self.REFRESH_ROWS) + t_head
        return refresh + (c["block"] - 1) * cached, cached, refresh, t_layer, t_slice, t_head


def _threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        return os.cpu_count()


def _sample_text(est, n):
    med = lambda i: statistics.median(e[i] for e in est)
    c = CFG
    L = c["prompt"] + c["gen"]
    return (f"{n} samples, float64 NumPy, one sequence: a cached step = {c['layers']} x one "
            f"layer of the block's {c['block']} rows over a {L}-row cache ({med(3):.3f} s) + the "
            f"full LM head ({med(5):.3f} s); the refresh = {c['layers']} x {L // 128} x one layer "
            f"on a {OracleSample.REFRESH_ROWS}-row slice ({med(4):.3f} s) + the LM head; a "
            f"block = refresh + {c['block'] - 1} cached steps (one position per step, as on the "
            f"GPU with random weights)")


def cpu_baseline(budget_s=20.0):
    smp = OracleSample()
    t0 = time.perf_counter()
    est, n = [], 0
    while time.perf_counter() - t0 < budget_s or n == 0:
        est.append(smp.block_seconds())
        n += 1
    block_s = statistics.median(e[0] for e in est)
    return {"value": CFG["block"] / block_s, "unit": "tokens/s", "cores": _threads(),
            "kind": "oracle", "host_cpus": os.cpu_count(), "sample": _sample_text(est, n)}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    smp = OracleSample()
    for _ in range(args.warmup):
        smp.block_seconds()
    t0 = time.perf_counter()
    est = [smp.block_seconds() for _ in range(args.steps)]
    wall = time.perf_counter() - t0
    ext = sum(e[0] for e in est)
    val = CFG["block"] * args.steps / ext
    out = {"impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": ext * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded random init)",
           "config": {"workload": WORKLOAD, "step": "one block: its refresh forward, then "
                                                    "cached steps until it is decoded",
                      "batch": CFG["batch"], "prompt": CFG["prompt"],
                      "gen": CFG["gen"], "block": CFG["block"], "tau": CFG["tau"],
                      "layers": CFG["layers"], "parallelism": "cpu oracle"},
           "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": _threads(),
                            "kind": "oracle", "host_cpus": os.cpu_count(),
                            "sample": _sample_text(est, args.steps) +
                            f" ({wall:.1f} s of CPU time for {args.steps} blocks)"},
           "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


# ----------------------------------------------------------------------------- sweeps
# The pages' ablations on synthetic inputs: block size, threshold and
# generation length (ICLR reviews, reviews 1-2: the block-size ablation), and
# the README evaluation table's four columns: the base decode (no cache, one
# position per step), +cache (DualCache, one position per step), +parallel
# (no cache, threshold rule) and both. All with the planted logit bias, so
# that the threshold rule fires as it would on a trained model's confident
# positions; tau = 1 decodes exactly one position per step. The bias is drawn
# from U(0, 24): with the random LM head's logit spread about 7% of U(0, 16)
# biases reach a confidence of 0.9, about 40% of U(0, 24) ones.
SWEEP_BIAS_HI = 24.0
SWEEP_GRID = (
    [dict(block=b, tau=0.9, gen=1024, cache="dual") for b in (8, 16, 32, 64, 128)]
    + [dict(block=32, tau=t, gen=1024, cache="dual") for t in (0.7, 1.0)]
    + [dict(block=32, tau=0.9, gen=g, cache="dual") for g in (256, 512)]
    + [dict(block=32, tau=t, gen=g, cache=m) for g in (256, 512)
       for m, t in (("none", 1.0), ("dual", 1.0), ("none", 0.9), ("prefix", 0.9),
                    ("prefix", 1.0))]
)


def run_sweep(args):
    """One whole decode per grid point (every step graph captured before the
    timed decode), CUDA events around it; one JSON line per point."""
    import torch
    from block_kv_cache_b200 import fdllm, synth
    from block_kv_cache_b200.model import BlockDecoder, DeviceWeights
    torch.cuda.set_device(0)
    base = dict(CFG)
    ctx = fdllm.Context(0)
    w = DeviceWeights.random(shape(), seed=1234)
    for pt in SWEEP_GRID:
        c = dict(base, **pt)
        L = c["prompt"] + c["gen"]
        bias = planted_bias(torch, c, 0, SWEEP_BIAS_HI)
        dec = BlockDecoder(ctx, w, c["batch"], L, c["block"], cache=c["cache"],
                           bias_tok=bias[0], bias_val=bias[1])
        prompt = torch.from_numpy(synth.prompt_ids(7, c["batch"], c["prompt"],
                                                   c["mask_id"])).cuda()
        dec.capture_all(c["prompt"], c["gen"], c["tau"])
        dec.begin(prompt, c["tau"])                 # untimed: every graph replayed once
        while not dec.done:
            dec.block()
        dec.begin(prompt, c["tau"])
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        kinds, toks = {}, 0
        e0.record()
        while not dec.done:
            n, steps = dec.block()
            toks += n
            for kind, _, _ in steps:
                kinds[kind] = kinds.get(kind, 0) + 1
        e1.record()
        torch.cuda.synchronize()
        ctx.device_status()
        ms = e0.elapsed_time(e1)
        nsteps = sum(kinds.values())
        print(json.dumps({"sweep": pt, "bias_hi": SWEEP_BIAS_HI, "tokens": toks,
                          "decode_steps": nsteps,
                          "tokens_per_step": toks / nsteps, "ms": ms,
                          "tokens_per_s": toks / (ms / 1e3), "steps_by_kind": kinds}),
              flush=True)
        dec.graphs.clear()
        del dec
        torch.cuda.empty_cache()
    ctx.close()


def main():
    global WORKLOAD
    args = parse()
    CFG.clear()
    CFG.update(CONFIGS[args.config])
    WORKLOAD = CFG["workload"]
    for k in ("block", "gen", "tau"):
        v = getattr(args, k)
        if v is not None and v != CFG[k]:
            CFG[k] = v
            WORKLOAD += f" [{k} {v}]"
    if args.impl == "reference":
        run_reference(args)
    elif args.sweep:
        run_sweep(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
