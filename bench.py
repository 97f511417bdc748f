#!/usr/bin/env python3
"""Benchmark: Fast-dLLM block decoding of a random-init LLaDA-8B-shaped model
on B200.

Workload: bidirectional transformer of the LLaDA-8B shape (32 layers, hidden
4096, 32 heads x 128, SwiGLU FFN 12288, RMSNorm, RoPE, vocab 126464), bf16,
batch 1, prompt 1024 uniform random ids, gen 1024, block 32, DualCache,
threshold 0.9. One step = one decoding step of the whole hot path:
  * the first step of every block is a refresh: a full forward over all 2048
    positions rewriting every layer's K/V cache, then the block's logits;
  * the others are cached DualCache steps: only the block's 32 rows go
    through the 32 layers (projection + RoPE + cache-slot write, attention
    over [prefix | block | masked suffix], O proj, SwiGLU FFN);
  each step ends with the fused LM-head confidence reduction and the
  threshold select/scatter; the host reads back 8 bytes (remaining and
  decoded counts) to decide refresh vs cached for the next step.
Each (step kind, block) is a CUDA graph captured before timing. Weights are
seeded random draws on the device (16 GB, larger than L2, streamed every
step), so no L2 flush is needed. With random weights no confidence reaches
0.9, so every step decodes one token (the fallback rule) and tokens/s equals
steps/s.

Prints one JSON line on rank 0. `--impl reference` times the CPU oracle on
the same workload instead (bounded sample per step, extrapolated).
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
    p.add_argument("--steps", type=int, default=64)
    p.add_argument("--warmup", type=int, default=4)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--e2e-steps", type=int, default=40)
    p.add_argument("--no-cpu-baseline", action="store_true")
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
    dec = BlockDecoder(ctx, w, c["batch"], L, c["block"])
    prompt = synth.prompt_ids(7 + rank, c["batch"], c["prompt"], c["mask_id"])
    t0 = time.perf_counter()
    dec.capture_all(c["prompt"], c["gen"], c["tau"], time_ffn=True)
    capture_s = time.perf_counter() - t0
    # kernels each step graph launches (kernel nodes of the captured graphs)
    for key in list(dec.graphs):
        dec.kernel_launches(*key)

    dec.begin(prompt, c["tau"])
    for _ in range(max(args.warmup, 3)):
        dec.step()
        if dec.done:
            dec.begin(prompt, c["tau"])
    ctx.device_status()

    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    toks, kinds, launches = 0, {"refresh": 0, "cached": 0}, 0
    sw_ms, sw_n = 0.0, 0
    step_ms = {"refresh": [], "cached": []}
    with ClockSampler(local) as clk:
        ev0.record()
        for _ in range(args.steps):
            h0 = time.perf_counter()
            toks += dec.step()
            step_ms[dec.last_kind].append((time.perf_counter() - h0) * 1e3)
            launches += dec.kernel_launches(*dec._last_key)
            kinds[dec.last_kind] += 1
            if dec.last_kind == "cached":
                for a, b in dec.last_timers():
                    sw_ms += a.elapsed_time(b)
                    sw_n += 1
            if dec.done:
                dec.begin(prompt, c["tau"])
        ev1.record()
        torch.cuda.synchronize()
    barrier()
    ms = ev0.elapsed_time(ev1)
    ctx.device_status()

    ms_max, toks_all = combine_ranks(dist, world, ms, toks, "cuda")
    e2e = run_e2e(torch, dec, prompt, args.e2e_steps)
    e2e_ms, e2e_toks = combine_ranks(dist, world, e2e["ms"], e2e["toks"], "cuda")
    e2e_val = e2e_toks / (e2e_ms / 1e3)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(budget_s=20.0)

    if rank == 0:
        peaks = read_peaks()
        peak = peaks.get("hbm_gbs") or 6650.0
        M = c["batch"] * c["block"]
        D, F = c["hidden"], c["ffn"]
        # algorithmic bytes of one FFN call: both weights once, the f32 residual
        # rows read for the norm and read + written by the down projection, x and
        # f each written and read back
        ffn_bytes = 3 * F * D * 2 + 2 * M * D * 2 + 2 * M * F * 2 + 3 * M * D * 4
        ffn_flops = 6.0 * M * D * F
        sw_avg_ms = sw_ms / max(sw_n, 1)
        if M <= 256:
            # few rows: the call streams its weights (HBM-bound)
            ach = ffn_bytes / (sw_avg_ms / 1e3) / 1e9 if sw_n else None
            bound, unit, kpeak, src = "hbm", "GB/s", peak, (
                "MEASURED_PEAKS.json hbm_gbs (measured)" if peaks.get("hbm_gbs")
                else "fallback 6650 GB/s")
        else:
            # a batch of blocks: the call is two dense GEMMs (tensor-bound), timed
            # inside a long step, so against the sustained bf16 peak
            ach = ffn_flops / (sw_avg_ms / 1e3) / 1e12 if sw_n else None
            kpeak = peaks.get("bf16_tflops_sustained") or 1400.0
            bound, unit, src = "tensor", "TFLOP/s", (
                "MEASURED_PEAKS.json bf16_tflops_sustained (measured)"
                if peaks.get("bf16_tflops_sustained") else "fallback 1400 TFLOP/s sustained")
        # DRAM bytes read + written by the two kernels of one such call, from an
        # ncu capture of the same kernels at the LLaDA-8B shape (kernel_cases ffn
        # --rows 32 --n 12288 --k 4096): 205.09 + 3.33 + 104.40 + 1.59 MB
        ffn_traffic = (205_085_184 + 3_330_560 + 104_400_896 + 1_594_624
                       if (M, D, F) == (32, 4096, 12288) else None)
        out = {
            "metric": METRIC, "value": toks_all / (ms_max / 1e3), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded random init)",
            "config": {"workload": WORKLOAD, "batch": c["batch"], "prompt": c["prompt"],
                       "gen": c["gen"], "block": c["block"], "tau": c["tau"],
                       "layers": c["layers"], "hidden": c["hidden"], "vocab": c["vocab"],
                       "parallelism": f"replicas x{world}",
                       "steps_by_kind": kinds, "tokens_decoded": toks,
                       "host_ms_per_step": {k: (statistics.median(v) if v else None)
                                            for k, v in step_ms.items()},
                       "host_ms_per_step_mean": {k: (statistics.fmean(v) if v else None)
                                                 for k, v in step_ms.items()},
                       "weights_gb": round(w.nbytes() / 1e9, 2),
                       "graph_capture_s": round(capture_s, 2),
                       "l2": f"no flush: {w.nbytes() / 1e9:.0f} GB of weights (> 126 MB L2) "
                             f"are streamed every step"},
            "gpu_launches": launches,
            "roofline": {"kernel": f"ffn call of layer 0 of a cached step (M={M}): RMSNorm, "
                                   f"gate/up GEMM {2 * F}x{D}, SwiGLU, down GEMM {D}x{F} "
                                   f"(with M <= 256 the RMSNorm and the SwiGLU run in the "
                                   f"GEMM kernels' prologues)",
                         "bytes_per_call": ffn_bytes, "flops_per_call": ffn_flops,
                         "bound": bound, "achieved": ach, "peak": kpeak, "unit": unit,
                         "frac": (ach / kpeak) if ach else None, "traffic": ffn_traffic,
                         "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum of "
                                           "the two kernels of one call" if ffn_traffic
                         else "no capture at this shape",
                         "peak_source": src,
                         "avg_launch_us": sw_avg_ms * 1e3, "launches_timed": sw_n},
            "e2e": {"value": e2e_val, "unit": "tokens/s",
                    "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"]},
            "clocks": clk.summary(),
            "cpu_baseline": cpu,
        }
        print(json.dumps(out), flush=True)
    if args.profile_steps and rank == 0:
        s0 = c["prompt"] + dec.blk * c["block"] if not dec.done else c["prompt"]
        prof = {k: dec.profile_step(k, s0, c["tau"]) for k in ("cached", "refresh")}
        print(json.dumps({"profile_us_per_step": prof}), flush=True)
    dec.graphs.clear()
    ctx.close()
    if world > 1:
        dist.destroy_process_group()


def run_e2e(torch, dec, prompt, steps):
    """The decode through the public API from a pinned host prompt to a host
    copy of the sequence: prompt upload, `steps` steps (each reads its 8-byte
    counters back), final sequence download."""
    c = CFG
    hp = torch.from_numpy(np.ascontiguousarray(prompt, dtype=np.int32)).pin_memory()
    hx = torch.empty((c["batch"], c["prompt"] + c["gen"]), dtype=torch.int32).pin_memory()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    dec.begin(hp, c["tau"])
    toks = 0
    for _ in range(steps):
        toks += dec.step()
        if dec.done:
            break
    hx.copy_(dec.x, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    n = max(dec.steps, 1)
    return {"ms": e0.elapsed_time(e1), "toks": toks,
            "h2d": hp.numel() * 4 / n, "d2h": 8 * c["batch"] + hx.numel() * 4 / n}


# ----------------------------------------------------------------------------- CPU oracle
class OracleSample:
    """A bounded sample of one decode step computed by the CPU oracle (float64
    NumPy): one transformer layer of a cached block step of one sequence (its
    block rows over its cache) and the full LM-head confidence of the block; a
    sequence's step is extrapolated as layers x layer + LM head. The rows of a
    batch are independent, so the batch's tokens per second equal one
    sequence's (batch tokens per step, batch times the work)."""

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
        self.lm = synth.lmhead_case(rows=c["block"], hidden=c["hidden"], vocab=c["vocab"],
                                    seed=seed, w_seed=0, mask_id=c["mask_id"])

    def step_seconds(self):
        O, P, c = self.O, self.P, CFG
        Lw = P.layers[0]
        s = c["prompt"]
        t0 = time.perf_counter()
        hn = O.rms_norm(self.h, Lw["attn_norm"], P.rms_eps)
        q, k, v = O._layer_qkv(P, Lw, hn, np.arange(s, s + c["block"]))
        self.k[:, s:s + c["block"]] = np.transpose(k, (1, 0, 2))
        self.v[:, s:s + c["block"]] = np.transpose(v, (1, 0, 2))
        o, _ = O.attention(q, self.k, self.v)
        O._layer_rest(P, Lw, self.h, o)
        t_layer = time.perf_counter() - t0
        t0 = time.perf_counter()
        r = O.lmhead_confidence(self.lm.h, self.lm.w, self.lm.bias_tok, self.lm.bias_val)
        O.select_positions(r.conf[:c["block"]], np.ones(c["block"], bool), c["tau"])
        t_head = time.perf_counter() - t0
        return c["layers"] * t_layer + t_head, t_layer, t_head


def _threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        return os.cpu_count()


def cpu_baseline(budget_s=20.0):
    smp = OracleSample()
    t0 = time.perf_counter()
    est, n = [], 0
    while time.perf_counter() - t0 < budget_s or n == 0:
        est.append(smp.step_seconds())
        n += 1
    step_s = statistics.median(e[0] for e in est)
    return {"value": 1.0 / step_s, "unit": "tokens/s", "cores": _threads(), "kind": "oracle",
            "host_cpus": os.cpu_count(),
            "sample": f"{n} samples of one layer of a cached block step of one sequence "
                      f"({CFG['block']} rows over a {CFG['prompt'] + CFG['gen']}-row cache) + "
                      f"the full LM head, float64 NumPy; step time extrapolated as "
                      f"{CFG['layers']} x layer ({statistics.median(e[1] for e in est):.3f} s)"
                      f" + LM head ({statistics.median(e[2] for e in est):.3f} s), 1 token "
                      f"per step as on the GPU"}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    smp = OracleSample()
    for _ in range(args.warmup):
        smp.step_seconds()
    t0 = time.perf_counter()
    ext = 0.0
    for _ in range(args.steps):
        ext += smp.step_seconds()[0]
    wall = time.perf_counter() - t0
    val = args.steps / ext
    out = {"impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": ext * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded random init)",
           "config": {"workload": WORKLOAD, "batch": CFG["batch"], "prompt": CFG["prompt"],
                      "gen": CFG["gen"], "block": CFG["block"], "tau": CFG["tau"],
                      "layers": CFG["layers"], "parallelism": "cpu oracle"},
           "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": _threads(),
                            "kind": "oracle", "host_cpus": os.cpu_count(),
                            "sample": f"each step: one layer of a cached block step of one "
                                      f"sequence + the full LM head, extrapolated to "
                                      f"{CFG['layers']} layers ({wall:.1f} s of CPU time for "
                                      f"{args.steps} steps)"},
           "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    global WORKLOAD
    args = parse()
    CFG.clear()
    CFG.update(CONFIGS[args.config])
    WORKLOAD = CFG["workload"]
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
