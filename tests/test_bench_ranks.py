"""The multi-rank path of bench.py on CPU: two gloo ranks combine their timed
figures the way the GPU arm does (slowest rank's time, all ranks' tokens)."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        # rank r: a step time of 10 (r + 1) ms and 32 (r + 1) tokens
        ms, toks = bench.combine_ranks(dist, world, 10.0 * (rank + 1), 32 * (rank + 1), "cpu")
        q.put((rank, ms, toks))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_ranks_combine_to_slowest_time_and_all_tokens(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    want_ms = 10.0 * world
    want_toks = 32.0 * world * (world + 1) / 2
    for rank, ms, toks in got:
        assert ms == want_ms and toks == want_toks, (rank, ms, toks)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.combine_ranks(None, 1, 12.5, 7, "cpu") == (12.5, 7.0)


def test_bench_configs_are_complete_and_switchable():
    """Both workloads carry every field the decoder and the bench read, and
    the model shape follows the selected one."""
    import bench
    keys = {"layers", "hidden", "heads", "kv_heads", "head_dim", "ffn", "vocab", "mask_id",
            "batch", "prompt", "gen", "block", "tau", "qkv_bias", "workload"}
    for name, c in bench.CONFIGS.items():
        assert keys <= set(c), name
        assert c["heads"] % c["kv_heads"] == 0 and 0 <= c["mask_id"] < c["vocab"]
        assert c["prompt"] % c["block"] == 0 and c["gen"] % c["block"] == 0
    saved = dict(bench.CFG)
    try:
        bench.CFG.clear()
        bench.CFG.update(bench.CONFIGS["dream"])
        sh = bench.shape()
        assert (sh.n_layers, sh.hidden, sh.n_kv_heads, sh.qkv_bias) == (28, 3584, 4, True)
    finally:
        bench.CFG.clear()
        bench.CFG.update(saved)
