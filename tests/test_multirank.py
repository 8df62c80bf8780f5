"""Host logic of the multi-rank path, on CPU with the gloo backend.

The path shards without a data-path collective: a one-layer workload gives
every rank its own layer (weak scaling), the 36-layer stack is split over
the ranks by layer, and the only cross-rank step is the max of the per-rank
times.  These tests run world_size 2 (and the split for 1..8 ranks) on CPU.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from post_int4_weight_b200 import pipeline
from post_int4_weight_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", range(1, 9))
def test_shard_layers_partition(world):
    n = wl.WORKLOADS["qwen3_8b_stack36"].layers
    shards = [pipeline.shard_layers(n, world, r) for r in range(world)]
    flat = sorted(l for s in shards for l in s)
    assert flat == list(range(n))                       # every layer exactly once
    sizes = [len(s) for s in shards]
    assert max(sizes) - min(sizes) <= 1                 # balanced


def test_shard_layers_rejects_bad_rank():
    with pytest.raises(ValueError):
        pipeline.shard_layers(36, 2, 2)
    with pytest.raises(ValueError):
        pipeline.shard_layers(36, 0, 0)


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        mine = pipeline.shard_layers(36, world, rank)
        every = [None] * world
        dist.all_gather_object(every, mine)
        t = pipeline.max_over_ranks(1.5 + rank)           # per-rank "times"
        # the weak-scaling seeds of a one-layer workload differ per rank
        work = wl.WORKLOADS["single_linear_256x512"]
        (_, Ws, X), = wl.group_inputs(work, 0, "cpu", work.seed + 1000 * rank)
        sig = [float(Ws[0].float().sum()), float(X.float().abs().sum())]
        sigs = [None] * world
        dist.all_gather_object(sigs, sig)
        q.put((rank, every, t, sigs))
    finally:
        dist.destroy_process_group()


def test_gloo_two_ranks_shard_and_max():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, every, t, sigs in res:
        assert sorted(l for s in every for l in s) == list(range(36))
        assert set(every[0]).isdisjoint(every[1])
        assert t == 2.5                                   # max over ranks, on every rank
        assert sigs[0] != sigs[1]                         # independent layers per rank


def test_max_over_ranks_without_group():
    assert pipeline.max_over_ranks(3.25) == 3.25


def test_reference_arm_two_ranks_prints_one_line():
    """bench.py --impl reference under torchrun with 2 ranks on CPU: rank 0
    prints exactly one JSON line, the other rank exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           "--nproc-per-node", "2", "--master-addr", "127.0.0.1", "--master-port",
           str(port), os.path.join(ROOT, "bench.py"), "--impl", "reference",
           "--gpus", "2", "--steps", "2", "--warmup", "0",
           "--workload", "single_linear_256x512"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2
    assert rec["value"] > 0 and rec["e2e"]["h2d_bytes_per_step"] == 0
