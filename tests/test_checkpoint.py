"""Checkpoint / resume of the layer-by-layer run (host logic, CPU).

Failures are made on the host: a compute function that raises at a chosen
layer (as a crashed or preempted run would stop), a layer file that is
damaged or half written.  A rerun must compute exactly the layers that are
not verified on disk and end with the same results as a run that never
stopped.  The two-rank case runs gloo ranks on CPU, each checkpointing its
own share of the layers.
"""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from post_int4_weight_b200 import checkpoint as ck
from post_int4_weight_b200 import pipeline

CONFIG = {"workload": "qwen3_8b_stack36", "group_size": 128, "n_grid": 20, "flags": 0}


def _results(layer):
    g = torch.Generator().manual_seed(1000 + layer)
    return {"qweight": torch.randint(-2**31, 2**31 - 1, (64, 8), dtype=torch.int32, generator=g),
            "scales": torch.randn(4, 64, generator=g).to(torch.float16),
            "err": torch.randn(20, dtype=torch.float64, generator=g)}


class Stop(RuntimeError):
    pass


def _compute(fail_at=None, calls=None):
    def f(layer):
        if calls is not None:
            calls.append(layer)
        if layer == fail_at:
            raise Stop(f"stopped at layer {layer}")
        return _results(layer)
    return f


def _same(a, b):
    assert a.keys() == b.keys()
    for k in a:
        assert set(a[k]) == set(b[k])
        for key in a[k]:
            assert torch.equal(a[k][key], b[k][key]), (k, key)


def test_interrupted_run_resumes_at_the_failed_layer(tmp_path):
    layers = list(range(8))
    c1 = ck.StackCheckpoint(str(tmp_path / "run"), CONFIG)
    calls = []
    with pytest.raises(Stop):
        ck.run_layers(layers, _compute(fail_at=5, calls=calls), c1)
    assert calls == [0, 1, 2, 3, 4, 5]
    c2 = ck.StackCheckpoint(str(tmp_path / "run"), CONFIG)
    assert c2.completed(layers) == [0, 1, 2, 3, 4]
    calls = []
    out = ck.run_layers(layers, _compute(calls=calls), c2)
    assert calls == [5, 6, 7]
    ref = ck.run_layers(layers, _compute(), ck.StackCheckpoint(str(tmp_path / "ref"), CONFIG))
    _same(out, ref)


def test_damaged_or_half_written_layer_is_recomputed(tmp_path):
    layers = list(range(4))
    c = ck.StackCheckpoint(str(tmp_path), CONFIG)
    ck.run_layers(layers, _compute(), c)
    # damage layer 1's file, leave a half-written temporary of layer 2
    p1 = os.path.join(str(tmp_path), "layer_0001.pt")
    with open(p1, "r+b") as f:
        f.seek(100)
        f.write(b"\x00\xff\x00\xff")
    p2 = os.path.join(str(tmp_path), "layer_0002.pt")
    os.replace(p2, p2 + ".tmp")
    c2 = ck.StackCheckpoint(str(tmp_path), CONFIG)
    assert c2.completed(layers) == [0, 3]
    calls = []
    out = ck.run_layers(layers, _compute(calls=calls), c2)
    assert calls == [1, 2]
    for l in layers:
        for k, v in _results(l).items():
            assert torch.equal(out[l][k], v)


def test_other_configuration_is_refused(tmp_path):
    c = ck.StackCheckpoint(str(tmp_path), CONFIG)
    ck.run_layers([0], _compute(), c)
    with pytest.raises(ck.CheckpointMismatch):
        ck.StackCheckpoint(str(tmp_path), dict(CONFIG, group_size=64))
    with pytest.raises(KeyError):
        c.load(7)


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, root, fail_layer, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        mine = pipeline.shard_layers(36, world, rank)
        c = ck.StackCheckpoint(os.path.join(root, f"rank{rank}"), CONFIG)
        ok = torch.tensor([1])
        calls = []
        try:
            ck.run_layers(mine, _compute(fail_at=fail_layer, calls=calls), c)
        except Stop:
            ok[0] = 0
        # every rank learns on the host whether the pass finished everywhere
        dist.all_reduce(ok, op=dist.ReduceOp.MIN)
        q.put((rank, int(ok[0]), calls))
    finally:
        dist.destroy_process_group()


def test_two_ranks_resume_their_own_layers(tmp_path):
    world = 2
    ctx = mp.get_context("spawn")
    # first pass: rank 1 stops at its third layer
    fail = pipeline.shard_layers(36, world, 1)[2]
    for attempt, fail_layer in enumerate((fail, None)):
        q = ctx.Queue()
        port = _port()
        procs = [ctx.Process(target=_rank,
                             args=(r, world, port, str(tmp_path), fail_layer if r == 1 else None,
                                   q)) for r in range(world)]
        for p in procs:
            p.start()
        res = sorted(q.get(timeout=120) for _ in procs)
        for p in procs:
            p.join(timeout=60)
            assert p.exitcode == 0
        oks = {r: ok for r, ok, _ in res}
        calls = {r: c for r, _, c in res}
        if attempt == 0:
            assert oks == {0: 0, 1: 0}                       # both learn of the stop
            assert calls[0] == pipeline.shard_layers(36, world, 0)
            assert calls[1] == pipeline.shard_layers(36, world, 1)[:3]
        else:
            assert oks == {0: 1, 1: 1}
            assert calls[0] == []                            # nothing redone on rank 0
            assert calls[1] == pipeline.shard_layers(36, world, 1)[2:]
    for r in range(world):
        c = ck.StackCheckpoint(os.path.join(str(tmp_path), f"rank{r}"), CONFIG)
        mine = pipeline.shard_layers(36, world, r)
        assert c.completed(mine) == mine
