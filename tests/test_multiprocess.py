"""Multi-process host logic on CPU (gloo, world size 2): the sharding of
independent (batch, kv-head) units across ranks and the max-over-ranks
timing reduction bench.py uses."""

import importlib.util
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from exact_attention_104_b200.workloads import shard_units

_ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(_ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, B, Hkv, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = shard_units(B, Hkv, rank, world)
        gathered = [None] * world
        dist.all_gather_object(gathered, mine)
        # per-rank elapsed time, reduced by bench.py's own helper (gloo on CPU
        # here; NCCL on CUDA tensors in the bench)
        tmax = _bench().reduce_max_over_ranks(float(rank + 1) * 1.5, world, "cpu")
        if rank == 0:
            q.put((gathered, tmax))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("B,Hkv", [(8, 16), (1, 3), (3, 1)])
def test_units_are_split_once_and_max_reduce(B, Hkv):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, B, Hkv, q)) for r in range(world)]
    for p in procs:
        p.start()
    gathered, tmax = q.get(timeout=120)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    flat = [u for part in gathered for u in part]
    assert sorted(flat) == [(b, h) for b in range(B) for h in range(Hkv)]
    assert len(set(flat)) == len(flat)
    assert abs(len(gathered[0]) - len(gathered[1])) <= 1
    assert tmax == 3.0


def test_shard_units_more_ranks_than_units():
    parts = [shard_units(1, 1, r, 4) for r in range(4)]
    assert sum(len(p) for p in parts) == 1 and parts[0] == [(0, 0)]
