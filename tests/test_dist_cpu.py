"""The multi-rank host logic of bench.py on CPU: two gloo ranks shard the batch
without overlap and agree on the slowest rank's time (max over ranks)."""
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


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    import bench
    from attention_learned_relative_b200.workloads import WORKLOADS
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    wl, span = bench.rank_workload(WORKLOADS["local_prefill_bf16"], rank, world)
    slowest = bench.max_over_ranks(1.5 + rank, torch.device("cpu"), world)
    out.put((rank, wl.seed, span, slowest))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_reduce():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    seeds = {r[1] for r in res}
    spans = [r[2] for r in res]
    assert len(seeds) == world                      # each rank draws its own shard
    assert spans == [(0, 2), (2, 4)]                # disjoint, covering the global batch
    assert all(r[3] == 2.5 for r in res)            # both see the slowest rank's time


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, torch.device("cpu"), 1) == 3.25
