"""Multi-GPU replicas, host logic only: two gloo ranks on the CPU.

The layer shards by tokens with no data-path collective (replicas); what the
ranks share is the barrier and the max-over-ranks timing that bench.py uses.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from combine_moe_route_14_b200 import inputs as I
from combine_moe_route_14_b200 import replicas as Rp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [12.5, 31.0][rank]
        m = Rp.max_over_ranks(local_ms)
        dist.barrier()
        X = I.random_bf16((8, 16), Rp.replica_token_seed(0, rank), "X")
        digest = float(X.float().sum())
        digests = [None] * world
        dist.all_gather_object(digests, digest)
        out.put((rank, m, digests))
    finally:
        dist.destroy_process_group()


def test_two_ranks_agree_on_the_slowest_time_and_own_batches():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [r[1] for r in res] == [31.0, 31.0]          # every rank sees the max
    d0, d1 = res[0][2]
    assert d0 != d1                                      # each rank has its own tokens


def test_weak_scaling_throughput():
    assert Rp.weak_scaling_throughput(4096, 20, 2, 40.0) == pytest.approx(4096 * 20 * 2 / 0.04)
    assert Rp.max_over_ranks(3.0) == 3.0                 # no process group: identity
    with pytest.raises(ValueError):
        Rp.weak_scaling_throughput(1, 1, 1, 0.0)
