"""Multi-process host logic of the benchmark on CPU (gloo, world size 2):
units shard across ranks with no data-path collective, and the timing is the
maximum over ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        lo, hi = bench.shard_units(17, world, rank)
        mine = [1.0 + rank, 10.0 - rank]
        mx = bench.max_over_ranks(mine, dist)
        got = [None] * world
        dist.all_gather_object(got, (lo, hi))
        q.put((rank, mx, got))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_sharding_and_max_timing(world):
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
    for rank, mx, shards in res:
        assert mx == [float(world), 10.0]
        covered = sorted(u for lo, hi in shards for u in range(lo, hi))
        assert covered == list(range(17))           # every unit exactly once
        assert all(hi - lo <= 9 for lo, hi in shards)
