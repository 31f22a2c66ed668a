"""The replicated (N > 1) bench path on CPU: two gloo ranks reduce their
timings (max) and work (sum) the way bench.py does over NCCL."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        times = [10.0 + rank, 20.0 - rank, 1.5 * (rank + 1), 0.25]
        out = bench.reduce_over_ranks(times, 1e12 * (rank + 1), world, torch.device("cpu"))
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_reduce_over_ranks_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want_times = [10.0 + world - 1, 20.0, 1.5 * world, 0.25]
    want_work = 1e12 * world * (world + 1) / 2
    for r in range(world):
        times, work = res[r]
        assert times == want_times and work == want_work


def test_reduce_single_rank_is_identity():
    import bench
    times, work = bench.reduce_over_ranks([1.0, 2.0], 5.0, 1, torch.device("cpu"))
    assert times == [1.0, 2.0] and work == 5.0
