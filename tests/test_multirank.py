"""The benchmark's multi-rank plumbing on CPU with gloo, world size 2: the
(b,h) units shard with no data-path collective, so the only cross-rank steps
are a barrier and the max-over-ranks time; the job value is the sum of all
ranks' tokens over that max."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, results):
    import datetime
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        local_ms = 10.0 * (rank + 1)  # rank 1 is the slow one
        value, total = bench.weak_scaling_value(world, tokens_per_step=1000, steps=5, local_ms=local_ms)
        results[rank] = (value, total)
    finally:
        dist.destroy_process_group()


def test_weak_scaling_max_over_ranks_gloo():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        results = m.dict()
        mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
        res = dict(results)
    assert set(res) == {0, 1}
    for rank in (0, 1):
        value, total = res[rank]
        assert total == pytest.approx(20.0)                       # max over ranks
        assert value == pytest.approx(2 * 1000 * 5 / 0.020)      # all ranks' tokens / job time


def test_single_rank_is_identity():
    import bench
    v, t = bench.weak_scaling_value(1, 100, 4, 8.0)
    assert t == 8.0 and v == pytest.approx(100 * 4 / 0.008)
