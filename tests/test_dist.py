"""Host-side multi-process path of bench.py, on CPU with gloo, world size 2:
the step time is the maximum over ranks and the work is the sum over ranks."""
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
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms, units = bench.reduce_max_sum(10.0 + 5.0 * rank, 100.0 * (rank + 1))
        results[rank] = (ms, units)
    finally:
        dist.destroy_process_group()


def test_reduce_max_sum_two_ranks():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, results)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert results[0] == (15.0, 300.0)
    assert results[1] == (15.0, 300.0)


def test_reduce_max_sum_single_process_is_identity():
    import bench
    assert bench.reduce_max_sum(3.5, 7.0) == (3.5, 7.0)
