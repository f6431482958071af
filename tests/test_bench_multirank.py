"""The bench's multi-rank aggregation on CPU: two gloo ranks (127.0.0.1),
each with its own timings; every rank must see the element-wise maximum and
the whole-job throughput must count both ranks' tokens over the slowest time."""
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


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    mine = [10.0 + rank, 20.0 - rank, 5.0 * (rank + 1)]
    got = bench.max_over_ranks(mine)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, got, bench.job_throughput(world, 7904, got[0])))


def test_max_over_ranks_and_job_throughput_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, thr in out:
        assert got == [11.0, 20.0, 10.0]
        assert thr == pytest.approx(2 * 7904 / 0.011)


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert bench.job_throughput(1, 100, 1000.0) == pytest.approx(100.0)
