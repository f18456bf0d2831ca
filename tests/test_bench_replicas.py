"""Host-side logic of the multi-replica bench on CPU: two gloo ranks with
different per-rank times must both see the slowest rank's time, and the
whole-job value counts every rank's bytes over that time."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    ms = bench.reduce_max(10.0 + 5.0 * rank, dist, "cpu")
    q.put((rank, ms, bench.whole_job_gbs(2e9, ms, world)))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_take_the_max():
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
    for rank, ms, gbs in res:
        assert ms == 15.0
        assert gbs == pytest.approx(2 * 2e9 / 15e-3 / 1e9)


def test_single_process_identity():
    import bench
    assert bench.reduce_max(3.5, None, "cpu") == 3.5
    assert bench.whole_job_gbs(1e9, 1.0, 1) == pytest.approx(1000.0)
