"""Multi-rank host logic of the benchmark, on CPU with two gloo ranks: the
timing reduction takes the slowest rank, and the whole-job value counts every
rank's replica of the workload."""
import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        local = [10.0 + rank, 30.0 - rank, 5.0 * (rank + 1)]
        got = bench.max_over_ranks(local, world, torch.device("cpu"))
        value = bench.whole_job_tflops(2e12, 4, world, got[0])
        dist.barrier()
        q.put((rank, got, value))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_whole_job_value():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, value in results:
        assert got == [11.0, 30.0, 10.0]           # element-wise max over the two ranks
        assert value == pytest.approx(2e12 * 4 * 2 / 0.011 / 1e12)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.5, 2.5], 1, torch.device("cpu")) == [1.5, 2.5]
    assert bench.whole_job_tflops(1e12, 10, 1, 1000.0) == pytest.approx(10.0)
