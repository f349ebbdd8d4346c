"""The multi-rank host logic of bench.py on CPU: two gloo ranks, max-over-ranks timing and the
whole-job (weak-scaling) rate. The data path has no collective; only these reductions cross ranks."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    import bench

    local_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
    m = bench.max_over_ranks(local_ms, dist, "cpu")
    rate = bench.whole_job_rate(1000, 4, world, m)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, m, rate))


def test_two_ranks_max_time_and_weak_scaling_rate():
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
    for rank, m, rate in res:
        assert m == 15.0
        assert rate == pytest.approx(1000 * 4 * 2 / 0.015)


def test_single_rank_needs_no_process_group():
    import bench

    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
