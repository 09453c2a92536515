"""The multi-rank plumbing of bench.py (replicas: no data-path collective) on
CPU with gloo, world size 2: the whole-job throughput counts every rank's
tokens over the slowest rank's time, and every rank takes the same collective
steps."""
import os

import pytest
import torch.multiprocessing as mp


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    elapsed = 100.0 if rank == 0 else 250.0           # rank 1 is the slow one
    value, emax = bench.job_throughput(1024.0, elapsed, world)
    bench.barrier(world)
    q.put((rank, value, emax))
    dist.destroy_process_group()


def test_job_throughput_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, value, emax in res:
        assert emax == 250.0
        assert value == pytest.approx(2 * 1024.0 / 0.25)


def test_single_rank_is_identity():
    import bench
    v, e = bench.job_throughput(256.0, 100.0, 1)
    assert e == 100.0 and v == pytest.approx(2560.0)
