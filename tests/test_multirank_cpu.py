"""The multi-rank plumbing of bench.py on CPU ranks (gloo, world size 2):
each rank runs its own batch, times are the slowest rank's, the throughput is
all ranks' tokens over that time, and the reference arm's extra ranks exit
without work."""
import datetime
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    ms = [10.0, 12.5][rank]
    m = bench.max_over_ranks(ms, world, "cpu")
    v = bench.whole_job_tokens_per_s(world, 64, 100, m)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, m, v))


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [12.5, 12.5]
    assert all(abs(r[2] - 2 * 64 * 100 / 0.0125) < 1e-6 for r in res)


def test_reference_arm_extra_ranks_exit_without_work(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")

    class A:
        tokens = 0
        steps = 3
        warmup = 3
        gpus = 2

    assert bench.run_reference(A()) == 0


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.0, 1) == 7.0
    assert bench.whole_job_tokens_per_s(1, 64, 10, 1000.0) == 640.0
