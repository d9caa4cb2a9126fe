"""The multi-process path of bench.py on CPU: 2 ranks over gloo.

Each rank times its own key switches (weak scaling, no data-path
collective); the job's time is the slowest rank's, found with one MAX
all-reduce after the timed region, and the whole-job rate counts every
rank's units.  The GPU path uses the same functions over NCCL.
"""
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


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w, r, lr = bench.dist_setup()
        ms = 10.0 + 5.0 * rank           # rank 1 is the slow one
        mx = bench.max_over_ranks(ms, dist, "cpu")
        rate = bench.whole_job_rate(3, 100, w, mx)
        dist.barrier()
        q.put((r, w, lr, mx, rate))
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_timing():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, (rank, w, lr, mx, rate) in enumerate(out):
        assert (rank, w, lr) == (r, 2, r)
        assert mx == 15.0                              # the slowest rank's time, on every rank
        assert rate == pytest.approx(3 * 100 * 2 / 15e-3)  # all ranks' units / slowest time


def test_single_process_defaults():
    import bench
    assert bench.max_over_ranks(7.5) == 7.5
    assert bench.whole_job_rate(1, 300, 1, 150.0) == pytest.approx(2000.0)
