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
        # the 16-pair batch split across the ranks: gather every rank's share
        plan = bench.rank_plan("batch16_n16", 16, w, r, lr)
        shares = [None] * w
        dist.all_gather_object(shares, (plan["device"], list(plan["items"]), plan["scaling"]))
        dist.barrier()
        q.put((r, w, lr, mx, rate, shares, bench.rank_plan("rot1_n16", 1, w, r, lr)["items"]))
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
    for r, (rank, w, lr, mx, rate, shares, replica) in enumerate(out):
        assert (rank, w, lr) == (r, 2, r)
        assert mx == 15.0                              # the slowest rank's time, on every rank
        assert rate == pytest.approx(3 * 100 * 2 / 15e-3)  # all ranks' units / slowest time
        # rank k's context is on GPU k; the batch's pairs are covered exactly once
        assert [d for d, _, _ in shares] == [0, 1]
        assert sorted(i for _, items, _ in shares for i in items) == list(range(16))
        assert all(sc == "strong" for _, _, sc in shares)
        assert list(replica) == [0]                    # other workloads run whole on every rank


def test_single_process_defaults():
    import bench
    assert bench.max_over_ranks(7.5) == 7.5
    assert bench.whole_job_rate(1, 300, 1, 150.0) == pytest.approx(2000.0)


@pytest.mark.parametrize("n,world", [(16, 1), (16, 2), (16, 3), (16, 8), (5, 8), (0, 2)])
def test_shard_covers_every_unit_once(n, world):
    import bench
    got = [list(bench.shard(n, world, r)) for r in range(world)]
    assert sorted(i for g in got for i in g) == list(range(n))
    assert max(map(len, got)) - min(map(len, got)) <= 1
