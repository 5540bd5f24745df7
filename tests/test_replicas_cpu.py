"""The multi-GPU path is replicas only (the decode weight stream has no exchange
step): ranks run independent copies, time themselves, and the job reports the
slowest rank's time.  This checks that host logic with world_size 2 over gloo
on the CPU: every rank sees the max, and the whole-job rate counts every
replica's bytes against that time."""
import os
import socket

import pytest


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        t_local = 0.25 if rank == 0 else 0.75          # rank 1 is the slow one
        t = bench.max_over_ranks(t_local, torch.device("cpu"), world)
        q.put((rank, t, bench.job_gbs(world, 10**9, 4, t)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_replicas_report_the_slowest_rank():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, t, gbs in got:
        assert t == pytest.approx(0.75)                  # the max over ranks, on every rank
        assert gbs == pytest.approx(2 * 4 * 1e9 / 0.75 / 1e9)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(0.5, None, 1) == 0.5
    assert bench.job_gbs(1, 2 * 10**9, 3, 2.0) == pytest.approx(3.0)
