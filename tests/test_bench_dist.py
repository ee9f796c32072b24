"""The multi-GPU path of bench.py is replicas only: each rank times its own
copy of the problem and rank 0 reports the whole job over the slowest rank's
device time.  These CPU tests run that host logic as two gloo ranks."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        t = bench.max_over_ranks(1.0 + rank * 0.25, world)   # rank 1 is the slow replica
        out.put((rank, t))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_takes_the_slowest_replica():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=10) for _ in range(world))
    assert got == {0: 1.25, 1: 1.25}


def _batches_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        calls = []

        def region(n):        # rank 0 fast, rank 1 slow: only the slow one alone would stop early
            calls.append(n)
            bench.barrier(world)
            secs = n * (0.001 if rank == 0 else 0.004)
            return secs, [secs / n] * n, 0.0, 1.0
        per, total, _, _ = bench.timed_batches(region, world, min_replays=10, min_secs=0.1, max_replays=1000)
        out.put((rank, len(calls), len(per), round(total, 6)))
    finally:
        dist.destroy_process_group()


def test_timed_batches_take_the_same_steps_on_every_rank():
    """Each timed region has barriers, so every rank must time the same
    number of batches even when the ranks run at different speeds."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_batches_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = dict((r, rest) for r, *rest in (q.get(timeout=10) for _ in range(world)))
    assert got[0] == got[1]
    calls, nper, total = got[0]
    assert nper >= 10 and total >= 0.1 and calls == 3    # 10 x 4 ms, then two more batches of 10


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")

    class Args:
        steps, warmup = 1, 1
    bench.run_reference(Args())          # rank 1: returns without work or output
    assert capsys.readouterr().out == ""
