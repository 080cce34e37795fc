"""Multi-rank host logic of bench.py on CPU: world size 2 over gloo.

Decode has no exchange step, so the only cross-rank logic is the timing
reduction (max over ranks) and the barrier around the timed region, plus
the reference arm running on rank 0 alone.
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


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    try:
        bench.barrier()
        got = bench.max_over_ranks(10.0 + 5.0 * rank)
        q.put((rank, "max", got))
        got2 = bench.max_over_ranks(-float(rank))
        q.put((rank, "max2", got2))
        bench.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = {}
    while not q.empty():
        r, k, v = q.get()
        res[(r, k)] = v
    assert res[(0, "max")] == res[(1, "max")] == 15.0
    assert res[(0, "max2")] == res[(1, "max2")] == 0.0


def test_max_over_ranks_without_group_is_identity():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5


def test_reference_arm_non_zero_rank_exits_without_work(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--gpus", "2"]) == 0
    assert capsys.readouterr().out == ""
