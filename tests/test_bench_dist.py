"""bench.py's replica logic across ranks, on CPU with gloo (world size 2):
the slowest rank's time and the sum of every rank's tokens."""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    dist = bench.init_dist("gloo", world)
    elapsed = [120.0, 180.0][rank]
    units = [1000.0, 3000.0][rank]
    t, u = bench.aggregate(elapsed, units, dist)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, t, u))


def test_aggregate_max_time_sum_units_two_ranks():
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
    assert res == [(0, 180.0, 4000.0), (1, 180.0, 4000.0)]


def test_reference_arm_other_ranks_exit_quietly(capsys):
    import bench
    os.environ["RANK"] = "1"
    try:
        assert bench.main(["--impl", "reference"]) == 0
    finally:
        os.environ.pop("RANK")
    assert capsys.readouterr().out == ""
