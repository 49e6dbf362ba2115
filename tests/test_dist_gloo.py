"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): the
whole-job throughput takes the slowest rank's time and every rank's units,
and the reference arm runs on rank 0 only."""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import bench
    ranks = bench.Ranks(backend="gloo")
    try:
        elapsed = 100.0 + 50.0 * rank          # rank 1 is the slow one
        units = 1000.0 * (rank + 1)
        value, tmax = bench.aggregate(ranks, elapsed, units)
        ranks.barrier()
        q.put((rank, value, tmax))
    finally:
        ranks.close()


def test_aggregate_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, value, tmax in res:
        assert tmax == 150.0                        # max over ranks
        assert value == pytest.approx(3000.0 / 0.150)   # all units / slowest time


def test_reference_arm_other_ranks_exit_without_work(monkeypatch):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]) == 0
