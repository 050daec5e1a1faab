"""Multi-process host logic of the benchmark on CPU (gloo, world size 2):
every rank runs its own replica, the timed region is bracketed by barriers,
the reported time is the max over ranks and the throughput aggregates all
ranks' units."""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    d = bench.Dist()
    d.init("gloo")
    d.barrier()
    elapsed = 1.0 + rank            # rank 1 is the slow one
    mx = d.max(elapsed)
    value = bench.aggregate(100, d.world, mx)
    d.barrier()
    d.close()
    q.put((rank, mx, value))


def test_two_rank_max_and_aggregate():
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
    assert [r[1] for r in res] == [2.0, 2.0]            # max over ranks, seen by every rank
    assert [r[2] for r in res] == [100.0, 100.0]        # 2 ranks x 100 units / 2 s


def test_reference_arm_other_ranks_exit(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    d = bench.Dist()
    assert bench.run_reference(bench.parse_args(["--impl", "reference"]), d) is None
