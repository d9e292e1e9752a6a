"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, one process each.

bench.py runs one process per GPU; with N > 1 every rank times its own batch
and rank 0 reports all ranks' tokens over the slowest rank's time.  Here the
same Dist/aggregate code runs over gloo on the host.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    d = bench.Dist()
    d.init("gloo")
    d.barrier()
    value, ms = bench.aggregate(d, ms_local=10.0 * (rank + 1), tokens_local=1000.0 * (rank + 1))
    out.put((rank, value, ms, d.max(rank), d.sum(1.0)))
    d.barrier()
    d.close()


def test_two_gloo_ranks_aggregate_weak_scaling():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, value, ms, mx, sm in res:
        assert ms == 20.0                      # the slowest rank's time
        assert value == pytest.approx(3000.0 / 20e-3)  # all tokens / slowest time
        assert mx == 1.0 and sm == 2.0


def test_reference_arm_other_ranks_exit_without_work(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = type("A", (), {"workload": "ce_gpt2", "steps": 1, "warmup": 3})()
    assert bench.reference_arm(args, bench.Dist()) == 0
