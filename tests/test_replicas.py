"""The multi-GPU bench path is replicas only (the products shard by rows or
experts with no exchange step): each rank times its own pool and rank 0
reports the units of all ranks over the slowest rank's time.  This checks
that host logic with two gloo ranks on the CPU."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, results):
    import datetime

    import torch
    import torch.distributed as dist

    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r took (r + 1) * 10 ms for its replica
        ms = bench.max_over_ranks(torch, dist, 10.0 * (rank + 1))
        results[rank] = (ms, bench.job_throughput(1000.0, 5, world, ms))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_replicas_report_the_slowest_rank_and_all_units():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        procs = [ctx.Process(target=_rank, args=(r, world, port, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(results)
    assert res[0][0] == res[1][0] == pytest.approx(20.0)          # max over ranks
    # 1000 units a step, 5 steps, on each of 2 ranks, in 20 ms
    assert res[0][1] == pytest.approx(1000.0 * 5 * 2 / 0.020)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import bench

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        workload = "q4_k_gemv_4096x4096"
        steps, warmup = 1, 0

    bench.run_reference(A())
    assert capsys.readouterr().out == ""
