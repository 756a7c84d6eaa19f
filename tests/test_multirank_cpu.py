"""The multi-GPU path of bench.py is replicas only (no data-path collective):
every rank runs its own layer calls on its own seeded inputs and the job's
time is the maximum over ranks.  These tests run that host logic as two
gloo ranks on the CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        # each rank's timed measurements, reduced to the job's (max) times
        mine = [1.0 + rank, 10.0 - rank, 0.5 * (rank + 1)]
        got = bench.max_over_ranks(mine, world, "cpu")
        # the replicas draw different routing (seed offset by rank)
        pool = bench.routing_pool(2, 8, 10_000 + 7919 * rank, 0.0, 0)
        ids = torch.from_numpy(pool[0][1]).flatten()
        all_ids = [torch.zeros_like(ids) for _ in range(world)]
        dist.all_gather(all_ids, ids)
        q.put((rank, got, [t.tolist() for t in all_ids]))
    finally:
        dist.destroy_process_group()


def test_replicas_max_over_ranks_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, all_ids in res:
        assert got == [2.0, 10.0, 1.0]            # every rank sees the same maxima
        assert all_ids[0] != all_ids[1]           # independent inputs per replica


def test_job_throughput_counts_every_rank():
    tokens, value = bench.job_throughput(1, 50, 4, 0.002)
    assert tokens == 200 and value == pytest.approx(100_000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        steps, warmup = 1, 3

    bench.run_reference(A())
    assert capsys.readouterr().out == ""
