"""Host-side logic of the multi-GPU bench (independent replicas), run as two
gloo ranks on CPU: per-rank batches are distinct, the reported time is the
slowest rank's, throughput counts the units of every rank, and the
reference arm runs on rank 0 only."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    try:
        w, r, local = bench.dist_env()
        ms = bench.max_over_ranks(10.0 * (rank + 1))  # rank 1 is the slower one
        case = workloads.make_case("tiny", seed=bench.rank_seed(rank))
        digest = float(case.target.astype("float64").sum())
        dist.barrier()
        out.put((rank, w, r, local, ms, digest))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_replica_logic():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, (r, w, r_env, local, ms, _) in enumerate(got):
        assert (r, w, r_env, local) == (rank, world, rank, rank)
        assert ms == 20.0  # every rank reports the slowest rank's time
    assert got[0][5] != got[1][5]  # independent batches per rank


def test_job_rate_counts_every_rank():
    assert bench.job_rate(256, 1, 1.0) == pytest.approx(256_000.0)
    assert bench.job_rate(256, 8, 2.0) == pytest.approx(256 * 8 / 0.002)


def test_max_over_ranks_without_process_group():
    assert not dist.is_initialized()
    assert bench.max_over_ranks(3.5) == 3.5


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        workload = "tiny"
        steps = 1
        warmup = 0

    assert bench.run_reference(A()) == 0
    assert capsys.readouterr().out == ""
