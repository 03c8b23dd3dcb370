"""bench.py's multi-GPU bookkeeping, exercised on CPU ranks (gloo, world size 2).

With N GPUs every rank runs an independent replica of the decode step (the path
has no exchange that crosses a device), so the whole-job figures are the units
all ranks processed over the slowest rank's time.  Checked here without a GPU:
the element-wise maximum over ranks that every timing goes through, the replica
value arithmetic, and that only rank 0 of the reference arm does any work.
"""
import os
import socket
from datetime import timedelta

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        # rank r took (1 + r) ms for the timed steps and 10 * (world - r) ms end to end
        got = bench.max_over_ranks([1.0 + rank, 10.0 * (world - rank)], world, dist)
        dist.barrier()
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        results = sorted(q.get(timeout=180) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [r for r, _ in results] == [0, 1]
    for _, got in results:
        assert got == [2.0, 20.0]          # each entry is the slowest rank's
    assert all(p.exitcode == 0 for p in procs)


def test_max_over_ranks_single_rank_is_identity():
    assert bench.max_over_ranks([3.5, 0.25], 1) == [3.5, 0.25]


def test_job_value_counts_every_replica():
    # 866,805,796 bytes per step, 8 replicas, 100 steps in 25 ms on the slowest rank
    v = bench.job_value(866_805_796, 8, 100, 25.0)
    assert v == pytest.approx(866_805_796 * 8 * 100 / 0.025 / 1e9)
    assert bench.job_value(1e9, 2, 10, 1000.0) == pytest.approx(20.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    args = type("A", (), {"gpus": 2, "steps": 3, "warmup": 3, "seed": 0})()
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""
