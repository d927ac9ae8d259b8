"""The benchmark's multi-rank host logic on CPU: two gloo ranks, as torchrun would start
them. Each rank times its own copy of the workload; the job time is the slowest rank's and
the throughput counts every rank's bytes (weak scaling, no data-path collective)."""
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        per_rank_ms = [1.5, 2.5][rank]
        t = bench.reduce_max(per_rank_ms, dist, "cpu")
        results[rank] = (t, bench.whole_job_gbs(1_000_000, world, t), bench.dist_env())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_count_all_bytes():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), results), nprocs=world,
                       start_method="spawn", join=True)
    for rank in range(world):
        t, gbs, env = results[rank]
        assert t == pytest.approx(2.5)
        assert gbs == pytest.approx(2 * 1_000_000 / 2.5e-3 / 1e9)
        assert env == (world, rank, rank)


def test_single_process_needs_no_group():
    assert bench.reduce_max(3.0, None, "cpu") == 3.0
    assert bench.whole_job_gbs(2_000_000, 1, 1.0) == pytest.approx(2.0)


def test_reference_arm_is_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        config = 1
        steps = 1
        warmup = 0
        gpus = 2

    assert bench.run_reference(Args()) == 0
    assert capsys.readouterr().out == ""
