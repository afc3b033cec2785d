"""The bench's multi-rank logic on CPU: two gloo ranks (127.0.0.1), replica seeds, max-over-ranks
timing and the whole-job throughput.  No GPU."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [3.0, 5.0][rank]            # rank 1 is the slow one
        job_ms = bench.max_over_ranks(local_ms, dist, torch.device("cpu"))
        value = bench.job_tokens_per_s(world, 32, job_ms)
        seeds = torch.tensor([bench.replica_seed(3002, rank)], dtype=torch.int64)
        gathered = [torch.zeros_like(seeds) for _ in range(world)]
        dist.all_gather(gathered, seeds)
        out[rank] = (job_ms, value, [int(g.item()) for g in gathered])
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank():
    world = 2
    out = mp.Manager().dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    for rank in range(world):
        job_ms, value, seeds = out[rank]
        assert job_ms == 5.0
        assert value == pytest.approx(world * 32 / 5e-3)
        assert len(set(seeds)) == world  # every replica draws its own inputs


def test_single_rank_is_identity():
    import bench

    assert bench.max_over_ranks(2.5, None, None) == 2.5
    assert bench.job_tokens_per_s(1, 32, 1.0) == pytest.approx(32000.0)


def test_reference_arm_other_ranks_exit_without_work(tmp_path, monkeypatch, capsys):
    import bench

    class A:
        steps, warmup, gpus = 1, 0, 2
    bench.run_reference(A(), rank=1, world=2)  # returns at once: only rank 0 runs the oracle
    assert capsys.readouterr().out == ""
