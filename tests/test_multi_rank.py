"""The benchmark's multi-rank plumbing on CPU: two gloo ranks, as torchrun
would start them (one process per rank, rendezvous on 127.0.0.1)."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        t = bench.job_time_ms(dist, times[rank], "cpu")
        out[rank] = t
    finally:
        dist.destroy_process_group()


def test_job_time_is_max_over_ranks():
    world = 2
    times = [12.5, 17.25]
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), times, out), nprocs=world, join=True)
    assert out[0] == out[1] == max(times)


def test_job_value_is_weak_scaling_sum():
    sys.path.insert(0, ROOT)
    import bench
    # two ranks each moving 1 GB per step in 1 ms: 2000 GB/s for the job
    assert bench.job_value(2, 1e9, 1.0) == pytest.approx(2000.0)
    assert bench.job_value(1, 1e9, 1.0) == pytest.approx(1000.0)


def test_reference_arm_prints_only_on_rank_zero(capsys, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"])
    bench.run_reference(bench.parse_args())
    assert capsys.readouterr().out == ""
