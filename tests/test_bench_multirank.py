"""Multi-rank host logic of bench.py on the CPU: two gloo ranks on 127.0.0.1.

Each rank runs a replica of the workload; the job's time is the slowest rank's and the
job's throughput counts every rank's FLOPs. The reference (oracle) arm runs on rank 0
only; other ranks return at once.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        elapsed = [12.5, 40.0][rank]
        m = bench.max_over_ranks(elapsed, dist, "cpu")
        out[rank] = (m, bench.whole_job_tflops(1e12, 10, world, m))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value_with_two_gloo_ranks():
    world = 2
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        m, v = out[rank]
        assert m == 40.0  # the slowest rank's time, on every rank
        assert v == pytest.approx(2 * 1e12 * 10 / 40e-3 / 1e12)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.0) == 3.0
    assert bench.whole_job_tflops(2e12, 5, 1, 10.0) == pytest.approx(1000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")

    class Args:
        workload = "hidream_tiny_321"
        steps = 1
        warmup = 3
        ref_step_seconds = 0.1

    assert bench.run_reference(Args()) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_line_on_rank_zero(monkeypatch, capsys):
    import json

    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setenv("RANK", "0")

    class Args:
        workload = "hidream_tiny_321"
        steps = 1
        warmup = 3
        ref_step_seconds = 0.05

    assert bench.run_reference(Args()) == 0
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
