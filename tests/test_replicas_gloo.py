"""Host-side multi-rank logic of bench.py on CPU with gloo, world size 2: the
timing reduction takes the slowest rank, the job throughput counts every
rank's work, and the reference arm runs on rank 0 only."""
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


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=__import__("datetime").timedelta(seconds=60))
    try:
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        got = bench.max_over_ranks(ms, torch.device("cpu"), dist)
        dist.barrier()
        results[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, results)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert results[0] == results[1] == 15.0


def test_single_rank_reduction_is_identity():
    assert bench.max_over_ranks(3.5, torch.device("cpu"), None) == 3.5


def test_job_throughput_counts_all_ranks():
    # 2 ranks x 10 steps of 1e12 FLOP in 100 ms (slowest rank) = 200 TFLOP/s
    assert bench.job_throughput(2, 1e12, 10, 100.0) == pytest.approx(200.0)
    assert bench.job_throughput(1, 1e12, 10, 100.0) == pytest.approx(100.0)


def test_reference_arm_runs_on_rank0_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    args = type("A", (), {"workload": "tiny_5x8x8_h12_b1", "steps": 1, "warmup": 0, "gpus": 2})()
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""
