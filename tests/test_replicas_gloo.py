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


def test_reference_arm_line_carries_the_contract_keys(monkeypatch, capsys):
    """Rank 0 prints one JSON line with the keys of the bench contract: the
    reference tag, the metric and its unit, the run's shape, a CPU-baseline
    object describing this run and an end-to-end object with no copies. The
    oracle's timing itself is stubbed (it runs for seconds by design)."""
    import json
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setattr(bench, "oracle_sample", lambda w, qkv, gq, gk, target_s: (0.02, 0.5, "stub sample"))
    args = type("A", (), {"workload": "tiny_5x8x8_h12_b1", "steps": 3, "warmup": 1, "gpus": 1})()
    assert bench.run_reference(args) == 0
    out = capsys.readouterr().out.strip().splitlines()
    assert len(out) == 1
    line = json.loads(out[0])
    assert line["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["value"] == pytest.approx(0.02) and line["unit"] == "TFLOP/s"
    assert line["steps"] == 3 and line["warmup"] == 1 and line["n_gpus"] == 1
    assert line["ms_per_step"] == pytest.approx(500.0)
    assert line["higher_is_better"] is True and line["vs_baseline"] is None
    assert line["config"]["workload"] == "tiny_5x8x8_h12_b1"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
