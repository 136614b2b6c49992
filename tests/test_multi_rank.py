"""The benchmark's multi-process host logic with world-size-2 gloo ranks on CPU:
process-group set-up, barriers, max-over-ranks timing, whole-job throughput,
and the reference arm's rank-0-only rule.  No GPU is touched."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch
    import torch.distributed as dist
    w, r, _ = bench.dist_env()
    assert (w, r) == (world, rank)
    assert bench.init_dist(w, r, backend="gloo")
    bench.barrier(True)
    # each rank reports a different time; everyone must see the maximum
    mx = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 0.5 * rank], True, torch.device("cpu"))
    results[rank] = mx
    dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, results), nprocs=world, join=True)
        got = dict(results)
    assert got[0] == got[1] == [2.0, 10.0, 0.5]


def test_job_throughput_is_all_ranks_over_slowest():
    # 4 ranks, each 1e12 FLOP per step, slowest step 2 ms -> 2e15 FLOP/s = 2e6 GFLOP/s
    assert bench.job_throughput(1e12, 4, 2e-3) == pytest.approx(2e6)


def test_single_rank_needs_no_process_group():
    assert bench.init_dist(1, 0) is False
    assert bench.max_over_ranks([3.0, 4.0], False, None) == [3.0, 4.0]


def test_reference_arm_runs_only_on_rank_zero(capsys, monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"])
    assert capsys.readouterr().out == ""


def test_reference_arm_json_line(capsys, monkeypatch):
    """Rank 0 prints one JSON line with the keys the benchmark contract needs
    for the CPU-oracle arm: the arm's own metric and unit, a cpu_baseline that
    describes the run, and an e2e with no host-device traffic."""
    import json
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.delenv("RANK", raising=False)
    bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"])
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["unit"] == "GFLOP/s" and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"] and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] and d["data"] == "synthetic"
