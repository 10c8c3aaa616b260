"""The multi-rank host logic of the benchmark on CPU: world size 2 over gloo.

Ranks process independent batches (replicas, weak scaling) with no data-path
collective; the only collectives are the timing reductions tested here.
"""
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # each rank's device time differs; the job is as slow as its slowest rank
        ms = bench.max_over_ranks(1.5 + rank)
        steps = int(bench.max_over_ranks(3 + 2 * rank))
        rate = bench.whole_job_rate(230, steps, world, ms / 1e3)
        out.put((rank, ms, steps, rate))
    finally:
        dist.destroy_process_group()


def test_timing_reductions_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms, steps, rate in got:
        assert ms == 2.5                  # max over ranks, seen by every rank
        assert steps == 5
        assert rate == pytest.approx(230 * 5 * 2 / 2.5e-3)


def test_without_process_group_values_pass_through():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(4.25) == 4.25
    assert bench.whole_job_rate(100, 10, 1, 0.5) == 2000.0


def test_reference_arm_only_rank0_prints(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("LOCAL_RANK", "1")
    assert bench.main(["--gpus", "2", "--impl", "reference", "--config", "1", "--steps", "1",
                       "--warmup", "3", "--cpu-seconds", "0.2"]) == 0
    assert capsys.readouterr().out == ""
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("LOCAL_RANK", "0")
    assert bench.main(["--gpus", "2", "--impl", "reference", "--config", "1", "--steps", "1",
                       "--warmup", "3", "--cpu-seconds", "0.2"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_gpus_must_match_the_launch(monkeypatch):
    """A multi-GPU request never runs (or reports) as a 1-GPU job: under a launcher
    whose world size differs from --gpus the script refuses."""
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setenv("RANK", "0")
    assert bench.main(["--gpus", "2", "--impl", "reference", "--config", "1", "--steps", "1",
                       "--warmup", "3", "--cpu-seconds", "0.2"]) == 2


def test_gpus_n_outside_a_launcher_spawns_n_ranks(monkeypatch, capfd):
    """--gpus 2 without torchrun relaunches the script with two ranks (here the reference
    arm, which needs no GPU): exactly one JSON line, from rank 0, saying n_gpus 2."""
    sys.path.insert(0, ROOT)
    import bench
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "LOCAL_WORLD_SIZE", "MASTER_ADDR", "MASTER_PORT"):
        monkeypatch.delenv(k, raising=False)
    assert bench.main(["--gpus", "2", "--impl", "reference", "--config", "1", "--steps", "1",
                       "--warmup", "3", "--cpu-seconds", "0.2"]) == 0
    lines = [l for l in capfd.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
