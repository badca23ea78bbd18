"""The multi-GPU bench path without GPUs: batch-1 decode runs independent
replicas, one per rank, so the only cross-rank step is the timing -- the
job's time is the slowest rank's and the value counts every rank's steps.
Two gloo ranks on the CPU check that arithmetic and the rank checks."""
import importlib.util
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as tmp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    return b


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b = _bench()
        ms = b.max_over_ranks(times[rank], dist, "cpu")
        out[rank] = (ms, b.job_rate(world, 64, ms))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time():
    world, times = 2, [10.0, 25.0]
    out = tmp.Manager().dict()
    tmp.spawn(_rank, args=(world, _free_port(), times, out), nprocs=world, join=True)
    for r in range(world):
        ms, rate = out[r]
        assert ms == 25.0
        assert rate == pytest.approx(world * 64 / 0.025)


def test_single_process_needs_no_group():
    b = _bench()
    assert b.max_over_ranks(12.5, None, "cpu") == 12.5
    assert b.job_rate(1, 128, 500.0) == pytest.approx(256.0)


def test_gpus_flag_must_match_the_launcher(monkeypatch):
    b = _bench()
    monkeypatch.setenv("WORLD_SIZE", "1")
    with pytest.raises(SystemExit):
        b.dist_setup(2)
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("LOCAL_RANK", "1")
    assert b.dist_setup(2) == (2, 1, 1)


def test_reference_arm_runs_on_rank_0_only(capsys):
    """Under torchrun the CPU reference runs once: ranks other than 0 return
    at once and print nothing."""
    import argparse
    b = _bench()
    ns = argparse.Namespace(workload="tiny", steps=1, warmup=0, gpus=2)
    assert b.run_reference(ns, 2, 1) is None
    assert capsys.readouterr().out == ""


def test_reference_arm_line(capsys):
    """Rank 0 prints one JSON line with the workload's config, the warm-up it
    ran, and an e2e block without host-device bytes (the oracle runs on the
    host)."""
    import argparse
    import json
    import synth
    b = _bench()
    ns = argparse.Namespace(workload="tiny", steps=3, warmup=3, gpus=1)
    b.run_reference(ns, 1, 0)
    lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["steps"] == 3 and d["warmup"] == 3
    assert d["config"] == b.workload_config(synth.WORKLOADS["tiny"])
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"] > 0
    assert d["unit"] == "steps/s" and d["higher_is_better"] is True
