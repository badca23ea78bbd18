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


def _shard_rank(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b = _bench()
        start, count = b.shard_sequences(16, world, rank)
        # every rank reports its slice; gather them to check the cover
        t = torch.tensor([start, count], dtype=torch.int64)
        got = [torch.zeros(2, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(got, t)
        ms = b.max_over_ranks(times[rank], dist, "cpu")
        out[rank] = ([tuple(int(x) for x in g) for g in got], ms, b.sharded_rate(64, ms))
    finally:
        dist.destroy_process_group()


def test_batched_workload_splits_sequences_across_two_ranks():
    """The 16-sequence workload is data parallel: two gloo ranks take
    disjoint contiguous slices that cover the batch once, and the job's rate
    counts whole-batch steps over the slowest rank's time."""
    world, times = 2, [40.0, 32.0]
    out = tmp.Manager().dict()
    tmp.spawn(_shard_rank, args=(world, _free_port(), times, out), nprocs=world, join=True)
    for r in range(world):
        slices, ms, rate = out[r]
        assert slices == [(0, 8), (8, 8)]
        assert ms == 40.0
        assert rate == pytest.approx(64 / 0.040)


def test_shard_slices_cover_the_batch():
    b = _bench()
    for world in (1, 2, 3, 4, 5, 8, 16):
        covered = []
        sizes = []
        for r in range(world):
            start, count = b.shard_sequences(16, world, r)
            covered += list(range(start, start + count))
            sizes.append(count)
        assert covered == list(range(16))
        assert max(sizes) - min(sizes) <= 1
    with pytest.raises(SystemExit):
        b.shard_sequences(16, 17, 0)
