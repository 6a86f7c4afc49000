"""Host-side logic of bench.py that runs without a GPU: the max-over-ranks
reduction of replica timings (two gloo ranks on CPU), the replica seeding,
and the reference arm (the CPU oracle on bounded samples, rank 0 only)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

from conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        got = bench.reduce_max([1.0 + rank, 10.0 - rank, 0.5 * rank], dist, torch.device("cpu"))
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        assert out[0] == out[1] == [2.0, 10.0, 0.5]


def test_reduce_max_without_group_is_identity():
    import torch

    assert bench.reduce_max([3.0, 4.0], None, torch.device("cpu")) == [3.0, 4.0]


def test_replica_seeds_differ():
    assert len({bench.replica_seed(0, r) for r in range(8)}) == 8


def test_reference_arm_other_ranks_exit_quietly():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "3",
                        "--warmup", "3", "--ref-tokens", "256"], env=dict(os.environ, RANK="1", WORLD_SIZE="2"),
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "3",
                        "--warmup", "3", "--ref-tokens", "512"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["config"]["workload"] == "large_table (fwd) + backward_stress (fwd+bwd)"
    assert [q["workload"] for q in d["config"]["parts"]] == ["large_table", "backward_stress"]
    assert "first 512 of 65536" in d["cpu_baseline"]["sample"]


def test_reference_arm_single_workload():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "3",
                        "--warmup", "3", "--ref-tokens", "512", "--workload", "single_layer_bf16"],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    d = json.loads(r.stdout.strip().splitlines()[-1])
    assert d["config"]["workload"] == "single_layer_bf16" and d["value"] > 0


def test_headline_parts():
    import argparse

    a = argparse.Namespace(workload="headline", fwd_only=False)
    assert bench.step_parts(a) == [("large_table", False), ("backward_stress", True)]
    a = argparse.Namespace(workload="tiny", fwd_only=True)
    assert bench.step_parts(a) == [("tiny", False)]


def test_bench_requires_three_warmups():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--warmup", "2"], capture_output=True,
                       text=True, timeout=120)
    assert r.returncode != 0
