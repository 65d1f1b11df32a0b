"""The bench's N > 1 host logic on CPU ranks (gloo, world size 2): the timing
is the slowest rank's, the value is the whole job's, and only rank 0 prints.
The path itself has no exchange step (replicas), so this is all the
multi-process logic there is."""
import importlib.util
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench = _bench()
        ms = bench.max_over_ranks(times[rank], world, torch.device("cpu"))
        out[rank] = ms
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    world = 2
    times = [3.25, 7.5]
    out = mp.Manager().dict()
    mp.spawn(_rank, args=(world, _free_port(), times, out), nprocs=world, join=True)
    assert out[0] == out[1] == max(times)


def test_whole_job_rate():
    bench = _bench()
    # 2 ranks x 10 steps x 6 units in 4 ms (the slowest rank) -> 30000 units/s
    assert bench.whole_job_rate(6.0, 2, 10, 4.0) == pytest.approx(30000.0)
    assert bench.max_over_ranks(1.5, 1, None) == 1.5


def test_reference_arm_prints_on_rank_zero_only():
    base = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
            "--steps", "1", "--warmup", "3", "--ref-rows", "16"]
    env = dict(os.environ, WORLD_SIZE="2", MASTER_ADDR="127.0.0.1")
    r1 = subprocess.run(base, env=dict(env, RANK="1", LOCAL_RANK="1"), capture_output=True, text=True, timeout=300)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = subprocess.run(base, env=dict(env, RANK="0", LOCAL_RANK="0"), capture_output=True, text=True, timeout=300)
    assert r0.returncode == 0
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["e2e"]["h2d_bytes_per_step"] == 0
    # the contract's keys, and the reference arm's own figures in cpu_baseline and e2e
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["steps"] == 1 and line["warmup"] == 3 and line["higher_is_better"] is True
    assert line["config"]["workload"] and line["value"] > 0
    cb, e2e = line["cpu_baseline"], line["e2e"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == line["value"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"] and e2e["d2h_bytes_per_step"] == 0
