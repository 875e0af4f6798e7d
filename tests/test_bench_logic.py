"""Host-side logic of bench.py, on CPU.

* Replicas: the timed region is the slowest rank's (max over ranks through
  torch.distributed), checked with two gloo processes; whole-job throughput is
  world x units / that time (weak scaling).
* The reference arm (the CPU oracle) prints one JSON line with the contract's
  keys, and under torchrun only rank 0 prints.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        mine = [3.5, 7.25][rank]
        out[rank] = bench.max_over_ranks(mine, world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_processes():
    port = _free_port()
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_rank_main, args=(2, port, out), nprocs=2, join=True)
    assert out[0] == 7.25 and out[1] == 7.25


def test_replica_throughput_is_weak_scaling():
    one = bench.replica_throughput(1, 1e9, 10, 20.0)
    assert one == pytest.approx(500.0)                          # 10 GB in 20 ms
    assert bench.replica_throughput(4, 1e9, 10, 20.0) == pytest.approx(4 * one)
    assert bench.replica_throughput(2, 1e9, 10, 40.0) == pytest.approx(one)


def _run_reference(env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--steps", "1", "--warmup", "0"] + (["--gpus", env_extra["WORLD_SIZE"]]
                                                               if "WORLD_SIZE" in env_extra else []),
                          capture_output=True, text=True, env=env, timeout=600)


def test_reference_arm_prints_contract_line():
    r = _run_reference({})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e", "impl"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "GB/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_are_silent():
    r = _run_reference({"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
