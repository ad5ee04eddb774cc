"""The multi-GPU bench logic on CPU: two gloo ranks, replicas with their own seeds, the slowest
rank's time and the whole-job throughput; and the reference arm (the CPU oracle) on rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        from paged_kv_cache_446_b200 import workloads as W
        wl = W.make("c2", small=True, seed=bench.rank_seed("c2", rank))
        local_ms = 1.0 + rank                        # a stand-in device time per rank
        ms = bench.max_over_ranks(local_ms, dist)
        value = bench.whole_job_gbs(bench.kv_bytes(wl), world, ms)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"ms": ms, "value": value, "bytes": bench.kv_bytes(wl),
                       "q0": float(wl.q.float().flatten()[0]), "ctx": [int(x) for x in wl.prior_lens]}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, join=True, start_method="spawn")
    r = [json.load(open(tmp_path / f"rank{i}.json")) for i in range(world)]
    assert r[0]["ms"] == r[1]["ms"] == 2.0                 # every rank sees the slowest rank's time
    assert r[0]["q0"] != r[1]["q0"] or r[0]["ctx"] != r[1]["ctx"]   # replicas draw their own data
    # weak scaling: rank 0 reports all ranks' bytes over the slowest time (its own bytes x world)
    assert abs(r[0]["value"] - world * r[0]["bytes"] / 2.0e-3 / 1e9) < 1e-9


def _run_bench(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                          env=env, timeout=600)


def test_reference_arm_runs_oracle_on_cpu():
    r = _run_bench(["--impl", "reference", "--config", "c1", "--steps", "2", "--warmup", "1"])
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "GB/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    r = _run_bench(["--impl", "reference", "--config", "c1", "--steps", "1", "--warmup", "1"],
                   {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
