"""Host-side multi-rank logic of bench.py, run as world_size-2 gloo groups on
CPU (no GPU): job-level timing is the maximum over ranks, launch counts add
up, the weak-scaling value counts every rank's work, and the CPU reference
arm runs on rank 0 only."""
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


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        times = [1.0 + rank, 0.5 * (rank + 1), 3.0 - rank, 0.25]
        got, n = bench.aggregate_over_ranks(times, 10 + rank, world, torch.device("cpu"))
        q.put((rank, got, n))
    finally:
        dist.destroy_process_group()


def test_aggregate_over_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, n in out:
        assert got == [2.0, 1.0, 3.0, 0.25]   # element-wise max over the ranks
        assert n == 21                        # launches summed


def test_single_rank_passthrough_and_weak_scaling():
    sys.path.insert(0, ROOT)
    import bench
    got, n = bench.aggregate_over_ranks([1.5, 2.5], 7, 1, torch.device("cpu"))
    assert got == [1.5, 2.5] and n == 7
    # 2 ranks x 1e12 ops in 1 ms each -> 2000 TOPS for the job
    assert bench.weak_scaling_value(1e12, 2, 1.0) == pytest.approx(2000.0)


def _run_bench(args, env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                          capture_output=True, text=True, env=env, timeout=600)


def test_reference_arm_runs_on_rank_zero_only():
    args = ["--impl", "reference", "--workload", "1", "--steps", "1", "--warmup", "3"]
    r1 = _run_bench(args, {"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"})
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = _run_bench(args, {"WORLD_SIZE": "2", "RANK": "0", "LOCAL_RANK": "0"})
    assert r0.returncode == 0, r0.stderr
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["unit"] == "TOPS" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
