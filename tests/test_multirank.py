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
    for key in ("metric", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config"):
        assert key in line, key
    assert line["steps"] == 1 and line["warmup"] == 3 and line["higher_is_better"] is True
    assert line["config"]["workload"] == "tiny-noncausal-B1H2L256d64"


def test_source_hash_ignores_comments_only():
    """The key of the recorded ncu traffic: comments and blank lines do not
    change it, code does."""
    import bench
    code = b"int f(int x) {\n  return x + 1;  // one more\n}\n"
    assert bench._code_only(code) == bench._code_only(
        b"/* header\n   block */\nint f(int x) {\n\n  return x + 1;\n}\n// end\n")
    assert bench._code_only(code) != bench._code_only(code.replace(b"x + 1", b"x + 2"))


def test_secondary_ceilings_arithmetic():
    """Closed forms: the LLM workload's 268,500,992 causal pairs at d = 128."""
    import bench
    pairs = 32 * 4096 * 4097 // 2
    c = bench.secondary_ceilings(128, pairs, attn_ms=0.1, t_roof_ms=0.05, fp8=False,
                                 sms=148, sm_mhz=1965.0)
    t_nom = (256 * pairs / 4.5e15 + 256 * pairs / 2.25e15) * 1e3
    assert c["datasheet"]["t_roof_ms"] == pytest.approx(t_nom)
    assert c["datasheet"]["frac"] == pytest.approx(t_nom / 0.1)
    t_exp2 = pairs / (16 * 148 * 1965e6) * 1e3          # ~0.0577 ms
    assert c["exp2"]["t_ms"] == pytest.approx(t_exp2)
    assert c["exp2"]["max_roofline_frac"] == pytest.approx(0.05 / t_exp2)
    assert c["exp2"]["frac_of_ceiling"] == pytest.approx(t_exp2 / 0.1)
    # FP8 P V is charged at the 8-bit datasheet rate; a roofline longer than
    # the exp2 time leaves the full fraction reachable
    c8 = bench.secondary_ceilings(128, pairs, 0.1, 1.0, True, 148, 1965.0)
    assert c8["datasheet"]["t_roof_ms"] == pytest.approx(512 * pairs / 4.5e15 * 1e3)
    assert c8["exp2"]["max_roofline_frac"] == 1.0


def test_cpu_baseline_sample_is_sized_by_pairs():
    import bench
    from bit_quantized_attention_mean_b200 import inputs
    for w in inputs.WORKLOADS.values():
        n = bench.cpu_sample_rows(w)
        total = w.B * w.H * w.Lq
        assert 64 <= n <= total or n == total
        per_row = w.pairs() / total
        if n < total:   # about the target, within one row
            assert abs(n * per_row - bench.CPU_BASELINE_PAIRS) <= per_row


def test_workload_pair_counts_closed_forms():
    """Unmasked (query, key) pairs: L^2 per head without a mask, L (L + 1) / 2
    with the causal one; ops = 4 d pairs."""
    from bit_quantized_attention_mean_b200 import inputs
    W = inputs.WORKLOADS
    assert W[1].pairs() == 2 * 256 * 256
    assert W[2].pairs() == 32 * 4096 * 4097 // 2 == 268_500_992
    assert W[3].pairs() == 2 * 24 * 16384 * 16384
    assert W[4].pairs() == 4 * 32 * 8192 * 8193 // 2
    assert W[5].pairs() == 16 * 32768 * 32769 // 2
    assert 4 * W[5].d * W[5].pairs() == pytest.approx(4.398e12, rel=1e-3)
    # bottom-right alignment when Lq != Lk: row i sees keys j <= i + Lk - Lq
    assert inputs.visible_pairs(1, 1, 4, 6, True) == 3 + 4 + 5 + 6
    assert inputs.visible_pairs(1, 1, 6, 4, True) == 0 + 0 + 1 + 2 + 3 + 4
    assert inputs.visible_pairs(2, 3, 5, 7, False) == 2 * 3 * 5 * 7


def test_combined_roofline_arithmetic():
    """The LLM workload at the measured 1640.7 TFLOP/s bf16 peak and twice it
    for INT8: t_roof = 2 d pairs / P_int8 + 2 d pairs / P_fp16 = 62.8 us, so
    an attention kernel of 143.8 us is at 0.437 of it."""
    import bench
    pairs = 268_500_992
    r = bench.combined_roofline(128, pairs, 0.1438, 3281.4, 1640.7, False)
    assert r["t_roof_ms"] == pytest.approx(256 * pairs / 3281.4e12 * 1e3
                                           + 256 * pairs / 1640.7e12 * 1e3)
    assert r["t_roof_ms"] == pytest.approx(0.0628, abs=5e-5)
    assert r["frac"] == pytest.approx(0.437, abs=1e-3)
    # the reported fraction is achieved / equivalent peak, the same number
    assert r["achieved"] / r["peak"] == pytest.approx(r["frac"])
    # equal QK and P V work: the equivalent peak is the harmonic mean
    assert r["peak"] == pytest.approx(2 / (1 / 3281.4 + 1 / 1640.7))
    # FP8 P V runs at the 8-bit rate
    r8 = bench.combined_roofline(128, pairs, 0.1438, 3281.4, 1640.7, True)
    assert r8["t_roof_ms"] == pytest.approx(512 * pairs / 3281.4e12 * 1e3)


def test_quant_algorithmic_bytes():
    """The GQA workload: 4 (32 + 8) 8192 128 = 168 M elements at 3 B each, plus
    the block scales (128-row Q, 64-row K blocks) and the K means, 4 B each."""
    import bench
    got = bench.quant_algorithmic_bytes(4, 32, 8, 8192, 8192, 128, 128)
    elems = 4 * (32 + 8) * 8192 * 128
    assert elems == 167_772_160
    scales = 4 * 32 * 64 + 4 * 8 * 128
    assert got == 3 * elems + 4 * scales + 4 * 4 * 8 * 128
    assert got == pytest.approx(503.3e6, rel=1e-3)
    # one Q scale per token at the long context
    assert bench.quant_algorithmic_bytes(1, 16, 16, 32768, 32768, 128, 1) == \
        3 * 2 * 16 * 32768 * 128 + 4 * (16 * 32768 + 16 * 512) + 4 * 16 * 128
