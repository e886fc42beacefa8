"""Benchmark of the 8-bit quantized attention forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload 1..5|all] [--q-block-rows 128|64|32|1]
                    [--pv-accum f32|f16|fp8] [--decode]

The default workload is the largest single-GPU configuration,
longctx-causal-B1H16L32768d128-t4 (heavy-tailed inputs, per-token Q blocks:
the Q granularity at which that workload meets the fp64 accuracy gate).
``--workload all`` prints one line per workload 2..5 instead.

A step is one pass of the whole hot path over the workload: K mean + Q/K
quantization (sage_quant_qk) and the fused attention kernel
(sage_attn_fwd_prequant) -- exactly what sage_attn_fwd runs, with the scratch
preallocated so the timed region holds only kernels.  Inputs are seeded
synthetic fp16 tensors resident in HBM before timing; L2 is flushed (256 MiB
write) before every timed step, outside the step's CUDA events.

Metric: TOPS = 4 * d * (unmasked query/key pairs) / step time, the QK^T and
PV work counted at 2*d each.  ``e2e`` is the same metric through the public
host-buffer call (sage_attn_fwd_host: H2D of q/k/v, forward pass, D2H of the
output, all inside the timed region).  ``--q-block-rows`` quantizes Q in
blocks finer than the 128-row attention tile (the _qblock entry points; e2e
then issues the same copies around sage_attn_fwd_ex); ``--pv-accum f16``
sums P V in fp16 as the SageAttention article states (sage_attn_fwd_ex /
sage_attn_fwd_prequant_ex with SAGE_PV_ACCUM_F16).  ``roofline`` reports the attention
kernel against the combined tensor roofline: QK at the INT8 peak and PV at the
FP16 peak, t_roof = 2*d*pairs/P_int8 + 2*d*pairs/P_fp16, with P_fp16 the
measured bf16 peak and P_int8 measured in the same run (torch._int_mm at
8192^3, best of 10); ``ceilings.nominal_int8`` repeats the fraction with
P_int8 = 2 x P_fp16 (the datasheet ratio).

Multi-GPU (torchrun, one process per GPU): every rank runs the same workload
on its own GPU (the path shards by batch and head with no exchange, so this
is weak scaling); value = all ranks' ops / the slowest rank's time.
``--impl reference`` times the CPU oracle (the only reference this path has)
on a bounded sample per step -- one (batch, head)'s Q/K quantization plus a
few hundred of its query rows of the quantized-path simulation -- on rank 0
only; its value is the sample's attention work over the sample's time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_quantized_attention_mean_b200 import inputs  # noqa: E402

METRIC = "quantized attention fwd TOPS at 1 B200 and % of INT8/FP16 tensor roofline"
DEFAULT_WORKLOAD = 5
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}
INT8_OVER_FP16 = 2.0  # nominal dense ratio (4.5 / 2.25 PFLOP/s)
# B200 datasheet dense peaks (TFLOP/s, per GPU) and the exp2 unit's rate
DATASHEET_TFLOPS = {"int8": 4500.0, "fp8": 4500.0, "fp16": 2250.0}
EX2_PER_CLK_PER_SM = 16  # MUFU ex2 results per clock per SM (measured 15.9)

# DRAM traffic of one attention launch from an ncu capture, valid only for the
# kernel source it was taken on (attn_source_hash); otherwise reported null.
NCU_TRAFFIC = {"attn_sha": "11cca823bf95dac9", "workload": "longctx-causal-B1H16L32768d128-t4",
               "q_block_rows": 1, "bytes_per_launch": 270883840 + 106859008}
# Same for the decoding kernel (decode.cu + PTX wrappers) on the --decode shape.
DECODE_NCU_TRAFFIC = {"sha": "6a43014109bd395c", "bytes_per_launch": 805530880 + 3755520}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


def _code_only(text: bytes) -> bytes:
    """C/C++ source without its comments and blank lines, so that a comment
    edit does not invalidate counters taken on unchanged code."""
    import re
    t = re.sub(rb"/\*.*?\*/", b"", text, flags=re.S)
    t = re.sub(rb"//[^\n]*", b"", t)
    return b"\n".join(ln.rstrip() for ln in t.split(b"\n") if ln.strip())


def decode_source_hash():
    """Hash of the decoding kernel's code and of the PTX wrappers."""
    csrc = os.path.join(ROOT, "bit_quantized_attention_mean_b200", "csrc")
    h = hashlib.sha256()
    for name in ("decode.cu", "sm100_ptx.cuh"):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(_code_only(f.read()))
    return h.hexdigest()[:16]


def attn_source_hash():
    """Hash of the attention kernel's device code (attn.cu up to its host
    section) and of the PTX wrappers it is built from, comments excluded."""
    csrc = os.path.join(ROOT, "bit_quantized_attention_mean_b200", "csrc")
    with open(os.path.join(csrc, "attn.cu"), "rb") as f:
        text = f.read()
    marker = b"// ------------------------------------------------------------------- host"
    h = hashlib.sha256(_code_only(text.split(marker)[0]))
    with open(os.path.join(csrc, "sm100_ptx.cuh"), "rb") as f:
        h.update(_code_only(f.read()))
    return h.hexdigest()[:16]


# ------------------------------------------------------------ clock sampler

class ClockSampler:
    """Samples SM clock, power and throttle reasons via NVML while running."""

    REASONS = {
        0x0000000000000001: "gpu_idle",
        0x0000000000000002: "applications_clocks_setting",
        0x0000000000000004: "sw_power_cap",
        0x0000000000000008: "hw_slowdown",
        0x0000000000000020: "sw_thermal_slowdown",
        0x0000000000000040: "hw_thermal_slowdown",
        0x0000000000000080: "hw_power_brake_slowdown",
    }

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples = []
        self.max_mhz = None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self._nvml = pynvml
            try:  # NVML indices ignore CUDA_VISIBLE_DEVICES; match by UUID
                uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
                self._h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - depends on the machine
            self._nvml = None
            self.error = str(e)

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                util = nv.nvmlDeviceGetUtilizationRates(self._h).gpu
                self.samples.append((mhz, reasons, util))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        if self._nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "error": getattr(self, "error", "nvml unavailable")}
        busy = [s for s in self.samples if s[2] > 0] or self.samples
        mask = 0
        for s in busy:
            mask |= s[1]
        reasons = [n for bit, n in self.REASONS.items() if mask & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median([s[0] for s in busy]) if busy else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(busy)}


def quant_algorithmic_bytes(B, H, Hkv, Lq, Lk, d, q_block_rows):
    """Bytes the quantization step must move: each fp16 Q and K element read
    once (2 B) and written once as int8 (1 B), plus the fp32 block scales of
    Q and K and the fp32 K mean.  The second read of K (mean, then quantize)
    is overhead, not part of it."""
    elems = B * H * Lq * d + B * Hkv * Lk * d
    scales = B * H * -(-Lq // q_block_rows) + B * Hkv * -(-Lk // 64)
    return 3 * elems + 4 * scales + 4 * B * Hkv * d


def combined_roofline(d, pairs, attn_ms, p_int8, p_fp16, fp8):
    """The attention kernel against its combined tensor roofline: 4 d ops per
    unmasked (query, key) pair, half of them (QK^T) at the INT8 peak and half
    (P V) at the FP16 peak, or at the 8-bit peak when P and V are FP8.
    Peaks in TOPS / TFLOP/s, times in ms."""
    p_pv = p_int8 if fp8 else p_fp16
    t_roof_ms = (2.0 * d * pairs / (p_int8 * 1e12) + 2.0 * d * pairs / (p_pv * 1e12)) * 1e3
    ops = 4.0 * d * pairs
    return {"t_roof_ms": t_roof_ms,
            "peak": ops / (t_roof_ms * 1e-3) / 1e12,          # equivalent combined peak
            "achieved": ops / (attn_ms * 1e-3) / 1e12,
            "frac": t_roof_ms / attn_ms}


def secondary_ceilings(d, pairs, attn_ms, t_roof_ms, fp8, sms, sm_mhz):
    """The two further bars of the attention kernel: the fraction of the
    datasheet dense peaks (QK at INT8, P V at FP16 or FP8), and the exp2
    ceiling -- one ex2 per unmasked pair on the SMs' ex2 units at the SM
    clock seen during the run -- as its time, the highest fraction of the
    (measured) combined roofline it leaves reachable, and how close the
    kernel comes to it."""
    pv = DATASHEET_TFLOPS["fp8" if fp8 else "fp16"]
    t_nom_ms = (2.0 * d * pairs / (DATASHEET_TFLOPS["int8"] * 1e12)
                + 2.0 * d * pairs / (pv * 1e12)) * 1e3
    t_exp2_ms = pairs / (EX2_PER_CLK_PER_SM * sms * sm_mhz * 1e6) * 1e3
    return {
        "datasheet": {"frac": t_nom_ms / attn_ms, "t_roof_ms": t_nom_ms,
                      "peaks_tflops": {"qk_int8": DATASHEET_TFLOPS["int8"],
                                       "pv": pv}},
        "exp2": {"t_ms": t_exp2_ms, "max_roofline_frac": min(1.0, t_roof_ms / t_exp2_ms),
                 "frac_of_ceiling": t_exp2_ms / attn_ms, "sms": sms, "sm_mhz": sm_mhz,
                 "ex2_per_clk_per_sm": EX2_PER_CLK_PER_SM},
    }


# ---------------------------------------------------------- distributed

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def aggregate_over_ranks(times_ms, launches, world, device):
    """Job-level numbers from per-rank ones: every time is the maximum over
    ranks (the slowest GPU sets the job's pace), the launch count is the sum.
    Works on any initialized torch.distributed backend (NCCL on GPUs, gloo
    on CPU); with world == 1 it returns the inputs unchanged."""
    import torch
    if world <= 1:
        return list(times_ms), int(launches)
    import torch.distributed as dist
    t = torch.tensor(list(times_ms), dtype=torch.float64, device=device)
    n = torch.tensor([int(launches)], dtype=torch.int64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(n, op=dist.ReduceOp.SUM)
    return t.tolist(), int(n.item())


def weak_scaling_value(ops_per_rank, world, ms_per_step):
    """Whole-job throughput in TOPS: every rank does ops_per_rank per step and
    a step takes ms_per_step (the maximum over ranks)."""
    return world * ops_per_rank / (ms_per_step * 1e-3) / 1e12


# ------------------------------------------------------------ CPU oracle

# The one-off CPU baseline beside our line: a sample of about this many
# query/key pairs of the quantized-path simulation (about 10 s on 16 host
# cores at d = 128), plus the quantization of the heads the rows fall in.
CPU_BASELINE_PAIRS = 1.2e8


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_sample_rows(w, target_pairs=CPU_BASELINE_PAIRS):
    """Query rows whose visible pairs add up to about target_pairs (at least
    64 rows, at most all of them)."""
    total_rows = w.B * w.H * w.Lq
    per_row = w.pairs() / total_rows
    return int(min(total_rows, max(64, round(target_pairs / per_row))))


def time_oracle_sample(w, q, k, v, n_rows, seed, qbr):
    """The oracle on a bounded sample of the workload: n_rows random query
    rows, spread over as few random (batch, head) pairs as hold them; for
    each head, its Q and its kv head's K are quantized (the oracle's
    quantization of that head alone, which is what it does for every head of
    the full problem) and the sampled rows run through the quantized-path
    simulation.  Returns (seconds, attention ops of the sampled rows, info)."""
    import oracle
    sm = float(np.float32(w.sm_scale))
    rng = np.random.default_rng(seed)
    heads = rng.permutation(w.B * w.H)
    t_quant = t_attn = 0.0
    pairs = 0
    left = n_rows
    used = 0
    for bh in heads:
        if left <= 0:
            break
        b, h = divmod(int(bh), w.H)
        hk = h // (w.H // w.Hkv)
        n = min(left, w.Lq)
        rows = np.sort(rng.choice(w.Lq, size=n, replace=False)).astype(np.int64)
        qh = np.ascontiguousarray(q[b:b + 1, h:h + 1])
        kh = np.ascontiguousarray(k[b:b + 1, hk:hk + 1])
        vh = np.ascontiguousarray(v[b:b + 1, hk:hk + 1])
        t0 = time.perf_counter()
        qk = oracle.quant_qk(qh, kh, sm, q_block_rows=qbr)
        t1 = time.perf_counter()
        oracle.attn_quant_sim(*qk[:4], vh, w.causal, rows=rows, q_block_rows=qbr)
        t2 = time.perf_counter()
        t_quant += t1 - t0
        t_attn += t2 - t1
        pairs += int(w.visible_keys(rows).sum())
        left -= n
        used += 1
    ops = 4.0 * w.d * pairs
    return t_quant + t_attn, ops, {"t_quant_s": t_quant, "t_attn_s": t_attn, "rows": n_rows,
                                   "heads": used, "pairs": pairs,
                                   "cores": oracle.num_threads()}


def run_reference(args, w):
    world, rank, _ = dist_setup()
    if rank != 0:
        return 0
    q, k, v = inputs.make_inputs(w)
    qbr = args.q_block_rows
    rows = args.ref_rows
    times, ops_l = [], []
    info = None
    for step in range(args.warmup + args.steps):
        t, ops, info = time_oracle_sample(w, q, k, v, rows, seed=step, qbr=qbr)
        if step >= args.warmup:
            times.append(t)
            ops_l.append(ops)
    t = float(np.mean(times))
    value = float(np.sum(ops_l) / np.sum(times) / 1e12)
    full_ms = 4.0 * w.d * w.pairs() / (value * 1e12) * 1e3
    sample = (f"per step: one random (batch, head)'s Q/K quantization + quantized-path "
              f"simulation of {rows} of its query rows (about "
              f"{info['pairs'] / rows:.0f} visible keys each); value = those rows' "
              f"attention ops / the step's time")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64 (int8 codes, int32 dot products)",
        "data": "synthetic (seeded numpy, fp16)",
        "config": dict(w.describe(), q_block_rows=qbr, pv_accum=args.pv_accum,
                       l2="n/a (CPU)"),
        "extrapolated_full_workload_ms": full_ms,
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": info["cores"],
                         "cpu_model": cpu_model(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def measure_int8_peak(dev, n=8192, reps=10):
    """Dense INT8 GEMM rate of this GPU through cuBLAS (torch._int_mm, int8 x
    int8 -> int32, n^3), best of `reps` CUDA-event timings, in TOPS."""
    import torch
    a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev)
    b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev).t().contiguous().t()
    for _ in range(3):
        torch._int_mm(a, b)
    torch.cuda.synchronize(dev)
    best = float("inf")
    for _ in range(reps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        torch._int_mm(a, b)
        e1.record()
        torch.cuda.synchronize(dev)
        best = min(best, e0.elapsed_time(e1))
    del a, b
    return 2.0 * n ** 3 / (best * 1e-3) / 1e12


# ---------------------------------------------------------------- ours

def run_ours(args, w):
    import torch
    import bit_quantized_attention_mean_b200 as sage

    world, rank, local = dist_setup()
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)

    p_int8_meas = measure_int8_peak(dev) if args.int8_peak else None
    qn, kn, vn = inputs.make_inputs(w)
    sm = float(np.float32(w.sm_scale))
    q = torch.from_numpy(qn).to(dev)
    k = torch.from_numpy(kn).to(dev)
    v = torch.from_numpy(vn).to(dev)
    out = torch.empty_like(q)
    B, H, Hkv, Lq, Lk, d = w.B, w.H, w.Hkv, w.Lq, w.Lk, w.d
    q_i8 = torch.empty(q.shape, dtype=torch.int8, device=dev)
    k_i8 = torch.empty(k.shape, dtype=torch.int8, device=dev)
    qbr = args.q_block_rows
    q_scale = torch.empty((B, H, -(-Lq // qbr)), dtype=torch.float32, device=dev)
    k_scale = torch.empty((B, Hkv, -(-Lk // 64)), dtype=torch.float32, device=dev)
    k_mean = torch.empty((B, Hkv, d), dtype=torch.float32, device=dev)
    fp8 = args.pv_accum == "fp8"
    if fp8:
        v8t = torch.empty((B, Hkv, d, -(-Lk // 64) * 64), dtype=torch.uint8, device=dev)
        v_scale = torch.empty((B, Hkv, d), dtype=torch.float32, device=dev)
        ws8 = torch.empty(sage.sage_quant_v_fp8_workspace_size(B, Hkv, d), dtype=torch.uint8,
                          device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    launches = 0

    def step():
        nonlocal launches
        if qbr == 128:
            sage.sage_quant_qk(q, k, q_i8, k_i8, q_scale, k_scale, k_mean, sm, stream=stream)
        else:
            sage.sage_quant_qk_qblock(q, k, q_i8, k_i8, q_scale, k_scale, k_mean, sm, qbr,
                                      stream=stream)
        launches += sage.sage_last_launch_count()
        if fp8:   # V to E4M3 is part of the quantization step
            sage.sage_quant_v_fp8(v, v8t, v_scale, workspace=ws8, stream=stream)
            launches += sage.sage_last_launch_count()
        ev_mid = torch.cuda.Event(enable_timing=True)
        ev_mid.record(stream)
        if fp8:
            sage.sage_attn_fwd_prequant_fp8pv(q_i8, k_i8, q_scale, k_scale, v8t, v_scale, out,
                                              w.causal, qbr, stream=stream)
        elif args.pv_accum != "f32":
            sage.sage_attn_fwd_prequant_ex(q_i8, k_i8, q_scale, k_scale, v, out, w.causal, qbr,
                                           args.pv_accum, stream=stream)
        elif qbr == 128:
            sage.sage_attn_fwd_prequant(q_i8, k_i8, q_scale, k_scale, v, out, w.causal,
                                        stream=stream)
        else:
            sage.sage_attn_fwd_prequant_qblock(q_i8, k_i8, q_scale, k_scale, v, out, w.causal,
                                               qbr, stream=stream)
        launches += sage.sage_last_launch_count()
        return ev_mid

    for _ in range(args.warmup):
        flush.zero_()
        step()
    sage.sage_check_device_status(stream)

    n = args.steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n)]
    mids = []
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    launches = 0
    with ClockSampler(local) as clocks:
        for i in range(n):
            flush.zero_()
            evs[i][0].record(stream)
            mids.append(step())
            evs[i][1].record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    sage.sage_check_device_status(stream)
    step_ms = [a.elapsed_time(b) for a, b in evs]
    attn_ms = [m.elapsed_time(b) for m, (a, b) in zip(mids, evs)]
    total_ms = float(sum(step_ms))
    attn_avg_ms = float(sum(attn_ms) / n)
    quant_avg_ms = float(sum(m0.elapsed_time(m) for (m0, _), m in zip(evs, mids)) / n)

    # e2e through the host-buffer entry point (pinned memory)
    hq = torch.from_numpy(qn).pin_memory()
    hk = torch.from_numpy(kn).pin_memory()
    hv = torch.from_numpy(vn).pin_memory()
    hout = torch.empty(qn.shape, dtype=torch.float16).pin_memory()
    e2e_steps = max(1, min(n, args.e2e_steps))

    def e2e_call():
        if args.pv_accum == "f32":
            sage.sage_attn_fwd_host_qblock(hq, hk, hv, hout, w.causal, sm, qbr, stream=stream)
            return
        # the other P V variants have no host-buffer entry point: the same
        # copies, issued from here on the same stream around the device call
        with torch.cuda.stream(stream):
            dq = hq.to(dev, non_blocking=True)
            dk = hk.to(dev, non_blocking=True)
            dv = hv.to(dev, non_blocking=True)
            dout = torch.empty_like(dq)
            sage.sage_attn_fwd_ex(dq, dk, dv, dout, w.causal, sm, qbr, args.pv_accum,
                                  stream=stream)
            hout.copy_(dout, non_blocking=True)

    for _ in range(2):
        e2e_call()
    torch.cuda.synchronize(dev)
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(e2e_steps)]
    for a, b in e2e_ev:
        a.record(stream)
        e2e_call()
        b.record(stream)
    torch.cuda.synchronize(dev)
    sage.sage_check_device_status(stream)
    e2e_ms = float(sum(a.elapsed_time(b) for a, b in e2e_ev) / e2e_steps)

    (total_ms, attn_avg_ms, e2e_ms, quant_avg_ms), n_launches = aggregate_over_ranks(
        [total_ms, attn_avg_ms, e2e_ms, quant_avg_ms], launches, world, dev)

    result = None
    if rank == 0:
        clk = clocks.summary()
        ops = 4.0 * d * w.pairs()
        ms_per_step = total_ms / n
        value = weak_scaling_value(ops, world, ms_per_step)
        peaks = load_peaks()
        p16 = float(peaks["bf16_tflops"])
        p8_nominal = INT8_OVER_FP16 * p16
        p8 = p_int8_meas if p_int8_meas else p8_nominal
        p8_note = (f"P_int8 = {p8:.1f} TOPS measured in this run (torch._int_mm int8 8192^3, "
                   f"best of 10)" if p_int8_meas else
                   f"P_int8 = {INT8_OVER_FP16} x P_fp16 (nominal ratio)")

        roof = combined_roofline(d, w.pairs(), attn_avg_ms, p8, p16, fp8)
        t_roof_ms, peak_eff, achieved = roof["t_roof_ms"], roof["peak"], roof["achieved"]
        traffic = None
        if NCU_TRAFFIC.get("attn_sha") == attn_source_hash() and \
                NCU_TRAFFIC.get("workload") == w.name and \
                NCU_TRAFFIC.get("q_block_rows", 128) == qbr and args.pv_accum == "f32":
            traffic = NCU_TRAFFIC.get("bytes_per_launch")
        quant_bytes = quant_algorithmic_bytes(B, H, Hkv, Lq, Lk, d, qbr)
        result = {
            "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
            "steps": n, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": ("int8 QK^T (int32 acc) + e4m3 PV (fp32 acc)" if fp8 else
                      f"int8 QK^T (int32 acc) + fp16 PV ({args.pv_accum} acc)"),
            "data": "synthetic (seeded numpy N(0,1)/t4 fp16, per-channel K offsets)",
            "config": dict(w.describe(), q_block_rows=qbr, pv_accum=args.pv_accum,
                           l2="flushed before every timed step (256 MiB write)",
                           parallelism=f"replicas x{world} (shard by batch/head)"),
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_eff,
                         "unit": "TFLOP/s", "frac": achieved / peak_eff, "traffic": traffic,
                         "kernel": "sage_attn_fwd_kernel",
                         "peak_note": (f"combined roofline (of measured), QK at P_int8, PV "
                                       f"at {'P_fp8 = P_int8' if fp8 else 'P_fp16'}: P_fp16 = "
                                       f"{p16} TFLOP/s ({peaks.get('source')} bf16 burst), "
                                       f"{p8_note}")},
            "kernel_ms": {"attention": attn_avg_ms, "quant": quant_avg_ms},
            "ceilings": dict(secondary_ceilings(
                d, w.pairs(), attn_avg_ms, t_roof_ms, fp8,
                torch.cuda.get_device_properties(dev).multi_processor_count,
                clk.get("sm_mhz") or clk.get("sm_max_mhz") or 1965.0),
                nominal_int8={"frac": combined_roofline(d, w.pairs(), attn_avg_ms,
                                                        p8_nominal, p16, fp8)["frac"],
                              "p_int8_tops": p8_nominal,
                              "note": "same kernel time, P_int8 = 2 x measured bf16 peak"}),
            "quant_hbm_gbs": quant_bytes / (quant_avg_ms * 1e-3) / 1e9,
            "e2e": {"value": weak_scaling_value(ops, world, e2e_ms), "unit": "TOPS",
                    "h2d_bytes_per_step": int(qn.nbytes + kn.nbytes + vn.nbytes),
                    "d2h_bytes_per_step": int(qn.nbytes)},
            "gpu_launches": n_launches,
            "clocks": clk,
        }
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n_rows = args.cpu_rows if args.cpu_rows else cpu_sample_rows(w)
        t, sample_ops, info = time_oracle_sample(w, qn, kn, vn, n_rows, seed=0, qbr=qbr)
        result["cpu_baseline"] = {
            "value": sample_ops / t / 1e12, "unit": "TOPS",
            "cores": info["cores"], "cpu_model": cpu_model(), "kind": "oracle",
            "sample": (f"{info['rows']} random query rows in {info['heads']} random "
                       f"(batch, head) pairs: the oracle's Q/K quantization of those heads "
                       f"({info['t_quant_s']:.2f} s) + quantized-path simulation of the rows "
                       f"({info['t_attn_s']:.2f} s, {info['pairs']} query/key pairs); value = "
                       f"the rows' attention ops / that time")}
    if rank == 0:
        print(json.dumps(result), flush=True)
    return 0


DECODE_SHAPE = {"B": 8, "H": 32, "Hkv": 8, "Lq": 1, "Lk": 32768, "d": 128}


def run_decode_bench(args):
    """Decoding step: one query token per head against a 32768-token KV cache
    that is already quantized (int8 K, fp16 V resident in HBM); times
    sage_attn_decode_prequant (decode kernel + split merge) against the HBM
    roofline.  Single GPU, rank 0 prints."""
    import torch
    import bit_quantized_attention_mean_b200 as sage

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    sh = DECODE_SHAPE
    B, H, Hkv, Lq, Lk, d = sh["B"], sh["H"], sh["Hkv"], sh["Lq"], sh["Lk"], sh["d"]
    qn, kn, vn = inputs.make_custom(B, H, Hkv, Lq, Lk, d, seed=93, k_offset_sigma=1.0)
    sm = float(np.float32(1 / np.sqrt(d)))
    q, k, v = (torch.from_numpy(x).to(dev) for x in (qn, kn, vn))
    qi, ki, qs, ks, km = sage.quant_qk(q, k, sm, q_block_rows=1)   # the cache, quantized once
    del k
    out = torch.empty_like(q)
    ws = torch.empty(max(16, sage.sage_attn_decode_workspace_size(B, H, Hkv, Lq, Lk, d)),
                     dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    launches = 0

    def step():
        nonlocal launches
        sage.sage_attn_decode_prequant(qi, ki, qs, ks, v, out, True, 1, workspace=ws,
                                       stream=stream)
        launches += sage.sage_last_launch_count()

    for _ in range(args.warmup):
        flush.zero_()
        step()
    sage.sage_check_device_status(stream)
    n = args.steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n)]
    torch.cuda.synchronize(dev)
    launches = 0
    with ClockSampler(local) as clocks:
        for i in range(n):
            flush.zero_()
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        torch.cuda.synchronize(dev)
    sage.sage_check_device_status(stream)
    ms = float(sum(a.elapsed_time(b) for a, b in evs) / n)
    if rank != 0:
        return 0
    pairs = inputs.visible_pairs(B, H, Lq, Lk, True)
    ops = 4.0 * d * pairs
    nbytes = (ki.numel() + 2 * v.numel() + qi.numel() + 2 * out.numel()
              + 4 * (qs.numel() + ks.numel()))
    peaks = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    gbs = nbytes / (ms * 1e-3) / 1e9
    line = {
        "metric": "quantized attention decode TOPS at 1 B200 and % of HBM roofline",
        "value": ops / (ms * 1e-3) / 1e12, "unit": "TOPS", "n_gpus": 1, "steps": n,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8 QK^T (int32 acc) + fp16 PV (fp32 acc)",
        "data": "synthetic (seeded numpy N(0,1) fp16, per-channel K offsets)",
        "config": {"workload": "decode-causal-B8H32Hkv8Lq1Lk32768d128", **sh, "causal": True,
                   "q_block_rows": 1, "kv_cache": "int8 K + fp16 V resident in HBM",
                   "l2": "flushed before every timed step (256 MiB write)"},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                     "frac": gbs / hbm,
                     "traffic": (DECODE_NCU_TRAFFIC["bytes_per_launch"]
                                 if DECODE_NCU_TRAFFIC["sha"] == decode_source_hash() else None),
                     "kernel": "sage_decode_kernel",
                     "bytes_per_launch": int(nbytes),
                     "peak_note": f"{peaks.get('source')} hbm_gbs (measured copy)"},
        "gpu_launches": launches,
        "clocks": clocks.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=str(DEFAULT_WORKLOAD),
                    choices=[str(i) for i in sorted(inputs.WORKLOADS)] + ["all"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-rows", type=int, default=0,
                    help="query rows of the CPU-baseline sample (0: about "
                         f"{CPU_BASELINE_PAIRS:.0e} query/key pairs' worth)")
    ap.add_argument("--ref-rows", type=int, default=512)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--q-block-rows", type=int, default=None, choices=[128, 64, 32, 1],
                    help="rows per Q quantization block (default: the workload's own, 128 "
                         "except per-token for the long-context workload)")
    ap.add_argument("--no-int8-peak", dest="int8_peak", action="store_false",
                    help="skip the INT8 GEMM peak measurement (roofline then uses 2 x bf16)")
    ap.add_argument("--pv-accum", default="f32", choices=["f32", "f16", "fp8"],
                    help="P V variant: fp16 P/V with fp32 sums (default), fp16 sums as the "
                         "article states, or P and V in FP8 E4M3 (SageAttention2)")
    ap.add_argument("--decode", action="store_true",
                    help="time the decoding layout on one query token per head against a "
                         "32768-token KV cache instead of the forward workloads")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)   # at least 3 untimed warm-up steps
    if args.decode:
        return run_decode_bench(args) if args.impl == "ours" else print(json.dumps(
            {"impl": "reference", "unavailable": "the decode timing has no CPU reference arm"}))
    ids = [2, 3, 4, 5] if args.workload == "all" else [int(args.workload)]
    qbr_arg = args.q_block_rows
    for i in ids:
        w = inputs.WORKLOADS[i]
        args.q_block_rows = qbr_arg if qbr_arg is not None else w.q_block_rows
        rc = run_reference(args, w) if args.impl == "reference" else run_ours(args, w)
        if rc:
            return rc
    return 0


if __name__ == "__main__":
    sys.exit(main())
