"""GPU parity of the CUDA path against the CPU oracle (needs a B200).

Quantization (int8 codes, fp32 scales, K mean) must match bit for bit.  The
attention output (fp16) must match the oracle's simulation of the quantized
algorithm to max-abs <= 1e-2 (widened to one fp16 spacing of the reference
where |O| >= 16, because the output format itself cannot resolve 1e-2 there)
and cosine >= 0.9999, and full-precision fp64 attention to cosine >= 0.999.
Small cases compare every element; the full-size workloads compare a seeded
sample of query rows that includes the first and last rows of every head and
both sides of each 128-row tile boundary of one head.  Each workload runs at
its own Q granularity (128-row blocks, or one row per block for the
heavy-tailed long-context workload, whose 128-row blocks miss the fp64 gate;
that 128-row result is printed, not asserted against the gate).
"""
import functools
import math

import numpy as np
import pytest

import oracle
import bit_quantized_attention_mean_b200 as sage
from bit_quantized_attention_mean_b200 import inputs

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
COS_SIM = 0.9999
COS_FP64 = 0.999


def torch_mod():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def to_dev(a):
    torch = torch_mod()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def cos(a, b):
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))


def assert_close(gpu_f16, sim, fp64=None, what=""):
    g = np.asarray(gpu_f16, dtype=np.float64)
    assert np.all(np.isfinite(g)), what
    ulp = np.spacing(np.abs(sim).astype(np.float16)).astype(np.float64)
    tol = np.maximum(MAX_ABS, ulp)
    err = np.abs(g - sim)
    worst = np.unravel_index(np.argmax(err - tol), err.shape)
    assert np.all(err <= tol), f"{what}: max err {err.max():.3e} at {worst}, ref {sim[worst]:.4f}"
    c = cos(g, sim)
    assert c >= COS_SIM, f"{what}: cos vs simulation {c}"
    if fp64 is not None:
        c64 = cos(g, fp64)
        print(f"{what}: cos vs sim {c:.6f}, vs fp64 {c64:.6f} (method {cos(sim, fp64):.6f})")
        assert c64 >= COS_FP64, f"{what}: cos vs fp64 {c64}"
    return c


def gpu_quant(q, k, sm, qbr=128):
    outs = sage.quant_qk(to_dev(q), to_dev(k), sm, q_block_rows=qbr)
    sage.sage_check_device_status()
    return [t.cpu().numpy() for t in outs]


def gpu_attention(q, k, v, causal, sm, qbr=128):
    torch = torch_mod()
    out = sage.attention(to_dev(q), to_dev(k), to_dev(v), causal, sm, q_block_rows=qbr)
    sage.sage_check_device_status()
    return out.cpu().numpy()


def assert_quant_bitexact(got, want, what):
    names = ("q_i8", "k_i8", "q_scale", "k_scale", "k_mean")
    for n, g, w in zip(names, got, want):
        assert g.shape == w.shape, (what, n)
        if g.dtype == np.float32:
            assert np.array_equal(g.view(np.uint32), w.view(np.uint32)), (what, n)
        else:
            assert np.array_equal(g, w), (what, n, int(np.sum(g != w)))


# --------------------------------------------------------- small shapes

SMALL = [
    # B, H, Hkv, Lq, Lk, d, causal
    (1, 2, 2, 256, 256, 64, False),
    (1, 2, 2, 300, 200, 64, False),     # ragged Q and K tails
    (2, 4, 2, 333, 333, 128, True),     # GQA + ragged causal
    (1, 3, 1, 130, 520, 128, True),     # Lq < Lk, bottom-right causal
    (1, 2, 2, 260, 70, 64, True),       # Lq > Lk: leading rows see no key
    (1, 1, 1, 1, 1, 128, False),        # single token
    (1, 2, 1, 64, 1000, 128, False),    # one partial Q tile, many K tiles
    (3, 2, 2, 129, 65, 64, True),
]


@pytest.mark.parametrize("shape", SMALL)
def test_quant_bitexact_small(shape):
    B, H, Hkv, Lq, Lk, d, causal = shape
    q, k, v = inputs.make_custom(B, H, Hkv, Lq, Lk, d, seed=Lq * 7 + Lk, k_offset_sigma=3.0)
    sm = float(np.float32(1 / math.sqrt(d)))
    assert_quant_bitexact(gpu_quant(q, k, sm), oracle.quant_qk(q, k, sm), str(shape))


@pytest.mark.parametrize("shape", SMALL)
def test_attention_small_full_compare(shape):
    B, H, Hkv, Lq, Lk, d, causal = shape
    q, k, v = inputs.make_custom(B, H, Hkv, Lq, Lk, d, seed=Lq * 7 + Lk, k_offset_sigma=3.0)
    sm = float(np.float32(1 / math.sqrt(d)))
    out = gpu_attention(q, k, v, causal, sm)
    sim, _ = oracle.attention(q, k, v, causal, sm)
    ref = oracle.attn_fp64(q, k, v, causal, sm)
    assert_close(out, sim, ref, str(shape))


MEDIUM = [
    # every row compared; enough CTAs that two share each SM and the tensor
    # core queue is long (short causal tiles finish while their last P V
    # products are still in flight)
    (1, 32, 32, 1024, 1024, 128, True),
    (2, 16, 4, 768, 768, 128, True),
    (1, 24, 24, 1024, 1024, 64, False),
    (1, 32, 32, 640, 640, 64, True),
]


@pytest.mark.parametrize("shape", MEDIUM)
def test_attention_medium_all_rows(shape):
    B, H, Hkv, Lq, Lk, d, causal = shape
    q, k, v = inputs.make_custom(B, H, Hkv, Lq, Lk, d, seed=Lq + H, k_offset_sigma=2.0)
    sm = float(np.float32(1 / math.sqrt(d)))
    for _ in range(2):   # twice: also checks run-to-run identity under load
        out = gpu_attention(q, k, v, causal, sm)
        if _ == 0:
            first = out
    assert np.array_equal(first, out)
    sim, _ = oracle.attention(q, k, v, causal, sm)
    assert_close(out, sim, None, str(shape))


def test_prequant_matches_whole_path():
    torch = torch_mod()
    q, k, v = inputs.make_custom(2, 4, 2, 300, 300, 128, seed=5)
    sm = 1 / math.sqrt(128)
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    qi, ki, qs, ks, km = sage.quant_qk(dq, dk, sm)
    out1 = torch.empty_like(dq)
    sage.sage_attn_fwd_prequant(qi, ki, qs, ks, dv, out1, True)
    out2 = sage.attention(dq, dk, dv, True, sm)
    sage.sage_check_device_status()
    assert torch.equal(out1, out2)


def test_deterministic():
    torch = torch_mod()
    q, k, v = inputs.make_custom(1, 4, 4, 512, 512, 128, seed=8)
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    a = sage.attention(dq, dk, dv, True, 0.088)
    b = sage.attention(dq, dk, dv, True, 0.088)
    sage.sage_check_device_status()
    assert torch.equal(a, b)


@pytest.mark.parametrize("shape", [(1, 2, 2, 384, 384, 64, False),
                                   (3, 8, 2, 300, 520, 128, True),    # 6 groups in 6 chunks
                                   (4, 32, 8, 256, 256, 64, True)])   # 32 groups, 8 chunks
def test_host_buffer_entry_point_matches_device(shape):
    """The host-buffer call processes (batch, kv head) groups in chunks on two
    side streams; its output must equal the device call's bit for bit."""
    torch = torch_mod()
    B, H, Hkv, Lq, Lk, d, causal = shape
    q, k, v = inputs.make_custom(B, H, Hkv, Lq, Lk, d, seed=9 + B)
    hq, hk, hv = (torch.from_numpy(x).pin_memory() for x in (q, k, v))
    hout = torch.empty(q.shape, dtype=torch.float16).pin_memory()
    sage.sage_attn_fwd_host(hq, hk, hv, hout, causal, 0.125)
    torch.cuda.current_stream().synchronize()
    dev = sage.attention(to_dev(q), to_dev(k), to_dev(v), causal, 0.125)
    sage.sage_check_device_status()
    assert torch.equal(hout, dev.cpu())


def test_host_buffer_entry_point_with_finer_q_blocks():
    """sage_attn_fwd_host_qblock equals the device call at the same Q
    granularity, bit for bit."""
    torch = torch_mod()
    q, k, v = inputs.make_custom(2, 8, 4, 300, 400, 128, seed=17)
    hq, hk, hv = (torch.from_numpy(x).pin_memory() for x in (q, k, v))
    for qbr in (1, 32):
        hout = torch.empty(q.shape, dtype=torch.float16).pin_memory()
        sage.sage_attn_fwd_host_qblock(hq, hk, hv, hout, True, 0.088, qbr)
        torch.cuda.current_stream().synchronize()
        dev = sage.attention(to_dev(q), to_dev(k), to_dev(v), True, 0.088, q_block_rows=qbr)
        sage.sage_check_device_status()
        assert torch.equal(hout, dev.cpu()), qbr


# ------------------------------------------------------------ closed forms

@pytest.mark.parametrize("causal", [False, True])
def test_closed_forms_on_gpu(causal):
    B, H, L, d = 1, 2, 320, 128
    q, k, v = inputs.make_custom(B, H, H, L, L, d, seed=77)
    sm = 1 / math.sqrt(d)
    # V constant along tokens -> O is that row (up to fp16 rounding of O)
    vc = np.broadcast_to(v[:, :, :1], v.shape).copy()
    out = gpu_attention(q, k, vc, causal, sm).astype(np.float64)
    exp = np.broadcast_to(vc[:, :, :1].astype(np.float64), out.shape)
    assert np.max(np.abs(out - exp)) <= 2e-3
    # all K rows equal -> smoothed K is 0 -> uniform weights over visible keys
    ke = np.broadcast_to(k[:, :, :1], k.shape).copy()
    out = gpu_attention(q, ke, v, causal, sm).astype(np.float64)
    vv = v.astype(np.float64)
    if causal:
        exp = np.cumsum(vv, axis=2) / np.arange(1, L + 1)[None, None, :, None]
    else:
        exp = np.broadcast_to(vv.mean(axis=2, keepdims=True), vv.shape)
    assert np.max(np.abs(out - exp)) <= 2e-3
    # causal row 0 sees only key 0 -> O = v0 exactly
    if causal:
        out = gpu_attention(q, k, v, True, sm)
        assert np.array_equal(out[:, :, 0], v[:, :, 0])


def test_invalid_arguments_are_rejected_before_launch():
    torch = torch_mod()
    q = torch.zeros((1, 3, 128, 64), dtype=torch.float16, device="cuda")
    k = torch.zeros((1, 2, 128, 64), dtype=torch.float16, device="cuda")
    out = torch.empty_like(q)
    with pytest.raises(sage.SageError) as e:
        sage.sage_attn_fwd(q, k, k, out, False, 0.125)      # H % Hkv != 0
    assert e.value.status == 1
    q96 = torch.zeros((1, 2, 128, 96), dtype=torch.float16, device="cuda")
    with pytest.raises(sage.SageError) as e:
        sage.sage_attn_fwd(q96, q96, q96, torch.empty_like(q96), False, 0.1)
    assert e.value.status == 2
    qq = torch.zeros((1, 2, 128, 64), dtype=torch.float16, device="cuda")
    with pytest.raises(sage.SageError) as e:
        sage.sage_attn_fwd(qq, qq, qq, torch.empty_like(qq), False, -1.0)
    assert e.value.status == 1
    base = torch.zeros(2 * 128 * 64 + 8, dtype=torch.float16, device="cuda")
    mis = base[1:1 + 2 * 128 * 64].view(1, 2, 128, 64)   # 2-byte offset
    with pytest.raises(sage.SageError) as e:
        sage.sage_attn_fwd(mis, qq, qq, torch.empty_like(qq), False, 0.1)
    assert e.value.status == 1
    sage.sage_check_device_status()


# ------------------------------------------------------ full-size workloads

@functools.lru_cache(maxsize=1)
def workload_data(idx):
    w = inputs.WORKLOADS[idx]
    q, k, v = inputs.make_inputs(w)
    return w, q, k, v


@pytest.mark.parametrize("idx", [1, 2, 3, 4, 5])
def test_workload(idx):
    """Full-size workload through sage_attn_fwd at the workload's Q
    granularity: quantization bit-exact over every element, output checked
    on the seeded row sample (all rows for the tiny workload), fp64 gate
    unrelaxed."""
    w, q, k, v = workload_data(idx)
    sm = float(np.float32(w.sm_scale))
    qbr = w.q_block_rows
    want_q = oracle.quant_qk(q, k, sm, q_block_rows=qbr)
    assert_quant_bitexact(gpu_quant(q, k, sm, qbr), want_q, w.name)
    out = gpu_attention(q, k, v, w.causal, sm, qbr).reshape(-1, w.d)
    rows = None if idx == 1 else inputs.sample_rows(w.B, w.H, w.Lq, 512, seed=idx)
    sim = oracle.attn_quant_sim(*want_q[:4], v, w.causal, rows=rows,
                                q_block_rows=qbr).reshape(-1, w.d)
    ref = oracle.attn_fp64(q, k, v, w.causal, sm, rows=rows).reshape(-1, w.d)
    got = out if rows is None else out[rows]
    assert_close(got, sim, ref, f"{w.name} (Q blocks of {qbr})")


def test_longctx_tile_granularity_reported():
    """The long-context workload at 128-row Q blocks (the attention tile):
    the kernel must match the oracle's simulation of that granularity; its
    accuracy against fp64 attention is printed as a reported number (the
    method itself falls short of 0.999 there, which is why the workload runs
    with per-token Q blocks)."""
    w, q, k, v = workload_data(5)
    sm = float(np.float32(w.sm_scale))
    want_q = oracle.quant_qk(q, k, sm)
    assert_quant_bitexact(gpu_quant(q, k, sm), want_q, w.name)
    out = gpu_attention(q, k, v, w.causal, sm).reshape(-1, w.d)
    rows = inputs.sample_rows(w.B, w.H, w.Lq, 512, seed=5)
    sim = oracle.attn_quant_sim(*want_q[:4], v, w.causal, rows=rows).reshape(-1, w.d)
    ref = oracle.attn_fp64(q, k, v, w.causal, sm, rows=rows).reshape(-1, w.d)
    assert_close(out[rows], sim, None, f"{w.name} (Q blocks of 128)")
    print(f"{w.name} with 128-row Q blocks: cos vs fp64 {cos(out[rows], ref):.6f} "
          f"(method {cos(sim, ref):.6f}; reported, not gated)")


def test_degenerate_blocks_zero_q_and_constant_k():
    """An all-zero 128-row Q block (scale 0) and a head whose K rows are all
    equal (smoothed K is 0, every K scale 0) quantize to zero codes with zero
    scales and give uniform attention over the visible keys."""
    torch = torch_mod()
    B, H, L, d = 1, 2, 300, 128
    q, k, v = inputs.make_custom(B, H, H, L, L, d, seed=71)
    q[0, 0, 128:256] = 0                            # zero Q block of head 0
    k[0, 1] = k[0, 1, :1]                           # constant K rows in head 1
    sm = 1 / math.sqrt(d)
    want = oracle.quant_qk(q, k, sm)
    got = gpu_quant(q, k, sm)
    assert_quant_bitexact(got, want, "degenerate blocks")
    assert got[2][0, 0, 1] == 0 and np.all(got[0][0, 0, 128:256] == 0)
    assert np.all(got[3][0, 1] == 0) and np.all(got[1][0, 1] == 0)
    out = gpu_attention(q, k, v, True, sm).astype(np.float64)
    vv = v.astype(np.float64)
    uniform = np.cumsum(vv, axis=2) / np.arange(1, L + 1)[None, None, :, None]
    assert np.abs(out[0, 0, 128:256] - uniform[0, 0, 128:256]).max() <= 2e-3
    assert np.abs(out[0, 1] - uniform[0, 1]).max() <= 2e-3
