"""GPU checks of the fp16 P V accumulator (the SageAttention article's
choice, selected by SAGE_PV_ACCUM_F16) against the oracle's simulation of the
quantized algorithm, whose P V sums are exact.

Tolerance: the accumulator is rounded to fp16 (unit roundoff u = 2^-11) after
each 16-key tensor-core step and at each rescale, and every partial sum is
bounded by sum_j P_ij |V_j| <= l_i max|V|, so the normalized output moves by at
most (steps + rescales) * u * max|V| with steps = ceil(visible keys / 16); the
test allows that bound on top of the fp32-path tolerance, and requires the
cosine to the simulation to stay >= 0.999.  The measured errors are far below
the bound (they grow like its square root)."""
import ctypes
import math

import numpy as np
import pytest

import oracle
import bit_quantized_attention_mean_b200 as sage
from bit_quantized_attention_mean_b200 import inputs

from test_gpu_parity import MAX_ABS, cos, to_dev, torch_mod, workload_data

pytestmark = pytest.mark.gpu

U16 = 2.0 ** -11


def f16acc_bound(v, lk, rows_rescaled=8):
    steps = -(-lk // 16) + rows_rescaled
    return MAX_ABS + steps * U16 * float(np.abs(v.astype(np.float64)).max())


def check(out, sim, v, lk, what, cos_min=0.999):
    g = np.asarray(out, np.float64)
    assert np.all(np.isfinite(g)), what
    err = np.abs(g - sim).max()
    bound = f16acc_bound(v, lk)
    c = cos(g, sim)
    print(f"{what}: fp16-accumulator max err {err:.3e} (bound {bound:.3e}), cos {c:.6f}")
    assert err <= bound, what
    assert c >= cos_min, what


SHAPES = [
    (1, 2, 2, 256, 256, 64, False),
    (2, 4, 2, 333, 333, 128, True),
    (1, 3, 1, 130, 520, 128, True),
    (1, 2, 2, 260, 70, 64, True),
    (1, 32, 32, 1024, 1024, 128, True),
]


@pytest.mark.parametrize("shape", SHAPES)
def test_f16_accumulator_small(shape):
    B, H, Hkv, Lq, Lk, d, causal = shape
    q, k, v = inputs.make_custom(B, H, Hkv, Lq, Lk, d, seed=Lq + 3 * Lk, k_offset_sigma=2.0)
    sm = float(np.float32(1 / math.sqrt(d)))
    out = sage.attention(to_dev(q), to_dev(k), to_dev(v), causal, sm, pv_accum="f16")
    sage.sage_check_device_status()
    sim, _ = oracle.attention(q, k, v, causal, sm)
    check(out.cpu().numpy(), sim, v, Lk, str(shape), cos_min=0.9999)


def test_flags_zero_is_the_default_path():
    torch = torch_mod()
    q, k, v = inputs.make_custom(2, 4, 2, 300, 300, 128, seed=25)
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    a = sage.attention(dq, dk, dv, True, 0.088)
    b = torch.empty_like(dq)
    sage.sage_attn_fwd_ex(dq, dk, dv, b, True, 0.088, 128, "f32")
    c = torch.empty_like(dq)
    sage.sage_attn_fwd_ex(dq, dk, dv, c, True, 0.088, 128, "f16")
    sage.sage_check_device_status()
    assert torch.equal(a, b)
    assert not torch.equal(a, c)   # the accumulator really changed


def test_prequant_ex_matches_whole_path_and_is_deterministic():
    torch = torch_mod()
    q, k, v = inputs.make_custom(1, 8, 8, 640, 640, 64, seed=26)
    sm = 0.125
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    qi, ki, qs, ks, km = sage.quant_qk(dq, dk, sm, q_block_rows=32)
    o1 = torch.empty_like(dq)
    sage.sage_attn_fwd_prequant_ex(qi, ki, qs, ks, dv, o1, True, 32, "f16")
    o2 = torch.empty_like(dq)
    sage.sage_attn_fwd_ex(dq, dk, dv, o2, True, sm, 32, "f16")
    o3 = torch.empty_like(dq)
    sage.sage_attn_fwd_ex(dq, dk, dv, o3, True, sm, 32, "f16")
    sage.sage_check_device_status()
    assert torch.equal(o1, o2) and torch.equal(o2, o3)


def test_unknown_flags_are_rejected():
    torch = torch_mod()
    lib = sage.load_library()
    q = torch.zeros((1, 1, 128, 64), dtype=torch.float16, device="cuda")
    out = torch.empty_like(q)
    P = ctypes.c_void_p
    for bad in (4, 8, 0x80000000, 3):   # 3 = both P V variants at once
        st = lib.sage_attn_fwd_ex(P(q.data_ptr()), P(q.data_ptr()), P(q.data_ptr()),
                                  P(out.data_ptr()), 1, 1, 1, 128, 128, 64, 0, 0.125, 128, bad,
                                  P(torch.cuda.current_stream().cuda_stream))
        assert st == 1, bad
    sage.sage_check_device_status()


@pytest.mark.parametrize("idx", [2, 3, 5])
def test_workload_f16_accumulator(idx):
    """Full-size workloads (seeded row sample): fp16 sums against the exact
    simulation, and the accuracy against fp64 attention of both accumulators
    side by side."""
    w, q, k, v = workload_data(idx)
    sm = float(np.float32(w.sm_scale))
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    o16 = sage.attention(dq, dk, dv, w.causal, sm, pv_accum="f16").cpu().numpy().reshape(-1, w.d)
    o32 = sage.attention(dq, dk, dv, w.causal, sm).cpu().numpy().reshape(-1, w.d)
    sage.sage_check_device_status()
    rows = inputs.sample_rows(w.B, w.H, w.Lq, 512, seed=idx)
    qk = oracle.quant_qk(q, k, sm)
    sim = oracle.attn_quant_sim(*qk[:4], v, w.causal, rows=rows).reshape(-1, w.d)
    ref = oracle.attn_fp64(q, k, v, w.causal, sm, rows=rows).reshape(-1, w.d)
    check(o16[rows], sim, v, w.Lk, w.name)
    print(f"{w.name}: cos vs fp64 {cos(o16[rows], ref):.6f} (fp16 sums) "
          f"{cos(o32[rows], ref):.6f} (fp32 sums); max err vs simulation "
          f"{np.abs(o16[rows] - sim).max():.3e} / {np.abs(o32[rows] - sim).max():.3e}")
