"""GPU checks of the fp16 P V accumulator (the SageAttention article's
choice, selected by SAGE_PV_ACCUM_F16) against the oracle's simulation of the
quantized algorithm, whose P V sums are exact.

Tolerance (pv_bounds.py): the accumulator is rounded to fp16 (unit roundoff
u = 2^-11) after each 16-key tensor-core step and at each rescale, and every
partial sum of element (i, c) is bounded by A_ic = sum_j P_ij |V_jc| / l_i,
that row's own absolute attention (the simulation run on |V|), so the element
moves by at most (steps + rescales) u A_ic with steps = ceil(visible keys /
16); each row's 2-norm error must also stay within the random-walk bound
4 sqrt(steps / 12) u |A_i|.  Small shapes must further meet the fp32 path's
max-abs 1e-2, and the cosine to the simulation must stay >= 0.999."""
import ctypes
import math

import numpy as np
import pytest

import oracle
import bit_quantized_attention_mean_b200 as sage
from bit_quantized_attention_mean_b200 import inputs

import pv_bounds
from test_gpu_parity import MAX_ABS, cos, to_dev, torch_mod, workload_data

pytestmark = pytest.mark.gpu

def check(out, sim, absatt, keys, what, cos_min=0.999, max_abs=None):
    g = np.asarray(out, np.float64).reshape(sim.shape)
    assert np.all(np.isfinite(g)), what
    elem, row = pv_bounds.f16acc_excess(g, sim, absatt, keys)
    err = np.abs(g - sim)
    c = cos(g, sim)
    print(f"{what}: fp16-accumulator max err {err.max():.3e}, largest error / own bound "
          f"{(err / (err - elem)).max():.3f}, cos {c:.6f}")
    pv_bounds.assert_within(elem, row, what)
    if max_abs is not None:
        assert err.max() <= max_abs, what
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
    qk = oracle.quant_qk(q, k, sm)
    sim = oracle.attn_quant_sim(*qk[:4], v, causal).reshape(-1, d)
    absatt = oracle.attn_quant_sim(*qk[:4], np.abs(v), causal).reshape(-1, d)
    keys = pv_bounds.visible_keys(np.arange(B * H * Lq) % Lq, Lq, Lk, causal)
    check(out.cpu().numpy(), sim, absatt, keys, str(shape), cos_min=0.9999, max_abs=MAX_ABS)


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
    absatt = oracle.attn_quant_sim(*qk[:4], np.abs(v), w.causal, rows=rows).reshape(-1, w.d)
    ref = oracle.attn_fp64(q, k, v, w.causal, sm, rows=rows).reshape(-1, w.d)
    keys = pv_bounds.visible_keys(rows % w.Lq, w.Lq, w.Lk, w.causal)
    check(o16[rows], sim, absatt, keys, w.name)
    print(f"{w.name}: cos vs fp64 {cos(o16[rows], ref):.6f} (fp16 sums) "
          f"{cos(o32[rows], ref):.6f} (fp32 sums); max err vs simulation "
          f"{np.abs(o16[rows] - sim).max():.3e} / {np.abs(o32[rows] - sim).max():.3e}")
