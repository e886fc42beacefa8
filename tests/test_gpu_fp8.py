"""GPU parity of the FP8 (E4M3) P V path (the SageAttention2 description:
P and V in FP8) against the oracle.

V quantization must match bit for bit.  The attention output is compared
with the oracle's FP8 simulation, which quantizes P against the exact row
max (e4m3(448 p)) while the kernel quantizes against its running max
(e4m3(1.75 p), p <= 2^8): each P is rounded at a different point, by at most
half an E4M3 unit (relative 2^-4), so element (i, c) moves by at most
2^-3 A_ic, A_ic = sum_j p_ij |V_jc| / sum_j p_ij, that row's own absolute
attention (the simulation run on |V|; pv_bounds.py), plus the fp16 output
rounding; the cosine to the simulation must stay >= 0.999."""
import ctypes
import math

import numpy as np
import pytest

import oracle
import bit_quantized_attention_mean_b200 as sage
from bit_quantized_attention_mean_b200 import inputs

import pv_bounds
from test_gpu_parity import cos, to_dev, torch_mod, workload_data

pytestmark = pytest.mark.gpu


def gpu_v8(v):
    v8t, vs = sage.quant_v_fp8(to_dev(v))
    sage.sage_check_device_status()
    return v8t.cpu().numpy(), vs.cpu().numpy()


@pytest.mark.parametrize("shape,tail", [((1, 2, 300, 64), False), ((2, 3, 130, 128), True),
                                        ((1, 1, 1000, 128), False), ((1, 2, 64, 64), False),
                                        ((1, 1, 1, 128), False)])
def test_quant_v_fp8_bitexact(shape, tail):
    rng = np.random.default_rng(shape[2])
    v = (rng.standard_t(4, size=shape) * 2).astype(np.float16)
    v[0, 0, :, 3] = 0                               # zero channel
    if tail:
        v[0, 0, 5, 7] = np.float16(60000)           # a large value
        v[0, 1, :, 9] = np.float16(2.0 ** -20)      # subnormal fp16 channel
    got8, gots = gpu_v8(v)
    want8, wants = oracle.quant_v_fp8(v)
    Lk = shape[2]
    assert np.array_equal(got8[..., :Lk], want8)
    assert np.all(got8[..., Lk:] == 0)
    assert np.array_equal(gots.view(np.uint32), wants.view(np.uint32))


def check(out, sim, absatt, what):
    g = np.asarray(out, np.float64).reshape(sim.shape)
    assert np.all(np.isfinite(g)), what
    elem, _ = pv_bounds.fp8_excess(g, sim, absatt)
    err = np.abs(g - sim)
    c = cos(g, sim)
    print(f"{what}: FP8 P V max err {err.max():.3e}, largest error / own bound "
          f"{(err / (err - elem)).max():.3f}, cos vs FP8 simulation {c:.6f}")
    pv_bounds.assert_within(elem, elem.max(axis=-1), what)
    assert c >= 0.999, what


SHAPES = [
    (1, 2, 2, 256, 256, 64, False),
    (2, 4, 2, 333, 333, 128, True),
    (1, 3, 1, 130, 520, 128, True),
    (1, 2, 2, 260, 70, 64, True),
    (1, 32, 32, 1024, 1024, 128, True),
]


@pytest.mark.parametrize("shape", SHAPES)
def test_fp8_attention_small(shape):
    B, H, Hkv, Lq, Lk, d, causal = shape
    q, k, v = inputs.make_custom(B, H, Hkv, Lq, Lk, d, seed=Lq + 11 * Lk, k_offset_sigma=2.0)
    sm = float(np.float32(1 / math.sqrt(d)))
    out = sage.attention(to_dev(q), to_dev(k), to_dev(v), causal, sm, pv_accum="fp8")
    sage.sage_check_device_status()
    qk = oracle.quant_qk(q, k, sm)
    v8t, vs = oracle.quant_v_fp8(v)
    sim = oracle.attn_fp8pv_sim(*qk[:4], v8t, vs, causal).reshape(-1, d)
    absatt = oracle.attn_fp8pv_sim(*qk[:4], v8t & 0x7F, vs, causal).reshape(-1, d)
    check(out.cpu().numpy(), sim, absatt, str(shape))


def test_fp8_equal_scores_give_the_mean_of_dequantized_v():
    """All K rows equal: every visible p is 1, which E4M3 holds exactly
    (1.75 in the kernel, 448 in the oracle), so the output is the mean of the
    dequantized V rows up to fp32 sums and the fp16 output."""
    B, H, L, d = 1, 2, 320, 128
    q, k, v = inputs.make_custom(B, H, H, L, L, d, seed=46)
    ke = np.broadcast_to(k[:, :, :1], k.shape).copy()
    sm = 1 / math.sqrt(d)
    out = sage.attention(to_dev(q), to_dev(ke), to_dev(v), True, sm, pv_accum="fp8")
    sage.sage_check_device_status()
    v8t, vs = oracle.quant_v_fp8(v)
    deq = np.swapaxes(np.vectorize(oracle.e4m3_decode)(v8t), 2, 3) * vs[:, :, None, :]
    exp = np.cumsum(deq, axis=2) / np.arange(1, L + 1)[None, None, :, None]
    g = out.cpu().numpy().astype(np.float64)
    assert np.abs(g - exp).max() <= 2e-3 * max(1.0, np.abs(exp).max())


def test_prequant_fp8pv_matches_whole_path():
    torch = torch_mod()
    q, k, v = inputs.make_custom(2, 4, 2, 300, 300, 128, seed=47)
    sm = 1 / math.sqrt(128)
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    qi, ki, qs, ks, km = sage.quant_qk(dq, dk, sm)
    v8t, vs = sage.quant_v_fp8(dv)
    o1 = torch.empty_like(dq)
    sage.sage_attn_fwd_prequant_fp8pv(qi, ki, qs, ks, v8t, vs, o1, True)
    o2 = torch.empty_like(dq)
    sage.sage_attn_fwd_ex(dq, dk, dv, o2, True, sm, 128, "fp8")
    sage.sage_check_device_status()
    assert torch.equal(o1, o2)


def test_fp8_flag_rules():
    torch = torch_mod()
    lib = sage.load_library()
    P = ctypes.c_void_p
    s = P(torch.cuda.current_stream().cuda_stream)
    q = torch.zeros((1, 1, 128, 64), dtype=torch.float16, device="cuda")
    out = torch.empty_like(q)
    qi = torch.zeros((1, 1, 128, 64), dtype=torch.int8, device="cuda")
    sc = torch.zeros(4, dtype=torch.float32, device="cuda")
    # both variants at once, and FP8 on the fp16-V prequant call, are refused
    assert lib.sage_attn_fwd_ex(P(q.data_ptr()), P(q.data_ptr()), P(q.data_ptr()),
                                P(out.data_ptr()), 1, 1, 1, 128, 128, 64, 0, 0.125, 128, 3, s) == 1
    assert lib.sage_attn_fwd_prequant_ex(P(qi.data_ptr()), P(qi.data_ptr()), P(sc.data_ptr()),
                                         P(sc.data_ptr()), P(q.data_ptr()), P(out.data_ptr()),
                                         1, 1, 1, 128, 128, 64, 0, 128, 2, s) == 1
    sage.sage_check_device_status()


@pytest.mark.parametrize("idx", [2, 3, 5])
def test_workload_fp8(idx):
    """Full-size workloads on the seeded row sample: FP8 P V against the FP8
    simulation, and the accuracy against fp64 attention next to the fp16 path."""
    w, q, k, v = workload_data(idx)
    sm = float(np.float32(w.sm_scale))
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    o8 = sage.attention(dq, dk, dv, w.causal, sm, pv_accum="fp8").cpu().numpy().reshape(-1, w.d)
    o16 = sage.attention(dq, dk, dv, w.causal, sm).cpu().numpy().reshape(-1, w.d)
    sage.sage_check_device_status()
    rows = inputs.sample_rows(w.B, w.H, w.Lq, 512, seed=idx)
    qk = oracle.quant_qk(q, k, sm)
    v8t, vs = oracle.quant_v_fp8(v)
    sim = oracle.attn_fp8pv_sim(*qk[:4], v8t, vs, w.causal, rows=rows).reshape(-1, w.d)
    absatt = oracle.attn_fp8pv_sim(*qk[:4], v8t & 0x7F, vs, w.causal,
                                   rows=rows).reshape(-1, w.d)
    ref = oracle.attn_fp64(q, k, v, w.causal, sm, rows=rows).reshape(-1, w.d)
    check(o8[rows], sim, absatt, w.name)
    print(f"{w.name}: cos vs fp64 {cos(o8[rows], ref):.6f} (FP8 P V) {cos(o16[rows], ref):.6f} "
          f"(fp16 P V); cos FP8 simulation vs fp64 {cos(sim, ref):.6f}")
