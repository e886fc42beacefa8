"""GPU parity of the padded-batch (variable-length) forward pass: entries
with different numbers of query rows and keys in one [B, H, Lq, d] /
[B, Hkv, Lk, d] batch.  Each entry must come out exactly as the oracle (and
the dense library call) computes it on that entry alone: its own K mean
(the K smoothing step of the SageAttention article's method), its own
ragged last Q and K blocks, causal masking aligned to its own lengths.
Padding must be neither read (NaN there) nor given weight, and padding
output rows must be zeros."""
import ctypes
import math

import numpy as np
import pytest

import oracle
import bit_quantized_attention_mean_b200 as sage
from bit_quantized_attention_mean_b200 import inputs

import pv_bounds
from test_gpu_parity import assert_close, assert_quant_bitexact, cos, to_dev, torch_mod

pytestmark = pytest.mark.gpu

# (B, H, Hkv, Lq, Lk, d, lens_q, lens_k): entries with full, ragged, one-row,
# one-key and empty extents; GQA in the second
CASES = [
    (4, 4, 4, 300, 333, 128, [300, 129, 1, 0], [333, 64, 70, 5]),
    (5, 8, 2, 256, 640, 64, [256, 100, 37, 256, 3], [640, 1, 200, 0, 639]),
]


def padded_inputs(B, H, Hkv, Lq, Lk, d, lens_q, lens_k, seed):
    """Seeded inputs whose padding would poison any read of it: Q and K hold
    NaN past each entry's length; V holds NaN past the entry's last 64-key
    tile and a large finite value inside it (those keys must get weight 0)."""
    q, k, v = inputs.make_custom(B, H, Hkv, Lq, Lk, d, seed=seed, k_offset_sigma=2.0)
    q, k, v = q.copy(), k.copy(), v.copy()
    for b in range(B):
        q[b, :, lens_q[b]:] = np.nan
        k[b, :, lens_k[b]:] = np.nan
        tile_end = -(-lens_k[b] // 64) * 64
        v[b, :, lens_k[b]:tile_end] = 1000.0
        v[b, :, tile_end:] = np.nan
    return q, k, v


def seqlens(lens):
    torch = torch_mod()
    return torch.tensor(lens, dtype=torch.int32, device="cuda")


@pytest.mark.parametrize("qbr", [128, 1])
@pytest.mark.parametrize("case", CASES)
def test_quant_varlen_bitexact_per_entry(case, qbr):
    torch = torch_mod()
    B, H, Hkv, Lq, Lk, d, lq, lk = case
    q, k, _ = padded_inputs(B, H, Hkv, Lq, Lk, d, lq, lk, seed=Lq + qbr)
    sm = float(np.float32(1 / math.sqrt(d)))
    dev = "cuda"
    q_i8 = torch.zeros((B, H, Lq, d), dtype=torch.int8, device=dev)
    k_i8 = torch.zeros((B, Hkv, Lk, d), dtype=torch.int8, device=dev)
    q_scale = torch.full((B, H, -(-Lq // qbr)), -1.0, dtype=torch.float32, device=dev)
    k_scale = torch.full((B, Hkv, -(-Lk // 64)), -1.0, dtype=torch.float32, device=dev)
    k_mean = torch.full((B, Hkv, d), -1.0, dtype=torch.float32, device=dev)
    sage.sage_quant_qk_varlen(to_dev(q), to_dev(k), q_i8, k_i8, q_scale, k_scale, k_mean,
                              seqlens(lq), seqlens(lk), sm, qbr)
    sage.sage_check_device_status()
    got = [t.cpu().numpy() for t in (q_i8, k_i8, q_scale, k_scale, k_mean)]
    for b in range(B):
        # the oracle needs one row and one key: an empty extent gets a zero
        # stand-in, and nothing of it is compared
        qb = q[b:b + 1, :, :lq[b]] if lq[b] else np.zeros((1, H, 1, d), np.float16)
        kb = k[b:b + 1, :, :lk[b]] if lk[b] else np.zeros((1, Hkv, 1, d), np.float16)
        want = oracle.quant_qk(qb, kb, sm, q_block_rows=qbr)
        nqs, nks = -(-lq[b] // qbr), -(-lk[b] // 64)
        mine = [got[0][b:b + 1, :, :lq[b]], got[1][b:b + 1, :, :lk[b]],
                got[2][b:b + 1, :, :nqs], got[3][b:b + 1, :, :nks], got[4][b:b + 1]]
        ref = [want[0][:, :, :lq[b]], want[1][:, :, :lk[b]], want[2][:, :, :nqs],
               want[3][:, :, :nks], want[4] if lk[b] > 0 else np.zeros_like(want[4])]
        assert_quant_bitexact(mine, ref, f"{case} qbr={qbr} entry {b}")
        # scales past the entry's blocks are left untouched (not written)
        assert np.all(got[2][b, :, nqs:] == -1.0) and np.all(got[3][b, :, nks:] == -1.0)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("qbr", [128, 32])
@pytest.mark.parametrize("case", CASES)
def test_attention_varlen_against_oracle(case, qbr, causal):
    B, H, Hkv, Lq, Lk, d, lq, lk = case
    q, k, v = padded_inputs(B, H, Hkv, Lq, Lk, d, lq, lk, seed=3 * Lk + qbr + causal)
    sm = float(np.float32(1 / math.sqrt(d)))
    out = sage.attention_varlen(to_dev(q), to_dev(k), to_dev(v), seqlens(lq), seqlens(lk),
                                causal, sm, q_block_rows=qbr)
    sage.sage_check_device_status()
    got = out.cpu().numpy().astype(np.float64)
    for b in range(B):
        assert np.all(got[b, :, lq[b]:] == 0), f"padding rows of entry {b}"
        if lq[b] == 0:
            continue
        if lk[b] == 0:
            assert np.all(got[b] == 0), f"entry {b} has no keys"
            continue
        qb, kb, vb = q[b:b + 1, :, :lq[b]], k[b:b + 1, :, :lk[b]], v[b:b + 1, :, :lk[b]]
        qk = oracle.quant_qk(qb, kb, sm, q_block_rows=qbr)
        sim = oracle.attn_quant_sim(*qk[:4], vb, causal, q_block_rows=qbr)
        ref = oracle.attn_fp64(qb, kb, vb, causal, sm)
        assert_close(got[b:b + 1, :, :lq[b]], sim, ref, f"{case} entry {b} causal={causal}")


@pytest.mark.parametrize("pv_accum", ["f32", "f16"])
def test_varlen_entry_equals_dense_call_on_that_entry(pv_accum):
    """Same arithmetic, different addressing: each entry of the padded call
    is bit-identical to the dense call on the entry alone."""
    torch = torch_mod()
    B, H, Hkv, Lq, Lk, d, lq, lk = CASES[1]
    q, k, v = padded_inputs(B, H, Hkv, Lq, Lk, d, lq, lk, seed=17)
    v = np.nan_to_num(v, nan=0.0).astype(np.float16)   # dense slices of V end at lk[b]
    sm = 0.125
    out = sage.attention_varlen(to_dev(q), to_dev(k), to_dev(v), seqlens(lq), seqlens(lk),
                                True, sm, q_block_rows=1, pv_accum=pv_accum)
    for b in range(B):
        if lq[b] == 0 or lk[b] == 0:
            continue
        one = sage.attention(to_dev(np.ascontiguousarray(q[b:b + 1, :, :lq[b]])),
                             to_dev(np.ascontiguousarray(k[b:b + 1, :, :lk[b]])),
                             to_dev(np.ascontiguousarray(v[b:b + 1, :, :lk[b]])),
                             True, sm, q_block_rows=1, pv_accum=pv_accum)
        assert torch.equal(out[b:b + 1, :, :lq[b]], one), f"entry {b}"
    sage.sage_check_device_status()


def test_full_lengths_equal_the_dense_call():
    torch = torch_mod()
    q, k, v = inputs.make_custom(2, 4, 2, 200, 300, 128, seed=23)
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    a = sage.attention(dq, dk, dv, True, 0.09)
    b = sage.attention_varlen(dq, dk, dv, seqlens([200, 200]), seqlens([300, 300]), True, 0.09)
    c = sage.attention_varlen(dq, dk, dv, None, None, True, 0.09)
    sage.sage_check_device_status()
    assert torch.equal(a, b) and torch.equal(a, c)


def test_prequant_varlen_matches_whole_path():
    torch = torch_mod()
    B, H, Hkv, Lq, Lk, d, lq, lk = CASES[0]
    q, k, v = padded_inputs(B, H, Hkv, Lq, Lk, d, lq, lk, seed=29)
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    sq, sk = seqlens(lq), seqlens(lk)
    sm = 0.088
    q_i8 = torch.empty((B, H, Lq, d), dtype=torch.int8, device="cuda")
    k_i8 = torch.empty((B, Hkv, Lk, d), dtype=torch.int8, device="cuda")
    q_scale = torch.empty((B, H, -(-Lq // 64)), dtype=torch.float32, device="cuda")
    k_scale = torch.empty((B, Hkv, -(-Lk // 64)), dtype=torch.float32, device="cuda")
    k_mean = torch.empty((B, Hkv, d), dtype=torch.float32, device="cuda")
    sage.sage_quant_qk_varlen(dq, dk, q_i8, k_i8, q_scale, k_scale, k_mean, sq, sk, sm, 64)
    o1 = torch.empty_like(dq)
    sage.sage_attn_fwd_prequant_varlen(q_i8, k_i8, q_scale, k_scale, dv, o1, sq, sk, False, 64)
    o2 = sage.attention_varlen(dq, dk, dv, sq, sk, False, sm, q_block_rows=64)
    sage.sage_check_device_status()
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("case", CASES)
def test_fp8_varlen_against_oracle(case, causal):
    """FP8 P V on a padded batch: each entry's V channel scales span its own
    keys (the oracle quantizes the entry's slice), the codes past its length
    are 0, so even NaN padding inside the last key tile is harmless here.
    Bound and cosine gate as the dense FP8 tests: P is rounded at a
    different point (running vs exact max), by at most half an E4M3 unit, so
    each element stays within 2^-3 of its row's own absolute attention."""
    B, H, Hkv, Lq, Lk, d, lq, lk = case
    q, k, v = padded_inputs(B, H, Hkv, Lq, Lk, d, lq, lk, seed=5 * Lk + causal)
    for b in range(B):
        v[b, :, lk[b]:] = np.nan
    sm = float(np.float32(1 / math.sqrt(d)))
    out = sage.attention_varlen(to_dev(q), to_dev(k), to_dev(v), seqlens(lq), seqlens(lk),
                                causal, sm, pv_accum="fp8")
    sage.sage_check_device_status()
    got = out.cpu().numpy().astype(np.float64)
    for b in range(B):
        assert np.all(got[b, :, lq[b]:] == 0), f"padding rows of entry {b}"
        if lq[b] == 0 or lk[b] == 0:
            assert np.all(got[b] == 0)
            continue
        qb, kb, vb = q[b:b + 1, :, :lq[b]], k[b:b + 1, :, :lk[b]], v[b:b + 1, :, :lk[b]]
        qk = oracle.quant_qk(qb, kb, sm)
        v8t, vs = oracle.quant_v_fp8(vb)
        sim = oracle.attn_fp8pv_sim(*qk[:4], v8t, vs, causal)
        absatt = oracle.attn_fp8pv_sim(*qk[:4], v8t & 0x7F, vs, causal)
        g = got[b:b + 1, :, :lq[b]]
        assert np.all(np.isfinite(g)), f"entry {b}"
        elem, row = pv_bounds.fp8_excess(g.reshape(-1, d), sim.reshape(-1, d),
                                         absatt.reshape(-1, d))
        pv_bounds.assert_within(elem, row, f"{case} entry {b}")
        if np.abs(sim).max() > 0:
            assert cos(g, sim) >= 0.999, f"{case} entry {b}"


def test_varlen_bad_args_rejected():
    torch = torch_mod()
    lib = sage.load_library()
    P = ctypes.c_void_p
    s = P(torch.cuda.current_stream().cuda_stream)
    q = torch.zeros((2, 2, 64, 64), dtype=torch.float16, device="cuda")
    out = torch.empty_like(q)
    sl = seqlens([64, 10])
    args = (P(q.data_ptr()), P(q.data_ptr()), P(q.data_ptr()), P(out.data_ptr()))
    st = lib.sage_attn_fwd_varlen(*args, P(0), P(sl.data_ptr()), 2, 2, 2, 64, 64, 64, 0, 0.125,
                                  7, 0, s)
    assert st == 1   # bad q_block_rows
    st = lib.sage_attn_fwd_varlen(*args, P(0), P(sl.data_ptr()), 2, 2, 2, 64, 64, 64, 0, 0.125,
                                  128, 3, s)
    assert st == 1   # both P V variants at once
    qi = torch.zeros((2, 2, 64, 64), dtype=torch.int8, device="cuda")
    sc = torch.zeros(8, dtype=torch.float32, device="cuda")
    st = lib.sage_attn_fwd_prequant_varlen(P(qi.data_ptr()), P(qi.data_ptr()), P(sc.data_ptr()),
                                           P(sc.data_ptr()), P(q.data_ptr()), P(out.data_ptr()),
                                           P(sl.data_ptr()), P(sl.data_ptr()), 2, 2, 2, 64, 64,
                                           64, 0, 128, sage.SAGE_PV_FP8, s)
    assert st == 1   # the prequant call takes fp16 V
    sage.sage_check_device_status()
