"""GPU parity of the finer Q granularity (Q quantization blocks of 64, 32 or
1 rows inside each 128-row attention tile) against the oracle run with the
same block height: quantization bit for bit, attention within the tolerances
of the tile-granularity tests, and on the heavy-tailed long-context workload
the accuracy gain over fp64 attention that per-token scales bring."""
import ctypes
import math

import numpy as np
import pytest

import oracle
import bit_quantized_attention_mean_b200 as sage
from bit_quantized_attention_mean_b200 import inputs

from test_gpu_parity import (COS_FP64, assert_close, assert_quant_bitexact, cos, to_dev,
                             torch_mod, workload_data)

pytestmark = pytest.mark.gpu

SHAPES = [
    # B, H, Hkv, Lq, Lk, d, causal
    (1, 2, 2, 300, 200, 64, False),     # ragged Q tail inside a 32-row block
    (2, 4, 2, 333, 333, 128, True),     # GQA + ragged causal
    (1, 3, 1, 130, 520, 128, True),     # Lq < Lk: a 2-row last tile
    (1, 2, 2, 260, 70, 64, True),       # Lq > Lk: rows that see no key
    (1, 1, 1, 1, 1, 128, False),        # single token
    (1, 32, 32, 1024, 1024, 128, True),  # many CTAs per SM
]


def gpu_quant(q, k, sm, qbr):
    outs = sage.quant_qk(to_dev(q), to_dev(k), sm, q_block_rows=qbr)
    sage.sage_check_device_status()
    return [t.cpu().numpy() for t in outs]


@pytest.mark.parametrize("qbr", [64, 32, 1])
@pytest.mark.parametrize("shape", SHAPES)
def test_quant_bitexact(shape, qbr):
    B, H, Hkv, Lq, Lk, d, causal = shape
    q, k, v = inputs.make_custom(B, H, Hkv, Lq, Lk, d, seed=Lq * 5 + qbr, k_offset_sigma=3.0)
    sm = float(np.float32(1 / math.sqrt(d)))
    want = oracle.quant_qk(q, k, sm, q_block_rows=qbr)
    assert_quant_bitexact(gpu_quant(q, k, sm, qbr), want, f"{shape} qbr={qbr}")


@pytest.mark.parametrize("qbr", [64, 32, 1])
@pytest.mark.parametrize("shape", SHAPES)
def test_attention_full_compare(shape, qbr):
    B, H, Hkv, Lq, Lk, d, causal = shape
    q, k, v = inputs.make_custom(B, H, Hkv, Lq, Lk, d, seed=Lq * 5 + qbr, k_offset_sigma=3.0)
    sm = float(np.float32(1 / math.sqrt(d)))
    out = sage.attention(to_dev(q), to_dev(k), to_dev(v), causal, sm, q_block_rows=qbr)
    sage.sage_check_device_status()
    qk = oracle.quant_qk(q, k, sm, q_block_rows=qbr)
    sim = oracle.attn_quant_sim(*qk[:4], v, causal, q_block_rows=qbr)
    ref = oracle.attn_fp64(q, k, v, causal, sm) if Lq * H * B <= 4096 else None
    assert_close(out.cpu().numpy(), sim, ref, f"{shape} qbr={qbr}")


@pytest.mark.parametrize("qbr", [128, 64, 32, 1])
def test_prequant_qblock_matches_whole_path(qbr):
    torch = torch_mod()
    q, k, v = inputs.make_custom(2, 4, 2, 300, 300, 128, seed=15)
    sm = 1 / math.sqrt(128)
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    qi, ki, qs, ks, km = sage.quant_qk(dq, dk, sm, q_block_rows=qbr)
    out1 = torch.empty_like(dq)
    sage.sage_attn_fwd_prequant_qblock(qi, ki, qs, ks, dv, out1, True, qbr)
    out2 = torch.empty_like(dq)
    sage.sage_attn_fwd_qblock(dq, dk, dv, out2, True, sm, qbr)
    sage.sage_check_device_status()
    assert torch.equal(out1, out2)
    if qbr == 128:   # the tile-granularity entry points are the same computation
        assert torch.equal(out2, sage.attention(dq, dk, dv, True, sm))
        sage.sage_check_device_status()


def test_invalid_block_height_is_rejected_by_the_library():
    torch = torch_mod()
    lib = sage.load_library()
    q = torch.zeros((1, 1, 128, 64), dtype=torch.float16, device="cuda")
    out = torch.empty_like(q)
    P = ctypes.c_void_p
    for bad in (0, 2, 16, 96, 256, -1):
        st = lib.sage_attn_fwd_qblock(P(q.data_ptr()), P(q.data_ptr()), P(q.data_ptr()),
                                      P(out.data_ptr()), 1, 1, 1, 128, 128, 64, 0, 0.125,
                                      bad, P(torch.cuda.current_stream().cuda_stream))
        assert st == 1, bad
    sage.sage_check_device_status()


@pytest.mark.parametrize("idx,qbr", [(5, 1), (5, 32), (2, 1)])
def test_workload_finer_q_blocks(idx, qbr):
    """Full-size workload with finer Q blocks: quantization bit-exact over
    every element, the output on the seeded row sample; on the heavy-tailed
    long-context workload per-token scales must lift the cosine to fp64
    attention above the tile-granularity method's own figure."""
    w, q, k, v = workload_data(idx)
    sm = float(np.float32(w.sm_scale))
    want = oracle.quant_qk(q, k, sm, q_block_rows=qbr)
    assert_quant_bitexact(gpu_quant(q, k, sm, qbr), want, f"{w.name} qbr={qbr}")
    out = sage.attention(to_dev(q), to_dev(k), to_dev(v), w.causal, sm, q_block_rows=qbr)
    sage.sage_check_device_status()
    out = out.cpu().numpy().reshape(-1, w.d)
    rows = inputs.sample_rows(w.B, w.H, w.Lq, 512, seed=idx)
    sim = oracle.attn_quant_sim(*want[:4], v, w.causal, rows=rows,
                                q_block_rows=qbr).reshape(-1, w.d)
    ref = oracle.attn_fp64(q, k, v, w.causal, sm, rows=rows).reshape(-1, w.d)
    assert_close(out[rows], sim, ref, f"{w.name} qbr={qbr}")
    if idx == 5:
        tile = oracle.quant_qk(q, k, sm)
        sim128 = oracle.attn_quant_sim(*tile[:4], v, w.causal, rows=rows).reshape(-1, w.d)
        c_fine, c_tile = cos(out[rows], ref), cos(sim128, ref)
        print(f"{w.name}: cos vs fp64 {c_fine:.6f} at {qbr}-row Q blocks, "
              f"{c_tile:.6f} at 128-row blocks")
        assert c_fine > c_tile
        if qbr == 1:
            assert c_fine >= COS_FP64
