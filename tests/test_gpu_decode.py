"""GPU parity of the decoding layout (few query tokens, query heads of a kv
group packed into one tile, keys split over CTAs and merged) against the CPU
oracle, with the tolerances of the forward tests: quantized inputs are the
same, and only the order of the softmax sums differs."""
import ctypes
import math

import numpy as np
import pytest

import oracle
import bit_quantized_attention_mean_b200 as sage
from bit_quantized_attention_mean_b200 import inputs

from test_gpu_parity import assert_close, cos, to_dev, torch_mod

pytestmark = pytest.mark.gpu

SHAPES = [
    # B, H, Hkv, Lq, Lk, d, causal, q_block_rows
    (1, 8, 2, 1, 1000, 128, False, 128),   # 4 heads per group, 16 splits of one tile
    (2, 32, 8, 1, 4096, 128, True, 1),     # per-token Q scales
    (1, 16, 16, 4, 777, 64, True, 1),      # 4 queries, bottom-right causal, ragged keys
    (2, 8, 1, 16, 2048, 128, True, 32),    # 8 heads x 16 queries = a full 128-row tile
    (4, 4, 4, 3, 130, 64, False, 128),     # three splits, ragged last tile
    (64, 8, 8, 1, 256, 128, False, 128),   # many groups: one split, no merge
    (1, 2, 2, 5, 3, 64, True, 1),          # fewer keys than queries: empty rows
]


def run_decode(q, k, v, causal, sm, qbr):
    out = sage.decode(to_dev(q), to_dev(k), to_dev(v), causal, sm, q_block_rows=qbr)
    sage.sage_check_device_status()
    return out.cpu().numpy()


@pytest.mark.parametrize("shape", SHAPES)
def test_decode_against_oracle(shape):
    B, H, Hkv, Lq, Lk, d, causal, qbr = shape
    q, k, v = inputs.make_custom(B, H, Hkv, Lq, Lk, d, seed=Lk + 7 * Lq, k_offset_sigma=2.0)
    sm = float(np.float32(1 / math.sqrt(d)))
    out = run_decode(q, k, v, causal, sm, qbr)
    qk = oracle.quant_qk(q, k, sm, q_block_rows=qbr)
    sim = oracle.attn_quant_sim(*qk[:4], v, causal, q_block_rows=qbr)
    ref = oracle.attn_fp64(q, k, v, causal, sm)
    assert_close(out, sim, ref, str(shape))


def test_decode_matches_forward_layout():
    torch = torch_mod()
    q, k, v = inputs.make_custom(2, 16, 4, 2, 3000, 128, seed=91)
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    a = sage.decode(dq, dk, dv, True, 0.088, q_block_rows=1)
    b = sage.attention(dq, dk, dv, True, 0.088, q_block_rows=1)
    sage.sage_check_device_status()
    a, b = a.cpu().numpy().astype(np.float64), b.cpu().numpy().astype(np.float64)
    assert np.abs(a - b).max() < 2e-3 and cos(a, b) > 0.99999


def test_prequant_with_caller_workspace():
    torch = torch_mod()
    B, H, Hkv, Lq, Lk, d = 1, 8, 2, 1, 5000, 128
    q, k, v = inputs.make_custom(B, H, Hkv, Lq, Lk, d, seed=92)
    sm = 0.088
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    qi, ki, qs, ks, km = sage.quant_qk(dq, dk, sm, q_block_rows=1)
    need = sage.sage_attn_decode_workspace_size(B, H, Hkv, Lq, Lk, d)
    assert need > 0
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    o1 = torch.empty_like(dq)
    sage.sage_attn_decode_prequant(qi, ki, qs, ks, dv, o1, False, 1, workspace=ws)
    o2 = torch.empty_like(dq)
    sage.sage_attn_decode_prequant(qi, ki, qs, ks, dv, o2, False, 1)
    o3 = sage.decode(dq, dk, dv, False, sm, q_block_rows=1)
    sage.sage_check_device_status()
    assert torch.equal(o1, o2) and torch.equal(o2, o3)


def test_unsupported_and_invalid_decode_shapes():
    torch = torch_mod()
    lib = sage.load_library()
    P = ctypes.c_void_p
    s = P(torch.cuda.current_stream().cuda_stream)
    q = torch.zeros((1, 16, 9, 64), dtype=torch.float16, device="cuda")   # 16 heads x 9 > 128
    k = torch.zeros((1, 1, 256, 64), dtype=torch.float16, device="cuda")
    out = torch.empty_like(q)
    st = lib.sage_attn_decode(P(q.data_ptr()), P(k.data_ptr()), P(k.data_ptr()),
                              P(out.data_ptr()), 1, 16, 1, 9, 256, 64, 0, 0.125, 128, s)
    assert st == 2
    assert lib.sage_attn_decode_workspace_size(1, 16, 1, 9, 256, 64) == 0
    st = lib.sage_attn_decode(P(q.data_ptr()), P(k.data_ptr()), P(k.data_ptr()),
                              P(out.data_ptr()), 1, 16, 1, 8, 256, 64, 0, 0.125, 7, s)
    assert st == 1   # bad q_block_rows
    sage.sage_check_device_status()


def test_decode_full_size_sampled_rows():
    """B=8, H=32, Hkv=8, one query token against 32768 keys (d = 128): the
    serving shape the decode layout is for; every output row checked."""
    B, H, Hkv, Lq, Lk, d = 8, 32, 8, 1, 32768, 128
    q, k, v = inputs.make_custom(B, H, Hkv, Lq, Lk, d, seed=93, k_offset_sigma=1.0)
    sm = float(np.float32(1 / math.sqrt(d)))
    out = run_decode(q, k, v, True, sm, 1).reshape(-1, d)
    qk = oracle.quant_qk(q, k, sm, q_block_rows=1)
    rows = np.arange(B * H * Lq, dtype=np.int64)
    sim = oracle.attn_quant_sim(*qk[:4], v, True, rows=rows, q_block_rows=1)
    ref = oracle.attn_fp64(q, k, v, True, sm, rows=rows)
    assert_close(out, sim, ref, "decode B8 H32 Hkv8 Lq1 Lk32768 d128")


@pytest.mark.parametrize("Lq,causal", [(1, True), (4, True), (3, False)])
def test_decode_varlen_against_oracle(Lq, causal):
    """Entries with 4096, 777, 65, 1 and 0 keys in one padded 4096-key cache:
    each entry's K is smoothed and quantized over its own keys (the oracle,
    per entry), and the kernel must read only those keys."""
    torch = torch_mod()
    B, H, Hkv, Lk, d = 5, 8, 2, 4096, 128
    lens = [4096, 777, 65, 1, 0]
    q, k, v = inputs.make_custom(B, H, Hkv, Lq, Lk, d, seed=94 + Lq, k_offset_sigma=2.0)
    sm = float(np.float32(1 / math.sqrt(d)))
    qbr = 1
    nkb = Lk // 64
    k_i8 = np.zeros((B, Hkv, Lk, d), np.int8)
    k_scale = np.zeros((B, Hkv, nkb), np.float32)
    q_i8 = np.zeros((B, H, Lq, d), np.int8)
    q_scale = np.zeros((B, H, Lq), np.float32)
    want = np.zeros((B, H, Lq, d))
    for b, L in enumerate(lens):
        Lb = max(L, 1)   # the oracle needs one key to quantize; length 0 reads none
        qk = oracle.quant_qk(q[b:b + 1], k[b:b + 1, :, :Lb], sm, q_block_rows=qbr)
        q_i8[b], q_scale[b] = qk[0][0], qk[2][0]
        k_i8[b, :, :Lb], k_scale[b, :, :-(-Lb // 64)] = qk[1][0], qk[3][0]
        if L > 0:
            want[b] = oracle.attn_quant_sim(qk[0], qk[1], qk[2], qk[3], v[b:b + 1, :, :L],
                                            causal, q_block_rows=qbr)[0]
    out = torch.empty((B, H, Lq, d), dtype=torch.float16, device="cuda")
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    sage.sage_attn_decode_prequant_varlen(to_dev(q_i8), to_dev(k_i8), to_dev(q_scale),
                                          to_dev(k_scale), to_dev(v), out, sl, causal, qbr)
    sage.sage_check_device_status()
    got = out.cpu().numpy().astype(np.float64)
    assert np.all(got[4] == 0)
    assert_close(got[:4], want[:4], None, f"varlen Lq={Lq} causal={causal}")


def test_decode_paged_equals_contiguous_varlen():
    """The same per-entry caches laid out as shuffled 64-key pages through a
    block table must give the contiguous variable-length result bit for bit
    (same arithmetic, different addressing)."""
    torch = torch_mod()
    B, H, Hkv, Lq, Lk, d = 4, 16, 4, 2, 2048, 128
    lens = [2048, 1000, 64, 3]
    q, k, v = inputs.make_custom(B, H, Hkv, Lq, Lk, d, seed=97, k_offset_sigma=2.0)
    sm, qbr = 0.088, 1
    nkb = Lk // 64
    k_i8 = np.zeros((B, Hkv, Lk, d), np.int8)
    k_scale = np.zeros((B, Hkv, nkb), np.float32)
    q_i8 = np.zeros((B, H, Lq, d), np.int8)
    q_scale = np.zeros((B, H, Lq), np.float32)
    for b, L in enumerate(lens):
        qk = oracle.quant_qk(q[b:b + 1], k[b:b + 1, :, :L], sm, q_block_rows=qbr)
        q_i8[b], q_scale[b] = qk[0][0], qk[2][0]
        k_i8[b, :, :L], k_scale[b, :, :-(-L // 64)] = qk[1][0], qk[3][0]
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    dq, dqs, dv = to_dev(q_i8), to_dev(q_scale), to_dev(v)
    ref = torch.empty((B, H, Lq, d), dtype=torch.float16, device="cuda")
    sage.sage_attn_decode_prequant_varlen(dq, to_dev(k_i8), dqs, to_dev(k_scale), dv, ref, sl,
                                          True, qbr)
    # pages: every used 64-key block of every entry gets a distinct page, shuffled
    rng = np.random.default_rng(5)
    used = [(b, t) for b, L in enumerate(lens) for t in range(-(-L // 64))]
    npages = len(used) + 7                      # a few pages nobody uses
    order = rng.permutation(npages)[:len(used)]
    k_pages = np.zeros((npages, Hkv, 64, d), np.int8)
    v_pages = np.zeros((npages, Hkv, 64, d), np.float16)
    ks_pages = np.zeros((npages, Hkv), np.float32)
    table = np.full((B, nkb), npages - 1, np.int32)  # unused slots point anywhere valid
    for (b, t), pg in zip(used, order):
        k_pages[pg] = k_i8[b, :, t * 64:(t + 1) * 64]
        v_pages[pg] = v[b, :, t * 64:(t + 1) * 64]
        ks_pages[pg] = k_scale[b, :, t]
        table[b, t] = pg
    out = torch.empty_like(ref)
    sage.sage_attn_decode_prequant_paged(dq, dqs, to_dev(k_pages), to_dev(ks_pages),
                                         to_dev(v_pages), to_dev(table), sl, out, True, qbr)
    sage.sage_check_device_status()
    assert torch.equal(out, ref)
