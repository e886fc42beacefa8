"""Pins of the CPU oracle to facts other than itself (no GPU needed).

Each test ties one oracle function to something the SageAttention article or
plain mathematics fixes: hand-derived quantized blocks (tests/golden), the
fp16 format as numpy implements it, brute-force fp64 attention written with
numpy matrix routines, closed forms and exact invariants.  A plausible slip in
the oracle (a dropped log2 e, a transposed operand, the wrong mean axis, a
wrong block index, round-half-up instead of half-even) fails at least one.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from bit_quantized_attention_mean_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "quant_blocks.json")


def f32_bits(x):
    return int(np.asarray(x, dtype=np.float32).view(np.uint32))


# ---------------------------------------------------------------- fp16 format

def test_half_to_double_matches_numpy_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits])
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.all(np.isnan(got[np.isnan(ref)]))
    assert np.array_equal(np.isinf(got), np.isinf(ref))


def test_double_to_half_matches_numpy_rne():
    rng = np.random.default_rng(7)
    xs = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-9, 5, 20000),
        # exact ties between consecutive fp16 values (normal and subnormal)
        (np.arange(0, 2048, dtype=np.float64) + 0.5) * 2.0 ** -24,
        (np.arange(1024, 2048, dtype=np.float64) + 0.5) * 2.0 ** -10,
        [65504.0, 65519.99, 65520.0, 1e6, 2.0 ** -25, 2.0 ** -25 * 1.0001, 0.0, -0.0],
    ])
    with np.errstate(over="ignore"):
        ref = xs.astype(np.float16).view(np.uint16)
    got = np.array([oracle.double_to_half(float(x)) for x in xs], dtype=np.uint16)
    assert np.array_equal(got, ref)


# ----------------------------------------------------------- golden blocks

def _golden_cases():
    with open(GOLDEN) as f:
        g = json.load(f)
    return g, g["cases"]


def _expand(case, key):
    if key in case:
        return np.array(case[key], dtype=np.float64)
    rule = case[key + "_rule"]
    n = int(np.prod(case["shape"]))
    name = case["name"]
    if name == "q_ragged_second_block":
        if key == "x":
            a = np.ones(n); a[5] = -4.0; a[128] = 0.75; a[129] = -0.25
        else:
            a = np.full(n, 32.0); a[5] = -127; a[128] = 127; a[129] = -42
        return a
    if name == "k_ragged_mean_over_all_tokens":
        t = np.arange(n)
        if key == "x":
            a = np.where(t % 2 == 0, 1.0, -1.0); a[64] = 5.0
        else:
            a = np.where(t % 2 == 0, 109.0, -127.0); a[64] = 127
        return a
    raise KeyError(rule)


@pytest.mark.parametrize("idx", range(6))
def test_golden_quant_blocks(idx):
    g, cases = _golden_cases()
    case = cases[idx]
    sm = g["sm_scale"]
    shape = case["shape"]
    x = _expand(case, "x").astype(np.float16).reshape(shape)
    qexp = _expand(case, "q").astype(np.int8).reshape(shape)
    dummy_shape = list(shape)
    dummy = np.zeros(dummy_shape, dtype=np.float16)
    if case["tensor"] == "q":
        q_i8, _, q_scale, _, _ = oracle.quant_qk(x, dummy, sm)
        assert np.array_equal(q_i8, qexp)
        got = [f32_bits(s) for s in q_scale.ravel()]
        assert got == [int(b, 16) for b in case["scale_bits"]]
    else:
        _, k_i8, _, k_scale, km = oracle.quant_qk(dummy, x, sm)
        assert np.array_equal(k_i8, qexp)
        if "k_mean" in case:
            assert np.array_equal(km.ravel(), np.array(case["k_mean"], dtype=np.float32))
        if "scale_bits" in case:
            got = [f32_bits(s) for s in k_scale.ravel()]
            assert got == [int(b, 16) for b in case["scale_bits"]]
        if "scale_exact" in case:
            m = Fraction(5, 65)
            exact = [(1 + m) / 127, (5 - m) / 127]
            for s, e in zip(k_scale.ravel(), exact):
                ulp = np.spacing(np.float32(float(e)))
                assert abs(float(s) - float(e)) <= ulp
        if "k_mean_exact" in case:
            assert km.ravel()[0] == np.float32(float(Fraction(5, 65)))


def test_golden_c_constant():
    g, _ = _golden_cases()
    # a Q block whose scale is exactly 1 exposes c itself
    q = np.zeros((1, 1, 1, 4), dtype=np.float16); q[..., 0] = 127
    _, _, qs, _, _ = oracle.quant_qk(q, np.zeros_like(q), g["sm_scale"])
    assert f32_bits(qs.ravel()[0]) == int(g["c_bits"], 16)
    assert abs(float(qs.ravel()[0]) - math.log2(math.e) / 8) < 1e-8


# --------------------------------------------------------------- K mean

def test_k_mean_equals_float64_sum_over_tokens():
    q, k, v = inputs.make_custom(2, 3, 3, 50, 333, 64, seed=3, k_offset_sigma=3.0)
    km = oracle.k_mean(k)
    # fp16 values are multiples of 2^-24 and small here, so the float64 sum is exact
    ref = (k.astype(np.float64).sum(axis=2) / k.shape[2]).astype(np.float32)
    assert np.array_equal(km, ref)
    # mean over channels (the other possible reading) is a different quantity
    assert not np.allclose(km, k.astype(np.float64).mean(axis=3, keepdims=False)[:, :, :1])


def test_k_mean_shift_invariance():
    # Lk a power of two: every mean is an exact dyadic, so the shift is exact
    rng = np.random.default_rng(11)
    k = rng.integers(-20, 20, size=(1, 2, 128, 16)).astype(np.float16)
    shift = rng.integers(-100, 100, size=16).astype(np.float16)
    km0 = oracle.k_mean(k)
    km1 = oracle.k_mean((k.astype(np.float32) + shift).astype(np.float16))
    assert np.array_equal(km1 - km0, np.broadcast_to(shift.astype(np.float32), km0.shape))


# ------------------------------------------------------------ quantizer

def _blocks(L, rows):
    return [(s, min(L, s + rows)) for s in range(0, L, rows)]


def test_quant_properties_random():
    q, k, v = inputs.make_custom(1, 2, 2, 300, 200, 64, seed=5, k_offset_sigma=4.0)
    sm = 1 / 8
    q_i8, k_i8, q_scale, k_scale, km = oracle.quant_qk(q, k, sm)
    c = np.float32(sm * math.log2(math.e))
    assert q_scale.shape == (1, 2, 3) and k_scale.shape == (1, 2, 4)
    for h in range(2):
        for bi, (s, e) in enumerate(_blocks(300, 128)):
            x = q[0, h, s:e].astype(np.float64)
            qq = q_i8[0, h, s:e].astype(np.int32)
            a = np.abs(x).max()
            assert np.abs(qq).max() == 127
            # round-to-nearest: |q - x*127/a| <= 1/2 (plus float32 slack)
            assert np.all(np.abs(qq - x * 127.0 / a) <= 0.5 + 1e-4)
            assert abs(q_scale[0, h, bi] / c - a / 127) <= 2e-7 * a
        kk = k[0, h].astype(np.float64) - km[0, h].astype(np.float64)
        for bi, (s, e) in enumerate(_blocks(200, 64)):
            x = kk[s:e]
            qq = k_i8[0, h, s:e].astype(np.int32)
            a = np.abs(x).max()
            assert np.abs(qq).max() == 127
            assert np.all(np.abs(qq - x * 127.0 / a) <= 0.5 + 1e-3)
            assert abs(k_scale[0, h, bi] - a / 127) <= 2e-7 * a


def test_quant_power_of_two_scaling_is_exact():
    q, k, v = inputs.make_custom(1, 2, 2, 256, 128, 64, seed=9)
    base = oracle.quant_qk(q, k, 0.125)
    for p in (1, 3):   # upward: no fp16 subnormal underflow
        q2 = (q.astype(np.float32) * 2.0 ** p).astype(np.float16)
        assert np.array_equal(q2.astype(np.float32), q.astype(np.float32) * 2.0 ** p)
        got = oracle.quant_qk(q2, k, 0.125)
        assert np.array_equal(got[0], base[0])
        assert np.array_equal(got[2], base[2] * np.float32(2.0 ** p))


def test_quant_blocks_are_independent():
    q, k, v = inputs.make_custom(1, 1, 1, 256, 128, 64, seed=4)
    base = oracle.quant_qk(q, k, 0.125)
    q2 = q.copy(); q2[0, 0, :128] *= np.float16(3)
    got = oracle.quant_qk(q2, k, 0.125)
    assert np.array_equal(got[0][0, 0, 128:], base[0][0, 0, 128:])
    assert got[2][0, 0, 1] == base[2][0, 0, 1]


@pytest.mark.parametrize("bq", [64, 32, 1])
def test_quant_properties_finer_q_blocks(bq):
    """Q blocks of bq rows obey the same per-block definition: the largest
    code of a non-zero block is 127, codes round x*127/amax to the nearest
    integer, and the scale is amax/127 times c; K does not depend on bq."""
    q, k, v = inputs.make_custom(1, 2, 2, 300, 200, 64, seed=5, k_offset_sigma=4.0)
    sm = 1 / 8
    q_i8, k_i8, q_scale, k_scale, km = oracle.quant_qk(q, k, sm, q_block_rows=bq)
    c = np.float32(sm * math.log2(math.e))
    assert q_scale.shape == (1, 2, -(-300 // bq))
    for h in range(2):
        for bi, (s, e) in enumerate(_blocks(300, bq)):
            x = q[0, h, s:e].astype(np.float64)
            qq = q_i8[0, h, s:e].astype(np.int32)
            a = np.abs(x).max()
            assert np.abs(qq).max() == 127
            assert np.all(np.abs(qq - x * 127.0 / a) <= 0.5 + 1e-4)
            assert abs(q_scale[0, h, bi] / c - a / 127) <= 2e-7 * a
    base = oracle.quant_qk(q, k, sm)
    for got, ref in zip((k_i8, k_scale, km), (base[1], base[3], base[4])):
        assert np.array_equal(got, ref)


def test_q_block_rows_one_is_per_token():
    """With one-row blocks, scaling one token by a power of two changes only
    that token's scale (its codes stay), and every other token is untouched;
    a 32-row block that contains it changes its codes elsewhere in the block."""
    q, k, v = inputs.make_custom(1, 1, 1, 96, 64, 64, seed=8)
    base = oracle.quant_qk(q, k, 0.125, q_block_rows=1)
    q2 = q.copy()
    q2[0, 0, 40] *= np.float16(4)
    got = oracle.quant_qk(q2, k, 0.125, q_block_rows=1)
    assert np.array_equal(got[0], base[0])
    assert got[2][0, 0, 40] == base[2][0, 0, 40] * np.float32(4)
    keep = np.arange(96) != 40
    assert np.array_equal(got[2][0, 0, keep], base[2][0, 0, keep])
    b32 = oracle.quant_qk(q, k, 0.125, q_block_rows=32)
    g32 = oracle.quant_qk(q2, k, 0.125, q_block_rows=32)
    assert not np.array_equal(g32[0][0, 0, 32:64], b32[0][0, 0, 32:64])
    assert np.array_equal(g32[0][0, 0, :32], b32[0][0, 0, :32])
    assert np.array_equal(g32[0][0, 0, 64:], b32[0][0, 0, 64:])
    # a single-token block is the whole tensor of that one token
    one = oracle.quant_qk(np.ascontiguousarray(q[:, :, 40:41]), k, 0.125)
    assert np.array_equal(one[0][0, 0, 0], base[0][0, 0, 40])
    assert one[2][0, 0, 0] == base[2][0, 0, 40]


def test_k_integer_shift_leaves_k_quant_unchanged():
    rng = np.random.default_rng(12)
    k = rng.integers(-30, 30, size=(1, 1, 128, 16)).astype(np.float16)
    shift = rng.integers(-50, 50, size=16).astype(np.float32)
    k2 = (k.astype(np.float32) + shift).astype(np.float16)
    q = np.ones((1, 1, 1, 16), dtype=np.float16)
    a = oracle.quant_qk(q, k, 0.125)
    b = oracle.quant_qk(q, k2, 0.125)
    assert np.array_equal(a[1], b[1]) and np.array_equal(a[3], b[3])


# --------------------------------------------------------- fp64 attention

def numpy_attention(q, k, v, causal, sm_scale):
    """Textbook attention with numpy matrix routines, float64."""
    q = q.astype(np.float64); k = k.astype(np.float64); v = v.astype(np.float64)
    B, H, Lq, d = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    g = H // Hkv
    out = np.zeros((B, H, Lq, d))
    for b in range(B):
        for h in range(H):
            s = q[b, h] @ k[b, h // g].T * sm_scale
            if causal:
                i = np.arange(Lq)[:, None]; j = np.arange(Lk)[None, :]
                s = np.where(j <= i + (Lk - Lq), s, -np.inf)
            for i in range(Lq):
                row = s[i]
                if np.all(np.isneginf(row)):
                    continue
                p = np.exp(row - row.max())
                out[b, h, i] = p @ v[b, h // g] / p.sum()
    return out


@pytest.mark.parametrize("shape,causal", [
    ((1, 2, 2, 37, 37, 16), False),
    ((2, 4, 2, 29, 41, 8), True),     # GQA, Lq < Lk, bottom-right causal
    ((1, 2, 1, 40, 23, 8), True),     # Lq > Lk: the first rows see no key
    ((1, 3, 3, 64, 64, 32), True),
])
def test_fp64_attention_matches_numpy(shape, causal):
    B, H, Hkv, Lq, Lk, d = shape
    q, k, v = inputs.make_custom(B, H, Hkv, Lq, Lk, d, seed=Lq + Lk)
    sm = 1 / math.sqrt(d)
    got = oracle.attn_fp64(q, k, v, causal, sm)
    ref = numpy_attention(q, k, v, causal, sm)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    rows = np.array([0, 5, B * H * Lq - 1], dtype=np.int64)
    got_rows = oracle.attn_fp64(q, k, v, causal, sm, rows=rows)
    np.testing.assert_allclose(got_rows, ref.reshape(-1, d)[rows], rtol=0, atol=1e-12)


def test_smoothing_identity_in_fp64():
    """softmax(QK^T) = softmax(Q(K - mean K)^T) for the token-axis mean only."""
    q, k, v = inputs.make_custom(1, 2, 2, 48, 48, 16, seed=21, k_offset_sigma=5.0)
    kk = k.astype(np.float64)
    qq = q.astype(np.float64)

    def probs(kmat):
        s = qq[0, 0] @ kmat.T
        p = np.exp(s - s.max(axis=1, keepdims=True))
        return p / p.sum(axis=1, keepdims=True)

    base = probs(kk[0, 0])
    tok = probs(kk[0, 0] - kk[0, 0].mean(axis=0, keepdims=True))
    chan = probs(kk[0, 0] - kk[0, 0].mean(axis=1, keepdims=True))
    assert np.max(np.abs(tok - base)) < 1e-12
    assert np.max(np.abs(chan - base)) > 1e-3


# ----------------------------------------------- quantized-path simulation

def _sim(q, k, v, causal, sm):
    out, qk = oracle.attention(q, k, v, causal, sm)
    return out, qk


def test_sim_exact_quantization_reduces_to_fp64_attention():
    """Integer Q and zero-mean integer K whose block maxima are 127 quantize
    without error (scales exactly 1), so the simulation must equal fp64
    softmax(sm_scale QK^T)V up to the fp16 rounding of P: this pins the
    dequantization product, the log2(e) fold and the base-2 softmax."""
    rng = np.random.default_rng(31)
    B, H, L, d = 1, 2, 256, 64
    q = rng.integers(-3, 4, size=(B, H, L, d)).astype(np.float64)
    q[:, :, ::128, 0] = 127                       # every 128-row block has max 127
    half = rng.integers(-8, 9, size=(B, H, L // 2, d)).astype(np.float64)
    half[:, :, ::32, 1] = 127                     # every 64-row K block has max 127
    k = np.empty((B, H, L, d))
    k[:, :, 0::2] = half
    k[:, :, 1::2] = -half                         # per-channel token mean is exactly 0
    v = rng.standard_normal((B, H, L, d))
    q, k, v = (t.astype(np.float16) for t in (q, k, v))
    sm = 1 / 512
    out, (q_i8, k_i8, qs, ks, km) = _sim(q, k, v, True, sm)
    assert np.all(km == 0) and np.all(ks == 1)
    assert np.array_equal(q_i8.astype(np.float16), q)
    ref = numpy_attention(q, k, v, True, float(np.float32(sm)))
    # fp16 rounding of p: relative error 2^-11 per weight
    assert np.max(np.abs(out - ref)) < 2.0 ** -10 * np.abs(v.astype(np.float64)).max()
    # and it is not the natural-exponent softmax (log2 e fold present)
    wrong = numpy_attention(q, k, v, True, float(np.float32(sm)) / math.log(2))
    assert np.max(np.abs(out - wrong)) > 1e-2


def test_sim_per_token_scales_are_exact_where_tile_scales_are_not():
    """Q rows that are 127-bounded integer vectors times a per-row power of
    two quantize without error at one scale per token, so the simulation
    then equals fp64 attention up to the fp16 rounding of P; one scale per
    128-row tile rounds the small rows coarsely and misses that bound.  This
    pins the row -> scale index of the simulation for every block height."""
    rng = np.random.default_rng(77)
    B, H, L, d = 1, 1, 256, 64
    q = rng.integers(-127, 128, size=(B, H, L, d)).astype(np.float64)
    q[..., 0] = 127
    q *= 2.0 ** rng.integers(-6, 1, size=(B, H, L, 1))
    half = rng.integers(-8, 9, size=(B, H, L // 2, d)).astype(np.float64)
    half[:, :, ::32, 1] = 127
    k = np.empty((B, H, L, d))
    k[:, :, 0::2] = half
    k[:, :, 1::2] = -half
    v = rng.standard_normal((B, H, L, d))
    q, k, v = (t.astype(np.float16) for t in (q, k, v))
    sm = 1 / 512
    ref = numpy_attention(q, k, v, False, float(np.float32(sm)))
    bound = 2.0 ** -10 * np.abs(v.astype(np.float64)).max()
    qk1 = oracle.quant_qk(q, k, sm, q_block_rows=1)
    assert np.array_equal(qk1[0].astype(np.float64) * (qk1[2][..., None] /
                          np.float32(sm * math.log2(math.e))).astype(np.float64),
                          q.astype(np.float64))
    out1 = oracle.attn_quant_sim(qk1[0], qk1[1], qk1[2], qk1[3], v, False, q_block_rows=1)
    assert np.max(np.abs(out1 - ref)) < bound
    qk128 = oracle.quant_qk(q, k, sm)
    out128 = oracle.attn_quant_sim(qk128[0], qk128[1], qk128[2], qk128[3], v, False)
    assert np.max(np.abs(out128 - ref)) > 4 * bound
    # reading the per-token scales as if they were per-tile ones is wrong
    wrong = oracle.attn_quant_sim(qk1[0], qk1[1], qk1[2][..., :2].copy(), qk1[3], v, False)
    assert np.max(np.abs(wrong - ref)) > 4 * bound


@pytest.mark.parametrize("causal", [False, True])
def test_sim_closed_forms(causal):
    B, H, L, d = 1, 2, 200, 64
    q, k, v = inputs.make_custom(B, H, H, L, L, d, seed=41)
    sm = 1 / 8
    # (a) V constant along tokens -> O equals that constant row
    vc = np.broadcast_to(v[:, :, :1], v.shape).copy()
    out, _ = _sim(q, k, vc, causal, sm)
    np.testing.assert_allclose(out, np.broadcast_to(vc[:, :, :1].astype(np.float64), out.shape),
                               rtol=0, atol=1e-12)
    # (b) all K rows equal -> smoothed K = 0 -> uniform weights over visible keys
    ke = np.broadcast_to(k[:, :, :1], k.shape).copy()
    out, (q_i8, k_i8, qs, ks, km) = _sim(q, ke, v, causal, sm)
    assert np.all(k_i8 == 0) and np.all(ks == 0)
    vv = v.astype(np.float64)
    if causal:
        ref = np.cumsum(vv, axis=2) / np.arange(1, L + 1)[None, None, :, None]
    else:
        ref = np.broadcast_to(vv.mean(axis=2, keepdims=True), vv.shape)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    # (c) causal row 0 sees only key 0
    out, _ = _sim(q, k, v, True, sm)
    np.testing.assert_array_equal(out[:, :, 0], v[:, :, 0].astype(np.float64))
    # (d) Lk = 1 -> O = v0 for every row that sees key 0; with bottom-right
    # causal alignment only the last query row does, the others output 0
    out, _ = _sim(q, k[:, :, :1], v[:, :, :1], causal, sm)
    ref = np.broadcast_to(v[:, :, :1].astype(np.float64), out.shape).copy()
    if causal:
        ref[:, :, :-1] = 0.0
    np.testing.assert_array_equal(out, ref)


@pytest.mark.parametrize("Lq,Lk", [(40, 100), (100, 40), (64, 64), (1, 70)])
def test_sim_bottom_right_alignment_closed_form(Lq, Lk):
    """All K rows equal: smoothed K is 0, every visible key gets the same
    weight, so causal row i is the mean of the first
    n_i = clamp(i + Lk - Lq + 1, 0, Lk) value rows (0 when n_i = 0), and a
    non-causal row is the mean of all Lk.  An off-by-one in the mask's
    alignment, or aligning at the top-left, changes n_i."""
    B, H, d = 1, 2, 32
    q, k, v = inputs.make_custom(B, H, H, Lq, Lk, d, seed=Lq * 7 + Lk)
    ke = np.broadcast_to(k[:, :, :1], k.shape).copy()
    vv = v.astype(np.float64)
    csum = np.concatenate([np.zeros((B, H, 1, d)), np.cumsum(vv, axis=2)], axis=2)
    out, _ = _sim(q, ke, v, True, 0.125)
    n = np.clip(np.arange(Lq) + Lk - Lq + 1, 0, Lk)
    ref = np.zeros((B, H, Lq, d))
    for i in range(Lq):
        if n[i] > 0:
            ref[:, :, i] = csum[:, :, n[i]] / n[i]
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    out, _ = _sim(q, ke, v, False, 0.125)
    np.testing.assert_allclose(out, np.broadcast_to(csum[:, :, Lk:] / Lk, out.shape),
                               rtol=0, atol=1e-12)


def _two_key_row(d=16):
    """One query row, two keys: int8 scores S = (0, -1) with q_scale
    fl32(1/3) and k_scale 1, so the base-2 scores are s = (0, -fl32(1/3))
    and the row max is 0.  V rows: v0 = 0, v1 = 1 in every channel."""
    q_i8 = np.zeros((1, 1, 1, d), np.int8); q_i8[..., 0] = 1
    k_i8 = np.zeros((1, 1, 2, d), np.int8); k_i8[0, 0, 1, 0] = -1
    q_scale = np.array([[[1 / 3]]], np.float32)
    k_scale = np.ones((1, 1, 1), np.float32)
    v = np.zeros((1, 1, 2, d), np.float16); v[0, 0, 1] = 1
    s1 = -float(np.float32(1 / 3))
    return q_i8, k_i8, q_scale, k_scale, v, s1


def test_sim_rounds_p_to_fp16():
    """P is held in fp16 (the FP16 P V step): with p1 = 2^s1 not an fp16
    value, the output is p1h / (1 + p1h) with p1h = fp16(p1), computed here
    with numpy's exp2 and float16 cast; the unrounded p1 moves it by ~1e-4."""
    q_i8, k_i8, qs, ks, v, s1 = _two_key_row()
    out = oracle.attn_quant_sim(q_i8, k_i8, qs, ks, v, False)
    p1 = np.exp2(np.float64(s1))
    p1h = float(np.float16(p1))
    assert p1h != p1
    np.testing.assert_allclose(out, np.full(out.shape, p1h / (1 + p1h)), rtol=0, atol=1e-15)
    assert abs(p1h / (1 + p1h) - p1 / (1 + p1)) > 1e-6


def test_fp8pv_sim_rounds_p_to_e4m3():
    """FP8 path: P = e4m3(fl32(fl32(p) * 448)) / 448 (torch's float8_e4m3fn
    conversion here), V = 1 is exact in E4M3 at scale 1/448, and the row sum
    takes the unquantized p: out = P1 / (1 + p1)."""
    import torch
    q_i8, k_i8, qs, ks, v, s1 = _two_key_row()
    v8t, vs = oracle.quant_v_fp8(v)
    out = oracle.attn_fp8pv_sim(q_i8, k_i8, qs, ks, v8t, vs, False)
    p1 = np.exp2(np.float64(s1))
    x = np.float32(np.float32(p1) * np.float32(448.0))
    p8 = float(torch.tensor([float(x)]).to(torch.float8_e4m3fn).float()[0]) / 448.0
    assert p8 != p1
    deq_v1 = float(torch.tensor([v8t[0, 0, 0, 1]], dtype=torch.uint8).view(
        torch.float8_e4m3fn).float()[0]) * float(vs[0, 0, 0])
    np.testing.assert_allclose(out, np.full(out.shape, p8 * deq_v1 / (1 + p1)), rtol=1e-15,
                               atol=0)


def test_sim_kv_block_permutation_invariance():
    q, k, v = inputs.make_custom(1, 1, 1, 64, 256, 64, seed=51)
    perm = np.array([2, 0, 3, 1])
    idx = (perm[:, None] * 64 + np.arange(64)[None, :]).ravel()
    out0, qk0 = _sim(q, k, v, False, 0.125)
    out1, qk1 = _sim(q, k[:, :, idx], v[:, :, idx], False, 0.125)
    assert np.array_equal(qk1[1], qk0[1][:, :, idx])
    assert np.array_equal(qk1[3], qk0[3][:, :, perm])
    np.testing.assert_allclose(out1, out0, rtol=0, atol=1e-12)


def test_sim_gqa_equals_repeated_kv():
    q, k, v = inputs.make_custom(2, 4, 2, 80, 96, 64, seed=61)
    out_g, _ = _sim(q, k, v, True, 0.125)
    k_rep = np.repeat(k, 2, axis=1)
    v_rep = np.repeat(v, 2, axis=1)
    out_r, _ = _sim(q, k_rep, v_rep, True, 0.125)
    np.testing.assert_array_equal(out_g, out_r)


def test_sim_row_subset_matches_full():
    q, k, v = inputs.make_custom(1, 2, 1, 150, 150, 64, seed=71)
    qk = oracle.quant_qk(q, k, 0.125)
    full = oracle.attn_quant_sim(*qk[:4], v, True)
    rows = np.array([0, 1, 127, 128, 149, 150, 299], dtype=np.int64)
    sub = oracle.attn_quant_sim(*qk[:4], v, True, rows=rows)
    np.testing.assert_array_equal(sub, full.reshape(-1, 64)[rows])


def test_sim_accuracy_and_smoothing_ablation():
    """Channel-outlier K (the article's motivation for smoothing): with
    smoothing the quantized path stays close to fp64 attention; without it,
    it is measurably worse."""
    w = inputs.WORKLOADS[1]
    q, k, v = inputs.make_inputs(w)
    sm = float(np.float32(w.sm_scale))
    ref = oracle.attn_fp64(q, k, v, w.causal, sm)
    out, _ = _sim(q, k, v, w.causal, sm)

    def cos(a, b):
        a = a.ravel(); b = b.ravel()
        return float(a @ b / np.linalg.norm(a) / np.linalg.norm(b))

    c_s = cos(out, ref)
    qk = oracle.quant_qk(q, k, sm, smooth=False)
    out_ns = oracle.attn_quant_sim(*qk[:4], v, w.causal)
    c_ns = cos(out_ns, ref)
    assert c_s >= 0.9999
    assert c_ns < c_s


def test_inputs_are_seeded_and_shaped():
    w = inputs.WORKLOADS[1]
    a = inputs.make_inputs(w)
    b = inputs.make_inputs(w)
    for x, y in zip(a, b):
        assert x.dtype == np.float16 and np.array_equal(x, y)
    assert a[0].shape == (1, 2, 256, 64) and a[1].shape == (1, 2, 256, 64)
    # the K offset is a per-channel constant: the token mean of K is far from 0
    assert np.abs(a[1].astype(np.float64).mean(axis=2)).max() > 1.0
    assert inputs.visible_pairs(1, 1, 4, 4, True) == 10
    assert inputs.visible_pairs(1, 1, 2, 4, True) == 7      # bottom-right: rows see 3, 4
    assert inputs.visible_pairs(1, 1, 4, 2, True) == 3      # rows see 0, 0, 1, 2


# ------------------------------------------------------ FP8 (E4M3) P V

def _torch_e4m3(values):
    import torch
    t = torch.tensor(np.asarray(values, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_decode_matches_torch_all_codes():
    import torch
    codes = [c for c in range(256) if c not in (0x7F, 0xFF)]     # the two NaN codes
    want = torch.tensor(codes, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    got = np.array([oracle.e4m3_decode(c) for c in codes])
    assert np.array_equal(got, want.astype(np.float64))


def test_e4m3_encode_matches_torch_rne_and_saturates():
    """Round to nearest even against torch's float8_e4m3fn conversion on every
    finite code, the midpoints between neighbouring codes (ties), points just
    off the midpoints and random magnitudes; values above 448 saturate."""
    import torch
    finite = np.array(sorted({oracle.e4m3_decode(c) for c in range(0x7F)}))   # 0 .. 448
    mids = (finite[:-1] + finite[1:]) / 2
    off = np.concatenate([mids * (1 + 2.0 ** -20), mids * (1 - 2.0 ** -20)])
    rng = np.random.default_rng(3)
    rand = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(448.0), size=4000))
    xs = np.concatenate([finite, mids, off, rand]).astype(np.float32)
    xs = np.concatenate([xs, -xs])
    got = np.array([oracle.e4m3_encode(float(x)) for x in xs], dtype=np.uint8)
    assert np.array_equal(got, _torch_e4m3(xs))
    for big in (448.01, 464.0, 1e6):
        assert oracle.e4m3_encode(big) == 0x7E and oracle.e4m3_encode(-big) == 0xFE


def test_quant_v_fp8_properties():
    rng = np.random.default_rng(8)
    v = (rng.standard_normal((1, 2, 300, 64)) * 3).astype(np.float16)
    v[0, 1, :, 5] = 0                                  # an all-zero channel
    v8t, vs = oracle.quant_v_fp8(v)
    assert v8t.shape == (1, 2, 64, 300) and vs.shape == (1, 2, 64)
    dec = np.vectorize(oracle.e4m3_decode)(v8t)       # [B, Hkv, d, Lk]
    vt = np.swapaxes(v.astype(np.float64), 2, 3)      # [B, Hkv, d, Lk]
    amax = np.abs(vt).max(axis=3)
    assert vs[0, 1, 5] == 0 and np.all(v8t[0, 1, 5] == 0)
    nz = amax > 0
    assert np.all(np.abs(dec).max(axis=3)[nz] == 448.0)
    assert np.allclose(vs[nz], (amax / 448)[nz], rtol=2 ** -23)
    # E4M3 keeps 3 mantissa bits: within half a unit in the last place of the
    # scaled value (relative 2^-4 for normals, 2^-10 absolute below 2^-6)
    scaled = vt * (448.0 / np.where(nz, amax, 1.0))[..., None]
    err = np.abs(dec - scaled)
    assert np.all(err <= np.maximum(np.abs(scaled) * 2.0 ** -4, 2.0 ** -10) * (1 + 1e-6))


def test_fp8pv_sim_closed_forms():
    """Equal scores give p = 1 for every visible key, which E4M3 holds
    exactly (448), so the FP8 path returns the plain mean of the dequantized
    V rows; causal row 0 returns the dequantized V row 0."""
    B, H, L, d = 1, 2, 200, 64
    q, k, v = inputs.make_custom(B, H, H, L, L, d, seed=44)
    ke = np.broadcast_to(k[:, :, :1], k.shape).copy()
    sm = 1 / 8
    qk = oracle.quant_qk(q, ke, sm)
    v8t, vs = oracle.quant_v_fp8(v)
    deq = np.swapaxes(np.vectorize(oracle.e4m3_decode)(v8t), 2, 3) * vs[:, :, None, :]
    out = oracle.attn_fp8pv_sim(*qk[:4], v8t, vs, True)
    exp = np.cumsum(deq, axis=2) / np.arange(1, L + 1)[None, None, :, None]
    assert np.allclose(out, exp, rtol=1e-12, atol=1e-12)
    out_nc = oracle.attn_fp8pv_sim(*qk[:4], v8t, vs, False)
    assert np.allclose(out_nc, np.broadcast_to(deq.mean(axis=2, keepdims=True), out_nc.shape),
                       rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("Lq,Lk", [(40, 100), (100, 40)])
def test_fp8pv_sim_bottom_right_alignment_closed_form(Lq, Lk):
    """The FP8 simulation's own causal mask, for Lq != Lk: with equal
    scores (P = 1 exactly in E4M3), row i is the mean of the first
    clamp(i + Lk - Lq + 1, 0, Lk) dequantized V rows, 0 when there are none."""
    B, H, d = 1, 2, 64
    q, k, v = inputs.make_custom(B, H, H, Lq, Lk, d, seed=Lq + 3 * Lk)
    ke = np.broadcast_to(k[:, :, :1], k.shape).copy()
    qk = oracle.quant_qk(q, ke, 0.125)
    v8t, vs = oracle.quant_v_fp8(v)
    deq = np.swapaxes(np.vectorize(oracle.e4m3_decode)(v8t), 2, 3)[:, :, :Lk] * vs[:, :, None, :]
    csum = np.concatenate([np.zeros((B, H, 1, d)), np.cumsum(deq, axis=2)], axis=2)
    out = oracle.attn_fp8pv_sim(*qk[:4], v8t, vs, True)
    n = np.clip(np.arange(Lq) + Lk - Lq + 1, 0, Lk)
    ref = np.zeros((B, H, Lq, d))
    for i in range(Lq):
        if n[i] > 0:
            ref[:, :, i] = csum[:, :, n[i]] / n[i]
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_fp8pv_sim_tracks_the_fp16_path_and_gqa():
    q, k, v = inputs.make_custom(1, 4, 2, 256, 256, 64, seed=45)
    sm = 1 / 8
    qk = oracle.quant_qk(q, k, sm)
    v8t, vs = oracle.quant_v_fp8(v)
    f8 = oracle.attn_fp8pv_sim(*qk[:4], v8t, vs, True)
    f16 = oracle.attn_quant_sim(*qk[:4], v, True)
    a, b = f8.ravel(), f16.ravel()
    assert a @ b / np.linalg.norm(a) / np.linalg.norm(b) > 0.999
    assert not np.allclose(f8, f16)            # the FP8 rounding is really applied
    # GQA: the same as repeating each kv head for its query heads
    rep = lambda t: np.repeat(t, 2, axis=1)
    qk2 = (qk[0], rep(qk[1]), qk[2], rep(qk[3]))
    v8t2, vs2 = oracle.quant_v_fp8(rep(v))
    assert np.array_equal(oracle.attn_fp8pv_sim(*qk2, v8t2, vs2, True), f8)
