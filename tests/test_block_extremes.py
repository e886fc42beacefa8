"""The shortcut behind the d = 64 quantization kernel's K scales, checked on
the CPU against the oracle (no GPU needed).

The SageAttention article's per-block INT8 step quantizes the smoothed key
fl32(K - m) with one scale per 64-row block, a = max |fl32(K - m)| over the
block.  fl32 rounding is monotonic, so within one channel c the largest
|fl32(k - m_c)| is taken at that channel's smallest or largest k.  The kernel
therefore keeps only each block's per-channel fp16 minimum and maximum from
its mean pass and forms a = max_c max(|fl32(max_c - m_c)|, |fl32(min_c -
m_c)|) once the mean is known.  These tests form the same quantities in numpy
float32 and require the oracle's block scales bit for bit, on inputs built to
stress the argument: large channel offsets, ragged last blocks, channels
whose extremes sit at equal distance from the mean, constant channels and
all-zero blocks.
"""
import numpy as np
import pytest

import oracle
from bit_quantized_attention_mean_b200 import inputs


def scales_from_extremes(k, mean):
    """k: fp16 [B, Hkv, Lk, d]; mean: float32 [B, Hkv, d] -> float32 block
    scales [B, Hkv, ceil(Lk / 64)] from per-channel extremes alone."""
    B, Hkv, Lk, d = k.shape
    nkb = -(-Lk // 64)
    out = np.empty((B, Hkv, nkb), dtype=np.float32)
    kf = k.astype(np.float32)
    for b in range(B):
        for h in range(Hkv):
            for j in range(nkb):
                blk = kf[b, h, 64 * j:min(Lk, 64 * j + 64)]
                hi = (blk.max(axis=0) - mean[b, h]).astype(np.float32)
                lo = (blk.min(axis=0) - mean[b, h]).astype(np.float32)
                a = np.float32(max(np.abs(hi).max(), np.abs(lo).max()))
                out[b, h, j] = a / np.float32(127.0) if a > 0 else np.float32(0.0)
    return out


def check(k):
    q = np.zeros((k.shape[0], k.shape[1], 1, k.shape[3]), dtype=np.float16)
    want = oracle.quant_qk(q, k, 0.125)
    got = scales_from_extremes(k, want[4])
    assert np.array_equal(got.view(np.uint32), want[3].view(np.uint32))


@pytest.mark.parametrize("shape", [(1, 2, 1000, 64), (2, 1, 64, 64), (1, 1, 130, 128),
                                   (1, 3, 1, 64)])
def test_extremes_give_the_oracle_block_scales(shape):
    B, Hkv, Lk, d = shape
    _, k, _ = inputs.make_custom(B, Hkv, Hkv, 1, Lk, d, seed=Lk + d, k_offset_sigma=40.0)
    check(k)


def test_extremes_with_equidistant_constant_and_zero_channels():
    rng = np.random.default_rng(7)
    Lk, d = 200, 64
    k = rng.standard_normal((1, 1, Lk, d)).astype(np.float32)
    # channel 0: values +-3 only, so max and min are equally far from a zero mean
    k[0, 0, :, 0] = np.where(np.arange(Lk) % 2 == 0, 3.0, -3.0)
    # channel 1 constant: k - m is 0 in every row
    k[0, 0, :, 1] = 5.5
    # channel 2: one large outlier in the ragged last block
    k[0, 0, :, 2] = 0.25
    k[0, 0, Lk - 1, 2] = 900.0
    check(k.astype(np.float16))
    # an all-zero block among nonzero ones
    z = k.copy()
    z[0, 0, 64:128, :] = 0.0
    check(z.astype(np.float16))
