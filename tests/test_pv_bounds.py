"""CPU checks that the FP8 and fp16-sum error bounds of the GPU tests
(pv_bounds.py) have teeth: an output that differs from the oracle's
simulation only by in-bound noise passes, and the same output with one
planted row-index error fails.  Everything here is the oracle on the CPU; the
"kernel output" is the simulation doctored on purpose."""
import math

import numpy as np
import pytest

import oracle
import pv_bounds
from bit_quantized_attention_mean_b200 import inputs

B, H, Hkv, L, D = 1, 4, 2, 384, 64


@pytest.fixture(scope="module")
def problem():
    q, k, v = inputs.make_custom(B, H, Hkv, L, L, D, seed=404, k_offset_sigma=2.0)
    # sharpen the scores so that many rows are dominated by a few keys, as in
    # the long-context workload
    q = (q.astype(np.float32) * 3).astype(np.float16)
    sm = float(np.float32(1 / math.sqrt(D)))
    return q, k, v, oracle.quant_qk(q, k, sm)


def planted(out, absatt, sim):
    """Row r (among rows with at least 64 visible keys, the one whose output
    is largest against its absolute attention) receives the output of the
    same position in a head of the other kv group: a wrong head index for
    one row."""
    bad = out.copy()
    ratio = np.linalg.norm(sim, axis=-1) / np.linalg.norm(absatt, axis=-1)
    ratio[np.arange(B * H * L) % L < 63] = 0
    r = int(np.argmax(ratio))
    other = (r + (H // Hkv) * L) % (B * H * L)
    bad[r] = out[other]
    return bad, r


def test_fp8_bound_passes_noise_and_catches_a_planted_row(problem):
    q, k, v, qk = problem
    v8t, vs = oracle.quant_v_fp8(v)
    sim = oracle.attn_fp8pv_sim(*qk[:4], v8t, vs, True).reshape(-1, D)
    absatt = oracle.attn_fp8pv_sim(*qk[:4], v8t & 0x7F, vs, True).reshape(-1, D)
    rng = np.random.default_rng(1)
    # in-bound stand-in for the kernel: every element moved by up to 2^-4 of
    # its absolute attention, then rounded to fp16
    noisy = (sim + rng.uniform(-1, 1, sim.shape) * 2.0 ** -4 * absatt)
    noisy = noisy.astype(np.float16).astype(np.float64)
    elem, row = pv_bounds.fp8_excess(noisy, sim, absatt)
    pv_bounds.assert_within(elem, row, "in-bound noise")
    bad, r = planted(noisy, absatt, sim)
    elem, row = pv_bounds.fp8_excess(bad, sim, absatt)
    assert elem[r].max() > 0 and np.all(np.delete(elem, r, axis=0) <= 0)
    with pytest.raises(AssertionError):
        pv_bounds.assert_within(elem, row, "planted row")


def test_f16acc_bound_passes_noise_and_catches_a_planted_row(problem):
    q, k, v, qk = problem
    sim = oracle.attn_quant_sim(*qk[:4], v, True).reshape(-1, D)
    absatt = oracle.attn_quant_sim(*qk[:4], np.abs(v), True).reshape(-1, D)
    keys = pv_bounds.visible_keys(np.arange(B * H * L) % L, L, L, True)
    rng = np.random.default_rng(2)
    # in-bound stand-in: a random walk of fp16 roundings per 16-key step
    steps = np.ceil(keys / 16.0)[:, None]
    walk = rng.standard_normal(sim.shape) * np.sqrt(steps / 12.0) * pv_bounds.U16 * absatt
    noisy = (sim + walk).astype(np.float16).astype(np.float64)
    elem, row = pv_bounds.f16acc_excess(noisy, sim, absatt, keys)
    pv_bounds.assert_within(elem, row, "in-bound noise")
    bad, r = planted(noisy, absatt, sim)
    elem, row = pv_bounds.f16acc_excess(bad, sim, absatt, keys)
    assert row[r] > 0 and np.all(np.delete(row, r) <= 0)
    with pytest.raises(AssertionError):
        pv_bounds.assert_within(elem, row, "planted row")
