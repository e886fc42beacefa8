"""Error bounds of the two P V variants whose rounding differs from the
oracle's simulation: P and V in FP8 E4M3, and fp16 P V sums.  Both bounds
are per row and per channel, and scale with that row's own absolute
attention A_ic = sum_j p_ij |v_jc| / l_i (the simulation run on |V|), not with
max |V| over the whole problem.

FP8 (E4M3) P.  The kernel rounds 1.75 p against its running max, the oracle
448 p against the exact row max; each rounding moves P by at most half an
E4M3 unit (relative 2^-4), the V codes are identical (bit-exact) and the row
sums use the unquantized p on both sides, so an element moves by at most
2^-3 A_ic.  (No tighter row-level bound holds: when the running max lags the
row max, even the dominant key's P is rounded, by up to 2^-4.)

fp16 sums.  The accumulator is rounded to fp16 (u = 2^-11) after each
16-key tensor-core step and at each rescale, and each partial sum is at most
A_ic (normalized), so an element moves by at most (steps + rescales) u A_ic
with steps = ceil(visible keys / 16).  Independent roundings add like a
random walk, so a row's 2-norm error stays within 4 sqrt(steps / 12) u |A_i|.

Both add h_ic, half an fp16 spacing of the reference (the kernel's output is
fp16), and a 1e-3 allowance for fp32 summation order and E4M3 subnormals.
"""
import numpy as np

U16 = 2.0 ** -11
E4M3_HALF_UNIT = 2.0 ** -4
SLACK = 1e-3
RESCALES = 8


def half_ulp16(ref):
    return 0.5 * np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64)


def fp8_excess(out, ref, absatt):
    """Per-element excess over the FP8 bound (<= 0 everywhere means within
    it), and a row excess that is the element bound's (no separate row
    bound).  out, ref, absatt: [rows, d]."""
    out = np.asarray(out, np.float64)
    err = np.abs(out - ref)
    h = half_ulp16(ref) + SLACK
    elem = err - (2 * E4M3_HALF_UNIT * absatt + h)
    return elem, elem.max(axis=-1)


def f16acc_excess(out, ref, absatt, keys):
    """Same for fp16 sums; keys[i] = visible keys of row i."""
    out = np.asarray(out, np.float64)
    steps = (np.ceil(np.asarray(keys, np.float64) / 16.0) + RESCALES)[:, None]
    err = np.abs(out - ref)
    h = half_ulp16(ref) + SLACK
    elem = err - (steps * U16 * absatt + h)
    row = (np.linalg.norm(out - ref, axis=-1)
           - (4.0 * np.sqrt(steps[:, 0] / 12.0) * U16 * np.linalg.norm(absatt, axis=-1)
              + np.linalg.norm(h, axis=-1)))
    return elem, row


def assert_within(elem, row, what):
    i = np.unravel_index(np.argmax(elem), elem.shape)
    assert elem.max() <= 0, f"{what}: element {i} exceeds its bound by {elem.max():.3e}"
    r = int(np.argmax(row))
    assert row.max() <= 0, f"{what}: row {r} exceeds its bound by {row.max():.3e}"


def visible_keys(rows_in_head, Lq, Lk, causal):
    rows_in_head = np.asarray(rows_in_head, np.int64)
    if not causal:
        return np.full(rows_in_head.shape, Lk, np.int64)
    return np.clip(rows_in_head + (Lk - Lq) + 1, 0, Lk)
