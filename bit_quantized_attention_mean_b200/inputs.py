"""Seeded synthetic workloads for 8-bit quantized attention.

This module only draws random numbers and casts them to fp16; it holds none of
the attention or quantization arithmetic.  Both the CUDA path and the CPU
oracle are fed from here, so that they see byte-identical inputs.

The SageAttention article (method section, K smoothing step: channel-wise
outliers in K for image/video models) motivates the per-channel K offsets below; the five
shapes stand in for the text (LLM, GQA, long-context) and video-diffusion
workloads the articles talk about.  No public dataset is used.

Recipe (fixed so that any run can regenerate the same bytes):
  * ``numpy.random.default_rng(seed)``, seed = the workload's index 1..5.
  * Draw order: Q, K, V (float32), then the K offset terms.
  * ``N(0, v)`` is read as variance v, so ``N(0, 4)`` has sigma 2.
  * The K offset is one length-d vector shared by every batch, head and token,
    added in float32 before the final cast.
  * Final cast float32 -> fp16 with round-to-nearest-even.  The long-context
    workload first rounds float32 -> bf16 (RNE), then bf16 -> fp16.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    index: int
    name: str
    B: int
    H: int
    Hkv: int
    L: int
    d: int
    causal: bool
    k_offset_sigma: float
    outlier_channels: int = 0
    outlier_magnitude: float = 0.0
    v_scale: float = 1.0
    student_t: bool = False
    # Q quantization block rows this workload is run with: the 128-row tile,
    # or one row per block where 128-row blocks miss the fp64 accuracy gate
    q_block_rows: int = 128

    @property
    def Lq(self) -> int:
        return self.L

    @property
    def Lk(self) -> int:
        return self.L

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def pairs(self) -> int:
        """Number of unmasked (query, key) pairs summed over B*H."""
        return visible_pairs(self.B, self.H, self.Lq, self.Lk, self.causal)

    def describe(self) -> dict:
        return {
            "workload": self.name,
            "B": self.B, "H": self.H, "Hkv": self.Hkv, "Lq": self.Lq,
            "Lk": self.Lk, "d": self.d, "causal": self.causal,
        }

    def visible_keys(self, rows: "np.ndarray") -> "np.ndarray":
        """Keys visible to each of the given within-head row indices."""
        rows = np.asarray(rows, dtype=np.int64)
        if not self.causal:
            return np.full(rows.shape, self.Lk, dtype=np.int64)
        return np.clip(rows + (self.Lk - self.Lq) + 1, 0, self.Lk)


def visible_pairs(B: int, H: int, Lq: int, Lk: int, causal: bool) -> int:
    """Count of (i, j) with key j visible to query i (bottom-right causal)."""
    if not causal:
        return B * H * Lq * Lk
    off = Lk - Lq
    total = 0
    # rows i with i + off + 1 keys visible, clipped to [0, Lk]
    for i in range(Lq):
        total += min(Lk, max(0, i + off + 1))
    return B * H * total


WORKLOADS = {
    1: Workload(1, "tiny-noncausal-B1H2L256d64", 1, 2, 2, 256, 64, False, 2.0),
    2: Workload(2, "llm-causal-B1H32L4096d128", 1, 32, 32, 4096, 128, True, 1.0,
                outlier_channels=4, outlier_magnitude=20.0),
    3: Workload(3, "video-noncausal-B2H24L16384d64", 2, 24, 24, 16384, 64, False, 5.0,
                v_scale=4.0),
    4: Workload(4, "gqa-causal-B4H32Hkv8L8192d128", 4, 32, 8, 8192, 128, True, 2.0),
    5: Workload(5, "longctx-causal-B1H16L32768d128-t4", 1, 16, 16, 32768, 128, True, 3.0,
                student_t=True, q_block_rows=1),
}


def _round_f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 (round to nearest even), returned as float32."""
    u = x.astype(np.float32).view(np.uint32).astype(np.uint64)
    bias = 0x7FFF + ((u >> 16) & 1)
    u = ((u + bias) & 0xFFFF0000).astype(np.uint32)
    return u.view(np.float32)


def _draw(rng: np.random.Generator, shape, student_t: bool) -> np.ndarray:
    if student_t:
        # Student-t with 4 dof has variance 4/(4-2) = 2; divide by sqrt(2).
        return (rng.standard_t(4, size=shape) / math.sqrt(2.0)).astype(np.float32)
    return rng.standard_normal(size=shape, dtype=np.float32)


def make_inputs(w: Workload, seed: int | None = None):
    """Return (q, k, v) as contiguous fp16 numpy arrays in [B, heads, L, d]."""
    rng = np.random.default_rng(w.index if seed is None else seed)
    q = _draw(rng, (w.B, w.H, w.Lq, w.d), w.student_t)
    k = _draw(rng, (w.B, w.Hkv, w.Lk, w.d), w.student_t)
    v = _draw(rng, (w.B, w.Hkv, w.Lk, w.d), w.student_t)
    offset = (rng.standard_normal(size=(w.d,), dtype=np.float32)
              * np.float32(w.k_offset_sigma))
    if w.outlier_channels:
        chans = rng.permutation(w.d)[: w.outlier_channels]
        signs = rng.choice(np.array([-1.0, 1.0], dtype=np.float32), size=w.outlier_channels)
        offset[chans] += signs * np.float32(w.outlier_magnitude)
    k += offset[None, None, None, :]
    if w.v_scale != 1.0:
        v *= np.float32(w.v_scale)
    out = []
    for t in (q, k, v):
        if w.student_t:
            t = _round_f32_to_bf16(t)
        out.append(np.ascontiguousarray(t.astype(np.float16)))
    return tuple(out)


def make_custom(B, H, Hkv, Lq, Lk, d, seed, k_offset_sigma=2.0, v_scale=1.0):
    """Small seeded problem of arbitrary shape for edge-case tests."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal(size=(B, H, Lq, d), dtype=np.float32)
    k = rng.standard_normal(size=(B, Hkv, Lk, d), dtype=np.float32)
    v = rng.standard_normal(size=(B, Hkv, Lk, d), dtype=np.float32) * np.float32(v_scale)
    k += (rng.standard_normal(size=(d,), dtype=np.float32)
          * np.float32(k_offset_sigma))[None, None, None, :]
    return tuple(np.ascontiguousarray(t.astype(np.float16)) for t in (q, k, v))


def sample_rows(w_B: int, w_H: int, Lq: int, n: int, seed: int, block: int = 128):
    """Seeded sample of flat row indices ((b*H + h)*Lq + i) over every (b, h).

    Always includes the first and last row and the rows on both sides of each
    128-row boundary of one head, plus ``n`` uniform random rows.
    """
    rng = np.random.default_rng(1000 + seed)
    rows = set()
    for bh in range(w_B * w_H):
        for i in (0, Lq - 1):
            rows.add(bh * Lq + i)
    bh0 = int(rng.integers(0, w_B * w_H))
    for t in range(block, Lq, block):
        rows.add(bh0 * Lq + t - 1)
        rows.add(bh0 * Lq + t)
    extra = rng.integers(0, w_B * w_H * Lq, size=n)
    rows.update(int(x) for x in extra)
    return np.array(sorted(rows), dtype=np.int64)
