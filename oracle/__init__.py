"""CPU oracle for 8-bit quantized attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product path (the CUDA library and its
binding) never calls it.  The arithmetic lives in ``sage_oracle.c``; this file
only compiles it (gcc, OpenMP, no fast-math, no FMA contraction) and marshals
numpy arrays through ctypes.

Functions and the passages they follow (SageAttention article, method section):
  k_mean          the K smoothing step
  quant_qk        the per-block INT8 quantization step, for Q and the
                  smoothed K
  attn_quant_sim  INT32-accumulated QK^T, dequantization, softmax with P kept
                  in FP16 (the FP16 P V step)
  attn_fp64       plain softmax(QK^T * sm_scale) V in fp64 (the full-precision
                  attention the article measures its accuracy against)
  e4m3_encode /   the FP8 (E4M3) format for P and V that the SageAttention2
  e4m3_decode     description (INT4 search results page, SageAttention2 entry)
                  proposes, round to nearest even, saturating
  quant_v_fp8     V to E4M3 with one scale per channel, stored channel-major
  attn_fp8pv_sim  the forward pass with P and V in E4M3 for the P V product
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sage_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
          "-shared", "-fPIC"]


def build(force: bool = False) -> str:
    """Compile sage_oracle.c into liboracle.so (if missing or stale)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        I64 = ctypes.c_int64
        D = ctypes.c_double
        lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_half_to_double.restype = D
        lib.oracle_double_to_half.argtypes = [D]
        lib.oracle_double_to_half.restype = ctypes.c_uint16
        lib.oracle_k_mean.argtypes = [P, I, I, I, I, P]
        lib.oracle_k_mean.restype = None
        lib.oracle_quant_qk.argtypes = [P, P, I, I, I, I, I, I, D, I, P, P, P, P, P]
        lib.oracle_quant_qk.restype = None
        lib.oracle_attn_quant_sim.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, P, I64, P]
        lib.oracle_attn_quant_sim.restype = None
        lib.oracle_quant_qk_blocks.argtypes = [P, P, I, I, I, I, I, I, D, I, I, P, P, P, P, P]
        lib.oracle_quant_qk_blocks.restype = None
        lib.oracle_attn_quant_sim_blocks.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, I, P,
                                                     I64, P]
        lib.oracle_attn_quant_sim_blocks.restype = None
        lib.oracle_attn_fp64.argtypes = [P, P, P, I, I, I, I, I, I, I, D, P, I64, P]
        lib.oracle_attn_fp64.restype = None
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_decode.restype = D
        lib.oracle_quant_v_fp8.argtypes = [P, I, I, I, I, P, P]
        lib.oracle_quant_v_fp8.restype = None
        lib.oracle_attn_fp8pv_sim.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, P, I64, P]
        lib.oracle_attn_fp8pv_sim.restype = None
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = I
        _lib = lib
        return lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _c(a: np.ndarray, dtype) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {a.dtype}")
    return np.ascontiguousarray(a)


def num_threads() -> int:
    return _load().oracle_num_threads()


def half_to_double(bits: int) -> float:
    return _load().oracle_half_to_double(int(bits))


def double_to_half(x: float) -> int:
    return _load().oracle_double_to_half(float(x))


def k_mean(k: np.ndarray) -> np.ndarray:
    """k: fp16 [B, Hkv, Lk, d] -> float32 [B, Hkv, d]."""
    k = _c(k, np.float16)
    B, Hkv, Lk, d = k.shape
    out = np.empty((B, Hkv, d), dtype=np.float32)
    _load().oracle_k_mean(_ptr(k), B, Hkv, Lk, d, _ptr(out))
    return out


def quant_qk(q: np.ndarray, k: np.ndarray, sm_scale: float, smooth: bool = True,
             q_block_rows: int = 128):
    """Returns (q_i8, k_i8, q_scale, k_scale, k_mean) as numpy arrays.
    q_block_rows: rows per Q quantization block (128 = the attention tile,
    1 = one scale per query token)."""
    q = _c(q, np.float16)
    k = _c(k, np.float16)
    B, H, Lq, d = q.shape
    Bk, Hkv, Lk, dk = k.shape
    assert Bk == B and dk == d
    nqb, nkb = -(-Lq // q_block_rows), -(-Lk // 64)
    q_i8 = np.empty(q.shape, dtype=np.int8)
    k_i8 = np.empty(k.shape, dtype=np.int8)
    q_scale = np.empty((B, H, nqb), dtype=np.float32)
    k_scale = np.empty((B, Hkv, nkb), dtype=np.float32)
    km = np.empty((B, Hkv, d), dtype=np.float32)
    _load().oracle_quant_qk_blocks(_ptr(q), _ptr(k), B, H, Hkv, Lq, Lk, d, float(sm_scale),
                                   1 if smooth else 0, int(q_block_rows), _ptr(q_i8),
                                   _ptr(k_i8), _ptr(q_scale), _ptr(k_scale), _ptr(km))
    return q_i8, k_i8, q_scale, k_scale, km


def attn_quant_sim(q_i8, k_i8, q_scale, k_scale, v, causal: bool, rows=None,
                   q_block_rows: int = 128):
    """Simulated quantized attention; returns float64 [n_rows, d]
    (or [B, H, Lq, d] when rows is None)."""
    q_i8 = _c(q_i8, np.int8)
    k_i8 = _c(k_i8, np.int8)
    q_scale = _c(q_scale, np.float32)
    k_scale = _c(k_scale, np.float32)
    v = _c(v, np.float16)
    B, H, Lq, d = q_i8.shape
    Hkv, Lk = k_i8.shape[1], k_i8.shape[2]
    if rows is None:
        out = np.empty((B, H, Lq, d), dtype=np.float64)
        rp, n = None, 0
    else:
        rows = _c(np.asarray(rows, dtype=np.int64), np.int64)
        out = np.empty((rows.shape[0], d), dtype=np.float64)
        rp, n = _ptr(rows), rows.shape[0]
    _load().oracle_attn_quant_sim_blocks(_ptr(q_i8), _ptr(k_i8), _ptr(q_scale),
                                         _ptr(k_scale), _ptr(v), B, H, Hkv, Lq, Lk, d,
                                         1 if causal else 0, int(q_block_rows), rp, n,
                                         _ptr(out))
    return out


def attn_fp64(q, k, v, causal: bool, sm_scale: float, rows=None):
    """Full-precision attention from fp16 inputs; float64 output."""
    q = _c(q, np.float16)
    k = _c(k, np.float16)
    v = _c(v, np.float16)
    B, H, Lq, d = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    if rows is None:
        out = np.empty((B, H, Lq, d), dtype=np.float64)
        rp, n = None, 0
    else:
        rows = _c(np.asarray(rows, dtype=np.int64), np.int64)
        out = np.empty((rows.shape[0], d), dtype=np.float64)
        rp, n = _ptr(rows), rows.shape[0]
    _load().oracle_attn_fp64(_ptr(q), _ptr(k), _ptr(v), B, H, Hkv, Lq, Lk, d,
                             1 if causal else 0, float(sm_scale), rp, n, _ptr(out))
    return out


def attention(q, k, v, causal: bool, sm_scale: float, rows=None):
    """Whole quantized path on the CPU: quantize, then simulate.
    Returns (out_f64, (q_i8, k_i8, q_scale, k_scale, k_mean))."""
    qk = quant_qk(q, k, sm_scale)
    return attn_quant_sim(qk[0], qk[1], qk[2], qk[3], v, causal, rows), qk


def e4m3_encode(x: float) -> int:
    return _load().oracle_e4m3_encode(float(x))


def e4m3_decode(code: int) -> float:
    return _load().oracle_e4m3_decode(int(code))


def quant_v_fp8(v: np.ndarray):
    """v: fp16 [B, Hkv, Lk, d] -> (v8t uint8 [B, Hkv, d, Lk], v_scale float32 [B, Hkv, d])."""
    v = _c(v, np.float16)
    B, Hkv, Lk, d = v.shape
    v8t = np.empty((B, Hkv, d, Lk), dtype=np.uint8)
    vs = np.empty((B, Hkv, d), dtype=np.float32)
    _load().oracle_quant_v_fp8(_ptr(v), B, Hkv, Lk, d, _ptr(v8t), _ptr(vs))
    return v8t, vs


def attn_fp8pv_sim(q_i8, k_i8, q_scale, k_scale, v8t, v_scale, causal: bool, rows=None,
                   q_block_rows: int = 128):
    """Quantized forward pass with P and V in E4M3; float64 [n_rows, d] (or
    [B, H, Lq, d] when rows is None)."""
    q_i8 = _c(q_i8, np.int8)
    k_i8 = _c(k_i8, np.int8)
    q_scale = _c(q_scale, np.float32)
    k_scale = _c(k_scale, np.float32)
    v8t = _c(v8t, np.uint8)
    v_scale = _c(v_scale, np.float32)
    B, H, Lq, d = q_i8.shape
    Hkv, Lk = k_i8.shape[1], k_i8.shape[2]
    if rows is None:
        out = np.empty((B, H, Lq, d), dtype=np.float64)
        rp, n = None, 0
    else:
        rows = _c(np.asarray(rows, dtype=np.int64), np.int64)
        out = np.empty((rows.shape[0], d), dtype=np.float64)
        rp, n = _ptr(rows), rows.shape[0]
    _load().oracle_attn_fp8pv_sim(_ptr(q_i8), _ptr(k_i8), _ptr(q_scale), _ptr(k_scale),
                                  _ptr(v8t), _ptr(v_scale), B, H, Hkv, Lq, Lk, d,
                                  1 if causal else 0, int(q_block_rows), rp, n, _ptr(out))
    return out
