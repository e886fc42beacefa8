"""ctypes marshalling for libsage_b200.so (C ABI in include/sage.h).

Argument marshalling only: shape/dtype/device checks, torch tensor -> device
pointer, torch's current CUDA stream -> cudaStream_t.  No arithmetic happens
here and there is no fallback path: a missing library raises on first use.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libsage_b200.so")
_lock = threading.Lock()
_lib = None

# Every symbol include/sage.h declares.
SYMBOLS = (
    "sage_quant_qk",
    "sage_workspace_size",
    "sage_attn_fwd_prequant",
    "sage_attn_fwd",
    "sage_attn_fwd_host",
    "sage_attn_fwd_host_qblock",
    "sage_check_device_status",
    "sage_status_string",
    "sage_last_launch_count",
    "sage_attn_fwd_noalloc",
    "sage_debug_wait_timeout",
    "sage_quant_qk_qblock",
    "sage_attn_fwd_prequant_qblock",
    "sage_attn_fwd_qblock",
    "sage_attn_fwd_ex",
    "sage_attn_fwd_prequant_ex",
    "sage_attn_decode_prequant",
    "sage_attn_decode_workspace_size",
    "sage_attn_decode",
    "sage_quant_v_fp8",
    "sage_quant_v_fp8_workspace_size",
    "sage_attn_fwd_prequant_fp8pv",
    "sage_attn_decode_prequant_varlen",
    "sage_attn_decode_prequant_paged",
    "sage_quant_qk_varlen",
    "sage_attn_fwd_prequant_varlen",
    "sage_attn_fwd_varlen",
    "sage_quant_k",
)

Q_BLOCK_ROWS = (128, 64, 32, 1)  # accepted Q quantization block heights
SAGE_PV_ACCUM_F16 = 1             # flag of the _ex calls: fp16 P V accumulator
SAGE_PV_FP8 = 2                   # flag of sage_attn_fwd_ex: P and V in FP8 E4M3
PV_ACCUM = {"f32": 0, "f16": SAGE_PV_ACCUM_F16, "fp8": SAGE_PV_FP8}

STATUS = {0: "SAGE_OK", 1: "SAGE_ERR_INVALID_ARG", 2: "SAGE_ERR_UNSUPPORTED",
          3: "SAGE_ERR_CUDA", 4: "SAGE_ERR_TIMEOUT"}


class SageError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where} failed: {STATUS.get(status, status)}")


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libsage_b200.so (raises if it was not built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"{_LIB_PATH} is missing: build it with "
                "`python -m bit_quantized_attention_mean_b200.build` (no fallback exists)")
        lib = ctypes.CDLL(_LIB_PATH)
        P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        lib.sage_quant_qk.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, F, P]
        lib.sage_quant_qk.restype = I
        lib.sage_attn_fwd_prequant.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, P]
        lib.sage_attn_fwd_prequant.restype = I
        lib.sage_attn_fwd.argtypes = [P, P, P, P, I, I, I, I, I, I, I, F, P]
        lib.sage_attn_fwd.restype = I
        lib.sage_attn_fwd_host.argtypes = [P, P, P, P, I, I, I, I, I, I, I, F, P]
        lib.sage_attn_fwd_host.restype = I
        lib.sage_attn_fwd_host_qblock.argtypes = [P, P, P, P, I, I, I, I, I, I, I, F, I, P]
        lib.sage_attn_fwd_host_qblock.restype = I
        lib.sage_workspace_size.argtypes = [I, I, I, I, I, I]
        lib.sage_workspace_size.restype = Z
        lib.sage_check_device_status.argtypes = [P]
        lib.sage_check_device_status.restype = I
        lib.sage_status_string.argtypes = [I]
        lib.sage_status_string.restype = ctypes.c_char_p
        lib.sage_attn_fwd_noalloc.argtypes = [P, P, P, P, I, I, I, I, I, I, I, F, P]
        lib.sage_attn_fwd_noalloc.restype = I
        lib.sage_debug_wait_timeout.argtypes = [I, P]
        lib.sage_debug_wait_timeout.restype = I
        lib.sage_quant_qk_qblock.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, P]
        lib.sage_quant_qk_qblock.restype = I
        lib.sage_attn_fwd_prequant_qblock.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I,
                                                      P]
        lib.sage_attn_fwd_prequant_qblock.restype = I
        lib.sage_attn_fwd_qblock.argtypes = [P, P, P, P, I, I, I, I, I, I, I, F, I, P]
        lib.sage_attn_fwd_qblock.restype = I
        U = ctypes.c_uint
        lib.sage_attn_fwd_ex.argtypes = [P, P, P, P, I, I, I, I, I, I, I, F, I, U, P]
        lib.sage_attn_fwd_ex.restype = I
        lib.sage_attn_fwd_prequant_ex.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, U, P]
        lib.sage_attn_fwd_prequant_ex.restype = I
        lib.sage_attn_decode_prequant.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, P, Z, P]
        lib.sage_attn_decode_prequant.restype = I
        lib.sage_attn_decode_workspace_size.argtypes = [I, I, I, I, I, I]
        lib.sage_attn_decode_workspace_size.restype = Z
        lib.sage_attn_decode.argtypes = [P, P, P, P, I, I, I, I, I, I, I, F, I, P]
        lib.sage_attn_decode.restype = I
        lib.sage_quant_v_fp8.argtypes = [P, P, P, I, I, I, I, P, Z, P]
        lib.sage_quant_v_fp8.restype = I
        lib.sage_quant_v_fp8_workspace_size.argtypes = [I, I, I]
        lib.sage_quant_v_fp8_workspace_size.restype = Z
        lib.sage_attn_fwd_prequant_fp8pv.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, P]
        lib.sage_attn_fwd_prequant_fp8pv.restype = I
        lib.sage_attn_decode_prequant_varlen.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I,
                                                         I, I, P, Z, P]
        lib.sage_attn_decode_prequant_varlen.restype = I
        lib.sage_attn_decode_prequant_paged.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I,
                                                        I, I, I, P, Z, P]
        lib.sage_attn_decode_prequant_paged.restype = I
        lib.sage_quant_qk_varlen.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, I,
                                             P]
        lib.sage_quant_qk_varlen.restype = I
        lib.sage_attn_fwd_prequant_varlen.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I,
                                                      I, I, U, P]
        lib.sage_attn_fwd_prequant_varlen.restype = I
        lib.sage_attn_fwd_varlen.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, F, I, U, P]
        lib.sage_attn_fwd_varlen.restype = I
        lib.sage_quant_k.argtypes = [P, P, P, P, I, I, I, I, P]
        lib.sage_quant_k.restype = I
        lib.sage_last_launch_count.argtypes = []
        lib.sage_last_launch_count.restype = I
        _lib = lib
        return lib


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dev(t, dtype, name, shape=None):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    return ctypes.c_void_p(t.data_ptr())


def _check(status: int, where: str):
    if status != 0:
        raise SageError(status, where)


def _dims(q, k):
    B, H, Lq, d = q.shape
    Bk, Hkv, Lk, dk = k.shape
    if Bk != B or dk != d:
        raise ValueError("q and k disagree on batch or head dim")
    return B, H, Hkv, Lq, Lk, d


# --------------------------------------------------------------- C ABI names

def sage_status_string(status: int) -> str:
    return load_library().sage_status_string(int(status)).decode()


def sage_last_launch_count() -> int:
    return load_library().sage_last_launch_count()


def sage_workspace_size(B, H, Hkv, Lq, Lk, d) -> int:
    """Bytes of device scratch sage_attn_fwd allocates for this shape."""
    return load_library().sage_workspace_size(B, H, Hkv, Lq, Lk, d)


def _quant_args(q, k, q_i8, k_i8, q_scale, k_scale, k_mean, q_block_rows):
    import torch
    B, H, Hkv, Lq, Lk, d = _dims(q, k)
    nqb, nkb = -(-Lq // q_block_rows), -(-Lk // 64)
    return [
        _dev(q, torch.float16, "q"), _dev(k, torch.float16, "k"),
        _dev(q_i8, torch.int8, "q_i8", q.shape), _dev(k_i8, torch.int8, "k_i8", k.shape),
        _dev(q_scale, torch.float32, "q_scale", (B, H, nqb)),
        _dev(k_scale, torch.float32, "k_scale", (B, Hkv, nkb)),
        _dev(k_mean, torch.float32, "k_mean", (B, Hkv, d)),
        B, H, Hkv, Lq, Lk, d,
    ]


def _workspace(workspace):
    import torch
    if workspace is None:
        return ctypes.c_void_p(0), 0
    return _dev(workspace, torch.uint8, "workspace"), workspace.numel()


def _check_qbr(q_block_rows):
    if q_block_rows not in Q_BLOCK_ROWS:
        raise ValueError(f"q_block_rows must be one of {Q_BLOCK_ROWS}, got {q_block_rows}")


def sage_quant_qk(q, k, q_i8, k_i8, q_scale, k_scale, k_mean, sm_scale, stream=None):
    """Smooth K and quantize Q/K per block into the given output tensors."""
    args = _quant_args(q, k, q_i8, k_i8, q_scale, k_scale, k_mean, 128)
    _check(load_library().sage_quant_qk(*args, float(sm_scale), _stream(stream)),
           "sage_quant_qk")


def sage_quant_qk_qblock(q, k, q_i8, k_i8, q_scale, k_scale, k_mean, sm_scale, q_block_rows,
                         stream=None):
    """sage_quant_qk with Q blocks of q_block_rows rows (128, 64, 32 or 1);
    q_scale has shape [B, H, ceil(Lq / q_block_rows)]."""
    _check_qbr(q_block_rows)
    args = _quant_args(q, k, q_i8, k_i8, q_scale, k_scale, k_mean, q_block_rows)
    _check(load_library().sage_quant_qk_qblock(*args, float(sm_scale), int(q_block_rows),
                                               _stream(stream)),
           "sage_quant_qk_qblock")


def _prequant_args(q_i8, k_i8, q_scale, k_scale, v, out, q_block_rows):
    import torch
    B, H, Hkv, Lq, Lk, d = _dims(q_i8, k_i8)
    nqb, nkb = -(-Lq // q_block_rows), -(-Lk // 64)
    return [
        _dev(q_i8, torch.int8, "q_i8"), _dev(k_i8, torch.int8, "k_i8"),
        _dev(q_scale, torch.float32, "q_scale", (B, H, nqb)),
        _dev(k_scale, torch.float32, "k_scale", (B, Hkv, nkb)),
        _dev(v, torch.float16, "v", k_i8.shape), _dev(out, torch.float16, "out", q_i8.shape),
        B, H, Hkv, Lq, Lk, d,
    ]


def sage_attn_fwd_prequant(q_i8, k_i8, q_scale, k_scale, v, out, causal, stream=None):
    """Attention kernel on pre-quantized Q/K (fp16 V, fp16 out)."""
    args = _prequant_args(q_i8, k_i8, q_scale, k_scale, v, out, 128)
    _check(load_library().sage_attn_fwd_prequant(*args, 1 if causal else 0, _stream(stream)),
           "sage_attn_fwd_prequant")


def sage_attn_fwd_prequant_qblock(q_i8, k_i8, q_scale, k_scale, v, out, causal, q_block_rows,
                                  stream=None):
    """sage_attn_fwd_prequant for Q quantized in blocks of q_block_rows rows."""
    _check_qbr(q_block_rows)
    args = _prequant_args(q_i8, k_i8, q_scale, k_scale, v, out, q_block_rows)
    _check(load_library().sage_attn_fwd_prequant_qblock(*args, 1 if causal else 0,
                                                        int(q_block_rows), _stream(stream)),
           "sage_attn_fwd_prequant_qblock")


def sage_attn_fwd(q, k, v, out, causal, sm_scale, stream=None):
    """Whole forward pass on fp16 device tensors, output written into `out`."""
    import torch
    lib = load_library()
    B, H, Hkv, Lq, Lk, d = _dims(q, k)
    _check(lib.sage_attn_fwd(
        _dev(q, torch.float16, "q"), _dev(k, torch.float16, "k"),
        _dev(v, torch.float16, "v", k.shape), _dev(out, torch.float16, "out", q.shape),
        B, H, Hkv, Lq, Lk, d, 1 if causal else 0, float(sm_scale), _stream(stream)),
        "sage_attn_fwd")


def sage_attn_fwd_qblock(q, k, v, out, causal, sm_scale, q_block_rows, stream=None):
    """sage_attn_fwd with Q quantized in blocks of q_block_rows rows."""
    import torch
    _check_qbr(q_block_rows)
    lib = load_library()
    B, H, Hkv, Lq, Lk, d = _dims(q, k)
    _check(lib.sage_attn_fwd_qblock(
        _dev(q, torch.float16, "q"), _dev(k, torch.float16, "k"),
        _dev(v, torch.float16, "v", k.shape), _dev(out, torch.float16, "out", q.shape),
        B, H, Hkv, Lq, Lk, d, 1 if causal else 0, float(sm_scale), int(q_block_rows),
        _stream(stream)), "sage_attn_fwd_qblock")


def _flags(pv_accum):
    if pv_accum not in PV_ACCUM:
        raise ValueError(f"pv_accum must be one of {tuple(PV_ACCUM)}, got {pv_accum!r}")
    return PV_ACCUM[pv_accum]


def sage_attn_fwd_ex(q, k, v, out, causal, sm_scale, q_block_rows=128, pv_accum="f32",
                     stream=None):
    """sage_attn_fwd with a Q block height and the P V variant: "f32" (fp16 P
    and V, fp32 sums; the default), "f16" (fp16 sums, as the SageAttention
    article states) or "fp8" (P and V in E4M3, as its SageAttention2
    description states)."""
    import torch
    _check_qbr(q_block_rows)
    flags = _flags(pv_accum)
    lib = load_library()
    B, H, Hkv, Lq, Lk, d = _dims(q, k)
    _check(lib.sage_attn_fwd_ex(
        _dev(q, torch.float16, "q"), _dev(k, torch.float16, "k"),
        _dev(v, torch.float16, "v", k.shape), _dev(out, torch.float16, "out", q.shape),
        B, H, Hkv, Lq, Lk, d, 1 if causal else 0, float(sm_scale), int(q_block_rows), flags,
        _stream(stream)), "sage_attn_fwd_ex")


def sage_attn_fwd_prequant_ex(q_i8, k_i8, q_scale, k_scale, v, out, causal, q_block_rows=128,
                              pv_accum="f32", stream=None):
    """sage_attn_fwd_prequant_qblock with the P V accumulator selectable
    ("f32" or "f16"; FP8 P V takes E4M3 V: sage_attn_fwd_prequant_fp8pv)."""
    _check_qbr(q_block_rows)
    flags = _flags(pv_accum)
    if flags == SAGE_PV_FP8:
        raise ValueError("sage_attn_fwd_prequant_ex takes fp16 V; use sage_attn_fwd_prequant_fp8pv")
    args = _prequant_args(q_i8, k_i8, q_scale, k_scale, v, out, q_block_rows)
    _check(load_library().sage_attn_fwd_prequant_ex(*args, 1 if causal else 0,
                                                    int(q_block_rows), flags, _stream(stream)),
           "sage_attn_fwd_prequant_ex")


def _seqlens(t, name, B):
    """Device pointer of an optional int32 [B] length tensor (None -> NULL)."""
    import torch
    if t is None:
        return ctypes.c_void_p(0)
    return _dev(t, torch.int32, name, (B,))


def sage_quant_qk_varlen(q, k, q_i8, k_i8, q_scale, k_scale, k_mean, seqlens_q, seqlens_k,
                         sm_scale, q_block_rows=128, stream=None):
    """sage_quant_qk_qblock on a padded batch: entry b quantizes its first
    seqlens_q[b] Q rows and smooths/quantizes its first seqlens_k[b] keys
    (int32 CUDA tensors [B], or None for all rows / all keys)."""
    _check_qbr(q_block_rows)
    args = _quant_args(q, k, q_i8, k_i8, q_scale, k_scale, k_mean, q_block_rows)
    B = q.shape[0]
    _check(load_library().sage_quant_qk_varlen(
        *args[:7], _seqlens(seqlens_q, "seqlens_q", B), _seqlens(seqlens_k, "seqlens_k", B),
        *args[7:], float(sm_scale), int(q_block_rows), _stream(stream)),
        "sage_quant_qk_varlen")


def sage_attn_fwd_prequant_varlen(q_i8, k_i8, q_scale, k_scale, v, out, seqlens_q, seqlens_k,
                                  causal, q_block_rows=128, pv_accum="f32", stream=None):
    """sage_attn_fwd_prequant_ex on a padded batch (lengths as
    sage_quant_qk_varlen); output rows past seqlens_q[b] are written as zeros."""
    _check_qbr(q_block_rows)
    flags = _flags(pv_accum)
    if flags == SAGE_PV_FP8:
        raise ValueError("sage_attn_fwd_prequant_varlen takes fp16 V (pv_accum 'f32' or 'f16')")
    args = _prequant_args(q_i8, k_i8, q_scale, k_scale, v, out, q_block_rows)
    B = q_i8.shape[0]
    _check(load_library().sage_attn_fwd_prequant_varlen(
        *args[:6], _seqlens(seqlens_q, "seqlens_q", B), _seqlens(seqlens_k, "seqlens_k", B),
        *args[6:], 1 if causal else 0, int(q_block_rows), flags, _stream(stream)),
        "sage_attn_fwd_prequant_varlen")


def sage_attn_fwd_varlen(q, k, v, out, seqlens_q, seqlens_k, causal, sm_scale, q_block_rows=128,
                         pv_accum="f32", stream=None):
    """The whole forward pass on a padded batch: entry b attends with its
    first seqlens_q[b] rows over its first seqlens_k[b] keys, exactly as the
    same call on that entry alone; padding output rows are zeros and (for
    pv_accum "f32" / "f16") the V padding inside an entry's last 64-key tile
    must be finite."""
    import torch
    _check_qbr(q_block_rows)
    flags = _flags(pv_accum)
    lib = load_library()
    B, H, Hkv, Lq, Lk, d = _dims(q, k)
    _check(lib.sage_attn_fwd_varlen(
        _dev(q, torch.float16, "q"), _dev(k, torch.float16, "k"),
        _dev(v, torch.float16, "v", k.shape), _dev(out, torch.float16, "out", q.shape),
        _seqlens(seqlens_q, "seqlens_q", B), _seqlens(seqlens_k, "seqlens_k", B),
        B, H, Hkv, Lq, Lk, d, 1 if causal else 0, float(sm_scale), int(q_block_rows), flags,
        _stream(stream)), "sage_attn_fwd_varlen")


def sage_quant_k(k, k_i8, k_scale, k_mean, stream=None):
    """Smooth K and quantize it in 64-row blocks (the K half of
    sage_quant_qk) into the given output tensors."""
    import torch
    B, Hkv, Lk, d = k.shape
    _check(load_library().sage_quant_k(
        _dev(k, torch.float16, "k"), _dev(k_i8, torch.int8, "k_i8", k.shape),
        _dev(k_scale, torch.float32, "k_scale", (B, Hkv, -(-Lk // 64))),
        _dev(k_mean, torch.float32, "k_mean", (B, Hkv, d)), B, Hkv, Lk, d,
        _stream(stream)), "sage_quant_k")


def sage_attn_decode_workspace_size(B, H, Hkv, Lq, Lk, d) -> int:
    return load_library().sage_attn_decode_workspace_size(B, H, Hkv, Lq, Lk, d)


def sage_attn_decode_prequant(q_i8, k_i8, q_scale, k_scale, v, out, causal, q_block_rows=128,
                              workspace=None, stream=None):
    """Few query tokens against a long key sequence, on pre-quantized Q/K
    ((H / Hkv) * Lq <= 128)."""
    _check_qbr(q_block_rows)
    args = _prequant_args(q_i8, k_i8, q_scale, k_scale, v, out, q_block_rows)
    _check(load_library().sage_attn_decode_prequant(*args, 1 if causal else 0,
                                                    int(q_block_rows), *_workspace(workspace),
                                                    _stream(stream)),
           "sage_attn_decode_prequant")


def sage_attn_decode_prequant_varlen(q_i8, k_i8, q_scale, k_scale, v, out, seqlens_k, causal,
                                     q_block_rows=128, workspace=None, stream=None):
    """sage_attn_decode_prequant with one key count per batch entry
    (seqlens_k: int32 CUDA tensor [B]) in a cache padded to Lk."""
    import torch
    _check_qbr(q_block_rows)
    args = _prequant_args(q_i8, k_i8, q_scale, k_scale, v, out, q_block_rows)
    sl = _dev(seqlens_k, torch.int32, "seqlens_k", (q_i8.shape[0],))
    _check(load_library().sage_attn_decode_prequant_varlen(
        *args[:6], sl, *args[6:], 1 if causal else 0, int(q_block_rows), *_workspace(workspace),
        _stream(stream)), "sage_attn_decode_prequant_varlen")


def sage_attn_decode_prequant_paged(q_i8, q_scale, k_pages, k_scale_pages, v_pages, block_table,
                                    seqlens_k, out, causal, q_block_rows=128, workspace=None,
                                    stream=None):
    """Decoding on a paged cache: k_pages int8 / v_pages fp16 [num_pages, Hkv,
    64, d], k_scale_pages [num_pages, Hkv], block_table int32 [B, max_blocks],
    seqlens_k int32 [B] (all CUDA tensors)."""
    import torch
    _check_qbr(q_block_rows)
    B, H, Lq, d = q_i8.shape
    num_pages, Hkv = k_pages.shape[0], k_pages.shape[1]
    max_blocks = block_table.shape[1]
    nqb = -(-Lq // q_block_rows)
    _check(load_library().sage_attn_decode_prequant_paged(
        _dev(q_i8, torch.int8, "q_i8"), _dev(q_scale, torch.float32, "q_scale", (B, H, nqb)),
        _dev(k_pages, torch.int8, "k_pages", (num_pages, Hkv, 64, d)),
        _dev(k_scale_pages, torch.float32, "k_scale_pages", (num_pages, Hkv)),
        _dev(v_pages, torch.float16, "v_pages", (num_pages, Hkv, 64, d)),
        _dev(block_table, torch.int32, "block_table", (B, max_blocks)),
        _dev(seqlens_k, torch.int32, "seqlens_k", (B,)),
        _dev(out, torch.float16, "out", q_i8.shape), B, H, Hkv, Lq, num_pages, max_blocks, d,
        1 if causal else 0, int(q_block_rows), *_workspace(workspace), _stream(stream)),
        "sage_attn_decode_prequant_paged")


def sage_attn_decode(q, k, v, out, causal, sm_scale, q_block_rows=128, stream=None):
    """Quantization + sage_attn_decode_prequant on fp16 device tensors."""
    import torch
    _check_qbr(q_block_rows)
    lib = load_library()
    B, H, Hkv, Lq, Lk, d = _dims(q, k)
    _check(lib.sage_attn_decode(
        _dev(q, torch.float16, "q"), _dev(k, torch.float16, "k"),
        _dev(v, torch.float16, "v", k.shape), _dev(out, torch.float16, "out", q.shape),
        B, H, Hkv, Lq, Lk, d, 1 if causal else 0, float(sm_scale), int(q_block_rows),
        _stream(stream)), "sage_attn_decode")


def decode(q, k, v, causal=False, sm_scale=None, q_block_rows=128, stream=None):
    """Allocate the output and run sage_attn_decode; returns the fp16 output."""
    import torch
    if sm_scale is None:
        sm_scale = q.shape[-1] ** -0.5
    out = torch.empty_like(q)
    sage_attn_decode(q, k, v, out, causal, sm_scale, q_block_rows, stream=stream)
    return out


def sage_quant_v_fp8_workspace_size(B, Hkv, d) -> int:
    return load_library().sage_quant_v_fp8_workspace_size(B, Hkv, d)


def sage_quant_v_fp8(v, v8t, v_scale, workspace=None, stream=None):
    """V fp16 [B, Hkv, Lk, d] -> E4M3 codes v8t uint8 [B, Hkv, d, 64*ceil(Lk/64)]
    (channel-major) and per-channel scales v_scale fp32 [B, Hkv, d]."""
    import torch
    B, Hkv, Lk, d = v.shape
    lkp = -(-Lk // 64) * 64
    _check(load_library().sage_quant_v_fp8(
        _dev(v, torch.float16, "v"), _dev(v8t, torch.uint8, "v8t", (B, Hkv, d, lkp)),
        _dev(v_scale, torch.float32, "v_scale", (B, Hkv, d)), B, Hkv, Lk, d,
        *_workspace(workspace), _stream(stream)), "sage_quant_v_fp8")


def sage_attn_fwd_prequant_fp8pv(q_i8, k_i8, q_scale, k_scale, v8t, v_scale, out, causal,
                                 q_block_rows=128, stream=None):
    """Attention on pre-quantized Q/K with P and V in FP8 E4M3 (V from
    sage_quant_v_fp8)."""
    import torch
    _check_qbr(q_block_rows)
    B, H, Hkv, Lq, Lk, d = _dims(q_i8, k_i8)
    nqb, nkb = -(-Lq // q_block_rows), -(-Lk // 64)
    _check(load_library().sage_attn_fwd_prequant_fp8pv(
        _dev(q_i8, torch.int8, "q_i8"), _dev(k_i8, torch.int8, "k_i8"),
        _dev(q_scale, torch.float32, "q_scale", (B, H, nqb)),
        _dev(k_scale, torch.float32, "k_scale", (B, Hkv, nkb)),
        _dev(v8t, torch.uint8, "v8t", (B, Hkv, d, nkb * 64)),
        _dev(v_scale, torch.float32, "v_scale", (B, Hkv, d)),
        _dev(out, torch.float16, "out", q_i8.shape), B, H, Hkv, Lq, Lk, d,
        1 if causal else 0, int(q_block_rows), _stream(stream)), "sage_attn_fwd_prequant_fp8pv")


def quant_v_fp8(v, stream=None):
    """Allocate outputs and run sage_quant_v_fp8; returns (v8t, v_scale)."""
    import torch
    B, Hkv, Lk, d = v.shape
    v8t = torch.empty((B, Hkv, d, -(-Lk // 64) * 64), dtype=torch.uint8, device=v.device)
    vs = torch.empty((B, Hkv, d), dtype=torch.float32, device=v.device)
    sage_quant_v_fp8(v, v8t, vs, stream=stream)
    return v8t, vs


NOALLOC_SCRATCH_BYTES = 64 << 20


def sage_attn_fwd_noalloc(q, k, v, out, causal, sm_scale, stream=None):
    """Whole forward pass without allocating device memory during the call.

    For callers that cannot allocate at call time (a server that reserved its
    memory budget up front, a plugin host without an allocator for the
    library).  The library's scratch is one fixed 64 MiB device array shared by
    all calls: order the calls on one stream, make the first call on a device
    before any stream capture, and keep problems within the array
    (sage_workspace_size(...) <= 64 MiB), else SageError is raised."""
    import torch
    lib = load_library()
    B, H, Hkv, Lq, Lk, d = _dims(q, k)
    status = lib.sage_attn_fwd_noalloc(
        _dev(q, torch.float16, "q"), _dev(k, torch.float16, "k"),
        _dev(v, torch.float16, "v", k.shape), _dev(out, torch.float16, "out", q.shape),
        B, H, Hkv, Lq, Lk, d, 1 if causal else 0, float(sm_scale), _stream(stream))
    if status != 0:
        need = lib.sage_workspace_size(B, H, Hkv, Lq, Lk, d)
        if status == 1 and need > NOALLOC_SCRATCH_BYTES:
            raise SageError(status, f"sage_attn_fwd_noalloc (needs {need} bytes of scratch, "
                                    f"the fixed array holds {NOALLOC_SCRATCH_BYTES})")
        raise SageError(status, "sage_attn_fwd_noalloc")


def sage_attn_fwd_host(q, k, v, out, causal, sm_scale, stream=None):
    """Whole forward pass on HOST fp16 tensors (pinned for async copies)."""
    sage_attn_fwd_host_qblock(q, k, v, out, causal, sm_scale, 128, stream)


def sage_attn_fwd_host_qblock(q, k, v, out, causal, sm_scale, q_block_rows, stream=None):
    """sage_attn_fwd_host with Q quantized in blocks of q_block_rows rows."""
    import torch
    _check_qbr(q_block_rows)
    lib = load_library()
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out)):
        if not isinstance(t, torch.Tensor) or t.is_cuda or t.dtype != torch.float16 \
                or not t.is_contiguous():
            raise ValueError(f"{name}: expected a contiguous fp16 host tensor")
    B, H, Hkv, Lq, Lk, d = _dims(q, k)
    if tuple(v.shape) != tuple(k.shape) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("v must match k and out must match q")
    _check(lib.sage_attn_fwd_host_qblock(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
        ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(out.data_ptr()),
        B, H, Hkv, Lq, Lk, d, 1 if causal else 0, float(sm_scale), int(q_block_rows),
        _stream(stream)), "sage_attn_fwd_host_qblock")


def sage_debug_wait_timeout(limit_ms, stream=None):
    """Launch the diagnostic kernel whose bounded wait must give up after
    limit_ms; the next sage_check_device_status then raises SAGE_ERR_TIMEOUT."""
    _check(load_library().sage_debug_wait_timeout(int(limit_ms), _stream(stream)),
           "sage_debug_wait_timeout")


def sage_check_device_status(stream=None):
    """Synchronize the stream and raise if a kernel's bounded wait gave up."""
    _check(load_library().sage_check_device_status(_stream(stream)),
           "sage_check_device_status")


# --------------------------------------------------------- conveniences

def quant_qk(q, k, sm_scale, q_block_rows=128, stream=None):
    """Allocate outputs and run sage_quant_qk (sage_quant_qk_qblock when
    q_block_rows != 128).
    Returns (q_i8, k_i8, q_scale, k_scale, k_mean) as CUDA tensors."""
    import torch
    _check_qbr(q_block_rows)
    B, H, Hkv, Lq, Lk, d = _dims(q, k)
    dev = q.device
    q_i8 = torch.empty(q.shape, dtype=torch.int8, device=dev)
    k_i8 = torch.empty(k.shape, dtype=torch.int8, device=dev)
    q_scale = torch.empty((B, H, -(-Lq // q_block_rows)), dtype=torch.float32, device=dev)
    k_scale = torch.empty((B, Hkv, -(-Lk // 64)), dtype=torch.float32, device=dev)
    k_mean = torch.empty((B, Hkv, d), dtype=torch.float32, device=dev)
    if q_block_rows == 128:
        sage_quant_qk(q, k, q_i8, k_i8, q_scale, k_scale, k_mean, sm_scale, stream=stream)
    else:
        sage_quant_qk_qblock(q, k, q_i8, k_i8, q_scale, k_scale, k_mean, sm_scale,
                             q_block_rows, stream=stream)
    return q_i8, k_i8, q_scale, k_scale, k_mean


def attention_varlen(q, k, v, seqlens_q=None, seqlens_k=None, causal=False, sm_scale=None,
                     q_block_rows=128, pv_accum="f32", stream=None):
    """Allocate the output and run sage_attn_fwd_varlen on a padded batch;
    returns the fp16 output (zeros past each entry's seqlens_q)."""
    import torch
    if sm_scale is None:
        sm_scale = q.shape[-1] ** -0.5
    out = torch.empty_like(q)
    sage_attn_fwd_varlen(q, k, v, out, seqlens_q, seqlens_k, causal, sm_scale, q_block_rows,
                         pv_accum, stream=stream)
    return out


def attention(q, k, v, causal=False, sm_scale=None, q_block_rows=128, pv_accum="f32",
              stream=None):
    """Allocate the output and run sage_attn_fwd (sage_attn_fwd_qblock when
    q_block_rows != 128, sage_attn_fwd_ex for an fp16 P V accumulator);
    returns the fp16 output."""
    import torch
    _check_qbr(q_block_rows)
    _flags(pv_accum)
    if sm_scale is None:
        sm_scale = q.shape[-1] ** -0.5
    out = torch.empty_like(q)
    if pv_accum != "f32":
        sage_attn_fwd_ex(q, k, v, out, causal, sm_scale, q_block_rows, pv_accum, stream=stream)
    elif q_block_rows == 128:
        sage_attn_fwd(q, k, v, out, causal, sm_scale, stream=stream)
    else:
        sage_attn_fwd_qblock(q, k, v, out, causal, sm_scale, q_block_rows, stream=stream)
    return out
