"""B200-native 8-bit quantized attention (SageAttention forward pass).

A thin Python binding over the C ABI of ``libsage_b200.so`` (declared in
``include/sage.h``).  Every function here only checks and marshals arguments
(torch CUDA tensors -> device pointers, torch's current stream) and calls the
library; all arithmetic runs in the library's sm_100a kernels.  There is no
CPU or PyTorch fallback: if the library is missing, every call raises.

Exported names mirror the C ABI:
    sage_quant_qk, sage_attn_fwd, sage_attn_fwd_prequant,
    sage_quant_qk_qblock, sage_attn_fwd_qblock, sage_attn_fwd_prequant_qblock,
    sage_attn_fwd_ex, sage_attn_fwd_prequant_ex,
    sage_attn_decode, sage_attn_decode_prequant, sage_attn_decode_workspace_size,
    sage_quant_v_fp8, sage_quant_v_fp8_workspace_size, sage_attn_fwd_prequant_fp8pv,
    sage_quant_qk_varlen, sage_attn_fwd_prequant_varlen, sage_attn_fwd_varlen,
    sage_quant_k, sage_attn_fwd_host, sage_attn_fwd_host_qblock, sage_attn_fwd_noalloc,
    sage_workspace_size,
    sage_check_device_status, sage_status_string, sage_last_launch_count
plus conveniences that allocate outputs: ``quant_qk``, ``attention``,
``attention_varlen`` and ``decode``.
"""
from __future__ import annotations

from ._lib import (  # noqa: F401
    SageError,
    SYMBOLS,
    library_path,
    load_library,
    sage_attn_fwd,
    sage_attn_fwd_host,
    sage_attn_fwd_host_qblock,
    sage_attn_fwd_noalloc,
    NOALLOC_SCRATCH_BYTES,
    sage_attn_fwd_prequant,
    sage_attn_fwd_prequant_qblock,
    sage_attn_fwd_qblock,
    sage_attn_fwd_ex,
    sage_attn_fwd_prequant_ex,
    SAGE_PV_ACCUM_F16,
    PV_ACCUM,
    sage_workspace_size,
    sage_check_device_status,
    sage_debug_wait_timeout,
    sage_last_launch_count,
    sage_quant_qk,
    sage_quant_qk_qblock,
    Q_BLOCK_ROWS,
    sage_status_string,
    quant_qk,
    attention,
    decode,
    sage_attn_decode,
    sage_attn_decode_prequant,
    sage_attn_decode_workspace_size,
    sage_attn_decode_prequant_varlen,
    sage_attn_decode_prequant_paged,
    sage_quant_v_fp8,
    sage_quant_v_fp8_workspace_size,
    sage_attn_fwd_prequant_fp8pv,
    quant_v_fp8,
    SAGE_PV_FP8,
    sage_quant_qk_varlen,
    sage_attn_fwd_prequant_varlen,
    sage_attn_fwd_varlen,
    attention_varlen,
    sage_quant_k,
)
