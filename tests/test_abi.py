"""CPU checks of the C ABI boundary: the library loads without a GPU and
exports exactly what include/sage.h declares (no compute calls here)."""
import ctypes
import os
import re
import pytest

import bit_quantized_attention_mean_b200 as sage

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_symbols():
    text = open(os.path.join(ROOT, "include", "sage.h")).read()
    return sorted(set(re.findall(r"^SAGE_API\s+[\w\s\*]*?\b(sage_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_binding_names():
    assert header_symbols() == sorted(sage.SYMBOLS)


def test_library_exports_every_declared_symbol():
    lib = sage.load_library()
    for name in header_symbols():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_host_only_helpers():
    assert sage.sage_status_string(0) == "SAGE_OK"
    assert sage.sage_status_string(4) == "SAGE_ERR_TIMEOUT"
    # workspace = int8 Q and K + scales + mean, 256-byte aligned pieces
    ws = sage.sage_attn_workspace_size(1, 2, 2, 256, 256, 64)
    assert ws >= 2 * 2 * 256 * 64 + 2 * 2 * 4 + 2 * 64 * 4
    assert sage.sage_attn_workspace_size(1, 2, 2, 256, 256, 96) == 0   # unsupported d
    assert sage.sage_attn_workspace_size(1, 3, 2, 256, 256, 64) == 0   # H % Hkv != 0
    # the K mean is reduced on chip: no scratch
    assert sage.sage_quant_workspace_size(2, 4, 1000, 128) == 0


def test_binding_rejects_unsupported_q_block_rows_before_any_call():
    import bit_quantized_attention_mean_b200 as sage
    assert sage.Q_BLOCK_ROWS == (128, 64, 32, 1)
    for bad in (0, 16, 100, 256):
        with pytest.raises(ValueError):
            sage.attention(None, None, None, q_block_rows=bad)
        with pytest.raises(ValueError):
            sage.quant_qk(None, None, 0.1, q_block_rows=bad)
