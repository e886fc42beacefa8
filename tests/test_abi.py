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
    # workspace = int8 Q and K + scales + mean, each a 256-byte aligned piece
    piece = lambda n: -(-n // 256) * 256
    ws = sage.sage_workspace_size(1, 2, 2, 256, 256, 64)
    assert ws == (piece(2 * 256 * 64) * 2 + piece(2 * 2 * 4) + piece(2 * 4 * 4)
                  + piece(2 * 64 * 4))
    assert sage.sage_workspace_size(1, 2, 2, 256, 256, 96) == 0   # unsupported d
    assert sage.sage_workspace_size(1, 3, 2, 256, 256, 64) == 0   # H % Hkv != 0


# The calls of the boundary the scope table names, with their argument
# lists as C types (ctypes names), in declaration order.
SCOPE_CALLS = {
    "sage_quant_qk": ["const void *", "const void *", "int8_t *", "int8_t *", "float *",
                      "float *", "float *", "int", "int", "int", "int", "int", "int", "float",
                      "void *"],
    "sage_attn_fwd": ["const void *", "const void *", "const void *", "void *", "int", "int",
                      "int", "int", "int", "int", "int", "float", "void *"],
    "sage_attn_fwd_prequant": ["const int8_t *", "const int8_t *", "const float *",
                               "const float *", "const void *", "void *", "int", "int", "int",
                               "int", "int", "int", "int", "void *"],
    "sage_workspace_size": ["int", "int", "int", "int", "int", "int"],
    "sage_check_device_status": ["void *"],
    "sage_status_string": ["sage_status"],
}


def _declared_params(name):
    text = open(os.path.join(ROOT, "include", "sage.h")).read()
    m = re.search(r"SAGE_API[^;(]*\b" + name + r"\s*\(([^)]*)\)\s*;", text)
    assert m, name
    params = []
    for p in m.group(1).split(","):
        p = " ".join(p.split())
        p = re.sub(r"\s*\w+$", "", p) if not p.endswith("*") else p   # drop the name
        p = re.sub(r"\*\s*\w+$", "*", p)
        params.append(p.replace(" *", " *").strip())
    return params


@pytest.mark.parametrize("name", sorted(SCOPE_CALLS))
def test_scope_table_calls_have_their_signatures(name):
    assert name in sage.SYMBOLS
    got = [re.sub(r"\s+\*", " *", p) for p in _declared_params(name)]
    assert got == SCOPE_CALLS[name], (name, got)


def test_binding_rejects_unsupported_q_block_rows_before_any_call():
    import bit_quantized_attention_mean_b200 as sage
    assert sage.Q_BLOCK_ROWS == (128, 64, 32, 1)
    for bad in (0, 16, 100, 256):
        with pytest.raises(ValueError):
            sage.attention(None, None, None, q_block_rows=bad)
        with pytest.raises(ValueError):
            sage.quant_qk(None, None, 0.1, q_block_rows=bad)
