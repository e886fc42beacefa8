"""CPU checks of the C ABI's argument validation: every call below carries
one invalid argument that the library rejects before it touches the device
(shape, block height, flags, causal flag, sm_scale, null or misaligned
pointer), so the stated status comes back without a GPU and the dummy
pointers are never dereferenced."""
import ctypes
import math

import pytest

import bit_quantized_attention_mean_b200 as sage

P = ctypes.c_void_p
A = P(1 << 20)          # a 16-byte aligned dummy address (never dereferenced)
M = P((1 << 20) + 4)    # misaligned
N = P(0)                # null
S = P(0)                # default stream
OK_, INVALID, UNSUPPORTED = 0, 1, 2


def quant_k(k=A, ki=A, ks=A, km=A, B=1, Hkv=2, Lk=128, d=64):
    return sage.load_library().sage_quant_k(k, ki, ks, km, B, Hkv, Lk, d, S)


def quant_qk_varlen(q=A, qs=A, B=1, H=2, Hkv=2, Lq=128, Lk=128, d=64, sm=0.125, qbr=128):
    return sage.load_library().sage_quant_qk_varlen(q, A, A, A, qs, A, A, A, A, B, H, Hkv, Lq,
                                                    Lk, d, sm, qbr, S)


def fwd_varlen(out=A, B=1, H=2, Hkv=2, Lq=128, Lk=128, d=64, causal=0, sm=0.125, qbr=128,
               flags=0):
    return sage.load_library().sage_attn_fwd_varlen(A, A, A, out, A, A, B, H, Hkv, Lq, Lk, d,
                                                    causal, sm, qbr, flags, S)


def prequant_varlen(qbr=128, flags=0, causal=0):
    return sage.load_library().sage_attn_fwd_prequant_varlen(A, A, A, A, A, A, A, A, 1, 2, 2,
                                                             128, 128, 64, causal, qbr, flags, S)


def quant_qk(Lk=128, d=64):
    return sage.load_library().sage_quant_qk(A, A, A, A, A, A, A, 1, 2, 2, 128, Lk, d, 0.125, S)


def quant_qk_qblock(Lk=128, qbr=1):
    return sage.load_library().sage_quant_qk_qblock(A, A, A, A, A, A, A, 1, 2, 2, 128, Lk, 64,
                                                    0.125, qbr, S)


def fwd(Lk=128, H=2, Lq=128):
    return sage.load_library().sage_attn_fwd(A, A, A, A, 1, H, 2, Lq, Lk, 64, 0, 0.125, S)


def fwd_host(Lk=128):
    return sage.load_library().sage_attn_fwd_host(A, A, A, A, 1, 2, 2, 128, Lk, 64, 0, 0.125, S)


def decode(Lk=1024):
    return sage.load_library().sage_attn_decode(A, A, A, A, 1, 8, 2, 1, Lk, 128, 1, 0.125, 1, S)


def noalloc(q=A, out=A, B=1, H=2, Hkv=2, Lq=128, Lk=128, d=64, causal=0, sm=0.125):
    return sage.load_library().sage_attn_fwd_noalloc(q, A, A, out, B, H, Hkv, Lq, Lk, d, causal,
                                                     sm, S)


LONG_K = (1 << 20) + 1   # one key past the quantizing calls' limit


def quant_v_fp8(v8t=A, vs=A, d=64, Lk=128):
    return sage.load_library().sage_quant_v_fp8(A, v8t, vs, 1, 2, Lk, d, N, 0, S)


def decode_varlen(H=8, Hkv=2, Lq=1, causal=0, qbr=1):
    return sage.load_library().sage_attn_decode_prequant_varlen(A, A, A, A, A, A, A, 1, H, Hkv,
                                                                Lq, 1024, 128, causal, qbr, N, 0,
                                                                S)


def decode_paged(num_pages=16, max_blocks=8, table=A, lens=A, H=8, Hkv=2, Lq=1, qbr=1):
    return sage.load_library().sage_attn_decode_prequant_paged(A, A, A, A, A, table, lens, A, 2,
                                                               H, Hkv, Lq, num_pages, max_blocks,
                                                               128, 1, qbr, N, 0, S)


CASES = [
    ("quant_k: no keys", lambda: quant_k(Lk=0), INVALID),
    ("quant_k: d = 96", lambda: quant_k(d=96), UNSUPPORTED),
    ("quant_k: null K", lambda: quant_k(k=N), INVALID),
    ("quant_k: misaligned k_i8", lambda: quant_k(ki=M), INVALID),
    ("quant_qk_varlen: sm_scale 0", lambda: quant_qk_varlen(sm=0.0), INVALID),
    ("quant_qk_varlen: block height 48", lambda: quant_qk_varlen(qbr=48), INVALID),
    ("quant_qk_varlen: null q_scale", lambda: quant_qk_varlen(qs=N), INVALID),
    ("quant_qk_varlen: H % Hkv != 0", lambda: quant_qk_varlen(H=3), INVALID),
    ("fwd_varlen: both P V variants", lambda: fwd_varlen(flags=3), INVALID),
    ("fwd_varlen: unknown flag", lambda: fwd_varlen(flags=8), INVALID),
    ("fwd_varlen: causal 2", lambda: fwd_varlen(causal=2), INVALID),
    ("fwd_varlen: sm_scale inf", lambda: fwd_varlen(sm=math.inf), INVALID),
    ("fwd_varlen: sm_scale nan", lambda: fwd_varlen(sm=math.nan), INVALID),
    ("fwd_varlen: d = 80", lambda: fwd_varlen(d=80), UNSUPPORTED),
    ("fwd_varlen: misaligned out", lambda: fwd_varlen(out=M), INVALID),
    ("fwd_varlen: no batch", lambda: fwd_varlen(B=0), INVALID),
    ("prequant_varlen: FP8 takes E4M3 V", lambda: prequant_varlen(flags=sage.SAGE_PV_FP8),
     INVALID),
    ("prequant_varlen: block height 0", lambda: prequant_varlen(qbr=0), INVALID),
    ("prequant_varlen: causal -1", lambda: prequant_varlen(causal=-1), INVALID),
    ("quant_v_fp8: d = 96", lambda: quant_v_fp8(d=96), UNSUPPORTED),
    ("quant_v_fp8: null v8t", lambda: quant_v_fp8(v8t=N), INVALID),
    ("quant_v_fp8: misaligned v_scale", lambda: quant_v_fp8(vs=M), INVALID),
    ("decode: 16 heads x 9 queries > one tile", lambda: decode_varlen(H=16, Hkv=1, Lq=9),
     UNSUPPORTED),
    ("decode: causal 3", lambda: decode_varlen(causal=3), INVALID),
    ("decode: block height 2", lambda: decode_varlen(qbr=2), INVALID),
    ("paged: no pages", lambda: decode_paged(num_pages=0), INVALID),
    ("paged: no block-table columns", lambda: decode_paged(max_blocks=0), INVALID),
    ("paged: null block table", lambda: decode_paged(table=N), INVALID),
    ("paged: null key counts", lambda: decode_paged(lens=N), INVALID),
    ("paged: 16 heads x 9 queries > one tile", lambda: decode_paged(H=16, Hkv=1, Lq=9),
     UNSUPPORTED),
    ("paged: H % Hkv != 0", lambda: decode_paged(H=6, Hkv=4), INVALID),
    # the Lk limit of the calls that smooth and quantize K
    ("quant_qk: Lk over the limit", lambda: quant_qk(Lk=LONG_K), UNSUPPORTED),
    ("quant_qk_qblock: Lk over the limit", lambda: quant_qk_qblock(Lk=LONG_K), UNSUPPORTED),
    ("quant_qk_varlen: Lk over the limit", lambda: quant_qk_varlen(Lk=LONG_K), UNSUPPORTED),
    ("quant_k: Lk over the limit", lambda: quant_k(Lk=LONG_K), UNSUPPORTED),
    ("fwd: Lk over the limit", lambda: fwd(Lk=LONG_K), UNSUPPORTED),
    ("fwd_varlen: Lk over the limit", lambda: fwd_varlen(Lk=LONG_K), UNSUPPORTED),
    ("fwd_host: Lk over the limit", lambda: fwd_host(Lk=LONG_K), UNSUPPORTED),
    ("decode: Lk over the limit", lambda: decode(Lk=LONG_K), UNSUPPORTED),
    ("noalloc: Lk over the limit", lambda: noalloc(Lk=LONG_K), UNSUPPORTED),
    # shapes whose element counts do not fit the kernels' index types
    ("fwd: over 2^40 query elements", lambda: fwd(H=1024, Lq=(1 << 31) - 1), INVALID),
    ("noalloc: huge B*H", lambda: noalloc(B=1 << 20, H=1 << 10, Hkv=1 << 10), INVALID),
    # the no-allocation entry point checks what sage_attn_fwd checks
    ("noalloc: H % Hkv != 0", lambda: noalloc(H=3), INVALID),
    ("noalloc: d = 96", lambda: noalloc(d=96), UNSUPPORTED),
    ("noalloc: null q", lambda: noalloc(q=N), INVALID),
    ("noalloc: misaligned out", lambda: noalloc(out=M), INVALID),
    ("noalloc: causal 2", lambda: noalloc(causal=2), INVALID),
    ("noalloc: sm_scale nan", lambda: noalloc(sm=math.nan), INVALID),
    ("noalloc: sm_scale -1", lambda: noalloc(sm=-1.0), INVALID),
    ("noalloc: scratch over 64 MiB", lambda: noalloc(H=64, Hkv=64, Lq=4096, Lk=4096, d=128),
     INVALID),
]


@pytest.mark.parametrize("what,call,want", CASES, ids=[c[0] for c in CASES])
def test_rejected_before_the_device(what, call, want):
    got = call()
    assert got == want, f"{what}: {sage.sage_status_string(got)}"
    assert sage.sage_last_launch_count() == 0


def test_workspace_sizes_of_the_newer_calls():
    # FP8 V maxima: one uint32 per (batch, kv head, channel), 256-byte rounded
    assert sage.sage_quant_v_fp8_workspace_size(2, 4, 128) == 4096
    assert sage.sage_quant_v_fp8_workspace_size(1, 1, 64) == 256
    # decoding layout: unsupported shapes report 0
    assert sage.sage_attn_decode_workspace_size(1, 16, 1, 9, 256, 64) == 0
    assert sage.sage_attn_decode_workspace_size(1, 8, 8, 1, 256, 96) == 0
