"""sage_attn_fwd_noalloc: the forward pass for callers that cannot allocate
device memory at call time (a server that reserved its memory budget at
start-up, a plugin host that gives the library no allocator).

Its scratch is one fixed array inside the library, shared by every call, so
the test makes two calls in a row with different problems (the second must
not see anything the first left behind) and checks each against the regular
sage_attn_fwd, within the parity tolerance the other GPU tests use.  It also
checks that a problem too large for the array is refused without touching the
output, and that a warm call really allocates nothing: the high-water mark of
the device's default memory pool (where cudaMallocAsync takes memory) does
not move across two no-allocation calls, while the same instrument does see
the allocating entry point's scratch.  This file is collected last and must
pass both alone in a fresh process and after the other tests.
"""
import ctypes
import math

import numpy as np
import pytest

import bit_quantized_attention_mean_b200 as sage
from bit_quantized_attention_mean_b200 import inputs

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
COS = 0.9999


def _torch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _close(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    tol = np.maximum(MAX_ABS, np.spacing(np.abs(b).astype(np.float16)).astype(np.float64))
    assert np.all(np.abs(a - b) <= tol), float(np.abs(a - b).max())
    c = float((a.ravel() @ b.ravel()) / (np.linalg.norm(a) * np.linalg.norm(b)))
    assert c >= COS, c


def _problem(B, H, Hkv, Lq, Lk, d, seed):
    torch = _torch()
    q, k, v = inputs.make_custom(B, H, Hkv, Lq, Lk, d, seed=seed)
    return tuple(torch.from_numpy(x).cuda() for x in (q, k, v))


def test_noalloc_matches_allocating_entry_point_twice_in_a_row():
    torch = _torch()
    cases = [
        ((1, 32, 32, 4096, 4096, 128), True, 11),    # the LLM-sized problem, ~34 MB scratch
        ((2, 8, 2, 700, 900, 64), False, 12),        # different shape, GQA, ragged tails
    ]
    for (B, H, Hkv, Lq, Lk, d), causal, seed in cases:
        assert sage.sage_workspace_size(B, H, Hkv, Lq, Lk, d) <= sage.NOALLOC_SCRATCH_BYTES
        q, k, v = _problem(B, H, Hkv, Lq, Lk, d, seed)
        sm = 1.0 / math.sqrt(d)
        out_fixed = torch.full_like(q, float("nan"))
        sage.sage_attn_fwd_noalloc(q, k, v, out_fixed, causal, sm)
        out_alloc = torch.empty_like(q)
        sage.sage_attn_fwd(q, k, v, out_alloc, causal, sm)
        sage.sage_check_device_status()
        assert bool(torch.isfinite(out_fixed).all())
        _close(out_fixed, out_alloc)


def test_noalloc_refuses_problems_larger_than_its_array():
    torch = _torch()
    B, H, Hkv, L, d = 1, 64, 64, 4096, 128      # ~68 MB of scratch
    assert sage.sage_workspace_size(B, H, Hkv, L, L, d) > sage.NOALLOC_SCRATCH_BYTES
    q = torch.zeros((B, H, L, d), dtype=torch.float16, device="cuda")
    out = torch.full_like(q, 7.0)
    with pytest.raises(sage.SageError) as e:
        sage.sage_attn_fwd_noalloc(q, q, q, out, False, 0.088)
    assert e.value.status == 1
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())


# CUmemPool_attribute values (cuda.h): memory of the pool in use now, and its
# high-water mark since the last reset (setting it to 0 resets it to "now").
CU_MEMPOOL_ATTR_USED_MEM_CURRENT = 7
CU_MEMPOOL_ATTR_USED_MEM_HIGH = 8


class _DefaultPool:
    """The current device's default memory pool, through the driver API."""

    def __init__(self):
        self.cu = ctypes.CDLL("libcuda.so.1")
        dev = ctypes.c_int()
        assert self.cu.cuCtxGetDevice(ctypes.byref(dev)) == 0
        self.pool = ctypes.c_void_p()
        assert self.cu.cuDeviceGetDefaultMemPool(ctypes.byref(self.pool), dev) == 0

    def _get(self, attr):
        v = ctypes.c_uint64()
        assert self.cu.cuMemPoolGetAttribute(self.pool, attr, ctypes.byref(v)) == 0
        return v.value

    def used(self):
        return self._get(CU_MEMPOOL_ATTR_USED_MEM_CURRENT)

    def high(self):
        return self._get(CU_MEMPOOL_ATTR_USED_MEM_HIGH)

    def reset_high(self):
        z = ctypes.c_uint64(0)
        assert self.cu.cuMemPoolSetAttribute(self.pool, CU_MEMPOOL_ATTR_USED_MEM_HIGH,
                                             ctypes.byref(z)) == 0


def test_noalloc_warm_calls_take_no_device_memory():
    torch = _torch()
    B, H, Hkv, L, d = 1, 8, 8, 2048, 128
    q, k, v = _problem(B, H, Hkv, L, L, d, seed=13)
    out = torch.empty_like(q)
    sage.sage_attn_fwd_noalloc(q, k, v, out, True, 0.088)      # warm: first-call set-up
    sage.sage_attn_fwd(q, k, v, out, True, 0.088)
    launches = sage.sage_last_launch_count()
    assert launches >= 2                                        # quantization + attention
    torch.cuda.synchronize()
    pool = _DefaultPool()
    # control: the instrument sees the allocating entry point's scratch
    pool.reset_high()
    base = pool.high()
    sage.sage_attn_fwd(q, k, v, out, True, 0.088)
    torch.cuda.synchronize()
    assert pool.high() >= base + sage.sage_workspace_size(B, H, Hkv, L, L, d)
    # the no-allocation entry point: two calls, no pool memory at all
    pool.reset_high()
    base = pool.high()
    assert base == pool.used()
    for _ in range(2):
        sage.sage_attn_fwd_noalloc(q, k, v, out, True, 0.088)
        assert sage.sage_last_launch_count() == launches
    torch.cuda.synchronize()
    assert pool.high() == base
    sage.sage_check_device_status()
