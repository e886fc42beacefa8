"""sage_attn_fwd_noalloc: the forward pass for callers that cannot allocate
device memory at call time (a server that reserved its memory budget at
start-up, a plugin host that gives the library no allocator).

Its scratch is one fixed array inside the library, shared by every call, so
the test makes two calls in a row with different problems (the second must
not see anything the first left behind) and checks each against the regular
sage_attn_fwd, within the parity tolerance the other GPU tests use.  It also
checks that a problem too large for the array is refused without touching the
output.  This file is collected last and must pass both alone in a fresh
process and after the other tests.
"""
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
        assert sage.sage_attn_workspace_size(B, H, Hkv, Lq, Lk, d) <= sage.NOALLOC_SCRATCH_BYTES
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
    assert sage.sage_attn_workspace_size(B, H, Hkv, L, L, d) > sage.NOALLOC_SCRATCH_BYTES
    q = torch.zeros((B, H, L, d), dtype=torch.float16, device="cuda")
    out = torch.full_like(q, 7.0)
    with pytest.raises(sage.SageError) as e:
        sage.sage_attn_fwd_noalloc(q, q, q, out, False, 0.088)
    assert e.value.status == 1
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())
