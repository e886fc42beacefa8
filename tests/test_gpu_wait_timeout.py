"""Failure detection on the GPU without a fault: a kernel's bounded wait on a
barrier that nothing completes gives up after its limit, records the event in
the device status word, and the context stays usable."""
import math

import numpy as np
import pytest

import oracle
import bit_quantized_attention_mean_b200 as sage
from bit_quantized_attention_mean_b200 import inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sage.sage_check_device_status()              # start from a clean status word
    sage.sage_debug_wait_timeout(50)
    with pytest.raises(sage.SageError) as e:
        sage.sage_check_device_status()
    assert e.value.status == 4                   # SAGE_ERR_TIMEOUT
    sage.sage_check_device_status()              # the check cleared it
    with pytest.raises(sage.SageError):
        sage.sage_debug_wait_timeout(0)          # outside 1..2000 ms
    # the context is still usable: a normal forward pass matches the oracle
    q, k, v = inputs.make_custom(1, 2, 2, 200, 200, 64, seed=3)
    out = sage.attention(*(torch.from_numpy(x).cuda() for x in (q, k, v)), True, 0.125)
    sage.sage_check_device_status()
    sim, _ = oracle.attention(q, k, v, True, 0.125)
    assert np.max(np.abs(out.cpu().numpy().astype(np.float64) - sim)) <= 1e-2
