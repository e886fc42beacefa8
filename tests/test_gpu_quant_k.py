"""GPU parity of the K-only quantization call (K smoothing and 64-row INT8
blocks, the K half of the SageAttention article's quantization step): bit
for bit the K outputs of the joint Q/K call and of the oracle."""
import numpy as np
import pytest

import oracle
import bit_quantized_attention_mean_b200 as sage
from bit_quantized_attention_mean_b200 import inputs

from test_gpu_parity import to_dev, torch_mod

pytestmark = pytest.mark.gpu

SHAPES = [
    # B, H, Hkv, Lq, Lk, d
    (1, 2, 2, 300, 200, 64),      # ragged last K block
    (2, 4, 2, 333, 333, 128),     # GQA
    (1, 3, 1, 130, 520, 128),     # one kv head: 16-CTA clusters
    (1, 2, 2, 260, 70, 64),
    (1, 1, 1, 1, 1, 128),         # a single key
    (1, 8, 8, 1024, 1024, 128),
    # more K blocks per CTA than the per-block extremes in shared memory
    # cover (32 at d = 128, 64 at d = 64): the two-blocks-at-a-time pass
    (1, 1, 1, 1, 40000, 128),
    (1, 2, 1, 1, 70001, 64),
]


@pytest.mark.parametrize("shape", SHAPES)
def test_quant_k_equals_joint_quantization_and_oracle(shape):
    torch = torch_mod()
    B, H, Hkv, Lq, Lk, d = shape
    q, k, _ = inputs.make_custom(B, H, Hkv, Lq, Lk, d, seed=Lk + 3, k_offset_sigma=3.0)
    dq, dk = to_dev(q), to_dev(k)
    ki = torch.empty(dk.shape, dtype=torch.int8, device="cuda")
    ks = torch.empty((B, Hkv, -(-Lk // 64)), dtype=torch.float32, device="cuda")
    km = torch.empty((B, Hkv, d), dtype=torch.float32, device="cuda")
    sage.sage_quant_k(dk, ki, ks, km)
    _, ki2, _, ks2, km2 = sage.quant_qk(dq, dk, 0.1)
    sage.sage_check_device_status()
    assert torch.equal(ki, ki2)
    assert torch.equal(ks.view(torch.int32), ks2.view(torch.int32))
    assert torch.equal(km.view(torch.int32), km2.view(torch.int32))
    want = oracle.quant_qk(q, k, 0.1)
    assert np.array_equal(ki.cpu().numpy(), want[1])
    assert np.array_equal(ks.cpu().numpy().view(np.uint32), want[3].view(np.uint32))
    assert np.array_equal(km.cpu().numpy().view(np.uint32), want[4].view(np.uint32))
