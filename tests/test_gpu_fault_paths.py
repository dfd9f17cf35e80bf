"""Error paths on the GPU without faulting it: an injected launch failure surfaces as MXError
(MX_ERR_CUDA) through the Python binding, writes nothing (canary bytes around and inside the
outputs stay), and the next call runs normally with correct results."""
import numpy as np
import pytest
import torch

import oracle
import fp4_microscaling_tensor_b200 as mx
from fp4_microscaling_tensor_b200 import _lib, inputs

from gpu_helpers import assert_same, u8

pytestmark = pytest.mark.gpu


def test_injected_failure_then_recovery(cuda_device):
    x = inputs.workload2(2, shape=(64, 1024), device=cuda_device)
    packed = torch.full((64, 512), 0xA5, dtype=torch.uint8, device=cuda_device)
    scales = torch.full((64, 32), 0xA5, dtype=torch.uint8, device=cuda_device)
    _lib.lib.mx_test_fail_next_calls(1)
    with pytest.raises(mx.MXError) as err:
        mx.quantize(x, 32, mx.E4M3, packed=packed, scales=scales)
    assert err.value.status == _lib.MX_ERR_CUDA
    torch.cuda.synchronize()
    assert bool((packed == 0xA5).all()) and bool((scales == 0xA5).all())
    mx.quantize(x, 32, mx.E4M3, packed=packed, scales=scales)
    po, so = oracle.quantize(inputs.to_oracle(x), 64, 1024, 32, mx.E4M3)
    assert_same(u8(packed), po, "packed after recovery")
    assert_same(u8(scales), so, "scales after recovery")
    assert _lib.lib.mx_test_fail_next_calls(0) == 0
