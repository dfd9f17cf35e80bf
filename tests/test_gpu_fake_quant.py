"""Fake quantization (quantize -> dequantize in one pass) against the oracle's quantize followed by
its dequantize: bit-exact output for every block size, format, input and output type, with
special values, global scales and the N = 4 tail; the straight-through gradient; and the
activation configuration (bf16 16384x8192, N = 16, E4M3) whole."""
import numpy as np
import pytest
import torch

import oracle
import fp4_microscaling_tensor_b200 as mx
from fp4_microscaling_tensor_b200 import inputs

from gpu_helpers import BLOCKS, FMTS, assert_same, bits, special_values_bf16

pytestmark = pytest.mark.gpu


def reference(x, block, fmt, g, out_bf16):
    rows, cols = x.shape
    xo = inputs.to_oracle(x)
    po, so = oracle.quantize(xo, rows, cols, block, fmt, g)
    yo = oracle.dequantize(po, so, rows, cols, block, fmt, g, out_bf16=out_bf16)
    return yo if out_bf16 else yo.view(np.uint32)


@pytest.mark.parametrize("block", BLOCKS)
@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("xdt", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("ydt", [torch.bfloat16, torch.float32])
def test_fake_quantize_matches_oracle(cuda_device, block, fmt, xdt, ydt):
    for g in (0x3C00, 0x3555, 0x0003):
        n = 3 * 4096 + (4 if block == 4 else 0)
        x = special_values_bf16(fmt, g, n, seed=block + 17 * fmt).to(xdt).reshape(1, -1)
        x = x.to(cuda_device)
        y = mx.fake_quantize(x, block, fmt, g, out_dtype=ydt)
        ref = reference(x, block, fmt, g, ydt == torch.bfloat16)
        assert_same(bits(y), ref, f"fake quantize N={block} fmt={fmt} {xdt}->{ydt} g={g:#x}")


def test_straight_through_gradient(cuda_device):
    x = inputs.workload2(2, shape=(64, 256), device=cuda_device).float().requires_grad_(True)
    y = mx.FakeQuantize.apply(x, 32, "e4m3")
    assert_same(bits(y.detach()),
                reference(x.detach(), 32, mx.E4M3, 0x3C00, out_bf16=False), "autograd forward")
    g = torch.randn_like(y)
    y.backward(g)
    assert torch.equal(x.grad, g)


def test_config4_round_trip(cuda_device):
    x = inputs.workload4(device=cuda_device)
    y = mx.fake_quantize(x, 16, mx.E4M3)
    assert_same(bits(y), reference(x, 16, mx.E4M3, 0x3C00, True), "config 4 round trip")
