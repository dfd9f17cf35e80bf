"""Parity at the workload configurations' full sizes, whole tensors, through the launches the
benchmark times.

Every tensor is drawn on the GPU with the seeded generators of `inputs.py` and copied to the host
for the oracle.  Every tensor is compared whole: codes, scales and dequantized bits bit-exact, and
the error record term by term (sse_elem, sse_max and sse_zero each within 1e-5 relative, the counts
exactly) against the oracle's record for the same codes.

Configurations (sizes as the workloads state them):
  2  bf16 4096x4096 x 5 sigma, N in {4..256} x {E4M3, UE5M3}: all 70 points, through the grouped
     fused pass and grouped dequantize the benchmark's sweep launches (one launch per (N, format)
     over the five sigma tensors).
  3  Llama-2-7B-shaped weights (32 layers x 7 tensors, Student-t rows), N = 32, UE5M3 + per-tensor
     global scale: all 224 tensors, per layer the grouped global scale, fused pass and dequantize
     with g kept in device memory.
  4  activations bf16 16384x8192 with outlier channels, N = 16, E4M3: quantize, dequantize and
     the error record.
  5  Llama-2-70B-shaped layers (2 x 8192^2, 2 x 1024x8192, 3 x 8192x28672), N = 32, UE5M3 + global
     scale: the eight layers 0, 1, 13, 27, 40, 53, 66, 79, through the benchmark's three grouped
     launches per layer (global scale -> fused pass -> dequantize, g in device memory).
"""
import numpy as np
import pytest
import torch

import oracle
import fp4_microscaling_tensor_b200 as mx
from fp4_microscaling_tensor_b200 import inputs

from gpu_helpers import assert_same, assert_stats, bits, u8

pytestmark = pytest.mark.gpu


def check_whole(x, p, s, st, y, block, fmt, g, what):
    """Codes, scales, dequantized bits and the error record of one tensor against the oracle."""
    rows, cols = x.shape
    xo = inputs.to_oracle(x)
    po, so = oracle.quantize(xo, rows, cols, block, fmt, g)
    assert_same(u8(s), so, f"{what} scales")
    assert_same(u8(p), po, f"{what} packed")
    yo = oracle.dequantize(po, so, rows, cols, block, fmt, g, out_bf16=True)
    assert_same(bits(y), yo, f"{what} dequant")
    ref = oracle.error_stats(xo, rows, cols, block, fmt, g, packed=po, scales=so)
    assert_stats(st, ref, f"{what} stats")


def layer_launches(xs, block, fmt):
    """The benchmark's three grouped launches over one layer: global scales into device memory,
    the fused pass and dequantize reading them there.  Returns (g bits, packed, scales, records,
    dequantized)."""
    g = mx.global_scale_group(xs, fmt)
    p, s, st = mx.quantize_with_stats_group(xs, block, fmt, g=g)
    y = mx.dequantize_group(p, s, block, fmt, g=g)
    gh = [int(v) for v in g.cpu().numpy().view(np.uint16)]
    return gh, p, s, [t.to_dict() for t in st], y


@pytest.mark.parametrize("block", inputs.SWEEP_BLOCKS)
@pytest.mark.parametrize("fmt", (mx.E4M3, mx.UE5M3))
def test_config2_sweep_whole(cuda_device, block, fmt):
    xs = [inputs.workload2(k, device=cuda_device) for k in range(len(inputs.SWEEP_SIGMAS))]
    p, s, st = mx.quantize_with_stats_group(xs, block, fmt)
    y = mx.dequantize_group(p, s, block, fmt)
    for k, x in enumerate(xs):
        what = f"config 2 sigma={inputs.SWEEP_SIGMAS[k]} N={block} fmt={fmt}"
        check_whole(x, p[k], s[k], st[k].to_dict(), y[k], block, fmt, 0x3C00, what)


@pytest.mark.parametrize("layer", range(32))
def test_config3_llama7b_weights_whole(cuda_device, layer):
    xs = [inputs.workload3_tensor(layer, j, device=cuda_device)
          for j in range(len(inputs.LLAMA7B_SHAPES))]
    gh, p, s, st, y = layer_launches(xs, 32, mx.UE5M3)
    for j, x in enumerate(xs):
        what = f"config 3 layer {layer} tensor {j}"
        assert gh[j] == oracle.global_scale(inputs.to_oracle(x), oracle.UE5M3), what
        check_whole(x, p[j], s[j], st[j], y[j], 32, mx.UE5M3, gh[j], what)


def test_config4_activations_whole(cuda_device):
    x = inputs.workload4(device=cuda_device)
    p, s, st = mx.quantize_with_stats(x, 16, mx.E4M3)
    y = mx.dequantize(p, s, 16, mx.E4M3)
    check_whole(x, p, s, st.to_dict(), y, 16, mx.E4M3, 0x3C00, "config 4")
    # the plain quantize kernel writes the same codes
    p2, s2 = mx.quantize(x, 16, mx.E4M3)
    assert torch.equal(p2, p) and torch.equal(s2, s)


@pytest.mark.parametrize("layer", [0, 1, 13, 27, 40, 53, 66, 79])
def test_config5_llama70b_layer_whole(cuda_device, layer):
    xs = [inputs.workload5_tensor(layer, j, device=cuda_device)
          for j in range(len(inputs.LLAMA70B_SHAPES))]
    gh, p, s, st, y = layer_launches(xs, 32, mx.UE5M3)
    for j, x in enumerate(xs):
        what = f"config 5 layer {layer} tensor {j}"
        assert gh[j] == oracle.global_scale(inputs.to_oracle(x), oracle.UE5M3), what
        check_whole(x, p[j], s[j], st[j], y[j], 32, mx.UE5M3, gh[j], what)
    del xs, p, s, y
    torch.cuda.empty_cache()
