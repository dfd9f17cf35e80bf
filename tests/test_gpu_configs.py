"""Parity at the workload configurations' full sizes, through the launches the benchmark times.

Every tensor is drawn on the GPU with the seeded generators of `inputs.py` and copied to the host
for the oracle.  A configuration is either compared with the oracle over whole tensors (codes,
scales and dequantized bits bit-exact, the error record within 1e-5 relative, counts exact) or,
where a whole-tensor oracle run would take too long, on sampled rows (first, last and seeded
random rows) plus properties that hold at any size:

* the three error sums add up to sum((x - y)^2) over the tensor, y the exact (fp32) dequantized
  output (checked in float64 on the device), and the zero-scale sum to sum(x^2) over zero-scale
  blocks;
* n_blocks = numel / N and n_zero_blocks = the number of zero scale bytes.

Configurations (sizes as the workloads state them):
  2  bf16 4096x4096 x 5 sigma, N in {4..256} x {E4M3, UE5M3}: the 14 points of sigma = 0.02 whole,
     the other 56 sampled + properties.
  3  Llama-2-7B-shaped weights (32 layers x 7 tensors, Student-t rows), N = 32, UE5M3 + global
     scale: layer 0 whole, every layer sampled.
  4  activations bf16 16384x8192 with outlier channels, N = 16, E4M3: whole.
  5  Llama-2-70B-shaped layer (2 x 8192^2, 2 x 1024x8192, 3 x 8192x28672), N = 32, UE5M3 + global
     scale, with the error record: layer 0 whole; layers 1, 13, 27, 40, 53, 66, 79 sampled +
     properties.
"""
import numpy as np
import pytest
import torch

import oracle
import fp4_microscaling_tensor_b200 as mx
from fp4_microscaling_tensor_b200 import inputs

from gpu_helpers import assert_same, assert_stats, bits, u8

pytestmark = pytest.mark.gpu


def bench_launches(x, block, fmt, g=0x3C00):
    """The benchmark's two launches for one tensor: fused pass, then dequantize (bf16 out)."""
    p, s, st = mx.quantize_with_stats(x, block, fmt, g)
    y = mx.dequantize(p, s, block, fmt, g)
    return p, s, st.to_dict(), y


def sample_rows(rows, seed, k=6):
    rng = np.random.default_rng(seed)
    extra = rng.choice(rows, size=min(k, rows), replace=False).tolist()
    return sorted(set([0, rows - 1] + extra))


def check_rows(x, p, s, y, block, fmt, g, row_ids, what):
    """Codes, scales and dequantized bits of the chosen rows against the oracle, row by row."""
    cols = x.shape[1]
    for r in row_ids:
        xr = inputs.to_oracle(x[r:r + 1])
        po, so = oracle.quantize(xr, 1, cols, block, fmt, g)
        assert_same(u8(s[r]), so, f"{what} scales row {r}")
        assert_same(u8(p[r]), po, f"{what} packed row {r}")
        yo = oracle.dequantize(po, so, 1, cols, block, fmt, g, out_bf16=True)
        assert_same(bits(y[r]), yo, f"{what} dequant row {r}")


def check_whole(x, p, s, st, y, block, fmt, g, what):
    rows, cols = x.shape
    xo = inputs.to_oracle(x)
    po, so = oracle.quantize(xo, rows, cols, block, fmt, g)
    assert_same(u8(s), so, f"{what} scales")
    assert_same(u8(p), po, f"{what} packed")
    yo = oracle.dequantize(po, so, rows, cols, block, fmt, g, out_bf16=True)
    assert_same(bits(y), yo, f"{what} dequant")
    ref = oracle.error_stats(xo, rows, cols, block, fmt, g, packed=po, scales=so)
    assert_stats(st, ref, f"{what} stats")


def check_properties(x, p, s, st, block, fmt, g, what):
    """Size-independent identities between the error record and the tensors themselves (y is the
    exact fp32 dequantization of the stored codes)."""
    y = mx.dequantize(p, s, block, fmt, g, out_dtype=torch.float32)
    numel = x.numel()
    assert st["numel"] == numel and st["n_blocks"] == numel // block, what
    zero = (s == 0)
    assert st["n_zero_blocks"] == int(zero.sum()), what
    xd = x.double().reshape(-1, block)
    d2 = (xd - y.double().reshape(-1, block)).square().sum(dim=1)
    total = float(d2.sum())
    got = st["sse_elem"] + st["sse_max"] + st["sse_zero"]
    assert abs(got - total) <= 1e-5 * total, (what, got, total)
    zsum = float(xd.square().sum(dim=1)[zero.reshape(-1)].sum())
    assert abs(st["sse_zero"] - zsum) <= 1e-5 * max(zsum, 1e-300), (what, st["sse_zero"], zsum)


def test_config2_sweep(cuda_device):
    for k in range(len(inputs.SWEEP_SIGMAS)):
        x = inputs.workload2(k, device=cuda_device)
        for n in inputs.SWEEP_BLOCKS:
            for fmt in (mx.E4M3, mx.UE5M3):
                what = f"config 2 sigma={inputs.SWEEP_SIGMAS[k]} N={n} fmt={fmt}"
                p, s, st, y = bench_launches(x, n, fmt)
                if k == 2:
                    check_whole(x, p, s, st, y, n, fmt, 0x3C00, what)
                else:
                    check_rows(x, p, s, y, n, fmt, 0x3C00, sample_rows(x.shape[0], 17 * k + n),
                               what)
                    check_properties(x, p, s, st, n, fmt, 0x3C00, what)


def test_config3_llama7b_weights(cuda_device):
    for layer in range(32):
        for j in range(len(inputs.LLAMA7B_SHAPES)):
            x = inputs.workload3_tensor(layer, j, device=cuda_device)
            what = f"config 3 layer {layer} tensor {j}"
            g = int(mx.global_scale(x, mx.UE5M3).item()) & 0xFFFF
            if layer == 0:
                assert g == oracle.global_scale(inputs.to_oracle(x), mx.UE5M3), what
            p, s = mx.quantize(x, 32, mx.UE5M3, g)
            y = mx.dequantize(p, s, 32, mx.UE5M3, g)
            if layer == 0:
                xo = inputs.to_oracle(x)
                rows, cols = x.shape
                po, so = oracle.quantize(xo, rows, cols, 32, mx.UE5M3, g)
                assert_same(u8(s), so, what + " scales")
                assert_same(u8(p), po, what + " packed")
                yo = oracle.dequantize(po, so, rows, cols, 32, mx.UE5M3, g, out_bf16=True)
                assert_same(bits(y), yo, what + " dequant")
            else:
                check_rows(x, p, s, y, 32, mx.UE5M3, g, sample_rows(x.shape[0], layer, k=2), what)


def test_config4_activations(cuda_device):
    x = inputs.workload4(device=cuda_device)
    rows, cols = x.shape
    p, s = mx.quantize(x, 16, mx.E4M3)
    y = mx.dequantize(p, s, 16, mx.E4M3)
    xo = inputs.to_oracle(x)
    po, so = oracle.quantize(xo, rows, cols, 16, mx.E4M3)
    assert_same(u8(s), so, "config 4 scales")
    assert_same(u8(p), po, "config 4 packed")
    yo = oracle.dequantize(po, so, rows, cols, 16, mx.E4M3, out_bf16=True)
    assert_same(bits(y), yo, "config 4 dequant")


@pytest.mark.parametrize("layer", [0, 1, 13, 27, 40, 53, 66, 79])
def test_config5_llama70b_layer(cuda_device, layer):
    for j in range(len(inputs.LLAMA70B_SHAPES)):
        x = inputs.workload5_tensor(layer, j, device=cuda_device)
        what = f"config 5 layer {layer} tensor {j}"
        g = int(mx.global_scale(x, mx.UE5M3).item()) & 0xFFFF
        p, s, st, y = bench_launches(x, 32, mx.UE5M3, g)
        if layer == 0:
            assert g == oracle.global_scale(inputs.to_oracle(x), mx.UE5M3), what
            check_whole(x, p, s, st, y, 32, mx.UE5M3, g, what)
        else:
            check_rows(x, p, s, y, 32, mx.UE5M3, g, sample_rows(x.shape[0], 79 * layer + j, k=2),
                       what)
            check_properties(x, p, s, st, 32, mx.UE5M3, g, what)
        del x, p, s, y
        torch.cuda.empty_cache()
