"""Blocks where the max element's error dominates, and items that mix huge and tiny blocks.

The fused kernels sum every element's squared error per block and then move the first max
element's share to SSE_max; where that share dominates the block, the elements below the maximum
are summed apart, and where fp32 squares could underflow (tiny blocks next to huge ones in one
item) the item is redone in double.  These inputs drive exactly those branches.

The dominant-max blocks have a closed form (scale 1.0 in both formats): the maximum 6.3125 sits
above 6 S = 6 (error 0.3125, one clipped element), one element 0.50390625 is one bf16 ulp above the
grid point 0.5 (error 2^-8), every other element is on the grid (error 0); rows of the second kind
repeat the maximum, whose copy goes to SSE_elem.  The CPU test pins the oracle to that closed form;
the GPU tests compare the CUDA path with the oracle (bit-exact codes, 1e-5 on the sums).
"""
import numpy as np
import pytest
import torch

import oracle

GRID = (0.5, -1.5, 3.0, -4.0, 1.0, 2.0, -0.5, 6.0, 0.0, -1.0, 1.5, -3.0, 4.0, -2.0, -6.0, 0.0)
A, OFF = 6.3125, 0.50390625
BLOCKS = (4, 8, 16, 32, 64, 128, 256)


def dominant_max_rows(block, rows):
    """rows x (2 block) values: per row two blocks, the first with one maximum, the second with a
    repeated maximum (tie); signs alternate by row."""
    out = np.zeros((rows, 2 * block), np.float32)
    for r in range(rows):
        sgn = -1.0 if r & 1 else 1.0
        for b in range(2):
            v = [sgn * A, OFF] + [GRID[(k + r) % len(GRID)] for k in range(block - 2)]
            if b == 1:
                v[block - 1] = -sgn * A  # the tie, opposite sign (same |x|)
            out[r, b * block:(b + 1) * block] = v
    return out


def to_bf16_bits(a):
    return torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("block", BLOCKS)
@pytest.mark.parametrize("fmt", (oracle.E4M3, oracle.UE5M3))
def test_oracle_dominant_max_closed_form(block, fmt):
    rows = 6
    x = dominant_max_rows(block, rows)
    xb = to_bf16_bits(x)
    assert np.array_equal(torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).float().numpy(), x)
    st = oracle.error_stats(xb.reshape(-1), rows, 2 * block, block, fmt)
    dmax2, off2 = 0.3125 ** 2, 2.0 ** -16
    nb = 2 * rows
    assert st["sse_max"] == nb * dmax2
    assert st["sse_elem"] == nb * off2 + rows * dmax2  # the ties' copies of dmax^2
    assert st["sse_zero"] == 0.0
    assert st["n_elem_sat"] == nb + rows  # every maximum (and its tie) is above 6 S = 6
    assert st["n_zero_blocks"] == 0 and st["n_scale_sat"] == 0
    _, scales = oracle.quantize(xb.reshape(-1), rows, 2 * block, block, fmt)
    assert np.all(scales == (0x38 if fmt == oracle.E4M3 else 0x78))  # the scale 1.0


@pytest.mark.gpu
@pytest.mark.parametrize("block", BLOCKS)
@pytest.mark.parametrize("fmt", (oracle.E4M3, oracle.UE5M3))
def test_gpu_dominant_max_blocks(cuda_device, block, fmt):
    from gpu_helpers import full_check
    rows = 67  # several CTAs' items and a ragged last warp
    x = torch.from_numpy(dominant_max_rows(block, rows)).to(torch.bfloat16).to(cuda_device)
    full_check(x, block, fmt)


@pytest.mark.gpu
@pytest.mark.parametrize("block", BLOCKS)
@pytest.mark.parametrize("fmt", (oracle.E4M3, oracle.UE5M3))
def test_gpu_huge_and_tiny_blocks(cuda_device, block, fmt):
    # consecutive blocks alternate between magnitudes near 1e30 and near 1e-30 (a zero-scale block
    # with E4M3), so one item of the small-block kernel holds both
    from gpu_helpers import full_check
    rng = np.random.default_rng(block + 10 * fmt)
    rows, nblk = 33, 4
    x = rng.standard_normal((rows, nblk * block)).astype(np.float32)
    for b in range(nblk):
        x[:, b * block:(b + 1) * block] *= 1e30 if b % 2 == 0 else 1e-30
    full_check(torch.from_numpy(x).to(torch.bfloat16).to(cuda_device), block, fmt)
