"""Parity of the bf16-activation x FP4-weight tensor-core product (mx_dequant_matmul) with the
oracle (oracle.dequant_matmul: the weights' bf16 dequantization, then a float64 multiply).

Weights are stored by the library's own quantizer (every block size, both scale formats, global
scales from the library's rule) or are seeded random codes and scales; activations are bf16.

* Exact cases: activations that are small integers and weights with unit scales and g = 1 give
  products that are multiples of 0.5 and partial sums far below 2^22, exact in float32 in any
  summation order: the result must equal the oracle bit for bit.
* General cases: each product of a bf16 activation and a bf16 weight is exact in float32; the
  tensor core sums k of them in float32 in an unspecified order, so the error is bounded by
  k * 2^-23 * sum |a w| (twice the round-to-nearest bound, allowing truncating adders), plus
  2^-8 |c| for bfloat16 output.
"""
import numpy as np
import pytest
import torch

import fp4_microscaling_tensor_b200 as mx
import oracle
from fp4_microscaling_tensor_b200 import inputs

pytestmark = pytest.mark.gpu

BLOCKS = (4, 8, 16, 32, 64, 128, 256)


def bits16(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1)


def magnitude(a, pw, sw, n, k, block, fmt, g):
    A = np.abs(oracle.bf16_values(bits16(a)).reshape(a.shape[0], k))
    W = np.abs(oracle.bf16_values(oracle.dequantize(pw, sw, n, k, block, fmt, g, out_bf16=True))
               ).reshape(n, k)
    return A @ W.T


def check(c, ref, mag, k, bf16):
    got = c.float().cpu().numpy().astype(np.float64)
    tol = k * 2.0 ** -23 * mag + (2.0 ** -8 * np.abs(ref) if bf16 else 0.0)
    err = np.abs(got - ref)
    worst = np.unravel_index(np.argmax(err - tol), err.shape)
    assert np.all(err <= tol), (f"max excess at {worst}: got {got[worst]}, oracle {ref[worst]}, "
                                f"bound {tol[worst]}")


def quantized_weights(n, k, block, fmt, seed, device, sigma=0.02):
    w = inputs.student_t4_rowgain((n, k), seed, sigma=sigma, device=device)
    g = int(mx.global_scale(w, fmt).item()) & 0xFFFF if fmt == mx.UE5M3 else 0x3C00
    pw, sw = mx.quantize(w, block, fmt, g)
    return pw, sw, g


@pytest.mark.parametrize("block", BLOCKS)
@pytest.mark.parametrize("fmt", (mx.E4M3, mx.UE5M3))
def test_every_block_size_and_format(cuda_device, block, fmt):
    m, n, k = 300, 520, 512  # m, n not multiples of the 256 x 256 tile
    pw, sw, g = quantized_weights(n, k, block, fmt, seed=block + 7 * fmt, device=cuda_device)
    a = inputs.normal((m, k), 1.0, seed=block, device=cuda_device)
    for out_dtype in (torch.float32, torch.bfloat16):
        c = mx.dequant_matmul(a, pw, sw, block, fmt, g, out_dtype=out_dtype)
        assert mx.matmul_gave_up() == 0  # (synchronizes) no wait ran out
        pwo, swo = pw.cpu().numpy().reshape(-1), sw.cpu().numpy().reshape(-1)
        ref = oracle.dequant_matmul(bits16(a), m, k, pwo, swo, n, block, fmt, g)
        check(c, ref, magnitude(a, pwo, swo, n, k, block, fmt, g), k,
              out_dtype == torch.bfloat16)
    assert mx.matmul_gave_up() == 0


def test_exact_integer_sums(cuda_device):
    rng = np.random.default_rng(5)
    m, n, k, block = 256, 256, 1024, 32
    a = torch.from_numpy(rng.integers(-3, 4, (m, k)).astype(np.float32)).to(torch.bfloat16)
    pw = rng.integers(0, 256, n * k // 2, dtype=np.uint8)
    sw = np.full(n * k // block, 0x38, np.uint8)  # E4M3 1.0
    c = mx.dequant_matmul(a.to(cuda_device), torch.from_numpy(pw).view(n, k // 2).to(cuda_device),
                          torch.from_numpy(sw).view(n, k // block).to(cuda_device), block,
                          mx.E4M3, out_dtype=torch.float32)
    ref = oracle.dequant_matmul(bits16(a), m, k, pw, sw, n, block, oracle.E4M3)
    assert np.array_equal(c.cpu().numpy().astype(np.float64), ref)
    assert mx.matmul_gave_up() == 0


def test_random_codes_all_scales(cuda_device):
    """Random code bytes and every scale code (UE5M3: all 256; E4M3: the finite 127) with a small
    and a large global scale."""
    rng = np.random.default_rng(9)
    m, n, k, block = 129, 257, 256, 16
    a = inputs.normal((m, k), 1.0, seed=3, device=cuda_device)
    for fmt, g in ((mx.UE5M3, 0x0001), (mx.E4M3, 0x5A00)):
        hi = 0x100 if fmt == mx.UE5M3 else 0x7F
        pw = rng.integers(0, 256, n * k // 2, dtype=np.uint8)
        sw = rng.integers(0, hi, n * k // block, dtype=np.uint8)
        c = mx.dequant_matmul(a, torch.from_numpy(pw).view(n, k // 2).to(cuda_device),
                              torch.from_numpy(sw).view(n, k // block).to(cuda_device), block,
                              fmt, g, out_dtype=torch.float32)
        ref = oracle.dequant_matmul(bits16(a), m, k, pw, sw, n, block, fmt, g)
        check(c, ref, magnitude(a, pw, sw, n, k, block, fmt, g), k, False)


def test_device_global_scale(cuda_device):
    """g read on the device (the output of the global-scale kernel) gives the same product as the
    same g passed by value."""
    m, n, k, block = 64, 384, 1024, 32
    w = inputs.workload5_tensor(0, 2, shape=(n, k), device=cuda_device)
    gd = mx.global_scale(w, mx.UE5M3)
    g = int(gd.item()) & 0xFFFF
    pw, sw = mx.quantize(w, block, mx.UE5M3, g)
    a = inputs.normal((m, k), 1.0, seed=4, device=cuda_device)
    c1 = mx.dequant_matmul(a, pw, sw, block, mx.UE5M3, g, out_dtype=torch.float32)
    c2 = mx.dequant_matmul(a, pw, sw, block, mx.UE5M3, gd, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(c1, c2)


def test_llama70b_layer_weights_sampled(cuda_device):
    """One 70B-shaped weight (8192 x 8192, N = 32, UE5M3 + its global scale) against 512 bf16
    activation rows; the oracle checks the first, last and seeded middle rows of C whole."""
    n = k = 8192
    m, block = 512, 32
    w = inputs.workload5_tensor(0, 0, device=cuda_device)
    g = int(mx.global_scale(w, mx.UE5M3).item()) & 0xFFFF
    pw, sw = mx.quantize(w, block, mx.UE5M3, g)
    a = inputs.normal((m, k), 1.0, seed=70, device=cuda_device)
    c = mx.dequant_matmul(a, pw, sw, block, mx.UE5M3, g, out_dtype=torch.float32)
    torch.cuda.synchronize()
    rows = sorted({0, m - 1, 255, 256, *np.random.default_rng(1).choice(m, 4, replace=False)})
    pwo, swo = pw.cpu().numpy().reshape(-1), sw.cpu().numpy().reshape(-1)
    yw = oracle.bf16_values(oracle.dequantize(pwo, swo, n, k, block, oracle.UE5M3, g,
                                              out_bf16=True)).reshape(n, k)
    A = oracle.bf16_values(bits16(a[rows])).reshape(len(rows), k)
    ref = A @ yw.T
    check(c[rows], ref, np.abs(A) @ np.abs(yw).T, k, False)
    assert mx.matmul_gave_up() == 0


def test_empty_and_unsupported(cuda_device):
    a = torch.zeros(4, 128, dtype=torch.bfloat16, device=cuda_device)
    pw = torch.zeros(8, 64, dtype=torch.uint8, device=cuda_device)
    sw = torch.zeros(8, 4, dtype=torch.uint8, device=cuda_device)
    assert mx.dequant_matmul(a[:0], pw, sw, 32, mx.E4M3).shape == (0, 8)
    with pytest.raises(mx.MXError):  # k = 96 is not a multiple of 64
        mx.dequant_matmul(torch.zeros(4, 96, dtype=torch.bfloat16, device=cuda_device),
                          torch.zeros(8, 48, dtype=torch.uint8, device=cuda_device),
                          torch.zeros(8, 3, dtype=torch.uint8, device=cuda_device), 32, mx.E4M3)
