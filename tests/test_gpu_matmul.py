"""Parity of the tensor-core block-scaled matrix product (mx_matmul) with the oracle.

Operands are seeded random E2M1 codes and E4M3 scales (or the oracle's quantization of seeded
Gaussian data), built on the host and copied to the device; the oracle multiplies the same bytes.

* Exact cases: with unit scales and g = 1 every value is a multiple of 0.5 and every partial sum a
  multiple of 0.25 far below 2^24, so the float32 result is exact in any summation order and must
  equal the oracle bit for bit.  Cases whose scales vary only by row or only by k-block (powers of
  two) stay exact too and pin the scale placement of each operand separately.
* General cases: the tensor core accumulates k products in float32 in an unspecified order; each
  product of two dequantized values is exact, so the error is bounded by the float32 summation
  bound k * 2^-23 * sum |a b| (twice the round-to-nearest bound, allowing truncating adders), plus
  one rounding of the final scaling by gA gB (2^-24 |c|) and, for bfloat16 output, 2^-8 |c|.
"""
import functools

import numpy as np
import pytest
import torch

import fp4_microscaling_tensor_b200 as mx
import oracle
from fp4_microscaling_tensor_b200 import _lib, inputs
from fp4_microscaling_tensor_b200 import api as mx_api

pytestmark = pytest.mark.gpu


@pytest.fixture(params=["one_cta", "cta_pairs"], autouse=True)
def kernel(request, monkeypatch):
    """Every test runs with both kernels: mx_matmul and mx_matmul_pair (CTA pairs for m > 128)."""
    monkeypatch.setattr(mx, "matmul", functools.partial(mx_api.matmul,
                                                        cta_pairs=request.param == "cta_pairs"))
    return request.param

ONE = 0x38  # E4M3 code of 1.0


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def run(pa, sa, pb, sb, m, n, k, ag=0x3C00, bg=0x3C00, out_dtype=torch.float32):
    c = mx.matmul(dev(pa).view(m, k // 2), dev(sa).view(m, k // 16), dev(pb).view(n, k // 2),
                  dev(sb).view(n, k // 16), a_g=ag, b_g=bg, out_dtype=out_dtype)
    torch.cuda.synchronize()
    return c.float().cpu().numpy().astype(np.float64)


def codes(rng, rows, k):
    return rng.integers(0, 256, rows * k // 2, dtype=np.uint8)


def magnitude(pa, sa, ag, pb, sb, bg, m, n, k):
    """sum_t |a_it| |b_jt|, from the oracle's dequantized operands."""
    ya = np.abs(oracle.dequantize(pa, sa, m, k, 16, oracle.E4M3, ag, out_bf16=False))
    yb = np.abs(oracle.dequantize(pb, sb, n, k, 16, oracle.E4M3, bg, out_bf16=False))
    return ya.astype(np.float64).reshape(m, k) @ yb.astype(np.float64).reshape(n, k).T


def check_bound(got, ref, mag, k, bf16):
    tol = k * 2.0 ** -23 * mag + 2.0 ** -24 * np.abs(ref)
    if bf16:
        tol = tol + 2.0 ** -8 * np.abs(ref)
    err = np.abs(got - ref)
    worst = np.unravel_index(np.argmax(err - tol), err.shape)
    assert np.all(err <= tol), (f"max excess at {worst}: got {got[worst]}, oracle {ref[worst]}, "
                                f"bound {tol[worst]}")


@pytest.mark.parametrize("case", ["unit", "a_rows", "a_kblocks", "b_rows", "b_kblocks"])
def test_exact_structured_scales(case):
    rng = np.random.default_rng(["unit", "a_rows", "a_kblocks", "b_rows", "b_kblocks"].index(case))
    m, n, k = 256, 256, 512
    pa, pb = codes(rng, m, k), codes(rng, n, k)
    sa = np.full((m, k // 16), ONE, np.uint8)
    sb = np.full((n, k // 16), ONE, np.uint8)
    pow2 = np.array([0x30, 0x38, 0x40, 0x48], np.uint8)  # 0.25, 1, 4, 16: sums stay exact
    if case == "a_rows":
        sa[:] = pow2[rng.integers(0, 4, m)][:, None]
    elif case == "a_kblocks":
        sa[:] = pow2[rng.integers(0, 4, k // 16)][None, :]
    elif case == "b_rows":
        sb[:] = pow2[rng.integers(0, 4, n)][:, None]
    elif case == "b_kblocks":
        sb[:] = pow2[rng.integers(0, 4, k // 16)][None, :]
    sa, sb = sa.reshape(-1), sb.reshape(-1)
    got = run(pa, sa, pb, sb, m, n, k)
    ref = oracle.matmul(pa, sa, 0x3C00, pb, sb, 0x3C00, m, n, k, 16, oracle.E4M3)
    assert np.array_equal(got, ref), f"{np.sum(got != ref)} of {got.size} differ"
    assert mx.matmul_gave_up() == 0


@pytest.mark.parametrize("shape", [(128, 128, 256), (256, 384, 4096), (200, 72, 768),
                                   (37, 45, 256), (1, 8, 512), (300, 1, 256)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_random_codes_and_scales(shape, out_dtype):
    m, n, k = shape
    rng = np.random.default_rng(m * 7 + n * 13 + k)
    pa, pb = codes(rng, m, k), codes(rng, n, k)
    # every finite E4M3 code but the extremes of the range, so sums stay far from overflow
    sa = rng.integers(0x10, 0x70, m * k // 16, dtype=np.uint8)
    sb = rng.integers(0x10, 0x70, n * k // 16, dtype=np.uint8)
    ag, bg = 0x4000, 0x3800  # 2.0, 0.5
    got = run(pa, sa, pb, sb, m, n, k, ag, bg, out_dtype)
    ref = oracle.matmul(pa, sa, ag, pb, sb, bg, m, n, k, 16, oracle.E4M3)
    check_bound(got, ref, magnitude(pa, sa, ag, pb, sb, bg, m, n, k), k,
                out_dtype == torch.bfloat16)
    assert mx.matmul_gave_up() == 0


def test_quantized_gaussian_layer():
    # a 512 x 2048 activation times a 768 x 2048 weight, both quantized by the oracle from seeded
    # Gaussian data with their own global scales
    m, n, k = 512, 768, 2048
    xa = inputs.normal((m, k), 0.5, seed=4100)
    xb = inputs.normal((n, k), 0.02, seed=4101)
    ga = oracle.global_scale(inputs.to_oracle(xa), oracle.E4M3)
    gb = oracle.global_scale(inputs.to_oracle(xb), oracle.E4M3)
    pa, sa = oracle.quantize(inputs.to_oracle(xa), m, k, 16, oracle.E4M3, ga)
    pb, sb = oracle.quantize(inputs.to_oracle(xb), n, k, 16, oracle.E4M3, gb)
    got = run(pa, sa, pb, sb, m, n, k, ga, gb)
    ref = oracle.matmul(pa, sa, ga, pb, sb, gb, m, n, k, 16, oracle.E4M3)
    check_bound(got, ref, magnitude(pa, sa, ga, pb, sb, gb, m, n, k), k, False)
    assert mx.matmul_gave_up() == 0


def test_large_square_sampled_rows():
    # 4096^3 in the launch configuration the benchmark times; the oracle recomputes 64 seeded rows
    m = n = k = 4096
    rng = np.random.default_rng(4096)
    pa, pb = codes(rng, m, k), codes(rng, n, k)
    sa = rng.integers(0x28, 0x48, m * k // 16, dtype=np.uint8)
    sb = rng.integers(0x28, 0x48, n * k // 16, dtype=np.uint8)
    got = run(pa, sa, pb, sb, m, n, k)
    rows = np.sort(rng.choice(m, 64, replace=False))
    pa_r = pa.reshape(m, k // 2)[rows].reshape(-1)
    sa_r = sa.reshape(m, k // 16)[rows].reshape(-1)
    ref = oracle.matmul(pa_r, sa_r, 0x3C00, pb, sb, 0x3C00, len(rows), n, k, 16, oracle.E4M3)
    check_bound(got[rows], ref, magnitude(pa_r, sa_r, 0x3C00, pb, sb, 0x3C00, len(rows), n, k), k,
                False)
    assert mx.matmul_gave_up() == 0


def test_consumes_quantize_output_directly():
    # the library's own quantizer writes the operands; the product equals the oracle's product of
    # the oracle's quantization of the same data (the quantizer is bit-exact, checked elsewhere)
    m, n, k = 256, 128, 1024
    xa = inputs.normal((m, k), 1.0, seed=4200)
    xb = inputs.normal((n, k), 1.0, seed=4201)
    pa_d, sa_d = mx.quantize(xa.cuda(), 16, "e4m3")
    pb_d, sb_d = mx.quantize(xb.cuda(), 16, "e4m3")
    got = mx.matmul(pa_d, sa_d, pb_d, sb_d, out_dtype=torch.float32).double().cpu().numpy()
    pa, sa = oracle.quantize(inputs.to_oracle(xa), m, k, 16, oracle.E4M3)
    pb, sb = oracle.quantize(inputs.to_oracle(xb), n, k, 16, oracle.E4M3)
    ref = oracle.matmul(pa, sa, 0x3C00, pb, sb, 0x3C00, m, n, k, 16, oracle.E4M3)
    check_bound(got, ref, magnitude(pa, sa, 0x3C00, pb, sb, 0x3C00, m, n, k), k, False)


def test_empty_and_unsupported():
    a = torch.zeros((0, 128), dtype=torch.uint8, device="cuda")
    s = torch.zeros((0, 16), dtype=torch.uint8, device="cuda")
    b = torch.zeros((8, 128), dtype=torch.uint8, device="cuda")
    bs = torch.zeros((8, 16), dtype=torch.uint8, device="cuda")
    assert mx.matmul(a, s, b, bs).shape == (0, 8)
    b2 = torch.zeros((8, 64), dtype=torch.uint8, device="cuda")
    s2 = torch.zeros((8, 8), dtype=torch.uint8, device="cuda")
    with pytest.raises((mx.MXError, ValueError)):
        mx.matmul(b2, s2, b2, s2)  # k = 128: not a multiple of 256
    with pytest.raises(mx.MXError):
        mx.matmul(b2, s2, b2, s2, prepared=True)


@pytest.mark.parametrize("rows,k", [(128, 256), (300, 768), (1, 512)])
def test_prepared_scale_layout(rows, k):
    # tensor-core order, written out here: tile t (256-row padded), step kt, group j, then
    # row 32 q + r of the tile at byte 16 r + 4 q, its 4 scales of group j in order
    rng = np.random.default_rng(rows + k)
    sc = rng.integers(0, 0x7F, (rows, k // 16), dtype=np.uint8)
    got = mx.prepare_scales(dev(sc), k).cpu().numpy()
    tiles = 2 * ((rows + 255) // 256)
    pad = np.zeros((tiles * 128, k // 16), np.uint8)
    pad[:rows] = sc
    ref = np.zeros((tiles, k // 256, 4, 32, 4, 4), np.uint8)
    for t in range(tiles):
        for kt in range(k // 256):
            for j in range(4):
                for q in range(4):
                    ref[t, kt, j, :, q, :] = pad[t * 128 + 32 * q: t * 128 + 32 * q + 32,
                                                 16 * kt + 4 * j: 16 * kt + 4 * j + 4]
    assert got.size == ref.size
    assert np.array_equal(got, ref.reshape(-1))


def test_abandoned_launch_leaves_later_launches_alone():
    """A launch marked as abandoned (as a thread block whose bounded waits ran out marks it) must
    not make a later launch stop waiting.  One long tile (k = 2^18: each CTA waits for its whole
    main loop, far beyond the polls after which an abandoned launch's waits give up) is run, its
    launch marked, then run again: the result is the same bit for bit and nothing gave up."""
    rng = np.random.default_rng(11)
    m, n, k = 256, 256, 1 << 18
    pa, pb = codes(rng, m, k), codes(rng, n, k)
    sa = np.full((m, k // 16), ONE, np.uint8)
    sb = np.full((n, k // 16), ONE, np.uint8)
    first = run(pa, sa, pb, sb, m, n, k)
    assert mx.matmul_gave_up() == 0
    assert _lib.lib.mx_test_matmul_abandon_last() == _lib.MX_OK
    second = run(pa, sa, pb, sb, m, n, k)
    assert mx.matmul_gave_up() == 0
    assert np.array_equal(first, second)
