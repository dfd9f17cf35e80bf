"""Pins of the oracle's block-scaled matrix product (dequantize both operands, then multiply).

The oracle's product is tied to decoders outside it: E2M1 codes through ml_dtypes, E4M3 scales
through torch.float8_e4m3fn, the global scales through numpy binary16, the nibble order and the
scale indexing written out here, and exact rational sums on tiny cases.  Special cases reduce the
product to a column selection and to a transpose.
"""
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle

E2M1 = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
E4M3 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()


def fp16(bits):
    return float(np.array([bits], np.uint16).view(np.float16)[0])


def decode(packed, scales, rows, cols, block, g_bits):
    """Values of a stored operand: element 2i is the low nibble of byte i, element 2i+1 the
    high nibble; block b of row r takes scales[r * cols / block + b]; everything times g."""
    codes = np.empty(rows * cols, np.uint8)
    codes[0::2] = packed & 0xF
    codes[1::2] = packed >> 4
    v = E2M1[codes].reshape(rows, cols)
    s = E4M3[scales].reshape(rows, cols // block)
    return v * np.repeat(s, block, axis=1) * fp16(g_bits)


def random_operand(rng, rows, cols, block):
    packed = rng.integers(0, 256, rows * cols // 2, dtype=np.uint8)
    scales = rng.integers(0, 0x7F, rows * cols // block, dtype=np.uint8)  # every finite E4M3 code
    return packed, scales


def test_brute_force_exact_sums():
    rng = np.random.default_rng(7)
    m, n, k, block = 3, 2, 32, 16
    ga, gb = 0x3C00, 0x3800  # 1.0 and 0.5
    pa, sa = random_operand(rng, m, k, block)
    pb, sb = random_operand(rng, n, k, block)
    A = decode(pa, sa, m, k, block, ga)
    B = decode(pb, sb, n, k, block, gb)
    C = oracle.matmul(pa, sa, ga, pb, sb, gb, m, n, k, block, oracle.E4M3)
    for i in range(m):
        for j in range(n):
            exact = sum(Fraction(float(A[i, t])) * Fraction(float(B[j, t])) for t in range(k))
            mag = sum(abs(Fraction(float(A[i, t])) * Fraction(float(B[j, t]))) for t in range(k))
            assert abs(Fraction(float(C[i, j])) - exact) <= mag * Fraction(1, 2 ** 48)


@pytest.mark.parametrize("shape", [(17, 9, 64), (5, 33, 256)])
def test_matches_independent_decode(shape):
    rng = np.random.default_rng(sum(shape))
    m, n, k = shape
    pa, sa = random_operand(rng, m, k, 16)
    pb, sb = random_operand(rng, n, k, 16)
    ga, gb = 0x3C00, 0x4400  # 1.0, 4.0
    C = oracle.matmul(pa, sa, ga, pb, sb, gb, m, n, k, 16, oracle.E4M3)
    ref = decode(pa, sa, m, k, 16, ga) @ decode(pb, sb, n, k, 16, gb).T
    mag = np.abs(decode(pa, sa, m, k, 16, ga)) @ np.abs(decode(pb, sb, n, k, 16, gb)).T
    assert np.all(np.abs(C - ref) <= mag * 2.0 ** -45)


def test_one_hot_columns_select_a():
    # row j of B holds 1.0 (code 0x2, scale 0x38 = 1.0) at column j and +0 elsewhere, so column
    # j of the product is column j of dequant(A)
    rng = np.random.default_rng(3)
    m, n, k = 9, 32, 64
    pa, sa = random_operand(rng, m, k, 16)
    codes = np.zeros((n, k), np.uint8)
    codes[np.arange(n), np.arange(n)] = 0x2
    flat = codes.reshape(-1)
    pb = (flat[0::2] | (flat[1::2] << 4)).astype(np.uint8)
    sb = np.full(n * k // 16, 0x38, np.uint8)
    C = oracle.matmul(pa, sa, 0x3C00, pb, sb, 0x3C00, m, n, k, 16, oracle.E4M3)
    A = decode(pa, sa, m, k, 16, 0x3C00)
    assert np.array_equal(C, A[:, :n])


def test_transpose_symmetry():
    rng = np.random.default_rng(11)
    m, n, k = 7, 12, 48
    pa, sa = random_operand(rng, m, k, 16)
    pb, sb = random_operand(rng, n, k, 16)
    C = oracle.matmul(pa, sa, 0x3C00, pb, sb, 0x3A00, m, n, k, 16, oracle.E4M3)
    Ct = oracle.matmul(pb, sb, 0x3A00, pa, sa, 0x3C00, n, m, k, 16, oracle.E4M3)
    assert np.array_equal(C, Ct.T)


def test_integer_sums_are_exact():
    # scales 1.0 and g = 1: every value is a multiple of 0.5 with |v| <= 6, so every partial sum
    # is a multiple of 0.25 below 2^24 and the product is exact in any order
    rng = np.random.default_rng(5)
    m, n, k = 8, 8, 256
    pa = rng.integers(0, 256, m * k // 2, dtype=np.uint8)
    pb = rng.integers(0, 256, n * k // 2, dtype=np.uint8)
    s1 = np.full(m * k // 16, 0x38, np.uint8)
    C = oracle.matmul(pa, s1, 0x3C00, pb, s1[: n * k // 16], 0x3C00, m, n, k, 16, oracle.E4M3)
    A = decode(pa, s1, m, k, 16, 0x3C00)
    B = decode(pb, s1[: n * k // 16], n, k, 16, 0x3C00)
    exact = [[sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(A[i], B[j]))
              for j in range(n)] for i in range(m)]
    assert all(Fraction(float(C[i, j])) == exact[i][j] for i in range(m) for j in range(n))


# ---- bf16 activations x stored FP4 weights (oracle.dequant_matmul) ----

_H = np.array([((c >> 3) << 10) | ((c & 7) << 7) for c in range(0xF8)], np.uint16).view(np.float16)
UE5M3 = np.concatenate([_H.astype(np.float64), 2 * _H[0xF0:0xF8].astype(np.float64)])


def decode_w_bf16(packed, scales, rows, cols, block, fmt, g_bits):
    """Weights as the product sees them: E2M1 (ml_dtypes) x scale (torch E4M3 / the UE5M3 table
    built from binary16 patterns) x g (numpy binary16), rounded to bfloat16 by torch."""
    codes = np.empty(rows * cols, np.uint8)
    codes[0::2] = packed & 0xF
    codes[1::2] = packed >> 4
    table = E4M3 if fmt == oracle.E4M3 else UE5M3
    v = E2M1[codes].reshape(rows, cols) * np.repeat(table[scales].reshape(rows, cols // block),
                                                    block, axis=1) * fp16(g_bits)
    return torch.from_numpy(v).to(torch.bfloat16).double().numpy()


def bf16_bits(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16).reshape(-1)


def random_weights(rng, rows, cols, block, fmt):
    packed = rng.integers(0, 256, rows * cols // 2, dtype=np.uint8)
    hi = 0x7F if fmt == oracle.E4M3 else 0x100
    scales = rng.integers(0, hi, rows * cols // block, dtype=np.uint8)
    return packed, scales


@pytest.mark.parametrize("block,fmt,g", [(4, oracle.UE5M3, 0x0003), (32, oracle.UE5M3, 0x1234),
                                         (256, oracle.E4M3, 0x3C00), (16, oracle.E4M3, 0x4400)])
def test_dequant_matmul_matches_independent_decode(block, fmt, g):
    rng = np.random.default_rng(block + 3 * fmt)
    m, n, k = 5, 9, 512
    a = rng.standard_normal((m, k)) * np.exp(rng.uniform(-4, 4, (m, 1)))
    ab = bf16_bits(a)
    pw, sw = random_weights(rng, n, k, block, fmt)
    C = oracle.dequant_matmul(ab, m, k, pw, sw, n, block, fmt, g)
    A = torch.from_numpy(ab.view(np.int16)).view(torch.bfloat16).double().numpy().reshape(m, k)
    W = decode_w_bf16(pw, sw, n, k, block, fmt, g)
    mag = np.abs(A) @ np.abs(W).T
    assert np.all(np.abs(C - A @ W.T) <= mag * 2.0 ** -45)


def test_dequant_matmul_exact_rational_sums():
    rng = np.random.default_rng(21)
    m, n, k, block = 3, 4, 64, 32
    ab = bf16_bits(rng.standard_normal((m, k)))
    pw, sw = random_weights(rng, n, k, block, oracle.UE5M3)
    C = oracle.dequant_matmul(ab, m, k, pw, sw, n, block, oracle.UE5M3, 0x2E66)
    A = torch.from_numpy(ab.view(np.int16)).view(torch.bfloat16).double().numpy().reshape(m, k)
    W = decode_w_bf16(pw, sw, n, k, block, oracle.UE5M3, 0x2E66)
    for i in range(m):
        for j in range(n):
            exact = sum(Fraction(float(A[i, t])) * Fraction(float(W[j, t])) for t in range(k))
            mag = sum(abs(Fraction(float(A[i, t])) * Fraction(float(W[j, t]))) for t in range(k))
            assert abs(Fraction(float(C[i, j])) - exact) <= mag * Fraction(1, 2 ** 48)


def test_dequant_matmul_one_hot_rows_select_weights():
    # row i of A is 1.0 at column i: row i of the product is column i of the bf16 weights
    rng = np.random.default_rng(8)
    n, k, block = 11, 128, 64
    m = 40
    a = np.zeros((m, k), np.float32)
    a[np.arange(m), np.arange(m)] = 1.0
    pw, sw = random_weights(rng, n, k, block, oracle.UE5M3)
    C = oracle.dequant_matmul(bf16_bits(a), m, k, pw, sw, n, block, oracle.UE5M3, 0x3555)
    yw = oracle.bf16_values(oracle.dequantize(pw, sw, n, k, block, oracle.UE5M3, 0x3555,
                                              out_bf16=True)).reshape(n, k)
    assert np.array_equal(C, yw[:, :m].T)


def test_dequant_matmul_reduces_to_the_fp4_product():
    # activations that are themselves a stored FP4 tensor (block 16, E4M3, g = 1: every value is
    # exact in bf16) against E4M3 weights with g = 1 (exact in bf16 too): the same product as
    # oracle.matmul of the two stored tensors
    rng = np.random.default_rng(13)
    m, n, k = 6, 10, 256
    pa, sa = random_operand(rng, m, k, 16)
    pb, sb = random_operand(rng, n, k, 16)
    ya = oracle.dequantize(pa, sa, m, k, 16, oracle.E4M3, out_bf16=True)
    C = oracle.dequant_matmul(ya, m, k, pb, sb, n, 16, oracle.E4M3)
    ref = oracle.matmul(pa, sa, 0x3C00, pb, sb, 0x3C00, m, n, k, 16, oracle.E4M3)
    assert np.array_equal(C, ref)
