"""Pins of the oracle's ragged last blocks (cols not a multiple of the block size N).

Reading: a row is cut into blocks of N from its first element and its last block holds the
cols mod N remaining elements, with its own absmax, scale and the same element rule.  Two facts
tie that to the (separately pinned) whole-block quantizer and to exact arithmetic:

* padding invariance: appending zeros to a row up to a whole number of blocks changes no scale,
  no code of a real element, no error sum and no count (a zero never raises the absmax, encodes to
  +0 exactly and adds nothing to any sum), so the ragged result must equal the padded result;
* brute force: short blocks of bf16 grid values (ties, thresholds, saturation) against the
  nearest-value rule in exact rational arithmetic, with candidate values from library decoders.

The byte layout (rows of ceil(cols/2) code bytes, an odd last element leaving the high nibble 0,
ceil(cols/N) scale bytes per row) is checked with an unpacker written here.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
from test_oracle_quantizer import E2M1_MAGS, SCALE_VALS, bf16_value, grid_values, nearest_even


def unpack_rows(packed, rows, cols):
    pb = (cols + 1) // 2
    p = packed.reshape(rows, pb)
    codes = np.empty((rows, 2 * pb), np.int64)
    codes[:, 0::2] = p & 15
    codes[:, 1::2] = p >> 4
    return codes


def bf16_rows(rng, rows, cols, scale):
    x = (rng.standard_normal((rows, cols)) * scale *
         np.exp(rng.uniform(-3, 1, (rows, 1)))).astype(np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)  # truncation to bf16 bits (any values do)


CASES = [(4, 7), (8, 13), (16, 9), (32, 45), (64, 100), (128, 129), (256, 300), (32, 3),
         (4, 2), (16, 1)]


@pytest.mark.parametrize("block,cols", CASES)
@pytest.mark.parametrize("fmt,g_bits", [(oracle.E4M3, 0x3C00), (oracle.UE5M3, 0x3C00),
                                        (oracle.E4M3, 0x2E66)])
def test_padding_invariance(block, cols, fmt, g_bits):
    rng = np.random.default_rng(block * 1000 + cols)
    rows = 5
    x = bf16_rows(rng, rows, cols, 0.05)
    nb = -(-cols // block)
    colsp = nb * block
    xp = np.zeros((rows, colsp), np.uint16)
    xp[:, :cols] = x
    p, s = oracle.quantize(x.reshape(-1), rows, cols, block, fmt, g_bits)
    pp, sp = oracle.quantize(xp.reshape(-1), rows, colsp, block, fmt, g_bits)
    assert p.size == rows * ((cols + 1) // 2) and s.size == rows * nb
    assert np.array_equal(s, sp)
    c, cp = unpack_rows(p, rows, cols), unpack_rows(pp, rows, colsp)
    assert np.array_equal(c[:, :cols], cp[:, :cols])
    if cols % 2:  # the spare high nibble of an odd row is 0
        assert np.all(c[:, cols] == 0)
    y = oracle.dequantize(p, s, rows, cols, block, fmt, g_bits, out_bf16=False).reshape(rows, cols)
    yp = oracle.dequantize(pp, sp, rows, colsp, block, fmt, g_bits,
                           out_bf16=False).reshape(rows, colsp)
    assert np.array_equal(y, yp[:, :cols])
    st = oracle.error_stats(x.reshape(-1), rows, cols, block, fmt, g_bits)
    stp = oracle.error_stats(xp.reshape(-1), rows, colsp, block, fmt, g_bits)
    for k in ("sse_elem", "sse_max", "sse_zero", "n_blocks", "n_zero_blocks", "n_scale_sat",
              "n_elem_sat"):
        assert st[k] == stp[k], k
    assert st["numel"] == rows * cols
    # stored codes give the same record
    assert oracle.error_stats(x.reshape(-1), rows, cols, block, fmt, g_bits, packed=p,
                              scales=s) == st


@pytest.mark.parametrize("fmt,g_bits", [(oracle.E4M3, 0x3C00), (oracle.UE5M3, 0x3C00)])
@pytest.mark.parametrize("length", [1, 2, 3, 5, 7])
def test_bruteforce_short_last_blocks(fmt, g_bits, length):
    # rows of 8 + length elements with N = 8: a whole block of zeros, then a short block drawn
    # from the 16-value grid (ties, thresholds, saturation)
    g = oracle.fp16_value(g_bits)
    gf = Fraction(g)
    gv = grid_values(fmt, g)
    vals = [bf16_value(int(b)) for b in gv]
    table = SCALE_VALS[fmt]
    rng = np.random.default_rng(length + 10 * fmt)
    rows, cols = 400, 8 + length
    pick = rng.integers(0, 16, (rows, length))
    x = np.zeros((rows, cols), np.uint16)
    x[:, 8:] = gv[pick]
    p, s = oracle.quantize(x.reshape(-1), rows, cols, 8, fmt, g_bits)
    codes = unpack_rows(p, rows, cols)
    s = s.reshape(rows, 2)
    for r in range(rows):
        blk = [Fraction(vals[i]) for i in pick[r]]
        a = max(abs(v) for v in blk)
        sc = nearest_even(a / (6 * gf), table)
        assert s[r, 1] == sc
        S = table[sc]
        for i, v in enumerate(blk):
            mag = 0 if S == 0 else nearest_even(abs(v) / (S * gf), E2M1_MAGS)
            sign = 8 if math.copysign(1, vals[pick[r, i]]) < 0 else 0
            assert codes[r, 8 + i] == (mag | sign)
