"""Pins of the oracle's block quantizer, dequantizer and error reduction.

* Exhaustive brute force: every N=4 block over a 16-value grid (65,536 blocks) that holds exact
  ties, the zero-scale threshold and saturation points is checked against a nearest-value rule
  evaluated in exact rational arithmetic, with the candidate values taken from library decoders.
* Invariants on seeded random tensors: |y| <= 6*S*g, zero scale => signed-zero block, the code's
  sign is x's sign, the three error sums add up to sum (x-y)^2 computed here with numpy, the max
  term equals a numpy argmax recomputation, counts, idempotence on normal scales.
"""
import math
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
from fp4_microscaling_tensor_b200 import inputs

# ----------------------------------------------------------------------------------------------
# candidate value tables from libraries (not from the oracle)
# ----------------------------------------------------------------------------------------------

E2M1_MAGS = [Fraction(float(v)) for v in
             np.arange(8, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)]
E4M3_VALS = [Fraction(float(v)) for v in
             torch.arange(0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()]
_h = np.array([((c >> 3) << 10) | ((c & 7) << 7) for c in range(0xF8)], np.uint16).view(np.float16)
UE5M3_VALS = [Fraction(float(v)) for v in _h.astype(np.float64)]
UE5M3_VALS += [2 * v for v in UE5M3_VALS[0xF0:0xF8]]  # exponent field 31 = twice field 30
SCALE_VALS = {oracle.E4M3: E4M3_VALS, oracle.UE5M3: UE5M3_VALS}


def nearest_even(u, table):
    """Index of the nearest table value to the Fraction u; ties -> even index; saturating."""
    if u >= table[-1]:
        return len(table) - 1
    best, bestd = 0, abs(u - table[0])
    for i, v in enumerate(table):
        d = abs(u - v)
        if d < bestd or (d == bestd and i % 2 == 0):
            best, bestd = i, d
    return best


def bf16_bits(v):
    return int(torch.tensor([v], dtype=torch.float64).to(torch.bfloat16).view(torch.int16)
               .numpy().view(np.uint16)[0])


def bf16_value(bits):
    return float(torch.tensor([bits], dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
                 .double()[0])


def grid_values(fmt, g):
    smin = float(SCALE_VALS[fmt][1])
    smax = float(SCALE_VALS[fmt][-1])
    t0 = bf16_bits(3 * smin * g)               # zero-scale threshold (or its bf16 neighbour)
    t1 = t0 + 1                                # one bf16 ulp above
    sat = bf16_bits(6 * smax * g)
    raw = [0.0, -0.0, bf16_value(t0), bf16_value(t1), -0.25 * g, 0.75 * g, 1.25 * g, -1.75 * g,
           2.5 * g, 3.5 * g, -5.0 * g, 6.0 * g, 0.3125 * g, bf16_value(sat),
           -bf16_value(bf16_bits(1.2 * 6 * smax * g)), bf16_value(bf16_bits(1e-3 * g))]
    bits = [bf16_bits(v) if not (v == 0 and math.copysign(1, v) < 0) else 0x8000 for v in raw]
    return np.array(bits, np.uint16)


CASES = [(oracle.E4M3, 0x3C00), (oracle.UE5M3, 0x3C00), (oracle.UE5M3, 0x0C00),
         (oracle.E4M3, 0x3A00)]


@pytest.mark.parametrize("fmt,g_bits", CASES)
def test_bruteforce_all_n4_blocks(fmt, g_bits):
    g = oracle.fp16_value(g_bits)
    gf = Fraction(g)
    gv = grid_values(fmt, g)
    vals = [bf16_value(int(b)) for b in gv]
    absf = [abs(Fraction(v)) for v in vals]
    table = SCALE_VALS[fmt]
    # scale code for each possible block max, element magnitude code for each (element, max)
    sc = [nearest_even(a / (6 * gf), table) for a in absf]
    ec = np.zeros((16, 16), np.int64)
    for j in range(16):
        S = table[sc[j]]
        for i in range(16):
            ec[i, j] = 0 if S == 0 else nearest_even(absf[i] / (S * gf), E2M1_MAGS)
    # every block of 4 grid values
    idx = np.stack(np.meshgrid(*[np.arange(16)] * 4, indexing="ij"), -1).reshape(-1, 4)
    x = gv[idx].reshape(-1)
    packed, scales = oracle.quantize(x, idx.shape[0], 4, 4, fmt, g_bits)
    A = np.array([float(a) for a in absf])
    jmax = idx[np.arange(idx.shape[0]), np.argmax(A[idx], axis=1)]
    exp_scale = np.array(sc)[jmax]
    assert np.array_equal(scales, exp_scale.astype(np.uint8))
    sign = (np.array([math.copysign(1, v) < 0 for v in vals])[idx]).astype(np.int64) << 3
    exp_codes = (ec[idx, jmax[:, None]] | sign).reshape(-1)
    codes = np.empty(x.size, np.int64)
    codes[0::2] = packed & 15
    codes[1::2] = packed >> 4
    assert np.array_equal(codes, exp_codes)


# ----------------------------------------------------------------------------------------------
# invariants on seeded random tensors
# ----------------------------------------------------------------------------------------------

def _codes(packed):
    c = np.empty(packed.size * 2, np.int64)
    c[0::2] = packed & 15
    c[1::2] = packed >> 4
    return c


RAND_CASES = [
    (0.005, 4, oracle.E4M3, 0x3C00), (0.005, 32, oracle.E4M3, 0x3C00),
    (0.02, 16, oracle.UE5M3, 0x3C00), (0.1, 256, oracle.E4M3, 0x3C00),
    (0.02, 32, oracle.UE5M3, 0x0003), (1.0, 8, oracle.E4M3, 0x2E66), (300.0, 64, oracle.E4M3, 0x3C00),
]


@pytest.mark.parametrize("sigma,block,fmt,g_bits", RAND_CASES)
def test_invariants_random(sigma, block, fmt, g_bits):
    rows, cols = 48, 1024
    xt = inputs.normal((rows, cols), sigma, seed=int(sigma * 1000) + block)
    x = inputs.to_oracle(xt)
    xd = xt.double().numpy().reshape(-1)
    g = oracle.fp16_value(g_bits)
    packed, scales = oracle.quantize(x, rows, cols, block, fmt, g_bits)
    y = oracle.dequantize(packed, scales, rows, cols, block, fmt, g_bits, out_bf16=False)
    yd = y.astype(np.float64)
    codes = _codes(packed)
    S = np.array([oracle.scale_value(s, fmt) for s in range(256)])[scales]
    Sel = np.repeat(S, block)
    # sign bit of every code is x's sign bit
    assert np.array_equal(codes >> 3, np.signbit(xd).astype(np.int64))
    # |y| <= 6 S g
    assert np.all(np.abs(yd) <= 6 * Sel * g)
    # zero scale -> signed zeros
    zb = Sel == 0
    assert np.all(yd[zb] == 0) and np.array_equal(np.signbit(yd[zb]), np.signbit(xd[zb]))
    # max element encodes to magnitude 6 whenever the scale is a normal value
    xb = xd.reshape(-1, block)
    first = np.argmax(np.abs(xb), axis=1)
    smin_normal = 2.0 ** -6 if fmt == oracle.E4M3 else 2.0 ** -14
    normal = S >= smin_normal
    mag_at_max = codes.reshape(-1, block)[np.arange(xb.shape[0]), first] & 7
    assert np.all(mag_at_max[normal] == 7)
    # the three sums against numpy recomputations
    st = oracle.error_stats(x, rows, cols, block, fmt, g_bits)
    err = (xd - yd) ** 2
    total = err.sum()
    assert math.isclose(st["sse_elem"] + st["sse_max"] + st["sse_zero"], total, rel_tol=1e-12,
                        abs_tol=1e-300)
    eb = err.reshape(-1, block)
    zero_blocks = S == 0
    sse_max = eb[np.arange(eb.shape[0]), first][~zero_blocks].sum()
    sse_zero = (xb[zero_blocks] ** 2).sum()
    assert math.isclose(st["sse_max"], sse_max, rel_tol=1e-12, abs_tol=1e-300)
    assert math.isclose(st["sse_zero"], sse_zero, rel_tol=1e-12, abs_tol=1e-300)
    # counts
    a = np.abs(xb).max(axis=1)
    assert st["numel"] == rows * cols and st["n_blocks"] == rows * cols // block
    assert st["n_zero_blocks"] == int(zero_blocks.sum())
    smax = 448.0 if fmt == oracle.E4M3 else 122880.0
    assert st["n_scale_sat"] == int((a > 6 * g * smax).sum())
    assert st["n_elem_sat"] == int(((np.abs(xd) > 6 * Sel * g) & (Sel > 0)).sum())
    # stats from the stored codes equal stats recomputed from x
    st2 = oracle.error_stats(x, rows, cols, block, fmt, g_bits, packed=packed, scales=scales)
    assert st2 == st
    # idempotence on blocks with a normal scale: re-quantizing y gives the same codes and scale
    p2, s2 = oracle.quantize(y, rows, cols, block, fmt, g_bits)
    c2 = _codes(p2).reshape(-1, block)
    assert np.array_equal(s2[normal], scales[normal])
    assert np.array_equal(c2[normal], codes.reshape(-1, block)[normal])


def test_constant_block_on_grid_has_zero_error():
    # a = 6 * S_k for a representable scale S_k: every element sits on the grid
    for fmt, s in ((oracle.E4M3, 0x38), (oracle.UE5M3, 0x78), (oracle.UE5M3, 0x03)):
        S = oracle.scale_value(s, fmt)
        row = np.array([6 * S, -3 * S, 1.5 * S, -0.5 * S, 0.0, 4 * S, -2 * S, S], np.float32)
        packed, scales = oracle.quantize(row, 1, 8, 8, fmt)
        assert scales[0] == s
        st = oracle.error_stats(row, 1, 8, 8, fmt)
        assert st["sse_elem"] == 0 and st["sse_max"] == 0 and st["sse_zero"] == 0


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.UE5M3])
@pytest.mark.parametrize("g_bits", [0x3C00, 0x4400])
def test_zero_scale_threshold(fmt, g_bits):
    # a block is zeroed iff a <= 3 * g * smin (ties go to the even code 0)
    g = oracle.fp16_value(g_bits)
    thr = 3 * g * oracle.scale_min(fmt)
    for a, zero in ((thr, True), (float(np.nextafter(np.float32(thr), np.float32(1))), False)):
        row = np.array([a, -a / 2, a / 4, 0.0], np.float32)
        packed, scales = oracle.quantize(row, 1, 4, 4, fmt, g_bits)
        assert (scales[0] == 0) == zero
        st = oracle.error_stats(row, 1, 4, 4, fmt, g_bits)
        assert (st["n_zero_blocks"] == 1) == zero
        if zero:
            assert st["sse_zero"] == float(np.sum(row.astype(np.float64) ** 2))


def test_signed_zero_codes():
    row = np.array([-0.0, 0.0, -1e-30, 1.0], np.float32)
    packed, scales = oracle.quantize(row, 1, 4, 4, oracle.E4M3)
    assert list(_codes(packed)) == [8, 0, 8, 7]
    row = np.array([-0.0, 0.0, -0.0, 0.0], np.float32)  # all-zero block: zero scale, signs kept
    packed, scales = oracle.quantize(row, 1, 4, 4, oracle.UE5M3)
    assert scales[0] == 0 and list(_codes(packed)) == [8, 0, 8, 0]
    y = oracle.dequantize(packed, scales, 1, 4, 4, oracle.UE5M3, out_bf16=True)
    assert list(y) == [0x8000, 0, 0x8000, 0]


def test_dequant_bf16_is_rounded_fp32():
    # bf16 output is the round-to-nearest-even of the exact fp32 reconstruction
    rng = np.random.default_rng(5)
    rows, cols, block = 16, 256, 32
    packed = rng.integers(0, 256, rows * cols // 2, dtype=np.uint8)
    scales = rng.integers(0, 0x7F, rows * cols // block, dtype=np.uint8)
    for g_bits in (0x3C00, 0x3555, 0x0001):
        y32 = oracle.dequantize(packed, scales, rows, cols, block, oracle.E4M3, g_bits, out_bf16=False)
        y16 = oracle.dequantize(packed, scales, rows, cols, block, oracle.E4M3, g_bits, out_bf16=True)
        ref = torch.from_numpy(y32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(y16, ref)


def test_bad_arguments_rejected():
    x = np.zeros(64, np.float32)
    with pytest.raises(ValueError):
        oracle.quantize(x, 2, 32, 12, oracle.E4M3)       # block not a power of two in 4..256
    with pytest.raises(ValueError):
        oracle.quantize(x, 1, 64, 512, oracle.E4M3)      # block too large
    with pytest.raises(ValueError):
        oracle.quantize(x, 1, 64, 32, oracle.E4M3, 0x0000)  # g = 0
    with pytest.raises(ValueError):
        oracle.quantize(x, 1, 64, 32, oracle.E4M3, 0x7C00)  # g = inf
    with pytest.raises(ValueError):
        oracle.quantize(x, 1, 64, 32, oracle.E4M3, 0xBC00)  # g < 0
