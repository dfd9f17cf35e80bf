"""Pins of the oracle's number formats.

The oracle decodes E2M1 / E4M3 / UE5M3 / FP16 from closed forms and rounds by a nearest-value
search.  These tests tie both to something outside the oracle: library converters (ml_dtypes
E2M1, torch E4M3 / E5M2, numpy binary16), the facts the microscaling pages print
(tests/golden/page_facts.txt), and exact scaling identities between the formats.
"""
import math
import os

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.txt")


def page_facts():
    facts = {}
    with open(GOLDEN, encoding="utf-8") as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            key, val = line.split()[:2]
            facts[key] = float(val)
    return facts


# ----------------------------------------------------------------------------------------------
# E2M1
# ----------------------------------------------------------------------------------------------

def test_e2m1_decode_matches_ml_dtypes():
    lib_vals = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    for c in range(16):
        v = oracle.e2m1_value(c)
        assert v == lib_vals[c] and math.copysign(1, v) == math.copysign(1, lib_vals[c]), c


def test_e2m1_page_facts():
    f = page_facts()
    mags = sorted({abs(oracle.e2m1_value(c)) for c in range(16)})
    assert mags[1] == f["e2m1_min_nonzero_magnitude"]
    assert mags[-1] == f["e2m1_max_magnitude"]
    # 1 sign + 2 exponent + 1 mantissa bits: 16 codes, all finite (no inf/NaN reading)
    assert 1 + f["e2m1_exponent_bits"] + f["e2m1_mantissa_bits"] == 4
    assert all(math.isfinite(oracle.e2m1_value(c)) for c in range(16))
    assert mags == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _e2m1_probe_values():
    vals = set()
    # every non-negative bf16 value up to 8 (covers all midpoints and saturation)
    bits = np.arange(0, 0x4101, dtype=np.uint32) << 16
    vals.update(bits.view(np.float32).astype(np.float64).tolist())
    # float32 neighbours of every midpoint
    for t in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0):
        t32 = np.float32(t)
        vals.update([float(np.nextafter(t32, np.float32(0))), float(t32),
                     float(np.nextafter(t32, np.float32(10)))])
    rng = np.random.default_rng(7)
    vals.update(rng.uniform(0, 7, 5000).astype(np.float32).astype(np.float64).tolist())
    return np.array(sorted(vals))


def test_e2m1_rounding_matches_ml_dtypes():
    v = _e2m1_probe_values()
    expect = v.astype(np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8)
    got = np.array([oracle.round_e2m1_mag(x) for x in v])
    bad = np.nonzero(got != expect)[0]
    assert bad.size == 0, [(v[i], got[i], expect[i]) for i in bad[:10]]


def test_e2m1_saturates_above_six():
    for v in (6.0, 6.5, 7.0, 100.0, 1e30):
        assert oracle.round_e2m1_mag(v) == 7


# ----------------------------------------------------------------------------------------------
# E4M3
# ----------------------------------------------------------------------------------------------

def test_e4m3_decode_matches_torch():
    lib = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    for c in range(256):
        v = oracle.e4m3_value(c)
        if math.isnan(lib[c]):
            assert math.isnan(v), c
        else:
            assert v == lib[c] and math.copysign(1, v) == math.copysign(1, lib[c]), c


def _scale_probe_values(hi):
    vals = set()
    bits = np.arange(0, 0x7F80, dtype=np.uint32) << 16  # every non-negative finite bf16
    b = bits.view(np.float32).astype(np.float64)
    vals.update(b[b <= hi].tolist())
    rng = np.random.default_rng(11)
    vals.update(np.exp(rng.uniform(math.log(1e-7), math.log(hi), 20000)).astype(np.float32)
                .astype(np.float64).tolist())
    return np.array(sorted(vals))


def test_e4m3_rounding_matches_torch():
    u = _scale_probe_values(448.0)
    # midpoints of consecutive E4M3 codes and their float32 neighbours
    mids = []
    for c in range(0x7E):
        t = np.float32((oracle.e4m3_value(c) + oracle.e4m3_value(c + 1)) / 2)
        mids += [np.nextafter(t, np.float32(0)), t, np.nextafter(t, np.float32(1e9))]
    u = np.unique(np.concatenate([u, np.array(mids, np.float32).astype(np.float64)]))
    u = u[u <= 448.0]
    expect = torch.from_numpy(u.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.round_scale(x, oracle.E4M3) for x in u])
    bad = np.nonzero(got != expect)[0]
    assert bad.size == 0, [(u[i], got[i], expect[i]) for i in bad[:10]]


def test_e4m3_saturates():
    # torch maps overflow to NaN; the method's reading saturates at 448 (code 0x7E)
    for u in (448.0, 460.0, 464.0, 480.0, 1e6):
        assert oracle.round_scale(u, oracle.E4M3) == 0x7E


def test_e4m3_zero_scale_tie_worked_case():
    # absmax 0.005859375 = 6 * 2^-10: u = 2^-10 sits half-way between 0 and 2^-9 -> even code 0
    assert oracle.round_scale(0.005859375 / 6.0, oracle.E4M3) == 0
    assert oracle.round_scale(np.nextafter(2.0 ** -10, 1.0), oracle.E4M3) == 1


# ----------------------------------------------------------------------------------------------
# UE5M3
# ----------------------------------------------------------------------------------------------

def test_ue5m3_special_values():
    assert oracle.ue5m3_value(0x00) == 0.0
    assert oracle.ue5m3_value(0x01) == 2.0 ** -17
    assert oracle.ue5m3_value(0x08) == 2.0 ** -14
    assert oracle.ue5m3_value(0x78) == 1.0
    assert oracle.ue5m3_value(0xFF) == 122880.0
    vals = [oracle.ue5m3_value(c) for c in range(256)]
    assert all(math.isfinite(v) for v in vals)
    assert all(b > a for a, b in zip(vals, vals[1:]))  # strictly increasing, unsigned


def test_ue5m3_matches_binary16_subset():
    # A UE5M3 code with exponent field e <= 30 is the binary16 number with the same exponent
    # field and the 3 mantissa bits on top: same bias (15), same subnormal spacing rule.
    for c in range(0xF8):
        e, m = c >> 3, c & 7
        h = np.array([(e << 10) | (m << 7)], np.uint16).view(np.float16)[0]
        assert oracle.ue5m3_value(c) == float(h), c


def test_ue5m3_matches_e5m2_on_even_mantissas():
    e5m2 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e5m2).double().numpy()
    for c in range(0xF8):
        e, m = c >> 3, c & 7
        if m % 2 == 0:
            assert oracle.ue5m3_value(c) == e5m2[(e << 2) | (m >> 1)], c


def _e4m3_round_value(x):
    return float(torch.tensor([x], dtype=torch.float64).to(torch.float32)
                 .to(torch.float8_e4m3fn).double()[0])


def test_ue5m3_rounding_matches_scaled_e4m3():
    # With 3 mantissa bits both formats round the same way inside a binade, and UE5M3 subnormals
    # (spacing 2^-17) are E4M3 subnormals (spacing 2^-9) scaled by 2^-8.  Power-of-two scaling is
    # exact, so torch's E4M3 conversion pins UE5M3 rounding everywhere below the top value.
    u = _scale_probe_values(122880.0)
    mids = []
    for c in range(0xFF):
        t = np.float32((oracle.ue5m3_value(c) + oracle.ue5m3_value(c + 1)) / 2)
        mids += [np.nextafter(t, np.float32(0)), t, np.nextafter(t, np.float32(1e9))]
    u = np.unique(np.concatenate([u, np.array(mids, np.float32).astype(np.float64)]))
    u = u[(u > 0) & (u <= 122880.0)]
    rng = np.random.default_rng(3)
    u = rng.choice(u, size=min(u.size, 20000), replace=False)
    for x in u:
        got = oracle.ue5m3_value(oracle.round_scale(x, oracle.UE5M3))
        if x < 2.0 ** -14:
            k = 8  # into the E4M3 subnormal range
        else:
            k = -math.floor(math.log2(x))  # x * 2^k in [1, 2)
        expect = _e4m3_round_value(x * 2.0 ** k) * 2.0 ** -k
        assert got == expect, (x, got, expect)


def test_ue5m3_saturates():
    for u in (122880.0, 126000.0, 1e12):
        assert oracle.round_scale(u, oracle.UE5M3) == 0xFF


# ----------------------------------------------------------------------------------------------
# the pages' printed facts about the scale formats
# ----------------------------------------------------------------------------------------------

def _normal_exponents(value_fn, codes):
    exps = set()
    for c in codes:
        v = value_fn(c)
        if v > 0 and math.isfinite(v):
            exps.add(math.frexp(v)[1] - 1)
    return exps


def test_scale_format_page_facts():
    f = page_facts()
    e4 = _normal_exponents(oracle.e4m3_value, range(0x08, 0x7F))
    ue = _normal_exponents(oracle.ue5m3_value, range(0x08, 0x100))
    assert max(e4) - min(e4) == f["e4m3_exponent_span"]       # -6 .. 8
    assert max(ue) - min(ue) == f["ue5m3_exponent_span"]      # -14 .. 16
    # dynamic range (largest / smallest normal) is about 10^4 and 10^9
    assert round(math.log10(448.0 / 2.0 ** -6)) == f["e4m3_log10_dynamic_range"]
    assert round(math.log10(oracle.scale_max(oracle.UE5M3) / 2.0 ** -14)) == \
        f["ue5m3_log10_dynamic_range"]
    # 3 mantissa bits: 8 codes per binade
    assert sum(1 for c in range(256) if 1.0 <= oracle.ue5m3_value(c) < 2.0) == \
        2 ** int(f["ue5m3_mantissa_bits"])


# ----------------------------------------------------------------------------------------------
# binary16 / bfloat16 decoders used for g and for x
# ----------------------------------------------------------------------------------------------

def test_fp16_decode_matches_numpy():
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    lib = h.view(np.float16).astype(np.float64)
    for b in range(0, 65536, 7):
        v = oracle.fp16_value(b)
        if math.isnan(lib[b]):
            assert math.isnan(v)
        else:
            assert v == lib[b], b


def test_bf16_decode_matches_torch():
    b = torch.arange(0, 65536, 13, dtype=torch.int32).to(torch.int16)
    lib = b.view(torch.bfloat16).double().numpy()
    for i, bits in enumerate(b.numpy().view(np.uint16)):
        v = oracle.lib.orc_bf16_value(int(bits))
        assert (math.isnan(v) and math.isnan(lib[i])) or v == lib[i]
