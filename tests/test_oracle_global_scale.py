"""Pin of the oracle's per-tensor FP16 scale rule against an exhaustive numpy binary16 search.

Reading: g is the smallest positive finite binary16 value with g * 6 * Smax >= max|x| (so no block
scale saturates), 1.0 for an all-zero tensor, 65504 when even that is too small.
"""
import numpy as np
import pytest

import oracle

POS_FP16 = np.arange(1, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)


def expected(A, smax):
    if A == 0:
        return 1.0
    ok = np.nonzero(POS_FP16 * (6 * smax) >= A)[0]
    return POS_FP16[ok[0]] if ok.size else 65504.0


@pytest.mark.parametrize("fmt,smax", [(oracle.E4M3, 448.0), (oracle.UE5M3, 122880.0)])
def test_global_scale_exhaustive_fp16(fmt, smax):
    rng = np.random.default_rng(17)
    As = list(np.exp(rng.uniform(np.log(1e-12), np.log(1e12), 300)).astype(np.float32))
    # values that land exactly on g * 6 * Smax for representable g, and one ulp around them
    for g in (2.0 ** -24, 3 * 2.0 ** -24, 0.5, 1.0, 1.5, 1000.0, 65504.0):
        t = np.float32(g * 6 * smax)
        As += [np.nextafter(t, np.float32(0)), t, np.nextafter(t, np.float32(np.inf))]
    As += [np.float32(0.0), np.float32(1e-45), np.float32(3e38)]
    for A in As:
        x = np.array([0.0, -A, A / 3], np.float32)
        g_bits = oracle.global_scale(x, fmt)
        assert oracle.fp16_value(g_bits) == expected(float(A), smax), (A, hex(g_bits))


def test_global_scale_bf16_input():
    x = np.array([0x3F80, 0xC2C8, 0x0000], np.uint16)  # 1.0, -100.0, 0
    g = oracle.fp16_value(oracle.global_scale(x, oracle.E4M3))
    assert g == expected(100.0, 448.0)
    assert g * 6 * 448 >= 100.0


def test_global_scale_prevents_scale_saturation():
    # with the chosen g no block scale of the tensor saturates
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(64 * 256) * 3e4).astype(np.float32)
    for fmt in (oracle.E4M3, oracle.UE5M3):
        g_bits = oracle.global_scale(x, fmt)
        st = oracle.error_stats(x, 64, 256, 32, fmt, g_bits)
        assert st["n_scale_sat"] == 0
