"""Shared checks for the GPU parity tests: the CUDA path (through the C ABI) against the oracle."""
import math

import numpy as np
import torch

import oracle
import fp4_microscaling_tensor_b200 as mx
from fp4_microscaling_tensor_b200 import inputs

FMTS = (mx.E4M3, mx.UE5M3)
BLOCKS = (4, 8, 16, 32, 64, 128, 256)
STATS_RTOL = 1e-5
COUNT_KEYS = ("numel", "n_blocks", "n_zero_blocks", "n_scale_sat", "n_elem_sat")
SSE_KEYS = ("sse_elem", "sse_max", "sse_zero")


def u8(t):
    return t.detach().reshape(-1).cpu().numpy()


def bits(t):
    """bf16 / fp32 tensor -> uint16 / uint32 bit patterns (numpy)."""
    t = t.detach().reshape(-1).cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.view(torch.int32).numpy().view(np.uint32)


def assert_same(got, ref, what):
    got, ref = np.asarray(got).reshape(-1), np.asarray(ref).reshape(-1)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    bad = np.nonzero(got != ref)[0]
    if bad.size:
        i = bad[0]
        raise AssertionError(f"{what}: {bad.size} of {got.size} differ; first at {i}: "
                             f"gpu={got[i]:#x} oracle={ref[i]:#x}")


def assert_stats(got, ref, what):
    for k in COUNT_KEYS:
        assert got[k] == ref[k], (what, k, got[k], ref[k])
    for k in SSE_KEYS:
        g, r = got[k], ref[k]
        assert abs(g - r) <= STATS_RTOL * abs(r), (what, k, g, r)


def to_dev(a, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def quantize_both(x, block, fmt, g=0x3C00):
    """x: 2-D CUDA tensor.  Returns gpu (packed, scales) and oracle (packed, scales), compared."""
    rows, cols = x.shape
    p, s = mx.quantize(x, block, fmt, g)
    po, so = oracle.quantize(inputs.to_oracle(x), rows, cols, block, fmt, g)
    assert_same(u8(s), so, f"scales N={block} fmt={fmt} g={g:#x}")
    assert_same(u8(p), po, f"packed N={block} fmt={fmt} g={g:#x}")
    return p, s, po, so


def dequantize_both(po, so, rows, cols, block, fmt, g=0x3C00):
    """Dequantize the oracle's codes on the GPU (bf16 and fp32 out) and compare bit patterns."""
    p = to_dev(po).reshape(rows, cols // 2)
    s = to_dev(so).reshape(rows, cols // block)
    for dt, bf in ((torch.bfloat16, True), (torch.float32, False)):
        y = mx.dequantize(p, s, block, fmt, g, out_dtype=dt)
        yo = oracle.dequantize(po, so, rows, cols, block, fmt, g, out_bf16=bf)
        ref = yo if bf else yo.view(np.uint32)
        assert_same(bits(y), ref, f"dequant {dt} N={block} fmt={fmt} g={g:#x}")


def stats_both(x, block, fmt, g=0x3C00, packed=None, scales=None, po=None, so=None):
    rows, cols = x.shape
    got = mx.error_stats(x, block, fmt, g, packed=packed, scales=scales).to_dict()
    ref = oracle.error_stats(inputs.to_oracle(x), rows, cols, block, fmt, g, packed=po, scales=so)
    assert_stats(got, ref, f"stats N={block} fmt={fmt} g={g:#x} given={packed is not None}")
    return got, ref


def fused_both(x, block, fmt, g, po, so):
    """mx_quantize_stats: codes and scales bit-exact, error sums as the oracle's."""
    rows, cols = x.shape
    p, s, st = mx.quantize_with_stats(x, block, fmt, g)
    assert_same(u8(s), so, f"fused scales N={block} fmt={fmt} g={g:#x}")
    assert_same(u8(p), po, f"fused packed N={block} fmt={fmt} g={g:#x}")
    ref = oracle.error_stats(inputs.to_oracle(x), rows, cols, block, fmt, g)
    assert_stats(st.to_dict(), ref, f"fused stats N={block} fmt={fmt} g={g:#x}")


def full_check(x, block, fmt, g=0x3C00):
    """Quantize, dequantize, stats (recomputed, from stored codes, fused) against the oracle."""
    rows, cols = x.shape
    p, s, po, so = quantize_both(x, block, fmt, g)
    dequantize_both(po, so, rows, cols, block, fmt, g)
    stats_both(x, block, fmt, g)
    stats_both(x, block, fmt, g, packed=p, scales=s, po=po, so=so)
    fused_both(x, block, fmt, g, po, so)


def special_values_bf16(fmt, g_bits, n, seed):
    """bf16 values mixing Gaussians of several widths with ties, thresholds, zeros and extremes."""
    g = oracle.fp16_value(g_bits)
    smin = oracle.scale_min(fmt)
    smax = oracle.scale_max(fmt)
    rng = np.random.default_rng(seed)
    base = rng.standard_normal(n) * np.exp(rng.uniform(math.log(1e-4), math.log(10), n)) * g
    picks = np.array([0.0, -0.0, 3 * smin * g, -3 * smin * g, 6 * g, 6 * smax * g, 7 * smax * g,
                      0.25 * g, 0.75 * g, 1.25 * g, 1.75 * g, 2.5 * g, 3.5 * g, 5 * g, 1e-30, -1e-38,
                      3e38, -3e38])
    mask = rng.random(n) < 0.08
    base[mask] = rng.choice(picks, mask.sum())
    t = torch.from_numpy(base.astype(np.float32)).to(torch.bfloat16)
    return t
