"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Bit-exact for packed codes, scale bytes and dequantized bit patterns (signed zeros included);
within 1e-5 relative for the three error sums, exact for the counts.  Small shapes span several
CTAs' worth of items and ragged tails; the exhaustive tests walk every bf16 value through the scale
rounding and every bf16 mantissa/exponent through the element rounding at every scale code.
"""
import numpy as np
import pytest
import torch

import oracle
import fp4_microscaling_tensor_b200 as mx
from fp4_microscaling_tensor_b200 import inputs

from gpu_helpers import (BLOCKS, FMTS, assert_same, assert_stats, bits, dequantize_both, full_check,
                         quantize_both, special_values_bf16, stats_both, to_dev, u8)

pytestmark = pytest.mark.gpu

G_CASES = (0x3C00, 0x3555, 0x0003, 0x5A00)  # 1.0, ~0.333, a subnormal, 192.0


def test_workload1_fp32_full(cuda_device):
    x = inputs.workload1(device="cpu").to(cuda_device)
    full_check(x, 32, mx.E4M3)


@pytest.mark.parametrize("block", BLOCKS)
@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_ragged_shapes_special_values(cuda_device, block, fmt, dtype):
    # rows x cols chosen so the item count is not a multiple of a warp and, for N <= 8, the element
    # count leaves 4, 8 or 12 elements after the last 16-element item (the tail paths)
    for i, (rows, k) in enumerate(((37, 5), (1, 1), (129, 3), (5, 2))):
        cols = block * k
        g = G_CASES[i % len(G_CASES)]
        x = special_values_bf16(fmt, g, rows * cols, seed=block * 7 + fmt + i).to(dtype)
        full_check(x.reshape(rows, cols).to(cuda_device), block, fmt, g)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("g", G_CASES)
def test_exhaustive_scale_rounding_bf16(cuda_device, fmt, g):
    # every positive finite bf16 value is the maximum of one block of 4
    a = np.arange(1, 0x7F80, dtype=np.uint16)
    blocks = np.zeros((a.size, 4), np.uint16)
    blocks[:, 0] = a
    blocks[:, 2] = a >> 1  # a smaller companion value
    x = to_dev(blocks.view(np.int16)).view(torch.bfloat16).reshape(-1, 4)
    p, s, po, so = quantize_both(x, 4, fmt, g)
    stats_both(x, 4, fmt, g)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("g", G_CASES)
def test_exhaustive_element_rounding_bf16(cuda_device, fmt, g):
    # For each scale code reachable with this g, one block of 256 per group of candidates: the block
    # maximum pins the scale; the other 255 values walk every bf16 mantissa over the 8 binades
    # below the maximum (both signs), so every (x mantissa, scale mantissa, g) combination is seen.
    gval = oracle.fp16_value(g)
    rows = []
    for s in range(1, 256 if fmt == mx.UE5M3 else 0x7F):
        S = oracle.scale_value(s, fmt)
        a = np.float32(6 * S * gval)
        if not np.isfinite(a) or a > 3e38:
            continue
        abits = int(torch.tensor([float(a)]).to(torch.bfloat16).view(torch.int16).item()) & 0xFFFF
        cand = []
        top = abits & 0x7F80
        for e in range(8):
            ex = top - (e << 7)
            if ex <= 0:
                break
            cand.append(np.arange(ex, ex + 128, dtype=np.int64))
        cand = np.concatenate(cand)
        cand = cand[cand < abits]
        signs = (np.arange(cand.size) & 1).astype(np.int64) << 15
        cand = (cand | signs).astype(np.uint16)
        for j in range(0, cand.size, 255):
            blk = np.zeros(256, np.uint16)
            blk[0] = abits
            chunk = cand[j:j + 255]
            blk[1:1 + chunk.size] = chunk
            rows.append(blk)
    x = to_dev(np.stack(rows).view(np.int16)).view(torch.bfloat16)
    p, s, po, so = quantize_both(x, 256, fmt, g)
    dequantize_both(po, so, x.shape[0], 256, 256, fmt, g)
    stats_both(x, 256, fmt, g)


@pytest.mark.parametrize("fmt", FMTS)
def test_fp32_near_ties(cuda_device, fmt):
    # fp32 values one ulp either side of every element midpoint t*S (g = 1), block max = 6 S
    rows = []
    for s in range(8, 0x7F if fmt == mx.E4M3 else 0xE0, 3):
        S = np.float32(oracle.scale_value(s, fmt))
        row = [6 * S]
        for t in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0):
            m = np.float32(t) * S
            row += [np.nextafter(m, np.float32(0)), m, np.nextafter(m, np.float32(1e30))]
        row += [0.0] * (32 - len(row))
        rows.append(np.array(row, np.float32)[:32] * np.where(np.arange(32) % 2, -1, 1).astype(np.float32))
    x = to_dev(np.stack(rows))
    full_check(x, 32, fmt)


@pytest.mark.parametrize("block", BLOCKS)
@pytest.mark.parametrize("fmt", FMTS)
def test_dequantize_every_code(cuda_device, block, fmt):
    rng = np.random.default_rng(block + 100 * fmt)
    rows, cols = 33, block * 3
    po = rng.integers(0, 256, rows * cols // 2, dtype=np.uint8)
    hi = 256 if fmt == mx.UE5M3 else 0x7F
    so = rng.integers(0, hi, rows * cols // block, dtype=np.uint8)
    so[: min(so.size, 8)] = [0, 1, 2, 8, 0x10, hi - 1, hi - 2, 0x40][: min(so.size, 8)]
    for g in G_CASES:
        dequantize_both(po, so, rows, cols, block, fmt, g)


@pytest.mark.parametrize("block", (4, 32, 256))
@pytest.mark.parametrize("fmt", FMTS)
def test_stats_given_arbitrary_codes(cuda_device, block, fmt):
    # codes that the quantizer would not produce: the max elements carry different errors
    rng = np.random.default_rng(block)
    rows, cols = 40, block * 4
    x = special_values_bf16(fmt, 0x3C00, rows * cols, seed=block).reshape(rows, cols).to(cuda_device)
    po = rng.integers(0, 256, rows * cols // 2, dtype=np.uint8)
    hi = 256 if fmt == mx.UE5M3 else 0x7F
    so = rng.integers(0, hi, rows * cols // block, dtype=np.uint8)
    p = to_dev(po).reshape(rows, cols // 2)
    s = to_dev(so).reshape(rows, cols // block)
    stats_both(x, block, fmt, 0x3C00, packed=p, scales=s, po=po, so=so)


@pytest.mark.parametrize("fmt", FMTS)
def test_adversarial_blocks(cuda_device, fmt):
    smin = oracle.scale_min(fmt)
    cases = {
        "zeros": np.zeros((8, 64), np.float32),
        "neg_zeros": -np.zeros((8, 64), np.float32),
        "constant": np.full((8, 64), 0.37, np.float32),
        "ties": np.tile(np.array([6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5], np.float32), (8, 8)),
        "threshold": np.tile(np.array([3 * smin, 3 * smin / 2, -3 * smin, 0], np.float32), (8, 16)),
        "saturating": np.tile(np.array([1e6, -3e5, 2688, 2689, 1, -1, 0, 5e4], np.float32), (8, 8)),
    }
    for name, arr in cases.items():
        x = torch.from_numpy(arr).to(torch.bfloat16).to(cuda_device)
        for block in (4, 16, 64):
            full_check(x, block, fmt)


def test_llama_mlp_cols_block256(cuda_device):
    x = inputs.workload3_tensor(0, 6, shape=(16, 11008)).to(cuda_device)
    for fmt in FMTS:
        full_check(x, 256, fmt)


def test_empty_tensor(cuda_device):
    x = torch.empty(0, 64, dtype=torch.bfloat16, device=cuda_device)
    p, s = mx.quantize(x, 32, mx.E4M3)
    assert p.numel() == 0 and s.numel() == 0
    y = mx.dequantize(p, s, 32, mx.E4M3)
    assert y.shape == (0, 64)
    st = mx.error_stats(x, 32, mx.E4M3).to_dict()
    assert st["numel"] == 0 and st["sse_elem"] == 0 and st["n_blocks"] == 0
    assert int(mx.global_scale(x, mx.UE5M3).item()) == 0x3C00


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_global_scale(cuda_device, fmt, dtype):
    rng = np.random.default_rng(3)
    for numel, scale in ((1, 1.0), (7, 1e-3), (4093, 1e5), (65536 + 5, 0.02), (1 << 20, 3e-9)):
        x = torch.from_numpy((rng.standard_normal(numel) * scale).astype(np.float32)).to(dtype)
        xd = x.reshape(1, -1).to(cuda_device)
        got = int(mx.global_scale(xd, fmt).item()) & 0xFFFF
        ref = oracle.global_scale(inputs.to_oracle(x), fmt)
        assert got == ref, (numel, scale, hex(got), hex(ref))
    for v in (0.0, 1e-45, 3.0e38):
        x = torch.full((1, 16), v, dtype=dtype)
        got = int(mx.global_scale(x.to(cuda_device), fmt).item()) & 0xFFFF
        assert got == oracle.global_scale(inputs.to_oracle(x), fmt)


def test_guard_bands_untouched(cuda_device):
    # outputs sit inside larger buffers filled with 0xA5; nothing outside the outputs may change
    for block, rows, cols in ((4, 3, 12), (32, 5, 96), (256, 2, 512)):
        x = torch.randn(rows, cols, device=cuda_device).to(torch.bfloat16)
        pad = 256
        nb, ns, ny = rows * cols // 2, rows * cols // block, rows * cols * 2
        pb = torch.full((nb + 2 * pad,), 0xA5, dtype=torch.uint8, device=cuda_device)
        sb = torch.full((ns + 2 * pad,), 0xA5, dtype=torch.uint8, device=cuda_device)
        yb = torch.full((ny + 2 * pad,), 0xA5, dtype=torch.uint8, device=cuda_device)
        p = pb[pad:pad + nb].view(rows, cols // 2)
        s = sb[pad:pad + ns].view(rows, cols // block)
        mx.quantize(x, block, mx.E4M3, packed=p, scales=s)
        y = yb[pad:pad + ny].view(torch.bfloat16).view(rows, cols)
        mx.dequantize(p, s, block, mx.E4M3, out=y)
        torch.cuda.synchronize()
        for buf, n in ((pb, nb), (sb, ns), (yb, ny)):
            h = u8(buf)
            assert np.all(h[:pad] == 0xA5) and np.all(h[pad + n:] == 0xA5)


def test_stats_deterministic(cuda_device):
    x = inputs.workload2(3, shape=(512, 4096), device="cpu").to(cuda_device)
    a = mx.error_stats(x, 32, mx.E4M3).to_dict()
    b = mx.error_stats(x, 32, mx.E4M3).to_dict()
    assert a == b


def test_kernel_launch_counter(cuda_device):
    x = torch.randn(64, 64, device=cuda_device).to(torch.bfloat16)
    n0 = mx.kernel_launches()
    mx.quantize(x, 32, mx.E4M3)
    assert mx.kernel_launches() == n0 + 1
