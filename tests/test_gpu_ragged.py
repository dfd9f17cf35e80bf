"""Parity of ragged tensors (cols not a multiple of the block size N) with the oracle.

Rows of cols values end in a block of cols mod N values; codes take ceil(cols/2) bytes per row and
scales ceil(cols/N).  Every output is written into a buffer with a guard band of 0xA5 bytes after
it, which must stay untouched.  Codes, scales and dequantized values are bit-exact; error sums
within 1e-5 relative, counts exact.
"""
import numpy as np
import pytest
import torch

import fp4_microscaling_tensor_b200 as mx
import oracle
from fp4_microscaling_tensor_b200 import inputs
from gpu_helpers import FMTS, assert_same, assert_stats, bits, special_values_bf16, u8

pytestmark = pytest.mark.gpu

GUARD = 64
SHAPES = [(5, 7, 4), (3, 13, 8), (17, 45, 32), (2, 300, 256), (9, 100, 64), (33, 129, 128),
          (4, 3, 32), (7, 1, 4), (64, 1000, 16), (300, 33, 32),
          # rows on 16-byte boundaries (cols % 8 == 0), bf16: the row-pitched modes and the
          # row-tile dequantize -- partial last tiles in both directions, a row shorter than one
          # block, one-block tensors
          (40, 8200, 32), (33, 520, 64), (65, 1000, 128), (31, 264, 256), (3, 24, 32),
          (1, 8, 256), (70, 776, 16), (129, 2056, 32)]
G_CASES = (0x3C00, 0x2E66)


def guarded(n, dtype=torch.uint8):
    t = torch.full((n * torch.empty((), dtype=dtype).element_size() + GUARD,), 0xA5,
                   dtype=torch.uint8, device="cuda")
    return t, t[: n * torch.empty((), dtype=dtype).element_size()].view(dtype)


def guard_ok(t, n_bytes, what):
    tail = t[n_bytes:].cpu().numpy()
    assert np.all(tail == 0xA5), f"{what}: write past the end"


@pytest.mark.parametrize("rows,cols,block", SHAPES)
@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_ragged_parity(rows, cols, block, fmt, dtype):
    g = G_CASES[(rows + cols) % 2]
    x = special_values_bf16(fmt, g, rows * cols, seed=rows * 31 + cols).to(dtype)
    x = x.reshape(rows, cols).cuda()
    xo = inputs.to_oracle(x)
    pb, nb = (cols + 1) // 2, -(-cols // block)
    po, so = oracle.quantize(xo, rows, cols, block, fmt, g)

    # quantize
    pbuf, p = guarded(rows * pb)
    sbuf, s = guarded(rows * nb)
    mx.quantize(x, block, fmt, g, packed=p.view(rows, pb), scales=s.view(rows, nb))
    torch.cuda.synchronize()
    assert_same(u8(s), so, "ragged scales")
    assert_same(u8(p), po, "ragged packed")
    guard_ok(pbuf, rows * pb, "packed")
    guard_ok(sbuf, rows * nb, "scales")

    # dequantize, both output types
    pd, sd = p.view(rows, pb), s.view(rows, nb)
    for dt, bf in ((torch.bfloat16, True), (torch.float32, False)):
        ybuf, y = guarded(rows * cols, dt)
        mx.dequantize(pd, sd, block, fmt, g, out=y.view(rows, cols), cols=cols)
        torch.cuda.synchronize()
        yo = oracle.dequantize(po, so, rows, cols, block, fmt, g, out_bf16=bf)
        assert_same(bits(y), yo if bf else yo.view(np.uint32), f"ragged dequant {dt}")
        guard_ok(ybuf, rows * cols * (2 if bf else 4), "y")
        # fake quantize = dequantize(quantize(x)) in one pass
        fbuf, yf = guarded(rows * cols, dt)
        mx.fake_quantize(x, block, fmt, g, out_dtype=dt, out=yf.view(rows, cols))
        torch.cuda.synchronize()
        assert_same(bits(yf), yo if bf else yo.view(np.uint32), f"ragged fake quantize {dt}")
        guard_ok(fbuf, rows * cols * (2 if bf else 4), "fake y")

    # error reduction: recomputed codes, stored codes, fused with quantize
    ref = oracle.error_stats(xo, rows, cols, block, fmt, g)
    got = mx.error_stats(x, block, fmt, g).to_dict()
    assert_stats(got, ref, "ragged stats (recomputed)")
    got = mx.error_stats(x, block, fmt, g, packed=pd, scales=sd).to_dict()
    assert_stats(got, ref, "ragged stats (stored codes)")
    p2buf, p2 = guarded(rows * pb)
    s2buf, s2 = guarded(rows * nb)
    _, _, st = mx.quantize_with_stats(x, block, fmt, g, packed=p2.view(rows, pb),
                                      scales=s2.view(rows, nb))
    assert_stats(st.to_dict(), ref, "ragged fused")
    assert_same(u8(p2), po, "ragged fused packed")
    assert_same(u8(s2), so, "ragged fused scales")
    guard_ok(p2buf, rows * pb, "fused packed")
    guard_ok(s2buf, rows * nb, "fused scales")


def test_ragged_aligned_rows_full_size():
    # 8192 x 8200, N = 32, UE5M3 with the tensor's global scale (256 whole blocks and a block of 8
    # per row; the row-pitched kernels and the row-tile dequantize): the error record of the whole tensor against the oracle,
    # codes, scales and dequantized bits on 256 seeded rows (the first and last included)
    rows, cols, block = 8192, 8200, 32
    x = inputs.normal((rows, cols), 0.015, seed=8200).cuda()
    xo = inputs.to_oracle(x)
    g = oracle.global_scale(xo, mx.UE5M3)
    p, s, st = mx.quantize_with_stats(x, block, "ue5m3", g)
    y = mx.dequantize(p, s, block, "ue5m3", g, cols=cols)
    yf = mx.fake_quantize(x, block, "ue5m3", g)
    rec = mx.error_stats(x, block, "ue5m3", g).to_dict()
    torch.cuda.synchronize()
    ref = oracle.error_stats(xo, rows, cols, block, mx.UE5M3, g)
    assert_stats(st.to_dict(), ref, "row tiles 8192x8200 fused")
    assert_stats(rec, ref, "row tiles 8192x8200 recomputed")
    sel = np.unique(np.concatenate([[0, rows - 1],
                                    np.random.default_rng(8).choice(rows, 254, replace=False)]))
    xs = xo.reshape(rows, cols)[sel].reshape(-1)
    po, so = oracle.quantize(xs, len(sel), cols, block, mx.UE5M3, g)
    idx = torch.from_numpy(sel).cuda()
    assert_same(u8(p.view(rows, -1)[idx]), po, "row tiles sampled packed")
    assert_same(u8(s.view(rows, -1)[idx]), so, "row tiles sampled scales")
    yo = oracle.dequantize(po, so, len(sel), cols, block, mx.UE5M3, g, out_bf16=True)
    assert_same(bits(y.view(rows, cols)[idx]), yo, "row tiles sampled dequant")
    assert_same(bits(yf.view(rows, cols)[idx]), yo, "row tiles sampled fake quantize")


def test_ragged_large_sampled_rows():
    # 4096 x 4100 (N = 32: 128 whole blocks and a block of 4 per row), N(0, 0.02^2): whole tensor
    # quantized on the GPU, 256 seeded rows compared with the oracle, the error record whole
    rows, cols, block = 4096, 4100, 32
    x = inputs.normal((rows, cols), 0.02, seed=4100).cuda()
    p, s, st = mx.quantize_with_stats(x, block, "e4m3")
    xo = inputs.to_oracle(x)
    ref = oracle.error_stats(xo, rows, cols, block, mx.E4M3)
    assert_stats(st.to_dict(), ref, "ragged 4096x4100")
    sel = np.sort(np.random.default_rng(7).choice(rows, 256, replace=False))
    xs = xo.reshape(rows, cols)[sel].reshape(-1)
    po, so = oracle.quantize(xs, len(sel), cols, block, mx.E4M3)
    assert_same(u8(p.view(rows, -1)[torch.from_numpy(sel).cuda()]), po, "sampled packed")
    assert_same(u8(s.view(rows, -1)[torch.from_numpy(sel).cuda()]), so, "sampled scales")


@pytest.mark.parametrize("block", [4, 16, 32, 256])
@pytest.mark.parametrize("fmt", (mx.E4M3, mx.UE5M3))
def test_grouped_calls_take_ragged_tensors(cuda_device, block, fmt):
    """A group mixing whole-block tensors and tensors whose rows the block size does not divide
    (odd row lengths included), with g by value and from device memory: every tensor's codes,
    scales, dequantized bits and error record equal the oracle's."""
    rng = np.random.default_rng(block + 5 * fmt)
    shapes = [(64, 2 * block), (33, 3 * block + 5), (7, block - 1 if block > 4 else 3),
              (0, block + 1), (129, 8 * block), (5, 2 * block + 1), (40, 3 * block + 8)]
    xs = []
    for r, c in shapes:
        x = rng.standard_normal((r, c)) * np.exp(rng.uniform(-3, 1, (r, 1)))
        xs.append(torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(cuda_device))
    for gmode in ("value", "device"):
        if gmode == "device":
            g = mx.global_scale_group(xs, fmt)
            gs = [int(v) for v in g.cpu().numpy().view(np.uint16)]
        else:
            gs = [0x3C00, 0x3555, 0x2E66, 0x3C00, 0x4400, 0x0003, 0x3C00][:len(xs)]
            g = gs
        p, s = mx.quantize_group(xs, block, fmt, g=g)
        p2, s2, st = mx.quantize_with_stats_group(xs, block, fmt, g=g)
        y = mx.dequantize_group(p, s, block, fmt, g=g, cols=[c for _, c in shapes])
        torch.cuda.synchronize()
        for k, x in enumerate(xs):
            rows, cols = shapes[k]
            what = f"ragged group N={block} fmt={fmt} g={gmode} tensor {k} {shapes[k]}"
            xo = inputs.to_oracle(x)
            if gmode == "device":
                assert gs[k] == oracle.global_scale(xo, fmt), what
            po, so = oracle.quantize(xo, rows, cols, block, fmt, gs[k])
            assert_same(u8(p[k]), po, what + " packed")
            assert_same(u8(s[k]), so, what + " scales")
            assert_same(u8(p2[k]), po, what + " fused packed")
            assert_same(u8(s2[k]), so, what + " fused scales")
            yo = oracle.dequantize(po, so, rows, cols, block, fmt, gs[k], out_bf16=True)
            assert_same(bits(y[k]), yo, what + " dequant")
            ref = oracle.error_stats(xo, rows, cols, block, fmt, gs[k], packed=po, scales=so)
            assert_stats(st[k].to_dict(), ref, what + " stats")
