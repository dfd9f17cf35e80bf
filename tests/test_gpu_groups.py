"""Grouped calls: one launch over several tensors gives, tensor by tensor, the oracle's codes,
scales and dequantized bits (bit-exact) and error records (within 1e-5 relative), with tensors of
different sizes and global scales in one group (an empty tensor, tensors whose size is not a
multiple of the kernels' item (tails, N <= 16), and sizes that give a tensor a single CTA among
many)."""
import numpy as np
import pytest
import torch

import oracle
import fp4_microscaling_tensor_b200 as mx
from fp4_microscaling_tensor_b200 import inputs

from gpu_helpers import BLOCKS, FMTS, assert_same, assert_stats, bits, u8

pytestmark = pytest.mark.gpu

G_MIX = (0x3C00, 0x3555, 0x0003, 0x5A00, 0x3C00, 0x2E66)


def make_group(block, dtype, device, seed):
    """Tensors of one group: sizes from tiny to a few CTAs' worth, one empty, plus (N = 4) one
    of 12 elements."""
    rng = np.random.default_rng(seed)
    shapes = [(3, 8 * block), (64, 4 * block), (1, block), (0, block), (257, 2 * block),
              (512, 1024)]
    if block == 4:
        shapes.append((3, 4))  # 12 elements: a tail after the last whole item (one item of 8 in
        #                        the quantize kernel, none in the error kernels' items of 16)
    xs = []
    for k, (r, c) in enumerate(shapes):
        x = rng.standard_normal((r, c)) * np.exp(rng.uniform(-3, 1, (r, 1)))
        xs.append(torch.from_numpy(x.astype(np.float32)).to(dtype).to(device))
    return xs


def oracle_tensor(x, block, fmt, g):
    rows, cols = x.shape
    xo = inputs.to_oracle(x)
    po, so = oracle.quantize(xo, rows, cols, block, fmt, g)
    yo = oracle.dequantize(po, so, rows, cols, block, fmt, g,
                           out_bf16=x.dtype == torch.bfloat16)
    st = oracle.error_stats(xo, rows, cols, block, fmt, g, packed=po, scales=so)
    return po, so, yo, st


@pytest.mark.parametrize("block", BLOCKS)
@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_groups_match_oracle(cuda_device, block, fmt, dtype):
    xs = make_group(block, dtype, cuda_device, seed=block * 7 + fmt)
    gs = [G_MIX[k % len(G_MIX)] for k in range(len(xs))]
    p, s = mx.quantize_group(xs, block, fmt, gs)
    y = mx.dequantize_group(p, s, block, fmt, gs, out_dtype=dtype)
    p2, s2, st = mx.quantize_with_stats_group(xs, block, fmt, gs)
    for k, x in enumerate(xs):
        what = f"group N={block} fmt={fmt} {dtype} tensor {k} {tuple(x.shape)} g={gs[k]:#x}"
        po, so, yo, sto = oracle_tensor(x, block, fmt, gs[k])
        assert_same(u8(s[k]), so, what + " scales")
        assert_same(u8(p[k]), po, what + " packed")
        assert_same(u8(s2[k]), so, what + " fused scales")
        assert_same(u8(p2[k]), po, what + " fused packed")
        ref = yo if dtype == torch.bfloat16 else yo.view(np.uint32)
        assert_same(bits(y[k]), ref, what + " dequant")
        assert_stats(st[k].to_dict(), sto, what + " stats")


def test_group_of_sixteen_bench_point(cuda_device):
    """The largest group, 16 tensors of the bench's point shape split among the CTAs."""
    xs = [inputs.workload2(k % 5, shape=(1024, 4096), device=cuda_device) for k in range(16)]
    p, s, st = mx.quantize_with_stats_group(xs, 32, mx.E4M3)
    y = mx.dequantize_group(p, s, 32, mx.E4M3)
    for k in (0, 7, 15):
        po, so, yo, sto = oracle_tensor(xs[k], 32, mx.E4M3, 0x3C00)
        assert_same(u8(p[k]), po, f"tensor {k} packed")
        assert_same(u8(s[k]), so, f"tensor {k} scales")
        assert_same(bits(y[k]), yo, f"tensor {k} dequant")
        assert_stats(st[k].to_dict(), sto, f"tensor {k} stats")


def test_group_rejects_mixed_dtypes(cuda_device):
    a = torch.zeros(4, 64, dtype=torch.bfloat16, device=cuda_device)
    b = torch.zeros(4, 64, dtype=torch.float32, device=cuda_device)
    with pytest.raises(ValueError):
        mx.quantize_group([a, b], 32, mx.E4M3)
    with pytest.raises(ValueError):
        mx.quantize_group([a] * (mx.MX_MAX_GROUP + 1), 32, mx.E4M3)


@pytest.mark.parametrize("block", [4, 16, 32, 256])
@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_device_global_scales_drive_the_group(cuda_device, block, fmt, dtype):
    """mx_global_scale_group writes every tensor's g to device memory; the other grouped calls
    read it there (no host round trip).  g equals the oracle's rule per tensor (1.0 for the empty
    tensor), and codes, scales, dequantized bits and error records equal the oracle's with it."""
    xs = make_group(block, dtype, cuda_device, seed=block * 11 + fmt + 3)
    xs[1] = xs[1] * 1e-4  # one tensor whose g sits far below 1
    g = mx.global_scale_group(xs, fmt)
    p, s = mx.quantize_group(xs, block, fmt, g=g)
    y = mx.dequantize_group(p, s, block, fmt, g=g, out_dtype=dtype)
    p2, s2, st = mx.quantize_with_stats_group(xs, block, fmt, g=g)
    gh = g.cpu().numpy().view(np.uint16)
    for k, x in enumerate(xs):
        gk = oracle.global_scale(inputs.to_oracle(x), fmt)
        what = f"device g N={block} fmt={fmt} {dtype} tensor {k} {tuple(x.shape)}"
        assert int(gh[k]) == gk, (what, hex(int(gh[k])), hex(gk))
        po, so, yo, sto = oracle_tensor(x, block, fmt, gk)
        assert_same(u8(s[k]), so, what + " scales")
        assert_same(u8(p[k]), po, what + " packed")
        assert_same(u8(s2[k]), so, what + " fused scales")
        assert_same(u8(p2[k]), po, what + " fused packed")
        ref = yo if dtype == torch.bfloat16 else yo.view(np.uint32)
        assert_same(bits(y[k]), ref, what + " dequant")
        assert_stats(st[k].to_dict(), sto, what + " stats")


def test_device_global_scales_in_a_graph(cuda_device):
    """The chain global scale -> fused pass -> dequantize captured in a CUDA graph and replayed on
    new inputs: the replay reads the g its own first launch wrote."""
    xs = [inputs.workload5_tensor(0, j, device=cuda_device, shape=(256, 1024)) for j in range(3)]
    g = torch.empty(3, dtype=torch.int16, device=cuda_device)
    p = [torch.empty(256, 512, dtype=torch.uint8, device=cuda_device) for _ in xs]
    s = [torch.empty(256, 32, dtype=torch.uint8, device=cuda_device) for _ in xs]
    y = [torch.empty(256, 1024, dtype=torch.bfloat16, device=cuda_device) for _ in xs]
    out = torch.empty(3, 64, dtype=torch.uint8, device=cuda_device)
    ws = mx.stats_workspace(cuda_device)

    def chain():
        mx.global_scale_group(xs, "ue5m3", out=g)
        mx.quantize_with_stats_group(xs, 32, "ue5m3", g=g, packed=p, scales=s, out=out,
                                     workspace=ws)
        mx.dequantize_group(p, s, 32, "ue5m3", g=g, out=y)

    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        chain()
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            chain()
    stream.synchronize()
    for scale in (1.0, 37.0):
        for x in xs:
            x.mul_(scale)
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        for k, x in enumerate(xs):
            gk = oracle.global_scale(inputs.to_oracle(x), oracle.UE5M3)
            po, so, yo, sto = oracle_tensor(x, 32, oracle.UE5M3, gk)
            assert_same(u8(p[k]), po, f"graph x{scale} tensor {k} packed")
            assert_same(u8(s[k]), so, f"graph x{scale} tensor {k} scales")
            assert_same(bits(y[k]), yo, f"graph x{scale} tensor {k} dequant")
            assert_stats(mx.ErrorStats(out[k]).to_dict(), sto, f"graph x{scale} tensor {k}")
    del graph
