"""Python API over the C ABI: quantize, dequantize, error_stats, global_scale, matmul.

Tensors are CUDA tensors, contiguous, row-major, with blocks along the last dimension.  Outputs are
allocated with torch on the tensor's device unless given.  Calls are asynchronous on the current
torch stream (or `stream=`); nothing here synchronizes except ErrorStats.to_dict().
"""
import ctypes
import struct

import numpy as np
import torch

from ._lib import (MX_BF16, MX_F32, MX_MAX_GROUP, MX_SCALE_E4M3, MX_SCALE_UE5M3,  # noqa: F401
                   MXError, Tensor, check, lib)

E4M3, UE5M3 = MX_SCALE_E4M3, MX_SCALE_UE5M3
_FMT = {"e4m3": E4M3, "ue5m3": UE5M3, E4M3: E4M3, UE5M3: UE5M3}
_DT = {torch.float32: MX_F32, torch.bfloat16: MX_BF16}
STATS_BYTES = 64
STATS_FIELDS = ("sse_elem", "sse_max", "sse_zero", "numel", "n_blocks", "n_zero_blocks",
                "n_scale_sat", "n_elem_sat")


def fmt_code(fmt):
    try:
        return _FMT[fmt.lower() if isinstance(fmt, str) else fmt]
    except KeyError:
        raise ValueError(f"unknown scale format {fmt!r}") from None


def g_bits(g):
    """binary16 bit pattern of the per-tensor scale: a float (rounded to fp16) or an int pattern."""
    if g is None:
        return 0x3C00
    if isinstance(g, (int, np.integer)) and not isinstance(g, bool):
        return int(g) & 0xFFFF
    return int(np.array([g], np.float16).view(np.uint16)[0])


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes_stream(stream)


def ctypes_stream(stream):
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _shape2d(t, what):
    if not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    if t.dim() == 0:
        raise ValueError(f"{what} must have at least one dimension")
    cols = t.shape[-1]
    rows = t.numel() // cols if cols else 0
    return rows, cols


def quantize(x, block=32, fmt="e4m3", g=None, packed=None, scales=None, stream=None):
    """Quantize + pack.  Returns (packed uint8 [..., cols/2], scales uint8 [..., cols/block])."""
    rows, cols = _shape2d(x, "x")
    if x.dtype not in _DT:
        raise ValueError("x must be float32 or bfloat16")
    lead = tuple(x.shape[:-1])
    if packed is None:
        packed = torch.empty(lead + ((cols + 1) // 2,), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(lead + (-(-cols // block) if block else 0,), dtype=torch.uint8,
                             device=x.device)
    check(lib.mx_quantize(x.data_ptr(), _DT[x.dtype], rows, cols, int(block), fmt_code(fmt),
                          g_bits(g), packed.data_ptr(), scales.data_ptr(),
                          _stream(stream, x.device)), "mx_quantize")
    return packed, scales


def dequantize(packed, scales, block=32, fmt="e4m3", g=None, out_dtype=torch.bfloat16, out=None,
               stream=None, cols=None):
    """Dequantize packed codes and block scales into a [..., cols] tensor of out_dtype.  cols
    defaults to 2 * packed.shape[-1]; give it for rows of odd length (ragged last blocks)."""
    if out_dtype not in _DT:
        raise ValueError("out_dtype must be float32 or bfloat16")
    prow, pcols = _shape2d(packed, "packed")
    _shape2d(scales, "scales")
    if cols is None:
        cols = 2 * pcols
    elif (cols + 1) // 2 != pcols:
        raise ValueError("cols does not match packed.shape[-1]")
    if out is None:
        out = torch.empty(tuple(packed.shape[:-1]) + (cols,), dtype=out_dtype, device=packed.device)
    check(lib.mx_dequantize(packed.data_ptr(), scales.data_ptr(), prow, cols, int(block),
                            fmt_code(fmt), g_bits(g), out.data_ptr(), _DT[out.dtype],
                            _stream(stream, packed.device)), "mx_dequantize")
    return out


def fake_quantize(x, block=32, fmt="e4m3", g=None, out_dtype=None, out=None, stream=None):
    """dequantize(quantize(x)) in one pass (x read once, only y written); out_dtype defaults to
    x's dtype.  No gradient: see FakeQuantize for the autograd version."""
    rows, cols = _shape2d(x, "x")
    if x.dtype not in _DT:
        raise ValueError("x must be float32 or bfloat16")
    out_dtype = out_dtype or x.dtype
    if out_dtype not in _DT:
        raise ValueError("out_dtype must be float32 or bfloat16")
    if out is None:
        out = torch.empty(x.shape, dtype=out_dtype, device=x.device)
    check(lib.mx_fake_quantize(x.data_ptr(), _DT[x.dtype], rows, cols, int(block), fmt_code(fmt),
                               g_bits(g), out.data_ptr(), _DT[out.dtype],
                               _stream(stream, x.device)), "mx_fake_quantize")
    return out


class FakeQuantize(torch.autograd.Function):
    """Quantization-aware training op: forward y = dequant(quant(x)) (one kernel pass), backward
    the straight-through estimator (the incoming gradient passes unchanged to x).  The pages give
    the forward only; straight-through is the plain reading for the backward."""

    @staticmethod
    def forward(ctx, x, block=32, fmt="e4m3", g=None):
        return fake_quantize(x.contiguous(), block, fmt, g)

    @staticmethod
    def backward(ctx, grad_y):
        return grad_y, None, None, None


def record_dict(raw):
    """An mx_error_stats_t record (64 bytes, host) as a dict of its fields plus the pages' mean
    squared errors (mse_elem, mse_max, mse_zero, mse_total), which the library computes from the
    sums (mx_error_stats_means)."""
    raw = bytes(raw)
    d = dict(zip(STATS_FIELDS, struct.unpack("<3d5q", raw)))
    buf = ctypes.create_string_buffer(raw, STATS_BYTES)
    mse = (ctypes.c_double * 4)()
    check(lib.mx_error_stats_means(ctypes.addressof(buf), mse), "mx_error_stats_means")
    d.update(mse_elem=mse[0], mse_max=mse[1], mse_zero=mse[2], mse_total=mse[3])
    return d


def record_bytes(d):
    """The 64-byte mx_error_stats_t of a dict with the record's fields."""
    return struct.pack("<3d5q", *(float(d[k]) for k in STATS_FIELDS[:3]),
                       *(int(d[k]) for k in STATS_FIELDS[3:]))


class ErrorStats:
    """Device-resident mx_error_stats_t (64 bytes); to_dict() copies it to the host."""

    def __init__(self, tensor):
        self.tensor = tensor

    def to_dict(self):
        return record_dict(self.tensor.cpu().numpy().tobytes())


def stats_workspace(device, rows=0, cols=0, block=32):
    n = lib.mx_error_stats_workspace_size(rows, cols, block)
    return torch.empty(n, dtype=torch.uint8, device=device)


def error_stats(x, block=32, fmt="e4m3", g=None, packed=None, scales=None, out=None,
                workspace=None, stream=None):
    """Three-term error sums of quantizing x (codes recomputed when packed is None)."""
    rows, cols = _shape2d(x, "x")
    if x.dtype not in _DT:
        raise ValueError("x must be float32 or bfloat16")
    if out is None:
        out = torch.empty(STATS_BYTES, dtype=torch.uint8, device=x.device)
    if workspace is None:
        workspace = stats_workspace(x.device, rows, cols, block)
    check(lib.mx_error_stats(x.data_ptr(), _DT[x.dtype], rows, cols, int(block), fmt_code(fmt),
                             g_bits(g), None if packed is None else packed.data_ptr(),
                             None if scales is None else scales.data_ptr(), out.data_ptr(),
                             workspace.data_ptr(), workspace.numel(), _stream(stream, x.device)),
          "mx_error_stats")
    return ErrorStats(out)


def quantize_with_stats(x, block=32, fmt="e4m3", g=None, packed=None, scales=None, out=None,
                        workspace=None, stream=None):
    """Quantize + pack with the three-term error reduction in the same pass over x.

    Returns (packed, scales, ErrorStats); the same values as quantize() followed by
    error_stats(x, packed=..., scales=...)."""
    rows, cols = _shape2d(x, "x")
    if x.dtype not in _DT:
        raise ValueError("x must be float32 or bfloat16")
    lead = tuple(x.shape[:-1])
    if packed is None:
        packed = torch.empty(lead + ((cols + 1) // 2,), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(lead + (-(-cols // block) if block else 0,), dtype=torch.uint8,
                             device=x.device)
    if out is None:
        out = torch.empty(STATS_BYTES, dtype=torch.uint8, device=x.device)
    if workspace is None:
        workspace = stats_workspace(x.device, rows, cols, block)
    check(lib.mx_quantize_stats(x.data_ptr(), _DT[x.dtype], rows, cols, int(block), fmt_code(fmt),
                                g_bits(g), packed.data_ptr(), scales.data_ptr(), out.data_ptr(),
                                workspace.data_ptr(), workspace.numel(),
                                _stream(stream, x.device)), "mx_quantize_stats")
    return packed, scales, ErrorStats(out)


def global_scale(x, fmt="e4m3", out=None, workspace=None, stream=None):
    """Per-tensor FP16 scale of x, as a device uint16 tensor of one element (bit pattern)."""
    rows, cols = _shape2d(x, "x")
    if x.dtype not in _DT:
        raise ValueError("x must be float32 or bfloat16")
    if out is None:
        out = torch.empty(8, dtype=torch.uint8, device=x.device)  # 16-byte aligned allocation
    if workspace is None:
        workspace = torch.empty(lib.mx_global_scale_workspace_size(rows, cols), dtype=torch.uint8,
                                device=x.device)
    check(lib.mx_global_scale(x.data_ptr(), _DT[x.dtype], rows, cols, fmt_code(fmt),
                              out.data_ptr(), workspace.data_ptr(), workspace.numel(),
                              _stream(stream, x.device)), "mx_global_scale")
    return out[:2].view(torch.uint16)


# ---- grouped calls: one launch for up to MX_MAX_GROUP tensors of the same dtype, block, format

def global_scale_group(xs, fmt="e4m3", out=None, workspace=None, stream=None):
    """global_scale() of every tensor of xs in one launch.  Returns a CUDA int16 tensor of
    len(xs) binary16 bit patterns, which the other grouped calls accept as g (read on the
    device)."""
    xs = list(xs)
    n = len(xs)
    desc = _group(n, "global_scale_group")
    dt = {x.dtype for x in xs}
    if len(dt) != 1 or next(iter(dt)) not in _DT:
        raise ValueError("all tensors float32 or all bfloat16")
    dev = xs[0].device
    if out is None:
        out = torch.empty(n, dtype=torch.int16, device=dev)
    if workspace is None:
        workspace = torch.empty(lib.mx_global_scale_workspace_size(0, 0), dtype=torch.uint8,
                                device=dev)
    for k, x in enumerate(xs):
        rows, cols = _shape2d(x, "x")
        desc[k].x, desc[k].rows, desc[k].cols = x.data_ptr(), rows, cols
        desc[k].global_scale_dev = out.data_ptr() + 2 * k
    check(lib.mx_global_scale_group(desc, n, _DT[xs[0].dtype], fmt_code(fmt), workspace.data_ptr(),
                                    workspace.numel(), _stream(stream, dev)),
          "mx_global_scale_group")
    return out


def _group(n, what):
    if not 1 <= n <= MX_MAX_GROUP:
        raise ValueError(f"{what}: between 1 and {MX_MAX_GROUP} tensors per call")
    return (Tensor * n)()


def _gs(g, n):
    """Per-tensor g of a grouped call: (bit patterns, device addresses).  g may be one value, one
    value per tensor, or a CUDA tensor of n 16-bit elements (e.g. from global_scale_group), whose
    values the kernels read on the device (they never visit the host)."""
    if isinstance(g, torch.Tensor):
        if not g.is_cuda or g.numel() != n or g.element_size() != 2 or not g.is_contiguous():
            raise ValueError("device global scales: a contiguous CUDA tensor of n 16-bit values")
        return [0] * n, [g.data_ptr() + 2 * k for k in range(n)]
    if isinstance(g, (list, tuple)):
        if len(g) != n:
            raise ValueError("one global scale per tensor")
        return [g_bits(v) for v in g], [None] * n
    return [g_bits(g)] * n, [None] * n


def _set_g(desc, gs, k):
    desc.global_scale_fp16 = gs[0][k]
    desc.global_scale_dev = gs[1][k]


def quantize_group(xs, block=32, fmt="e4m3", g=None, packed=None, scales=None, stream=None):
    """quantize() of every tensor of xs in one launch; g: one value or one per tensor.
    Returns (list of packed, list of scales)."""
    xs = list(xs)
    n = len(xs)
    desc = _group(n, "quantize_group")
    dt = {x.dtype for x in xs}
    if len(dt) != 1 or next(iter(dt)) not in _DT:
        raise ValueError("all tensors float32 or all bfloat16")
    gs = _gs(g, n)
    packed = list(packed) if packed is not None else [None] * n
    scales = list(scales) if scales is not None else [None] * n
    for k, x in enumerate(xs):
        rows, cols = _shape2d(x, "x")
        lead = tuple(x.shape[:-1])
        if packed[k] is None:
            packed[k] = torch.empty(lead + ((cols + 1) // 2,), dtype=torch.uint8,
                                    device=x.device)
        if scales[k] is None:
            scales[k] = torch.empty(lead + (-(-cols // block) if block else 0,),
                                    dtype=torch.uint8, device=x.device)
        desc[k].x, desc[k].packed, desc[k].scales = (x.data_ptr(), packed[k].data_ptr(),
                                                     scales[k].data_ptr())
        desc[k].rows, desc[k].cols = rows, cols
        _set_g(desc[k], gs, k)
    check(lib.mx_quantize_group(desc, n, _DT[xs[0].dtype], int(block), fmt_code(fmt),
                                _stream(stream, xs[0].device)), "mx_quantize_group")
    return packed, scales


def dequantize_group(packed, scales, block=32, fmt="e4m3", g=None, out_dtype=torch.bfloat16,
                     out=None, stream=None, cols=None):
    """dequantize() of every (packed, scales) pair in one launch.  cols: the row length of each
    tensor (default 2 * packed.shape[-1]; give it for rows of odd length).  Returns the list of
    outputs."""
    packed, scales = list(packed), list(scales)
    n = len(packed)
    if len(scales) != n:
        raise ValueError("one scales tensor per packed tensor")
    if out_dtype not in _DT:
        raise ValueError("out_dtype must be float32 or bfloat16")
    desc = _group(n, "dequantize_group")
    gs = _gs(g, n)
    out = list(out) if out is not None else [None] * n
    cols = list(cols) if cols is not None else [None] * n
    for k in range(n):
        prow, pcols = _shape2d(packed[k], "packed")
        _shape2d(scales[k], "scales")
        ck = 2 * pcols if cols[k] is None else int(cols[k])
        if (ck + 1) // 2 != pcols:
            raise ValueError("cols does not match packed.shape[-1]")
        if out[k] is None:
            out[k] = torch.empty(tuple(packed[k].shape[:-1]) + (ck,), dtype=out_dtype,
                                 device=packed[k].device)
        desc[k].y, desc[k].packed, desc[k].scales = (out[k].data_ptr(), packed[k].data_ptr(),
                                                     scales[k].data_ptr())
        desc[k].rows, desc[k].cols = prow, ck
        _set_g(desc[k], gs, k)
    check(lib.mx_dequantize_group(desc, n, int(block), fmt_code(fmt), _DT[out_dtype],
                                  _stream(stream, packed[0].device)), "mx_dequantize_group")
    return out


def quantize_with_stats_group(xs, block=32, fmt="e4m3", g=None, packed=None, scales=None,
                              out=None, workspace=None, stream=None):
    """quantize_with_stats() of every tensor of xs in one launch.  out: a uint8 tensor of
    len(xs) x 64 bytes for the records (allocated when None).  Returns (packed list, scales list,
    list of ErrorStats)."""
    xs = list(xs)
    n = len(xs)
    desc = _group(n, "quantize_with_stats_group")
    dt = {x.dtype for x in xs}
    if len(dt) != 1 or next(iter(dt)) not in _DT:
        raise ValueError("all tensors float32 or all bfloat16")
    gs = _gs(g, n)
    dev = xs[0].device
    if out is None:
        out = torch.empty(n, STATS_BYTES, dtype=torch.uint8, device=dev)
    if workspace is None:
        workspace = stats_workspace(dev)
    packed = list(packed) if packed is not None else [None] * n
    scales = list(scales) if scales is not None else [None] * n
    for k, x in enumerate(xs):
        rows, cols = _shape2d(x, "x")
        lead = tuple(x.shape[:-1])
        if packed[k] is None:
            packed[k] = torch.empty(lead + ((cols + 1) // 2,), dtype=torch.uint8,
                                    device=x.device)
        if scales[k] is None:
            scales[k] = torch.empty(lead + (-(-cols // block) if block else 0,),
                                    dtype=torch.uint8, device=x.device)
        desc[k].x, desc[k].packed, desc[k].scales = (x.data_ptr(), packed[k].data_ptr(),
                                                     scales[k].data_ptr())
        desc[k].stats = out[k].data_ptr()
        desc[k].rows, desc[k].cols = rows, cols
        _set_g(desc[k], gs, k)
    check(lib.mx_quantize_stats_group(desc, n, _DT[xs[0].dtype], int(block), fmt_code(fmt),
                                      workspace.data_ptr(), workspace.numel(),
                                      _stream(stream, dev)), "mx_quantize_stats_group")
    return packed, scales, [ErrorStats(out[k]) for k in range(n)]


def prepare_scales(scales, k, out=None, stream=None):
    """Scales of a rows x k operand (uint8 [rows, k/16], block 16) in tensor-core order for
    matmul; returns a uint8 tensor of mx_matmul_scales_size(rows, k) bytes."""
    rows = scales.shape[0] if scales.dim() == 2 else 0
    _shape2d(scales, "scales")
    size = int(lib.mx_matmul_scales_size(rows, int(k)))
    if size == 0 and rows:
        raise ValueError("k must be a positive multiple of 256")
    if out is None:
        out = torch.empty(max(size, 16), dtype=torch.uint8, device=scales.device)
    check(lib.mx_matmul_prepare_scales(scales.data_ptr(), rows, int(k), out.data_ptr(), out.numel(),
                                       _stream(stream, scales.device)), "mx_matmul_prepare_scales")
    return out


def matmul(a_packed, a_scales, b_packed, b_scales, a_g=None, b_g=None, out_dtype=torch.bfloat16,
           out=None, prepared=False, stream=None, cta_pairs=False):
    """C = dequant(A) dequant(B)^T on the tensor cores (block 16, E4M3 scales, as quantize writes
    them): a_packed [m, k/2] of an m x k tensor, b_packed [n, k/2] of an n x k tensor; a_scales /
    b_scales are the quantizer's [rows, k/16] arrays, or (prepared=True) the outputs of
    prepare_scales.  cta_pairs: the CTA-pair kernel (mx_matmul_pair).  Returns C [m, n] of
    out_dtype."""
    if out_dtype not in _DT:
        raise ValueError("out_dtype must be float32 or bfloat16")
    for t, what in ((a_packed, "a_packed"), (b_packed, "b_packed")):
        if t.dim() != 2:
            raise ValueError(f"{what} must be 2-D")
        _shape2d(t, what)
    m, n, k = a_packed.shape[0], b_packed.shape[0], 2 * a_packed.shape[1]
    if 2 * b_packed.shape[1] != k:
        raise ValueError("A and B must have the same k")
    if not prepared and m and n:
        a_scales = prepare_scales(a_scales, k, stream=stream)
        b_scales = prepare_scales(b_scales, k, stream=stream)
    if out is None:
        out = torch.empty((m, n), dtype=out_dtype, device=a_packed.device)
    fn = lib.mx_matmul_pair if cta_pairs else lib.mx_matmul
    check(fn(a_packed.data_ptr(), a_scales.data_ptr(), g_bits(a_g), b_packed.data_ptr(),
             b_scales.data_ptr(), g_bits(b_g), m, n, k, 16, E4M3, out.data_ptr(), _DT[out.dtype],
             _stream(stream, a_packed.device)), "mx_matmul")
    return out


def dequant_matmul(a, w_packed, w_scales, block=32, fmt="ue5m3", g=None, out_dtype=torch.bfloat16,
                   out=None, stream=None):
    """C = a dequant(W)^T on the tensor cores: a [m, k] bfloat16 activations, W an n x k weight
    tensor as quantize() stores it (w_packed [n, k/2], w_scales [n, k/block]) with any block size,
    E4M3 or UE5M3 scales and global scale g (a value, or a CUDA tensor of one 16-bit bit pattern
    read on the device, e.g. from global_scale).  The weights enter as their bf16 dequantization.
    Returns C [m, n] of out_dtype."""
    if out_dtype not in _DT:
        raise ValueError("out_dtype must be float32 or bfloat16")
    if a.dtype != torch.bfloat16 or a.dim() != 2 or w_packed.dim() != 2:
        raise ValueError("a must be a 2-D bfloat16 tensor and w_packed 2-D")
    _shape2d(a, "a")
    _shape2d(w_packed, "w_packed")
    _shape2d(w_scales, "w_scales")
    m, k = a.shape
    n = w_packed.shape[0]
    if 2 * w_packed.shape[1] != k:
        raise ValueError("w_packed must hold n x k codes (k / 2 bytes per row)")
    g_dev = None
    if isinstance(g, torch.Tensor):
        if not g.is_cuda or g.numel() < 1 or g.element_size() != 2:
            raise ValueError("device global scale: a CUDA tensor of 16-bit values")
        g_dev, gb = g.data_ptr(), 0
    else:
        gb = g_bits(g)
    if out is None:
        out = torch.empty((m, n), dtype=out_dtype, device=a.device)
    check(lib.mx_dequant_matmul(a.data_ptr(), m, k, w_packed.data_ptr(), w_scales.data_ptr(), n,
                                int(block), fmt_code(fmt), gb, g_dev, out.data_ptr(),
                                _DT[out.dtype], _stream(stream, a.device)), "mx_dequant_matmul")
    return out


def matmul_gave_up():
    """Number of matmul thread blocks whose bounded waits ran out since the last call (0 normally);
    synchronizes the device."""
    c = ctypes.c_uint(0)
    check(lib.mx_matmul_gave_up(ctypes.byref(c)), "mx_matmul_gave_up")
    return int(c.value)


def kernel_launches():
    """Number of kernels the library has enqueued in this process (diagnostic)."""
    return int(lib.mx_kernel_launches())
