"""mx_error_stats_noalloc: the error reduction for callers that cannot allocate a workspace (its
scratch is a fixed array inside the library).  Called through the C ABI and checked against the
workspace entry point mx_error_stats and against the oracle on two calls in a row, so the second
call runs over the scratch contents the first one left behind.  Whole-block tensors and ragged ones
(cols not a multiple of the block, the row-wise path with its own scratch layout) are both run.
Collected last on purpose (file name)."""
import ctypes
import struct

import numpy as np
import pytest
import torch

import oracle
from fp4_microscaling_tensor_b200 import _lib, inputs
import fp4_microscaling_tensor_b200 as mx

pytestmark = pytest.mark.gpu

RTOL = 1e-5
FIELDS = ("sse_elem", "sse_max", "sse_zero", "numel", "n_blocks", "n_zero_blocks", "n_scale_sat",
          "n_elem_sat")


def unpack(buf):
    return dict(zip(FIELDS, struct.unpack("<3d5q", buf.cpu().numpy().tobytes())))


def noalloc(x, block, fmt, g=0x3C00, packed=None, scales=None):
    out = torch.empty(64, dtype=torch.uint8, device=x.device)
    rows, cols = x.shape
    xt = _lib.MX_BF16 if x.dtype == torch.bfloat16 else _lib.MX_F32
    st = _lib.lib.mx_error_stats_noalloc(
        x.data_ptr(), xt, rows, cols, block, fmt, g,
        None if packed is None else packed.data_ptr(),
        None if scales is None else scales.data_ptr(), out.data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    assert st == _lib.MX_OK, _lib.lib.mx_status_string(st)
    return unpack(out)


def same(got, ref):
    for k in FIELDS[3:]:
        assert got[k] == ref[k], (k, got[k], ref[k])
    for k in FIELDS[:3]:
        assert abs(got[k] - ref[k]) <= RTOL * abs(ref[k]), (k, got[k], ref[k])


def test_noalloc_matches_workspace_entry_point_twice(cuda_device):
    cases = [  # (rows, cols, block, fmt, dtype, scale): later cases are smaller than the first
        (2048, 4096, 32, mx.E4M3, torch.bfloat16, 0.02),
        (37, 20, 4, mx.UE5M3, torch.bfloat16, 1e-3),
        (256, 256, 32, mx.E4M3, torch.float32, 0.02),
        (33, 100, 32, mx.UE5M3, torch.bfloat16, 0.02),   # ragged: 100 = 3 * 32 + 4
        (5, 7, 4, mx.E4M3, torch.float32, 0.5),          # ragged: 7 = 4 + 3
    ]
    gen = torch.Generator(device=cuda_device)
    gen.manual_seed(7)
    for rows, cols, block, fmt, dtype, scale in cases:
        x = (torch.randn(rows, cols, generator=gen, device=cuda_device) * scale).to(dtype)
        packed, scales = mx.quantize(x, block, fmt)
        xo = inputs.to_oracle(x)
        po, so = oracle.quantize(xo, rows, cols, block, fmt)
        for given in (False, True):
            p, s = (packed, scales) if given else (None, None)
            ref = mx.error_stats(x, block, fmt, packed=p, scales=s).to_dict()
            orc = oracle.error_stats(xo, rows, cols, block, fmt,
                                     packed=po if given else None, scales=so if given else None)
            first = noalloc(x, block, fmt, packed=p, scales=s)
            second = noalloc(x, block, fmt, packed=p, scales=s)
            torch.cuda.synchronize()
            for got in (first, second):
                same(got, ref)
                same(got, orc)
            assert first == second
