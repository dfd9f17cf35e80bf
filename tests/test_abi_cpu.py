"""The C-ABI library loads, exports every symbol include/mx.h declares, and rejects bad arguments
on the host before enqueueing anything (no compute call is made: every call here is invalid)."""
import ctypes
import os
import re

import pytest

from fp4_microscaling_tensor_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
L = _lib.lib
OK, INV, UNS, MIS, WS = (_lib.MX_OK, _lib.MX_ERR_INVALID_ARG, _lib.MX_ERR_UNSUPPORTED,
                         _lib.MX_ERR_MISALIGNED, _lib.MX_ERR_WORKSPACE)
A = 0x10000  # a fake 16-byte-aligned device address; never dereferenced (every call fails first)
BF16, F32, E4, UE = _lib.MX_BF16, _lib.MX_F32, _lib.MX_SCALE_E4M3, _lib.MX_SCALE_UE5M3


def declared_symbols():
    with open(os.path.join(ROOT, "include", "mx.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"MX_API\s+[\w\s\*]+?\b(mx_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = declared_symbols()
    assert len(names) >= 8
    for n in names:
        assert hasattr(L, n), n
    assert sorted(_lib.EXPORTS) == names


def test_status_strings():
    for s in range(6):
        assert L.mx_status_string(s)
    assert b"unknown" in L.mx_status_string(99)


def test_workspace_sizes():
    assert L.mx_error_stats_workspace_size(4096, 4096, 32) >= 64
    assert L.mx_global_scale_workspace_size(4096, 4096) >= 4


def q(x=A, xt=BF16, rows=4, cols=64, block=32, fmt=E4, g=0x3C00, p=A, s=A):
    return L.mx_quantize(x, xt, rows, cols, block, fmt, g, p, s, None)


def test_quantize_rejects_bad_arguments():
    assert q(x=None) == INV
    assert q(p=None) == INV
    assert q(s=None) == INV
    assert q(rows=-1) == INV
    assert q(cols=-8) == INV                      # negative size
    assert q(block=12) == UNS
    assert q(block=512) == UNS
    assert q(block=2) == UNS
    assert q(xt=7) == INV
    assert q(fmt=3) == INV
    for g in (0x0000, 0x8000, 0xBC00, 0x7C00, 0x7E00, 0xFC00):  # 0, -0, <0, inf, nan, -inf
        assert q(g=g) == INV
    assert q(x=A + 8) == MIS
    assert q(p=A + 4) == MIS
    assert q(s=A + 1) == MIS
    assert q(rows=1 << 40, cols=1 << 40) == INV   # element count overflows


def test_dequantize_rejects_bad_arguments():
    def dq(p=A, s=A, rows=4, cols=64, block=32, fmt=E4, g=0x3C00, y=A, yt=BF16):
        return L.mx_dequantize(p, s, rows, cols, block, fmt, g, y, yt, None)
    assert dq(p=None) == INV
    assert dq(y=None) == INV
    assert dq(cols=-40) == INV
    assert dq(block=24) == UNS
    assert dq(yt=2) == INV
    assert dq(g=0) == INV
    assert dq(y=A + 2) == MIS
    assert dq(s=A + 3) == MIS


def test_error_stats_rejects_bad_arguments():
    ws = L.mx_error_stats_workspace_size(4, 64, 32)

    def st(x=A, p=None, s=None, out=A, w=A, n=ws, block=32, cols=64, g=0x3C00):
        return L.mx_error_stats(x, BF16, 4, cols, block, E4, g, p, s, out, w, n, None)
    assert st(out=None) == INV
    assert st(x=None) == INV
    assert st(p=A, s=None) == INV                 # packed and scales go together
    assert st(p=None, s=A) == INV
    assert st(w=None) == WS
    assert st(n=ws - 1) == WS
    assert st(cols=-50) == INV
    assert st(block=3) == UNS
    assert st(g=0xFFFF) == INV
    assert st(out=A + 8) == MIS
    assert st(w=A + 4) == MIS
    assert st(p=A + 1, s=A) == MIS


def test_quantize_stats_rejects_bad_arguments():
    ws = L.mx_error_stats_workspace_size(4, 64, 32)

    def qs(x=A, p=A, s=A, out=A, w=A, n=ws, block=32, cols=64, g=0x3C00, xt=BF16):
        return L.mx_quantize_stats(x, xt, 4, cols, block, E4, g, p, s, out, w, n, None)
    assert qs(x=None) == INV
    assert qs(p=None) == INV
    assert qs(s=None) == INV
    assert qs(out=None) == INV
    assert qs(w=None) == WS
    assert qs(n=ws - 1) == WS
    assert qs(cols=-48) == INV
    assert qs(block=64 * 8) == UNS
    assert qs(g=0x7C00) == INV
    assert qs(xt=5) == INV
    assert qs(p=A + 2) == MIS
    assert qs(out=A + 4) == MIS


def test_global_scale_rejects_bad_arguments():
    ws = L.mx_global_scale_workspace_size(4, 64)

    def gs(x=A, out=A, w=A, n=ws, fmt=UE):
        return L.mx_global_scale(x, BF16, 4, 64, fmt, out, w, n, None)
    assert gs(out=None) == INV
    assert gs(x=None) == INV
    assert gs(fmt=9) == INV
    assert gs(w=None) == WS
    assert gs(n=ws - 1) == WS
    assert gs(x=A + 2) == MIS


def test_python_binding_marshalling_errors():
    import torch
    import fp4_microscaling_tensor_b200 as mx
    with pytest.raises(ValueError):
        mx.quantize(torch.zeros(4, 64, dtype=torch.bfloat16))  # CPU tensor: not accepted
    with pytest.raises(ValueError):
        mx.fmt_code("e5m2")
    assert mx.g_bits(None) == 0x3C00 and mx.g_bits(1.0) == 0x3C00 and mx.g_bits(0x1234) == 0x1234


def group(n, rows=4, cols=64, x=A, y=A, p=A, s=A, st=A, g=0x3C00, reserved=0, gdev=None):
    d = (_lib.Tensor * max(n, 1))()
    for k in range(max(n, 1)):
        d[k].x, d[k].y, d[k].packed, d[k].scales, d[k].stats = x, y, p, s, st
        d[k].rows, d[k].cols, d[k].global_scale_fp16 = rows, cols, g
        d[k].global_scale_dev = gdev
        d[k].reserved[0] = reserved
    return d


def test_group_calls_reject_bad_arguments():
    ws = L.mx_error_stats_workspace_size(4, 64, 32)
    for n in (0, _lib.MX_MAX_GROUP + 1):
        assert L.mx_quantize_group(group(n), n, BF16, 32, E4, None) == INV
        assert L.mx_dequantize_group(group(n), n, 32, E4, BF16, None) == INV
        assert L.mx_quantize_stats_group(group(n), n, BF16, 32, E4, A, ws, None) == INV
    assert L.mx_quantize_group(None, 1, BF16, 32, E4, None) == INV
    assert L.mx_quantize_group(group(2), 2, 9, 32, E4, None) == INV           # dtype
    assert L.mx_quantize_group(group(2), 2, BF16, 12, E4, None) == UNS        # block
    L.mx_test_fail_next_calls(1)  # ragged rows (48 % 32 != 0) are accepted: stop before launch
    assert L.mx_quantize_group(group(2, cols=48), 2, BF16, 32, E4, None) == _lib.MX_ERR_CUDA
    assert L.mx_test_fail_next_calls(0) == 0
    assert L.mx_quantize_group(group(2, g=0x7C00), 2, BF16, 32, E4, None) == INV
    assert L.mx_quantize_group(group(2, reserved=1), 2, BF16, 32, E4, None) == INV
    assert L.mx_quantize_group(group(2, x=None), 2, BF16, 32, E4, None) == INV
    assert L.mx_quantize_group(group(2, x=A + 8), 2, BF16, 32, E4, None) == MIS
    assert L.mx_quantize_group(group(2, s=A + 1), 2, BF16, 32, E4, None) == MIS
    assert L.mx_dequantize_group(group(2, y=None), 2, 32, E4, BF16, None) == INV
    assert L.mx_dequantize_group(group(2, y=A + 2), 2, 32, E4, BF16, None) == MIS
    assert L.mx_dequantize_group(group(2), 2, 32, E4, 7, None) == INV
    assert L.mx_quantize_stats_group(group(2, st=None), 2, BF16, 32, E4, A, ws, None) == INV
    assert L.mx_quantize_stats_group(group(2, st=A + 8), 2, BF16, 32, E4, A, ws, None) == MIS
    assert L.mx_quantize_stats_group(group(2), 2, BF16, 32, E4, None, ws, None) == WS
    assert L.mx_quantize_stats_group(group(2), 2, BF16, 32, E4, A, ws - 1, None) == WS
    assert L.mx_quantize_stats_group(group(2), 2, BF16, 32, E4, A + 4, ws, None) == MIS
    # one bad tensor among good ones rejects the whole call
    d = group(3)
    d[2].rows = -1
    assert L.mx_quantize_group(d, 3, BF16, 32, E4, None) == INV


def test_device_global_scales_in_groups():
    gws = L.mx_global_scale_workspace_size(4, 64)
    # g read from device memory: the bit-pattern field is then not checked, the address must be
    # 2-byte aligned
    L.mx_test_fail_next_calls(1)  # valid arguments on fake pointers: stop before any launch
    assert L.mx_quantize_group(group(2, g=0, gdev=A + 2), 2, BF16, 32, E4, None) == \
        _lib.MX_ERR_CUDA
    assert L.mx_quantize_group(group(2, g=0, gdev=A + 3), 2, BF16, 32, E4, None) == MIS
    assert L.mx_dequantize_group(group(2, g=0, gdev=A + 1), 2, 32, E4, BF16, None) == MIS
    assert L.mx_quantize_group(group(2, g=0), 2, BF16, 32, E4, None) == INV  # neither form
    # the grouped global scale writes g: the address is required, the bit pattern ignored
    assert L.mx_global_scale_group(group(2, gdev=None), 2, BF16, E4, A, gws, None) == INV
    assert L.mx_global_scale_group(group(2, gdev=A + 1), 2, BF16, E4, A, gws, None) == MIS
    assert L.mx_global_scale_group(group(2, gdev=A, x=None), 2, BF16, E4, A, gws, None) == INV
    assert L.mx_global_scale_group(group(2, gdev=A, x=A + 4), 2, BF16, E4, A, gws, None) == MIS
    assert L.mx_global_scale_group(group(2, gdev=A), 2, 5, E4, A, gws, None) == INV
    assert L.mx_global_scale_group(group(2, gdev=A), 2, BF16, 7, A, gws, None) == INV
    assert L.mx_global_scale_group(group(2, gdev=A), 2, BF16, E4, None, gws, None) == WS
    assert L.mx_global_scale_group(group(2, gdev=A), 2, BF16, E4, A, gws - 1, None) == WS
    assert L.mx_global_scale_group(group(0, gdev=A), 0, BF16, E4, A, gws, None) == INV
    L.mx_test_fail_next_calls(1)  # any cols is fine for the global scale (it has no block)
    assert L.mx_global_scale_group(group(2, gdev=A, cols=40), 2, BF16, E4, A, gws, None) == \
        _lib.MX_ERR_CUDA
    assert L.mx_test_fail_next_calls(0) == 0


def test_error_stats_means_on_the_host():
    import fp4_microscaling_tensor_b200 as mx
    rec = mx.api.record_bytes(dict(sse_elem=3.0, sse_max=1.5, sse_zero=0.5, numel=8, n_blocks=1,
                                   n_zero_blocks=0, n_scale_sat=0, n_elem_sat=0))
    d = mx.api.record_dict(rec)
    assert (d["mse_elem"], d["mse_max"], d["mse_zero"], d["mse_total"]) == \
        (3.0 / 8, 1.5 / 8, 0.5 / 8, 5.0 / 8)
    empty = mx.api.record_dict(mx.api.record_bytes(dict.fromkeys(mx.api.STATS_FIELDS, 0)))
    assert empty["mse_total"] == 0.0
    out = (ctypes.c_double * 4)()
    assert L.mx_error_stats_means(None, out) == INV
    buf = ctypes.create_string_buffer(rec, 64)
    assert L.mx_error_stats_means(ctypes.addressof(buf), None) == INV


def test_fake_quantize_rejects_bad_arguments():
    def fq(x=A, xt=BF16, rows=4, cols=64, block=32, fmt=E4, g=0x3C00, y=A, yt=BF16):
        return L.mx_fake_quantize(x, xt, rows, cols, block, fmt, g, y, yt, None)
    assert fq(x=None) == INV
    assert fq(y=None) == INV
    assert fq(yt=3) == INV
    assert fq(xt=3) == INV
    assert fq(cols=-40) == INV
    assert fq(block=24) == UNS
    assert fq(g=0xFC00) == INV
    assert fq(x=A + 2) == MIS
    assert fq(y=A + 8) == MIS
    assert fq(rows=0, x=None, y=None) == OK      # empty: nothing to do


def test_matmul_rejects_bad_arguments():
    def mm(ap=A, as_=A, ag=0x3C00, bp=A, bs=A, bg=0x3C00, m=128, n=64, k=256, block=16, fmt=E4,
           c=A, ct=BF16):
        return L.mx_matmul(ap, as_, ag, bp, bs, bg, m, n, k, block, fmt, c, ct, None)
    assert mm(block=32) == UNS                   # no native tensor-core form
    assert mm(fmt=1) == UNS                      # UE5M3 scales
    assert mm(k=128) == UNS                      # k % 256 != 0
    assert mm(k=0) == UNS
    assert mm(fmt=5) == INV
    assert mm(ct=4) == INV
    assert mm(ag=0x7C00) == INV                  # g must be finite and positive
    assert mm(bg=0x8000) == INV
    assert mm(m=-1) == INV
    assert mm(n=1 << 31) == INV
    assert mm(ap=None) == INV
    assert mm(bs=None) == INV
    assert mm(c=None) == INV
    assert mm(ap=A + 8) == MIS
    assert mm(bs=A + 4) == MIS
    assert mm(c=A + 2) == MIS
    assert mm(m=0, ap=None, as_=None, c=None) == OK   # empty product: nothing to do
    assert mm(n=0) == OK
    assert L.mx_matmul_gave_up(None) == INV
    # the CTA-pair entry point checks the same arguments
    args = (A, A, 0x3C00, A, A, 0x3C00, 128, 64, 256, 32, E4, A, BF16, None)
    assert L.mx_matmul_pair(*args) == UNS


def test_dequant_matmul_rejects_bad_arguments():
    def dm(a=A, m=128, k=256, pw=A, sw=A, n=64, block=32, fmt=UE, g=0x3C00, gdev=None, c=A,
           ct=BF16):
        return L.mx_dequant_matmul(a, m, k, pw, sw, n, block, fmt, g, gdev, c, ct, None)
    assert dm(k=96) == UNS                       # k not a multiple of 64
    assert dm(k=128, block=256) == UNS           # k not a multiple of the block
    assert dm(block=12) == UNS
    assert dm(k=0) == UNS
    assert dm(fmt=3) == INV
    assert dm(ct=9) == INV
    assert dm(g=0x7C00) == INV                   # g must be finite and positive ...
    L.mx_test_fail_next_calls(1)
    assert dm(g=0, gdev=A + 2) == _lib.MX_ERR_CUDA   # ... unless read from device memory
    assert dm(g=0, gdev=A + 1) == MIS
    assert dm(m=-1) == INV
    assert dm(n=1 << 31) == INV
    assert dm(k=1 << 31) == INV
    assert dm(a=None) == INV
    assert dm(sw=None) == INV
    assert dm(c=None) == INV
    assert dm(a=A + 8) == MIS
    assert dm(pw=A + 4) == MIS
    assert dm(c=A + 2) == MIS
    assert dm(m=0, a=None, c=None) == OK       # empty product: nothing to do
    assert dm(n=0) == OK
    for blk in (4, 8, 16, 32, 64, 128, 256):     # every block size is accepted
        L.mx_test_fail_next_calls(1)
        assert dm(k=512, block=blk) == _lib.MX_ERR_CUDA
    assert L.mx_test_fail_next_calls(0) == 0


def test_matmul_scale_preparation_arguments():
    assert L.mx_matmul_scales_size(128, 256) == 256 * 16        # rows padded to 256
    assert L.mx_matmul_scales_size(300, 512) == 512 * 32
    assert L.mx_matmul_scales_size(0, 256) == 0
    assert L.mx_matmul_scales_size(128, 128) == 0               # k not a multiple of 256
    assert L.mx_matmul_scales_size(-1, 256) == 0
    size = L.mx_matmul_scales_size(128, 256)
    def prep(s=A, rows=128, k=256, out=A, nbytes=size):
        return L.mx_matmul_prepare_scales(s, rows, k, out, nbytes, None)
    assert prep(k=128) == UNS
    assert prep(k=0) == UNS
    assert prep(rows=-1) == INV
    assert prep(s=None) == INV
    assert prep(out=None) == INV
    assert prep(nbytes=size - 1) == WS
    assert prep(s=A + 4) == MIS
    assert prep(out=A + 8) == MIS
    assert prep(rows=0, s=None, out=None) == OK


def test_injected_cuda_failure_is_reported_before_any_launch():
    # valid arguments on fake pointers: the armed failures are consumed before anything is
    # enqueued, so nothing touches the (fake) buffers; the status is MX_ERR_CUDA
    assert L.mx_test_fail_next_calls(2) == 0
    assert q() == _lib.MX_ERR_CUDA
    ws = L.mx_error_stats_workspace_size(4, 64, 32)
    assert L.mx_quantize_stats(A, BF16, 4, 64, 32, E4, 0x3C00, A, A, A, A, ws, None) == \
        _lib.MX_ERR_CUDA
    assert L.mx_test_fail_next_calls(0) == 0           # both consumed
    # argument checks come first: an invalid call does not consume an armed failure
    assert L.mx_test_fail_next_calls(1) == 0
    assert q(block=12) == UNS
    assert L.mx_test_fail_next_calls(0) == 1           # still pending, now disarmed
