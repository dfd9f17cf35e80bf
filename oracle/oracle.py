"""ctypes wrapper of the C oracle (TEST INFRASTRUCTURE ONLY).

Arrays are numpy: bf16 tensors are passed as their uint16 bit patterns, float32 as float32.
"""
import ctypes
import os

import numpy as np

from .build import build

F32, BF16 = 0, 1
E4M3, UE5M3 = 0, 1


class Stats(ctypes.Structure):
    _fields_ = [("sse_elem", ctypes.c_double), ("sse_max", ctypes.c_double),
                ("sse_zero", ctypes.c_double), ("numel", ctypes.c_int64),
                ("n_blocks", ctypes.c_int64), ("n_zero_blocks", ctypes.c_int64),
                ("n_scale_sat", ctypes.c_int64), ("n_elem_sat", ctypes.c_int64)]

    def as_dict(self):
        return {k: getattr(self, k) for k, _ in self._fields_}


def _load():
    L = ctypes.CDLL(build())
    d, i, u16, i64, vp = ctypes.c_double, ctypes.c_int, ctypes.c_uint16, ctypes.c_int64, ctypes.c_void_p
    for name in ("orc_e2m1_value", "orc_e4m3_value", "orc_ue5m3_value"):
        getattr(L, name).restype = d
        getattr(L, name).argtypes = [i]
    L.orc_scale_value.restype = d
    L.orc_scale_value.argtypes = [i, i]
    L.orc_fp16_value.restype = d
    L.orc_fp16_value.argtypes = [u16]
    L.orc_bf16_value.restype = d
    L.orc_bf16_value.argtypes = [u16]
    L.orc_round_scale.restype = i
    L.orc_round_scale.argtypes = [d, i]
    L.orc_round_e2m1_mag.restype = i
    L.orc_round_e2m1_mag.argtypes = [d]
    L.orc_scale_max.restype = d
    L.orc_scale_max.argtypes = [i]
    L.orc_scale_min.restype = d
    L.orc_scale_min.argtypes = [i]
    L.orc_quantize.restype = i
    L.orc_quantize.argtypes = [vp, i, i64, i64, i, i, u16, vp, vp, i]
    L.orc_dequantize.restype = i
    L.orc_dequantize.argtypes = [vp, vp, i64, i64, i, i, u16, vp, i, i]
    L.orc_error_stats.restype = i
    L.orc_error_stats.argtypes = [vp, i, i64, i64, i, i, u16, vp, vp, ctypes.POINTER(Stats), i]
    L.orc_global_scale.restype = u16
    L.orc_global_scale.argtypes = [vp, i, i64, i]
    return L


lib = _load()
_THREADS = int(os.environ.get("MX_ORACLE_THREADS", os.cpu_count() or 1))


def e2m1_value(c): return lib.orc_e2m1_value(int(c))
def e4m3_value(c): return lib.orc_e4m3_value(int(c))
def ue5m3_value(c): return lib.orc_ue5m3_value(int(c))
def scale_value(c, fmt): return lib.orc_scale_value(int(c), int(fmt))
def fp16_value(bits): return lib.orc_fp16_value(int(bits))
def round_scale(u, fmt): return lib.orc_round_scale(float(u), int(fmt))
def round_e2m1_mag(v): return lib.orc_round_e2m1_mag(float(v))
def scale_max(fmt): return lib.orc_scale_max(int(fmt))
def scale_min(fmt): return lib.orc_scale_min(int(fmt))


def _xarg(x):
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.uint16:
        return x, BF16
    raise TypeError("x must be float32 or uint16 (bf16 bit patterns)")


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def quantize(x, rows, cols, block, fmt, g_bits=0x3C00, threads=None):
    """Return (packed uint8[rows*ceil(cols/2)], scales uint8[rows*ceil(cols/block)]): rows of
    ceil(cols/2) code bytes and ceil(cols/block) scale bytes (the last block of a row holds
    cols mod block elements when block does not divide cols)."""
    x, xt = _xarg(x)
    assert x.size == rows * cols
    packed = np.zeros(rows * ((cols + 1) // 2), np.uint8)
    scales = np.zeros(rows * (-(-cols // block) if block > 0 else 0), np.uint8)
    rc = lib.orc_quantize(_ptr(x), xt, rows, cols, block, fmt, g_bits, _ptr(packed), _ptr(scales),
                          threads or _THREADS)
    if rc != 0:
        raise ValueError("oracle quantize rejected its arguments")
    return packed, scales


def dequantize(packed, scales, rows, cols, block, fmt, g_bits=0x3C00, out_bf16=True, threads=None):
    """Return y as uint16 bf16 bit patterns (out_bf16) or float32."""
    packed = np.ascontiguousarray(packed, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    y = np.zeros(rows * cols, np.uint16 if out_bf16 else np.float32)
    rc = lib.orc_dequantize(_ptr(packed), _ptr(scales), rows, cols, block, fmt, g_bits, _ptr(y),
                            BF16 if out_bf16 else F32, threads or _THREADS)
    if rc != 0:
        raise ValueError("oracle dequantize rejected its arguments")
    return y


def error_stats(x, rows, cols, block, fmt, g_bits=0x3C00, packed=None, scales=None, threads=None):
    """Three-term error sums and counts as a dict (recomputes the codes when packed is None)."""
    x, xt = _xarg(x)
    if packed is not None:
        packed = np.ascontiguousarray(packed, np.uint8)
        scales = np.ascontiguousarray(scales, np.uint8)
    out = Stats()
    rc = lib.orc_error_stats(_ptr(x), xt, rows, cols, block, fmt, g_bits, _ptr(packed),
                             _ptr(scales), ctypes.byref(out), threads or _THREADS)
    if rc != 0:
        raise ValueError("oracle error_stats rejected its arguments")
    return out.as_dict()


def global_scale(x, fmt):
    """Per-tensor FP16 scale bit pattern."""
    x, xt = _xarg(x)
    return lib.orc_global_scale(_ptr(x), xt, x.size, fmt)


def matmul(a_packed, a_scales, a_g_bits, b_packed, b_scales, b_g_bits, m, n, k, block, fmt):
    """C = dequant(A) dequant(B)^T in float64 (m x n), A m x k and B n x k in the library's layout.

    The 4-bit float quantization article (gtnt.cn/news/16247, §3.1, the inference step that
    dequantizes the stored weights before the matrix multiply) dequantizes, then multiplies.  Here both operands are stored block-quantized along k (the reduction dimension);
    each is dequantized exactly (E2M1 x scale x g fits float32 exactly) and the product is one
    float64 matrix multiply, whose rounding error (at most k 2^-53 relative to sum |a b|) is far
    below any float32 accumulation.
    """
    ya = dequantize(a_packed, a_scales, m, k, block, fmt, a_g_bits, out_bf16=False)
    yb = dequantize(b_packed, b_scales, n, k, block, fmt, b_g_bits, out_bf16=False)
    A = ya.astype(np.float64).reshape(m, k)
    B = yb.astype(np.float64).reshape(n, k)
    return A @ B.T



def bf16_values(bits):
    """float64 values of bf16 bit patterns: a bf16 value is the float32 whose upper 16 bits are
    the pattern and whose lower 16 bits are zero."""
    bits = np.ascontiguousarray(bits, np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def dequant_matmul(a_bits, m, k, w_packed, w_scales, n, block, fmt, w_g_bits=0x3C00):
    """C = A dequant(W)^T in float64 (m x n): A an m x k bf16 tensor (uint16 bit patterns), W an
    n x k tensor stored by the quantizer.

    The 4-bit float quantization article (gtnt.cn/news/16247, §3.1) runs inference by dequantizing
    the stored weights to the activations' type and multiplying.  Here the weights' values are
    their bf16 dequantization (round to nearest even of E2M1 x S x g, what dequantize() returns
    with out_bf16=True), the activations their exact bf16 values, and the product is one float64
    matrix multiply, whose rounding (at most k 2^-53 relative to sum |a w|) is far below any
    float32 accumulation.
    """
    A = bf16_values(a_bits).reshape(m, k)
    yw = dequantize(w_packed, w_scales, n, k, block, fmt, w_g_bits, out_bf16=True)
    W = bf16_values(yw).reshape(n, k)
    return A @ W.T
