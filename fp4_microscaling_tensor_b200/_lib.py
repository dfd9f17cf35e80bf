"""ctypes binding of libmxfp4_b200.so (the C ABI in include/mx.h).

Argument marshalling only: every step of the method runs in the library's CUDA kernels.  PyTorch is
used for device memory and streams.  Importing this module fails loudly when the library has not
been built; there is no fallback.
"""
import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmxfp4_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m fp4_microscaling_tensor_b200.build` "
        "(nvcc, sm_100a) or __graft_entry__.build()")

lib = ctypes.CDLL(LIB_PATH)

MX_OK, MX_ERR_INVALID_ARG, MX_ERR_UNSUPPORTED, MX_ERR_MISALIGNED, MX_ERR_WORKSPACE, MX_ERR_CUDA = \
    range(6)
MX_F32, MX_BF16 = 0, 1
MX_SCALE_E4M3, MX_SCALE_UE5M3 = 0, 1

# every symbol declared in include/mx.h
EXPORTS = ("mx_quantize", "mx_dequantize", "mx_error_stats_workspace_size", "mx_error_stats",
           "mx_quantize_stats",
           "mx_global_scale_workspace_size", "mx_global_scale", "mx_error_stats_noalloc",
           "mx_quantize_group", "mx_dequantize_group", "mx_quantize_stats_group",
           "mx_global_scale_group", "mx_error_stats_means",
           "mx_fake_quantize", "mx_matmul_scales_size", "mx_matmul_prepare_scales",
           "mx_matmul", "mx_matmul_pair", "mx_dequant_matmul", "mx_matmul_gave_up",
           "mx_test_matmul_abandon_last",
           "mx_test_fail_next_calls", "mx_status_string", "mx_kernel_launches")
MX_MAX_GROUP = 16


class Tensor(ctypes.Structure):
    """mx_tensor_t (72 bytes): one tensor of a grouped call."""
    _fields_ = [("x", ctypes.c_void_p), ("y", ctypes.c_void_p), ("packed", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("stats", ctypes.c_void_p),
                ("global_scale_dev", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("global_scale_fp16", ctypes.c_uint16), ("reserved", ctypes.c_uint16 * 3)]


assert ctypes.sizeof(Tensor) == 72

_i, _i64, _u16, _vp, _sz = ctypes.c_int, ctypes.c_int64, ctypes.c_uint16, ctypes.c_void_p, ctypes.c_size_t

lib.mx_quantize.restype = _i
lib.mx_quantize.argtypes = [_vp, _i, _i64, _i64, _i, _i, _u16, _vp, _vp, _vp]
lib.mx_dequantize.restype = _i
lib.mx_dequantize.argtypes = [_vp, _vp, _i64, _i64, _i, _i, _u16, _vp, _i, _vp]
lib.mx_error_stats_workspace_size.restype = _sz
lib.mx_error_stats_workspace_size.argtypes = [_i64, _i64, _i]
lib.mx_error_stats.restype = _i
lib.mx_error_stats.argtypes = [_vp, _i, _i64, _i64, _i, _i, _u16, _vp, _vp, _vp, _vp, _sz, _vp]
lib.mx_quantize_stats.restype = _i
lib.mx_quantize_stats.argtypes = [_vp, _i, _i64, _i64, _i, _i, _u16, _vp, _vp, _vp, _vp, _sz, _vp]
lib.mx_global_scale_workspace_size.restype = _sz
lib.mx_global_scale_workspace_size.argtypes = [_i64, _i64]
lib.mx_global_scale.restype = _i
lib.mx_global_scale.argtypes = [_vp, _i, _i64, _i64, _i, _vp, _vp, _sz, _vp]
lib.mx_error_stats_noalloc.restype = _i
lib.mx_error_stats_noalloc.argtypes = [_vp, _i, _i64, _i64, _i, _i, _u16, _vp, _vp, _vp, _vp]
lib.mx_test_fail_next_calls.restype = _i
lib.mx_test_fail_next_calls.argtypes = [_i]
lib.mx_fake_quantize.restype = _i
lib.mx_fake_quantize.argtypes = [_vp, _i, _i64, _i64, _i, _i, _u16, _vp, _i, _vp]
_tp = ctypes.POINTER(Tensor)
lib.mx_quantize_group.restype = _i
lib.mx_quantize_group.argtypes = [_tp, _i, _i, _i, _i, _vp]
lib.mx_dequantize_group.restype = _i
lib.mx_dequantize_group.argtypes = [_tp, _i, _i, _i, _i, _vp]
lib.mx_quantize_stats_group.restype = _i
lib.mx_quantize_stats_group.argtypes = [_tp, _i, _i, _i, _i, _vp, _sz, _vp]
lib.mx_global_scale_group.restype = _i
lib.mx_global_scale_group.argtypes = [_tp, _i, _i, _i, _vp, _sz, _vp]
lib.mx_error_stats_means.restype = _i
lib.mx_error_stats_means.argtypes = [_vp, ctypes.POINTER(ctypes.c_double)]
lib.mx_matmul.restype = _i
lib.mx_matmul.argtypes = [_vp, _vp, _u16, _vp, _vp, _u16, _i64, _i64, _i64, _i, _i, _vp, _i, _vp]
lib.mx_matmul_pair.restype = _i
lib.mx_matmul_pair.argtypes = lib.mx_matmul.argtypes
lib.mx_dequant_matmul.restype = _i
lib.mx_dequant_matmul.argtypes = [_vp, _i64, _i64, _vp, _vp, _i64, _i, _i, _u16, _vp, _vp, _i, _vp]
lib.mx_test_matmul_abandon_last.restype = _i
lib.mx_test_matmul_abandon_last.argtypes = []
lib.mx_matmul_scales_size.restype = _sz
lib.mx_matmul_scales_size.argtypes = [_i64, _i64]
lib.mx_matmul_prepare_scales.restype = _i
lib.mx_matmul_prepare_scales.argtypes = [_vp, _i64, _i64, _vp, _sz, _vp]
lib.mx_matmul_gave_up.restype = _i
lib.mx_matmul_gave_up.argtypes = [ctypes.POINTER(ctypes.c_uint)]
lib.mx_status_string.restype = ctypes.c_char_p
lib.mx_status_string.argtypes = [_i]
lib.mx_kernel_launches.restype = ctypes.c_longlong
lib.mx_kernel_launches.argtypes = []


class MXError(RuntimeError):
    """A non-OK mx_status returned by the library."""

    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {lib.mx_status_string(status).decode()}")


def check(status, where):
    if status != MX_OK:
        raise MXError(status, where)
