"""FP4 (E2M1) microscaling with FP8 (E4M3 / UE5M3) block scales on B200 (sm_100a).

The CUDA library (libmxfp4_b200.so, C ABI in include/mx.h) does the work: quantize + pack,
dequantize, the three-term block-error reduction, the per-tensor FP16 scale and the block-scaled
matrix product on the tensor cores.  This package is a thin binding over it.

The binding (``api``) is loaded on first use of any of its names, so that the seeded input
generators (``fp4_microscaling_tensor_b200.inputs``) can be imported without the CUDA library.
Using the API raises ImportError when the library is missing: there is no fallback.
"""
import importlib

_API_NAMES = ("E4M3", "MX_MAX_GROUP", "UE5M3", "ErrorStats", "FakeQuantize", "MXError",
              "dequant_matmul", "dequantize", "dequantize_group", "error_stats", "fake_quantize", "fmt_code",
              "g_bits", "global_scale", "global_scale_group", "kernel_launches", "matmul",
              "matmul_gave_up", "prepare_scales", "quantize", "quantize_group",
              "quantize_with_stats", "quantize_with_stats_group", "stats_workspace")

__all__ = list(_API_NAMES)


_SUBMODULES = ("api", "dist", "error_model", "inputs")


def __getattr__(name):
    if name in _SUBMODULES:
        return importlib.import_module("." + name, __name__)
    if name in _API_NAMES:
        api = importlib.import_module(".api", __name__)
        value = getattr(api, name)
        globals()[name] = value
        return value
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")


def __dir__():
    return sorted(list(globals()) + list(_API_NAMES))
