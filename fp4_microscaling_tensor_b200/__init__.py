"""FP4 (E2M1) microscaling with FP8 (E4M3 / UE5M3) block scales on B200 (sm_100a).

The CUDA library (libmxfp4_b200.so, C ABI in include/mx.h) does the work: quantize + pack,
dequantize, the three-term block-error reduction, the per-tensor FP16 scale and the block-scaled
matrix product on the tensor cores.  This package is a
thin binding over it; importing it fails when the library is missing.
"""
from .api import (E4M3, MX_MAX_GROUP, UE5M3, ErrorStats, FakeQuantize, MXError,  # noqa: F401
                  dequantize, dequantize_group, error_stats, fake_quantize, fmt_code, g_bits,
                  global_scale, kernel_launches, matmul, matmul_gave_up, prepare_scales,
                  quantize, quantize_group, quantize_with_stats, quantize_with_stats_group,
                  stats_workspace)
