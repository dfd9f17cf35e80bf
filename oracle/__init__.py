"""CPU oracle for FP4 microscaling -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package.  It wraps the plain C definition in ``mx_oracle.c`` (see its header for the sources
and readings) and shares nothing with the CUDA library.
"""
from .oracle import (  # noqa: F401
    F32, BF16, E4M3, UE5M3, Stats, lib, e2m1_value, e4m3_value, ue5m3_value, scale_value,
    fp16_value, round_scale, round_e2m1_mag, scale_max, scale_min, quantize, dequantize,
    error_stats, global_scale, matmul, bf16_values, dequant_matmul,
)
