"""Block-scaled FP8 (E4M3, power-of-two 1x128 / 128x128 scales) linear layer
for NVIDIA B200 (sm_100a): quantizers and fprop/dgrad/wgrad GEMMs behind a
C ABI (include/puro_fp8.h, libpuro_fp8.so).

Importing the package loads nothing; the first call into the library loads
libpuro_fp8.so and raises if it is missing.  There is no CPU fallback.
"""
from __future__ import annotations

_API = ("quant_act", "quant_weight", "blocked_scale_bytes", "gemm_fprop", "gemm_dgrad", "gemm_wgrad",
        "gemm_dgrad_wgrad", "device_status", "linear_forward", "linear_backward", "QuantAct",
        "QuantWeight")


def __getattr__(name):
    if name in _API:
        from . import linear
        return getattr(linear, name)
    raise AttributeError(name)
