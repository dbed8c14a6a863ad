"""Block-scaled FP4 (NVFP4 / MXFP4) quantization and W4A4 GEMM for B200.

The compute lives in ``libfp4.so`` (hand-written sm_100a CUDA behind the C ABI
of ``include/fp4.h``); ``fp4`` is its ctypes binding and ``synth`` the seeded
input generator used by tests and benchmarks.
"""
from .fp4 import (  # noqa: F401
    NVFP4, MXFP4, ROWWISE, COLWISE, GEMM_AUTO, GEMM_PREFILL, GEMM_DECODE, Fp4Error,
    fp4_status_string, fp4_packed_bytes, fp4_scale_bytes, fp4_compute_global_scale,
    fp4_quantize, fp4_alpha_from_global_scales, fp4_gemm, fp4_gemm_workspace_bytes,
    fp4_get_device_status, quantize, global_scale, gemm, lib,
)
