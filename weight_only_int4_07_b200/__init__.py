"""W4A16 weight-only INT4 linear layer for NVIDIA B200 (sm_100a).

The compute lives in the CUDA library libw4a16.so (C ABI: include/w4a16.h); `native` is its
thin Python binding. `synthetic` draws the seeded inputs the tests and the benchmark use.
"""
from .native import (  # noqa: F401
    BF16,
    F16,
    KERNEL_AUTO,
    KERNEL_GEMV,
    KERNEL_TC,
    LAYOUT_PLAIN,
    LAYOUT_TILED,
    W4A16Error,
    w4a16_dequantize,
    w4a16_awq_quantize,
    w4a16_awq_workspace_bytes,
    w4a16_fp8_gemm,
    w4a16_fp8_quantize_acts,
    w4a16_fp8_quantize_weights,
    w4a16_gemm,
    w4a16_gptq_quantize,
    w4a16_gptq_workspace_bytes,
    w4a16_quantize,
    w4a16_repack,
    w4a16_repack_bytes,
    w4a16_select_kernel,
    w4a16_status_str,
    w4a16_version,
    w4a16_workspace_bytes,
)
