"""NVFP4 (W4A4) group-limited mixture-of-experts layer for NVIDIA B200 (sm_100a).

The layer and its contracts are documented in include/nvfp4moe.h; this package is the
thin Python binding of libnvfp4moe.so (ctypes; torch supplies device memory and
streams).  Build the library with ``python -m nvfp4_quantized_moe_group_b200.build``.
"""
from ._lib import (  # noqa: F401
    Cfg, Experts, NvFp4MoeError, cfg_default, make_cfg, quantize, quantize_weights_lh, route, forward,
    forward_residual, status_read, quantize_fp8, Fp8Experts, forward_fp8, forward_fp8_workspace_bytes,
    forward_partial, finalize,
    status_string, last_launch_count, forward_workspace_bytes, route_workspace_bytes,
    quantize_workspace_bytes, swizzled_scale_bytes, declared_symbols, lib, LIB_PATH, StageTimer, STAGES,
    OK, ERR_ARG, ERR_SHAPE, ERR_CUDA, ERR_WORKSPACE, ERR_NONFINITE, ERR_TIMEOUT, ERR_DEVICE,
)
