"""NVFP4 (W4A4) group-limited mixture-of-experts layer for NVIDIA B200 (sm_100a).

The layer and its contracts are documented in include/nvfp4moe.h; this package is the
thin Python binding of libnvfp4moe.so (ctypes; torch supplies device memory and
streams).  Build the library with ``python -m nvfp4_quantized_moe_group_b200.build``.

Typical use (all tensors on one CUDA device; the current stream is used)::

    import nvfp4_quantized_moe_group_b200 as moe
    cfg = moe.cfg_default()                       # 256 experts, 8 groups, top-4/top-8, x2.5
    experts = moe.Experts(cfg)                    # library-owned NVFP4 weights
    for e in range(cfg.E):                        # BF16 gate/up [I, H], down [H, I], static g_h
        experts.set_from_bf16(e, gate[e], up[e], down[e], g_h[e])
    ws = torch.empty(moe.forward_workspace_bytes(cfg, T_max), dtype=torch.uint8, device="cuda")
    out = moe.forward(experts, x_bf16, w_router_fp32, ws=ws)    # [T, H] BF16
    assert moe.status_read(ws) == moe.OK

Also: ``quantize`` / ``route`` / ``route_noalloc`` (the layer's steps alone), ``forward_residual`` (RMSNorm in,
weighted residual add out), ``quantize_weights_lh`` (local-Hessian weight scales),
``Fp8Experts`` / ``forward_fp8`` (the FP8 W8A8 variant), and ``ep.ExpertParallelLayer`` with
``forward_partial`` / ``finalize``, ``forward_partial_peer`` / ``ipc_handle`` / ``ipc_open`` or ``amax`` /
``ep_dispatch`` / ``ep_experts`` / ``ep_combine`` (experts spread over the ranks of a process group;
a gather exchange, the same with the combine into the owners' memory inside the down GEMM, or an
all-to-all one), and ``tp.TensorParallelLayer`` (every expert's intermediate features split over
the ranks, an all-reduce of the FP32 sums).
"""
from ._lib import (  # noqa: F401
    Cfg, Experts, NvFp4MoeError, cfg_default, make_cfg, quantize, quantize_weights_lh, route, route_noalloc, forward,
    forward_residual, status_read, last_device_status, workspace_bytes, quantize_fp8, Fp8Experts, forward_fp8, forward_fp8_workspace_bytes,
    forward_partial, finalize, amax, ep_dispatch, ep_dispatch_workspace_bytes, ep_experts, ep_experts_workspace_bytes,
    ep_combine, forward_partial_peer, ipc_handle, ipc_open, ipc_close,
    status_string, last_launch_count, forward_workspace_bytes, route_workspace_bytes,
    quantize_workspace_bytes, swizzled_scale_bytes, declared_symbols, lib, LIB_PATH, StageTimer, STAGES,
    OK, ERR_ARG, ERR_SHAPE, ERR_CUDA, ERR_WORKSPACE, ERR_NONFINITE, ERR_TIMEOUT, ERR_DEVICE,
)
