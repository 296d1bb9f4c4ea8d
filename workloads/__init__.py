"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This package generates numbers only: activations, router weights, expert weights
(BF16, before any quantisation), the per-expert router bias of the skewed
workload and the layer shapes.  It holds none of the layer's arithmetic
(no quantisation, routing or expert math), so the CUDA path and the CPU oracle
can both consume it without sharing any of the method.
"""
from .synthetic import (  # noqa: F401
    LayerShape,
    TINY,
    BEAM,
    approx_normal,
    activations,
    router_weight,
    expert_weight,
    zipf_bias,
    workload,
    WORKLOADS,
)
