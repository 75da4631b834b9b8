"""Seeded synthetic inputs for the LLSA hot path.

This package holds only random-number recipes and token placement. It holds none
of the attention method's arithmetic, so both the CUDA path's tests and the CPU
oracle can draw identical inputs from it without sharing any method code.
"""
from .configs import WORKLOADS, WorkloadConfig, workload  # noqa: F401
from .generate import (  # noqa: F401
    make_config_inputs,
    make_inputs,
    make_tensor,
    morton_order,
    quadtree_order_recursive,
    smooth_field_tokens,
    to_f32_numpy,
    to_f64_numpy,
)
