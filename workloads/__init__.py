"""Seeded synthetic workloads for the EPLB hot path (inputs only).

This package holds no EPLB arithmetic: it draws routed top-k expert indices
and per-step load histograms shaped like the DeepSeek-V3 setting the pages
describe, and is the only code that the CUDA path's tests, the bench and the
CPU oracle share.
"""
from .gen import (  # noqa: F401
    DSV3_PREFILL,
    GLOBAL_POLICY,
    HBM_STREAM,
    TINY,
    WINDOW_SWEEP,
    WORKLOADS,
    Workload,
    global_policy_loads,
    group_limited_indices,
    histogram_steps,
    routed_indices,
    seed_for,
    tiny_indices,
    window_sweep_steps,
    zipf_indices,
)
