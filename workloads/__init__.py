"""Seeded synthetic workloads for the EPLB hot path (inputs only).

This package holds no EPLB arithmetic: it draws routed top-k expert indices
and per-step load histograms shaped like the DeepSeek-V3 setting the pages
describe, and is the only code that the CUDA path's tests, the bench and the
CPU oracle share.
"""
from .gen import (  # noqa: F401
    CONFIGS,
    Config,
    c1_indices,
    c3_loads,
    c4_steps,
    group_limited_indices,
    histogram_steps,
    routed_indices,
    seed_for,
    zipf_indices,
)
