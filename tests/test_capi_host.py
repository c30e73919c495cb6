"""Host-only checks of the C ABI (no GPU needed).

The library must load, export every entry point ``include/eplb.h`` declares,
and reject bad arguments on the host before any CUDA call.
"""
from __future__ import annotations

import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "eplb.h")


@pytest.fixture(scope="module")
def lib():
    from moe_expert_load_eplb_b200 import build, load_library
    build.build()
    return load_library()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+char\s*\*|eplb_status|int32_t)\s*(eplb_\w+)\s*\(",
                                 text, flags=re.M)))


def test_header_declares_the_four_stages():
    names = declared_symbols()
    for n in ("eplb_count_loads", "eplb_window_accumulate", "eplb_rebalance", "eplb_redirect",
              "eplb_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    from moe_expert_load_eplb_b200 import lib_path
    out = subprocess.run(["nm", "-D", "--defined-only", lib_path()], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT\s+(\w+)$", out, flags=re.M))
    for name in declared_symbols():
        assert name in exported, name
        assert getattr(lib, name) is not None


def test_status_strings(lib):
    from moe_expert_load_eplb_b200 import STATUS
    for code, name in STATUS.items():
        assert lib.eplb_status_string(code).decode() == name
    assert lib.eplb_status_string(1234).decode() == "EPLB_ERR_UNKNOWN"
    assert lib.eplb_abi_version() >> 16 == 2


def test_host_argument_checks(lib):
    p = ctypes.c_void_p
    one = p(16)  # never dereferenced: every call below fails its checks first
    # count: bad shapes, limits, null, alignment
    assert lib.eplb_count_loads(one, -1, 4, 2, 8, one, 0, None, None) == 2
    assert lib.eplb_count_loads(one, 1, 4, 0, 8, one, 0, None, None) == 2
    assert lib.eplb_count_loads(one, 1, 4, 2, 2000, one, 0, None, None) == 9
    assert lib.eplb_count_loads(None, 1, 4, 2, 8, one, 1, None, None) == 1
    assert lib.eplb_count_loads(p(20), 1, 4, 2, 8, one, 1, None, None) == 8
    assert lib.eplb_count_loads(one, 0, 4, 2, 8, None, 0, None, None) == 0  # nothing to do
    # window
    assert lib.eplb_window_accumulate(one, 4, 2, 3, 0, 0, one, -1, None) == 2
    assert lib.eplb_window_accumulate(one, 4, 2, 3, 2, 4, one, -1, None) == 2
    assert lib.eplb_window_accumulate(one, 4, 2, 3, 2, 0, one, 4, None) == 2   # zero_row >= S
    assert lib.eplb_window_accumulate(one, 4, 2, 3, 2, 0, one, -2, None) == 2
    assert lib.eplb_window_accumulate(None, 4, 2, 3, 2, 0, one, -1, None) == 1
    # rebalance: divisibility, shape, limits; R == 0 needs no device
    rb = lib.eplb_rebalance
    assert rb(one, 1, 12, 16, 5, 2, 8, 5, one, one, one, one, None, None, None, None) == 3   # 12 % 5
    assert rb(one, 1, 12, 18, 4, 2, 8, 5, one, one, one, one, None, None, None, None) == 3   # 18 % 8
    assert rb(one, 1, 12, 8, 4, 2, 8, 5, one, one, one, one, None, None, None, None) == 2    # P < E
    assert rb(one, 1, 12, 18, 4, 4, 6, 5, one, one, one, one, None, None, None, None) == 3   # hier: 6 % 4
    assert rb(one, 1, 2048, 4096, 8, 4, 32, 5, one, one, one, one, None, None, None, None) == 9
    assert rb(one, 1, 12, 16, 4, 2, 8, 0, one, one, one, one, None, None, None, None) == 2   # X < 1
    assert rb(one, 0, 12, 18, 3, 2, 3, 7, None, None, None, None, None, None, None, None) == 0  # global, R = 0
    assert rb(None, 1, 12, 16, 4, 2, 8, 5, one, one, one, one, None, None, None, None) == 1
    # redirect: shape, limits, alignment
    rd = lib.eplb_redirect
    assert rd(one, 1, 4, 2, 8, one, 0, one, 0, one, None, None, None) == 2
    assert rd(one, 1, 4, 2, 8, one, 3, one, -1, one, None, None, None) == 2
    assert rd(one, 1, 4, 2, 1024, one, 64, one, 0, one, None, None, None) == 9    # E * X > 32768
    assert rd(one, 1, 4, 2, 8, one, 3, one, (1 << 31) - 2, one, None, None, None) == 9
    assert rd(one, 1, 4, 2, 8, one, 3, one, 0, p(20), None, None, None) == 8
    assert rd(None, 1, 4, 2, 8, one, 3, one, 0, one, None, None, None) == 1


def test_binding_fails_loudly_without_a_gpu_tensor():
    import torch
    import moe_expert_load_eplb_b200 as eplb
    with pytest.raises(TypeError):
        eplb.count_loads(torch.zeros((1, 4, 2), dtype=torch.int32), 8)


def test_missing_library_fails_loudly(monkeypatch):
    """No CPU fallback: without libeplb.so every call raises."""
    import moe_expert_load_eplb_b200 as eplb
    monkeypatch.setattr(eplb, "_lib", None)
    monkeypatch.setattr(eplb, "_LIB_PATH", "/nonexistent/libeplb.so")
    with pytest.raises(ImportError, match="build"):
        eplb.load_library()


def test_host_tensors_are_refused():
    """The binding never computes on host tensors: it refuses them."""
    import torch

    import moe_expert_load_eplb_b200 as eplb
    idx = torch.zeros((1, 4, 2), dtype=torch.int32)
    with pytest.raises(TypeError, match="CUDA"):
        eplb.count_loads(idx, 8)
    with pytest.raises(TypeError, match="CUDA"):
        eplb.rebalance(torch.zeros((1, 8), dtype=torch.int64), 8, 1, 1, 1)
