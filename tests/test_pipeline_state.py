"""Checkpoint / resume of the serving step's state (host logic, CPU).

The window keeps per-step counts in a ring; the plan is an exact function of
the ring, so the ring, the plan in force and the step count are the whole
state.  These tests check the round trip through torch.save / torch.load and
the shape check; the GPU test in test_gpu_parity.py checks that a restored
step continues bit for bit.
"""
from __future__ import annotations

import io

import pytest
import torch

from moe_expert_load_eplb_b200.pipeline import EplbStep


def _step(window=3):
    # buffers only: nothing here launches a kernel
    return EplbStep(2, 16, 2, 12, 16, 4, 2, 8, window=window, device="cpu")


def test_state_round_trip():
    a = _step()
    g = torch.Generator().manual_seed(5)
    a.ring.copy_(torch.randint(0, 100, a.ring.shape, generator=g))
    a.cur = 1
    for t in a.plans[1]:
        t.copy_(torch.randint(-1, 9, t.shape, generator=g, dtype=torch.int32))
    a.steps_done, a.primed, a.token_offset = 7, True, 123
    buf = io.BytesIO()
    torch.save(a.state_dict(), buf)
    buf.seek(0)
    b = _step()
    b.load_state_dict(torch.load(buf))
    assert torch.equal(b.ring, a.ring)
    assert (b.cur, b.steps_done, b.primed, b.token_offset) == (1, 7, True, 123)
    for x, y in zip(b.plan, a.plan):
        assert torch.equal(x, y)


def test_state_of_another_shape_is_refused():
    with pytest.raises(ValueError):
        _step(window=4).load_state_dict(_step(window=3).state_dict())
