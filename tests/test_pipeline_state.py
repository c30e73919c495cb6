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


@pytest.mark.parametrize("window,rows,steps_done", [(3, 5, None), (3, 5, 7), (4, 2, 9), (5, 4, 4),
                                                    (1, 3, 11), (16, 15, 40)])
def test_history_lands_where_the_steps_would_have_left_it(window, rows, steps_done):
    """load_history puts step u's counts in ring slot u mod W and clears the
    slot the next step counts into, for any step count: the ring then holds
    the window of the last W - 1 steps, which is what the plan is built from
    (the oracle's window sum over the same history is the check)."""
    import numpy as np

    import oracle
    a = _step(window=window)
    g = torch.Generator().manual_seed(window * 100 + rows)
    hist = torch.randint(0, 1000, (rows, a.L, a.E), generator=g, dtype=torch.int64)
    a.load_history(hist, steps_done)
    n = min(rows, window - 1)
    s = n if steps_done is None else steps_done
    assert a.steps_done == s
    for i in range(n):
        u = s - n + i  # the step that made history row rows - n + i
        assert torch.equal(a.ring[u % window], hist[rows - n + i])
    assert int(a.ring[s % window].abs().sum()) == 0
    # the ring's sum is the oracle's window sum ending at the last history row
    want = oracle.window(hist.numpy(), window - 1, rows - 1)[0] if n else np.zeros((a.L, a.E), np.int64)
    assert np.array_equal(a.ring.sum(0).numpy(), want)


def test_history_needs_as_many_steps_as_rows():
    a = _step(window=4)
    with pytest.raises(ValueError):
        a.load_history(torch.zeros((3, a.L, a.E), dtype=torch.int64), steps_done=2)
