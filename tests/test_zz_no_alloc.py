"""eplb_serve_step_noalloc: the serving step with library-owned per-layer
counters.  Collected last on purpose: its GPU test also shows that the
library's counters are still zero after every other test ran."""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import moe_expert_load_eplb_b200 as eplb
import oracle


def test_noalloc_rejects_too_many_layers_before_touching_anything():
    lib = eplb.load_library()
    # null pointers everywhere: the layer limit is checked first
    rc = lib.eplb_serve_step_noalloc(None, 4097, 16, 4, 24, None, 17, None, 0, None, None, None,
                                     2, 0, -1, 40, 6, 2, 4, None, None, None, None, None, None,
                                     None, None, None)
    assert rc == 9  # EPLB_ERR_LIMIT


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda:0")


@pytest.mark.gpu
@pytest.mark.parametrize("shape", [(3, 70001, 8, 24, 40, 6, 2, 4), (58, 8192, 8, 256, 288, 8, 4, 32)])
def test_noalloc_matches_serve_step_on_two_calls_in_a_row(shape):
    L, T, K, E, P, G, N, gpus = shape
    X = P - E + 1
    W = 3
    rng = np.random.default_rng(L + T)
    ring0 = rng.integers(0, 5000, (W, L, E)).astype(np.int64)
    ring0[0] = 0
    plan_in = oracle.rebalance(rng.integers(0, 10000, (L, E)), P, G, N, gpus, slots=X)
    batches = [rng.integers(-1, E + 1, (L, T, K)).astype(np.int32) for _ in range(2)]

    def run(noalloc):
        ring = _dev(ring0)
        plans = [eplb.Plan(*[_dev(a) for a in plan_in]),
                 eplb.Plan(*[torch.zeros(a.shape, dtype=torch.int32, device="cuda:0") for a in plan_in])]
        done = torch.zeros(L, dtype=torch.uint32, device="cuda:0")
        st = torch.zeros(1, dtype=torch.int32, device="cuda:0")
        outs = []
        for k, idx in enumerate(batches):  # two calls in a row, the plans swapping
            used, nxt = plans[k % 2], plans[1 - k % 2]
            if noalloc:
                o = eplb.serve_step_noalloc(_dev(idx), used, ring, k, nxt, G, N, gpus,
                                            zero_slot=k + 1, token_offset=100 * k, status=st)
            else:
                o = eplb.serve_step(_dev(idx), used, ring, k, nxt, done, G, N, gpus,
                                    zero_slot=k + 1, token_offset=100 * k, status=st)
            torch.cuda.synchronize()
            assert int(st.item()) == 0
            outs.append([o.cpu().numpy()] + [t.cpu().numpy() for t in nxt] + [ring.cpu().numpy()])
        return outs

    ref = run(False)
    got = run(True)
    for k in range(2):
        for a, b in zip(got[k], ref[k]):
            assert np.array_equal(a, b), f"call {k}"
    # and the first call's plan is the oracle's
    counts, _ = oracle.count_loads(batches[0], E)
    loads = ring0.sum(axis=0) + counts
    want = oracle.rebalance(loads, P, G, N, gpus, slots=X)
    for a, b in zip(ref[0][1:5], want):
        assert np.array_equal(a, b)
