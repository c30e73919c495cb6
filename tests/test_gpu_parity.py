"""GPU parity: every CUDA stage against the CPU oracle, bit for bit.

All comparisons are exact (integer and index work).  Inputs come from the
seeded generators in ``workloads``; the oracle consumes the same bytes copied
to the host.  Calls go through the C ABI (ctypes binding).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests._invariants import check_plan

pytestmark = pytest.mark.gpu

eplb = pytest.importorskip("moe_expert_load_eplb_b200")
DEV = "cuda:0"


def _np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def _status():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def _oracle_rows(loads_np, P, G, N, gpus, X):
    """Oracle plan; rows the oracle rejects as not exactly representable
    (status RANGE) come back as error rows (-1 / 0), the GPU's convention."""
    try:
        return oracle.rebalance(loads_np, P, G, N, gpus, slots=X), 0
    except oracle.OracleError as err:
        if err.code != oracle.ERR_RANGE:
            raise
    R, E = loads_np.shape
    out = [np.full((R, P), -1, np.int32), np.full((R, P), -1, np.int32),
           np.zeros((R, E), np.int32), np.full((R, E, X), -1, np.int32)]
    for r in range(R):
        try:
            row = oracle.rebalance(loads_np[r:r + 1], P, G, N, gpus, slots=X)
        except oracle.OracleError as err:
            assert err.code == oracle.ERR_RANGE
            continue
        for o, x in zip(out, row):
            o[r] = x[0]
    return tuple(out), oracle.ERR_RANGE


def _rebalance_both(loads_np, P, G, N, gpus, slots=None):
    loads = torch.from_numpy(np.ascontiguousarray(loads_np)).to(DEV)
    st = _status()
    plan = eplb.rebalance(loads, P, G, N, gpus, slots=slots, status=st)
    torch.cuda.synchronize()
    ref, ref_status = _oracle_rows(np.ascontiguousarray(loads_np, dtype=np.int64), P, G, N, gpus,
                                   plan.log2phy.shape[2])
    got_status = int(st.item())
    assert got_status == ref_status, (got_status, ref_status)
    return plan, ref, got_status


def _assert_plan_equal(plan, ref):
    for name, got, want in zip(("phy2log", "phyrank", "logcnt", "log2phy"), plan, ref):
        g = _np(got)
        assert g.shape == want.shape, f"{name}: shape {g.shape}, oracle {want.shape}"
        if not np.array_equal(g, want):
            bad = np.argwhere(g != want)
            raise AssertionError(f"{name} differs at {len(bad)} places, first {bad[:5].tolist()}")


# ---------------------------------------------------------------- fixtures --

@pytest.fixture(scope="module")
def tiny_idx():
    return W.tiny_indices(device=DEV)


@pytest.fixture(scope="module")
def dsv3_idx():
    return W.routed_indices("dsv3_prefill", device=DEV)


@pytest.fixture(scope="module")
def hbm_idx():
    torch.cuda.empty_cache()
    return W.routed_indices("hbm_stream", device=DEV)


# ------------------------------------------------------------------ count --

@pytest.mark.parametrize("cfg", ["tiny", "dsv3_prefill", "hbm_stream"])
def test_count_workloads(cfg, request):
    idx = request.getfixturevalue({"tiny": "tiny_idx", "dsv3_prefill": "dsv3_idx", "hbm_stream": "hbm_idx"}[cfg])
    E = W.WORKLOADS[cfg].E
    bad = torch.zeros(1, dtype=torch.int64, device=DEV)
    counts = eplb.count_loads(idx, E, bad=bad)
    ref, nbad = oracle.count_loads(_np(idx), E)
    assert np.array_equal(_np(counts), ref)
    assert int(bad.item()) == nbad == 0
    assert int(counts.sum()) == idx.numel()


@pytest.mark.parametrize("shape", [(1, 1, 1), (3, 1001, 3), (2, 4097, 8), (5, 3, 7), (4, 4096, 1),
                                   (1, 70001, 5), (2, 0, 8), (7, 12345, 2)])
@pytest.mark.parametrize("E", [1, 12, 256, 1024])
def test_count_ragged_and_bad(shape, E):
    L, T, K = shape
    g = torch.Generator(device=DEV).manual_seed(L * 131 + T * 7 + K + E)
    idx = torch.randint(-2, E + 2, (L, T, K), generator=g, device=DEV, dtype=torch.int32)
    bad = torch.zeros(1, dtype=torch.int64, device=DEV)
    counts = eplb.count_loads(idx, E, bad=bad)
    ref, nbad = oracle.count_loads(_np(idx), E)
    assert np.array_equal(_np(counts), ref)
    assert int(bad.item()) == nbad
    again = eplb.count_loads(idx, E, counts=counts, accumulate=True, bad=bad)
    assert np.array_equal(_np(again), 2 * ref)
    assert int(bad.item()) == 2 * nbad


def test_count_skewed_single_expert():
    # every index equal: the worst case for same-address atomics
    idx = torch.full((3, 50000, 8), 7, dtype=torch.int32, device=DEV)
    counts = eplb.count_loads(idx, 256)
    ref, _ = oracle.count_loads(_np(idx), 256)
    assert np.array_equal(_np(counts), ref)


def test_count_misaligned_pointer_rejected():
    base = torch.zeros(1 + 4 * 16, dtype=torch.int32, device=DEV)
    with pytest.raises(eplb.EplbError) as e:
        eplb.count_loads(base[1:].view(1, 16, 4), 8)
    assert e.value.code == 8


# ----------------------------------------------------------------- window --

@pytest.fixture(scope="module")
def sweep_steps():
    return W.window_sweep_steps(device=DEV)


@pytest.mark.parametrize("window", [1000, 128, 1])
def test_window_sweep(sweep_steps, window):
    snaps = eplb.window_accumulate(sweep_steps, window)
    ref = oracle.window(_np(sweep_steps), window)
    assert np.array_equal(_np(snaps), ref)


@pytest.mark.parametrize("S,L,E,window,s_first", [(1, 1, 1, 1, 0), (7, 3, 5, 2, 0), (100, 2, 12, 7, 0),
                                                  (33, 1, 1, 100, 10), (65, 58, 256, 16, 64),
                                                  (16, 58, 256, 16, 15), (300, 3, 3, 40, 299),
                                                  (129, 5, 77, 64, 1)])
def test_window_shapes(S, L, E, window, s_first):
    g = torch.Generator(device=DEV).manual_seed(S * 1000 + E)
    steps = torch.randint(0, 1 << 40, (S, L, E), generator=g, device=DEV, dtype=torch.int64)
    snaps = eplb.window_accumulate(steps, window, s_first=s_first)
    ref = oracle.window(_np(steps), window, s_first)
    assert np.array_equal(_np(snaps), ref)


@pytest.mark.parametrize("S,W_,zero_row", [(16, 16, 3), (16, 16, 15), (1, 1, 0), (1000, 1000, 999),
                                            (300, 40, 0), (7, 2, 6)])
def test_window_zero_row(S, W_, zero_row):
    """The window sum is taken before the row is cleared; only that row changes."""
    g = torch.Generator(device=DEV).manual_seed(S + zero_row)
    L, E = 3, 77
    steps = torch.randint(0, 1 << 30, (S, L, E), generator=g, device=DEV, dtype=torch.int64)
    before = _np(steps).copy()
    snaps = eplb.window_accumulate(steps, W_, s_first=S - 1, zero_row=zero_row)
    assert np.array_equal(_np(snaps), oracle.window(before, W_, S - 1))
    after = before.copy()
    after[zero_row] = 0
    assert np.array_equal(_np(steps), after)


# -------------------------------------------------------------- rebalance --

def test_rebalance_readme_example():
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "eplb_readme_example.json")) as f:
        ex = json.load(f)
    w = np.array(ex["weight"], dtype=np.int64)
    for G in (4, 3):
        plan, ref, st = _rebalance_both(w, 16, G, 2, 8)
        assert st == 0
        _assert_plan_equal(plan, ref)
    plan, _, _ = _rebalance_both(w, 16, 4, 2, 8)
    assert _np(plan.phy2log).tolist() == ex["phy2log"]["value"]


@pytest.mark.parametrize("cfg", ["tiny", "dsv3_prefill", "hbm_stream"])
def test_rebalance_on_counted_loads(cfg, request):
    idx = request.getfixturevalue({"tiny": "tiny_idx", "dsv3_prefill": "dsv3_idx", "hbm_stream": "hbm_idx"}[cfg])
    c = W.WORKLOADS[cfg]
    loads = _np(eplb.count_loads(idx, c.E))
    plan, ref, st = _rebalance_both(loads, c.P, c.G, c.N, c.gpus)
    assert st == 0
    _assert_plan_equal(plan, ref)
    check_plan(loads[:4], *(p[:4] for p in ref), c.P, c.G, c.N, c.gpus)


def test_rebalance_global_policy():
    c = W.GLOBAL_POLICY
    loads = W.global_policy_loads()
    plan, ref, st = _rebalance_both(loads, c.P, c.G, c.N, c.gpus)
    assert st == 0
    _assert_plan_equal(plan, ref)


def test_rebalance_window_sweep_rows(sweep_steps):
    c = W.WINDOW_SWEEP
    snaps = eplb.window_accumulate(sweep_steps, c.W)
    loads = _np(snaps).reshape(-1, c.E)
    plan, ref, st = _rebalance_both(loads, c.P, c.G, c.N, c.gpus)
    assert st == 0
    _assert_plan_equal(plan, ref)


SHAPES = [
    (12, 4, 16, 2, 8), (12, 3, 16, 2, 8), (16, 4, 16, 2, 4), (16, 4, 32, 4, 8), (8, 2, 16, 2, 16),
    (24, 6, 36, 3, 6), (256, 8, 288, 4, 32), (256, 1, 288, 2, 144), (64, 8, 96, 8, 16),
    (1, 1, 1, 1, 1), (1, 1, 64, 1, 4), (2, 2, 2, 2, 2), (1024, 32, 2048, 8, 64), (1024, 1, 1024, 1, 1),
    (384, 12, 448, 4, 64), (160, 10, 200, 5, 40), (128, 16, 160, 16, 32), (256, 8, 320, 1, 160),
    (96, 3, 2048, 2, 8), (300, 5, 602, 7, 7),
    # two groups per node over 16+ nodes / two replicas per GPU over 16+ GPUs
    # per node: the balanced_packing closed form for two items per pack
    (64, 32, 128, 16, 32), (96, 48, 192, 24, 48), (64, 16, 128, 1, 64),
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("dist", ["uniform", "ties", "zeros", "huge", "skew", "onehot"])
def test_rebalance_shapes(shape, dist):
    E, G, P, N, gpus = shape
    rng = np.random.default_rng(abs(hash((E, G, P, N, gpus))) % (1 << 31) + len(dist))
    R = 5
    if dist == "uniform":
        w = rng.integers(0, 5000, (R, E))
    elif dist == "ties":
        w = rng.integers(0, 3, (R, E)) * 12
    elif dist == "zeros":
        w = np.zeros((R, E), dtype=np.int64)
    elif dist == "huge":
        w = rng.integers((1 << 40) - 100000, 1 << 40, (R, E))
    elif dist == "skew":
        w = np.round(1e4 * (rng.pareto(1.1, (R, E)) + 1)).astype(np.int64)
    else:
        w = np.zeros((R, E), dtype=np.int64)
        w[np.arange(R), rng.integers(0, E, R)] = (1 << 40) - 1
    plan, ref, st = _rebalance_both(w.astype(np.int64), P, G, N, gpus)
    assert st in (0, 4)
    _assert_plan_equal(plan, ref)


@pytest.mark.parametrize("shape", [(256, 8, 288, 4, 32), (64, 8, 96, 4, 16), (24, 6, 36, 3, 6)])
@pytest.mark.parametrize("edge", [-1, 0])
def test_rebalance_replica_ranking_widths(shape, edge):
    """The replica ranking takes 32-bit arithmetic while a node's heaviest
    candidate times R + 1 stays below 2^31 and 64-bit arithmetic from there:
    loads at that edge (one below it, and at it), many of them exact
    multiples of each other so that w_k2 * d == w_k * d2 ties are common,
    give the oracle's plans on both sides."""
    E, G, P, N, gpus = shape
    R = P // N - E // N
    top = (1 << 31) // (R + 1) + edge  # heaviest load of every node
    rng = np.random.default_rng(R * 7 + edge)
    rows = []
    for _ in range(6):
        base = top // 12
        w = base * rng.choice([12, 6, 4, 3, 2, 1], E)  # exact ratios among the loads
        w[rng.integers(0, E, E // 8)] = rng.integers(0, base, E // 8)
        for n in range(N):
            w[n * (E // N) + rng.integers(0, E // N)] = top
        rows.append(w)
    plan, ref, st = _rebalance_both(np.stack(rows).astype(np.int64), P, G, N, gpus)
    assert st == 0
    _assert_plan_equal(plan, ref)


def _random_shape(rng):
    while True:
        N = int(rng.choice([1, 2, 3, 4, 5, 8]))
        hier = rng.random() < 0.7
        G = N * int(rng.integers(1, 5)) if hier else int(rng.choice([3, 5, 7, 9])) * (1 if N == 1 else 1)
        if not hier and G % N == 0:
            G += 1
        gs = int(rng.integers(1, 9))
        E = G * gs
        gpus = (N if hier else 1) * int(rng.integers(1, 9))
        ppg = int(rng.integers(1, 6))
        P = gpus * ppg
        while P < E:
            P += gpus
        if E <= 1024 and P <= 2048:
            return E, G, P, N, gpus


@pytest.mark.parametrize("seed", range(60))
def test_rebalance_fuzz(seed):
    rng = np.random.default_rng(1000 + seed)
    E, G, P, N, gpus = _random_shape(rng)
    R = int(rng.integers(1, 6))
    kind = seed % 4
    if kind == 0:
        w = rng.integers(0, 100, (R, E))
    elif kind == 1:
        w = rng.integers(0, 1 << 40, (R, E))
    elif kind == 2:
        w = rng.integers(0, 4, (R, E)) * int(rng.integers(1, 1000))
    else:
        w = np.round(1e3 * (rng.pareto(1.2, (R, E)) + 1)).astype(np.int64)
    plan, ref, st = _rebalance_both(w.astype(np.int64), P, G, N, gpus)
    assert st in (0, 4), (E, G, P, N, gpus)
    _assert_plan_equal(plan, ref)


def test_rebalance_range_error_row():
    w = np.full((3, 12), 10, dtype=np.int64)
    w[1, 5] = 1 << 40
    loads = torch.from_numpy(w).to(DEV)
    st = _status()
    plan = eplb.rebalance(loads, 16, 4, 2, 8, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 4
    assert (_np(plan.phy2log[1]) == -1).all() and (_np(plan.logcnt[1]) == 0).all()
    ref, code = _oracle_rows(w, 16, 4, 2, 8, plan.log2phy.shape[2])
    assert code == 4
    _assert_plan_equal(plan, ref)


def test_rebalance_slots_error():
    w = np.array([[1000, 1, 1, 1]], dtype=np.int64)
    loads = torch.from_numpy(w).to(DEV)
    st = _status()
    plan = eplb.rebalance(loads, 8, 1, 1, 4, slots=2, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 5
    ref = oracle.rebalance(w, 8, 1, 1, 4)  # full width
    assert np.array_equal(_np(plan.phy2log), ref[0])
    assert np.array_equal(_np(plan.log2phy), ref[3][:, :, :2])


def test_rebalance_host_errors():
    loads = torch.ones((1, 12), dtype=torch.int64, device=DEV)
    for args, code in [((16, 5, 2, 8), 3), ((18, 4, 2, 8), 3), ((8, 4, 2, 8), 2), ((16, 4, 4, 6), 3)]:
        with pytest.raises(eplb.EplbError) as e:
            eplb.rebalance(loads, *args)
        assert e.value.code == code


# --------------------------------------------------------------- redirect --

@pytest.mark.parametrize("cfg", ["tiny", "dsv3_prefill", "hbm_stream"])
def test_redirect_workloads(cfg, request):
    idx = request.getfixturevalue({"tiny": "tiny_idx", "dsv3_prefill": "dsv3_idx", "hbm_stream": "hbm_idx"}[cfg])
    c = W.WORKLOADS[cfg]
    counts = eplb.count_loads(idx, c.E)
    plan = eplb.rebalance(counts, c.P, c.G, c.N, c.gpus)
    bad = torch.zeros(1, dtype=torch.int64, device=DEV)
    st = _status()
    out = eplb.redirect(idx, plan.log2phy, plan.logcnt, bad=bad, status=st)
    ref, nbad = oracle.redirect(_np(idx), _np(plan.log2phy), _np(plan.logcnt))
    assert np.array_equal(_np(out), ref)
    assert int(bad.item()) == nbad == 0 and int(st.item()) == 0


@pytest.mark.parametrize("shape", [(1, 1, 1), (3, 1001, 3), (2, 4097, 8), (5, 3, 7), (2, 70001, 5),
                                   (1, 9999, 1), (4, 2048, 6)])
@pytest.mark.parametrize("t0", [0, 17, (1 << 31) - 80000])
def test_redirect_ragged(shape, t0):
    L, T, K = shape
    E, P, G, N, gpus = 24, 40, 6, 2, 4
    rng = np.random.default_rng(L + T + K)
    w = rng.integers(0, 1000, (L, E))
    ref_plan = oracle.rebalance(w, P, G, N, gpus)
    l2p = torch.from_numpy(ref_plan[3]).to(DEV)
    cnt = torch.from_numpy(ref_plan[2]).to(DEV)
    g = torch.Generator(device=DEV).manual_seed(T)
    idx = torch.randint(-1, E + 1, (L, T, K), generator=g, device=DEV, dtype=torch.int32)
    bad = torch.zeros(1, dtype=torch.int64, device=DEV)
    out = eplb.redirect(idx, l2p, cnt, token_offset=t0, bad=bad)
    ref, nbad = oracle.redirect(_np(idx), ref_plan[3], ref_plan[2], t0)
    assert np.array_equal(_np(out), ref)
    assert int(bad.item()) == nbad


def test_redirect_invalid_logcnt_reports_range():
    idx = torch.zeros((1, 8, 4), dtype=torch.int32, device=DEV)
    l2p = torch.zeros((1, 4, 2), dtype=torch.int32, device=DEV)
    cnt = torch.tensor([[0, 1, 3, 1]], dtype=torch.int32, device=DEV)
    st = _status()
    out = eplb.redirect(idx, l2p, cnt, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 4 and (_np(out) == -1).all()


@pytest.mark.parametrize("E,X,K", [(1, 1, 4), (7, 40, 4), (7, 40, 3), (1024, 32, 4), (300, 9, 8),
                                   (16, 2048, 5), (33, 6, 4)])
@pytest.mark.parametrize("fused", [False, True])
def test_redirect_arbitrary_tables(E, X, K, fused):
    """Any int32 log2phy entries and any logcnt in [1, X]: replicas held in the
    per-expert descriptor (<= 5, index < 2048) and the rest must all agree."""
    L, T = 3, 3001
    rng = np.random.default_rng(E * 31 + X * 7 + K + fused)
    l2p = rng.integers(-2 ** 31, 2 ** 31, (L, E, X)).astype(np.int32)
    l2p[:, ::2] = rng.integers(0, 2048, (L, (E + 1) // 2, X))
    l2p[:, 1::4] = rng.integers(2040, 2056, (L, len(range(1, E, 4)), X))
    cnt = rng.integers(1, X + 1, (L, E)).astype(np.int32)
    cnt[:, ::3] = rng.integers(1, min(5, X) + 1, (L, (E + 2) // 3))
    idx = rng.integers(-3, E + 3, (L, T, K)).astype(np.int32)
    t0 = 123457
    l2p_d, cnt_d = torch.from_numpy(l2p).to(DEV), torch.from_numpy(cnt).to(DEV)
    idx_d = torch.from_numpy(idx).to(DEV)
    bad = torch.zeros(1, dtype=torch.int64, device=DEV)
    st = _status()
    if fused:
        counts, out = eplb.count_redirect(idx_d, E, l2p_d, cnt_d, token_offset=t0, bad=bad, status=st)
        assert np.array_equal(_np(counts), oracle.count_loads(idx, E)[0])
    else:
        out = eplb.redirect(idx_d, l2p_d, cnt_d, token_offset=t0, bad=bad, status=st)
    ref, nbad = oracle.redirect(idx, l2p, cnt, t0)
    assert np.array_equal(_np(out), ref)
    assert int(bad.item()) == nbad and int(st.item()) == 0


@pytest.mark.parametrize("fused", [False, True])
def test_redirect_mixed_table_periods(fused):
    """Layers whose replica counts all divide 24 take the short table, layers
    with a count of 5 the 120-entry one, a count of 7 the descriptors: all in
    one call, each equal to the oracle."""
    L, T, K, E, X = 4, 5003, 8, 256, 9
    rng = np.random.default_rng(77)
    cnt = np.empty((L, E), np.int32)
    cnt[0] = rng.choice([1, 2, 3, 4, 6, 8], E)   # period 24
    cnt[1] = rng.choice([1, 2, 3, 4], E)
    cnt[1, 17] = 5                                  # period 120
    cnt[2] = 1
    cnt[2, 200] = 7                                 # descriptors
    cnt[3] = rng.choice([1, 2, 4, 8], E)            # period 24
    l2p = np.full((L, E, X), -1, np.int32)
    for l in range(L):
        for e in range(E):
            l2p[l, e, :cnt[l, e]] = rng.integers(0, 288, cnt[l, e])
    idx = rng.integers(-1, E + 1, (L, T, K)).astype(np.int32)
    d = lambda a: torch.from_numpy(a).to(DEV)
    st = _status()
    bad = torch.zeros(1, dtype=torch.int64, device=DEV)
    if fused:
        counts, out = eplb.count_redirect(d(idx), E, d(l2p), d(cnt), 11, bad=bad, status=st)
        assert np.array_equal(_np(counts), oracle.count_loads(idx, E)[0])
    else:
        out = eplb.redirect(d(idx), d(l2p), d(cnt), 11, bad=bad, status=st)
    ref, nbad = oracle.redirect(idx, l2p, cnt, 11)
    assert np.array_equal(_np(out), ref)
    assert int(bad.item()) == nbad and int(st.item()) == 0


def test_redirect_sharded_equals_whole(dsv3_idx):
    c = W.DSV3_PREFILL
    counts = eplb.count_loads(dsv3_idx, c.E)
    plan = eplb.rebalance(counts, c.P, c.G, c.N, c.gpus)
    whole = eplb.redirect(dsv3_idx, plan.log2phy, plan.logcnt)
    h = c.T // 2
    a = eplb.redirect(dsv3_idx[:, :h].contiguous(), plan.log2phy, plan.logcnt, 0)
    b = eplb.redirect(dsv3_idx[:, h:].contiguous(), plan.log2phy, plan.logcnt, h)
    assert torch.equal(torch.cat([a, b], dim=1), whole)


# ---------------------------------------------------- fused count + redirect --

def _plan_in_force(c, seed):
    loads = W.histogram_steps(1, c.L, c.E, max(c.T, 1) * max(c.K, 1), seed, device=DEV)[0]
    return eplb.rebalance(loads, c.P, c.G, c.N, c.gpus)


@pytest.mark.parametrize("cfg", ["tiny", "dsv3_prefill", "hbm_stream"])
def test_count_redirect_workloads(cfg, request):
    idx = request.getfixturevalue({"tiny": "tiny_idx", "dsv3_prefill": "dsv3_idx", "hbm_stream": "hbm_idx"}[cfg])
    c = W.WORKLOADS[cfg]
    plan = _plan_in_force(c, 100 + c.stream)
    bad = torch.zeros(1, dtype=torch.int64, device=DEV)
    st = _status()
    counts, out = eplb.count_redirect(idx, c.E, plan.log2phy, plan.logcnt, bad=bad, status=st)
    idx_h = _np(idx)
    ref_c, nb = oracle.count_loads(idx_h, c.E)
    ref_o, nb2 = oracle.redirect(idx_h, _np(plan.log2phy), _np(plan.logcnt))
    assert np.array_equal(_np(counts), ref_c)
    assert np.array_equal(_np(out), ref_o)
    assert int(bad.item()) == nb == nb2 == 0 and int(st.item()) == 0


@pytest.mark.parametrize("shape", [(1, 200003, 8), (2, 333331, 3), (3, 65537, 7)])
def test_count_redirect_many_parts_per_layer(shape):
    """Layers split over many CTAs that take the layer's slices in turn, with
    a ragged layer length (not a multiple of 4): every index counted and
    redirected once, as the oracle does."""
    L, T, K = shape
    E, P, G, N, gpus = 256, 288, 8, 4, 32
    rng = np.random.default_rng(L * 13 + T)
    ref_plan = oracle.rebalance(rng.integers(0, 100000, (L, E)), P, G, N, gpus)
    l2p = torch.from_numpy(ref_plan[3]).to(DEV)
    cnt = torch.from_numpy(ref_plan[2]).to(DEV)
    g = torch.Generator(device=DEV).manual_seed(T)
    idx = torch.randint(-1, E + 1, (L, T, K), generator=g, device=DEV, dtype=torch.int32)
    bad = torch.zeros(1, dtype=torch.int64, device=DEV)
    counts, out = eplb.count_redirect(idx, E, l2p, cnt, token_offset=5, bad=bad)
    idx_h = _np(idx)
    ref_c, nb = oracle.count_loads(idx_h, E)
    ref_o, _ = oracle.redirect(idx_h, ref_plan[3], ref_plan[2], 5)
    assert np.array_equal(_np(counts), ref_c)
    assert np.array_equal(_np(out), ref_o)
    assert int(bad.item()) == nb
    only = eplb.count_loads(idx, E)
    assert np.array_equal(_np(only), ref_c)


@pytest.mark.parametrize("shape", [(1, 1, 1), (3, 1001, 3), (2, 4097, 8), (5, 3, 7), (2, 70001, 5),
                                   (4, 2048, 6), (7, 12345, 2)])
@pytest.mark.parametrize("t0", [0, 19, (1 << 31) - 80000])
def test_count_redirect_ragged(shape, t0):
    L, T, K = shape
    E, P, G, N, gpus = 24, 40, 6, 2, 4
    rng = np.random.default_rng(L * 7 + T + K)
    ref_plan = oracle.rebalance(rng.integers(0, 1000, (L, E)), P, G, N, gpus)
    l2p = torch.from_numpy(ref_plan[3]).to(DEV)
    cnt = torch.from_numpy(ref_plan[2]).to(DEV)
    g = torch.Generator(device=DEV).manual_seed(T + 1)
    idx = torch.randint(-2, E + 2, (L, T, K), generator=g, device=DEV, dtype=torch.int32)
    bad = torch.zeros(1, dtype=torch.int64, device=DEV)
    counts, out = eplb.count_redirect(idx, E, l2p, cnt, token_offset=t0, bad=bad)
    idx_h = _np(idx)
    ref_c, nb = oracle.count_loads(idx_h, E)
    ref_o, _ = oracle.redirect(idx_h, ref_plan[3], ref_plan[2], t0)
    assert np.array_equal(_np(counts), ref_c)
    assert np.array_equal(_np(out), ref_o)
    assert int(bad.item()) == nb
    counts2, _ = eplb.count_redirect(idx, E, l2p, cnt, token_offset=t0, counts=counts, accumulate=True)
    assert np.array_equal(_np(counts2), 2 * ref_c)


# --------------------------------------------------------------- pipeline --

def _oracle_plan_from_ring(ring, c, X):
    loads = oracle.window(ring, ring.shape[0], ring.shape[0] - 1)[0]
    return oracle.rebalance(loads, c.P, c.G, c.N, c.gpus, slots=X)


def test_pipeline_fresh_order_dsv3_prefill(dsv3_idx):
    from moe_expert_load_eplb_b200.pipeline import EplbStep
    c = W.DSV3_PREFILL
    hist = W.histogram_steps(15, c.L, c.E, c.T * c.K, c.stream, device=DEV)
    step = EplbStep(c.L, c.T, c.K, c.E, c.P, c.G, c.N, c.gpus, window=16, device=DEV, fused=False)
    step.fill_history(hist)
    plan, out = step(dsv3_idx)
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0
    counts, _ = oracle.count_loads(_np(dsv3_idx), c.E)
    ref = _oracle_plan_from_ring(np.concatenate([_np(hist), counts[None]], axis=0), c, step.X)
    _assert_plan_equal(plan, ref)
    red, _ = oracle.redirect(_np(dsv3_idx), ref[3], ref[2])
    assert np.array_equal(_np(out), red)


@pytest.mark.parametrize("single", [True, False])
def test_pipeline_serving_order_dsv3_prefill(dsv3_idx, single):
    """Three serving steps: each redirects with the plan in force, then rebuilds it
    (one launch per step, or count_redirect + rebalance_window)."""
    from moe_expert_load_eplb_b200.pipeline import EplbStep
    c = W.DSV3_PREFILL
    W_ = 4
    hist = W.histogram_steps(W_ - 1, c.L, c.E, c.T * c.K, c.stream, device=DEV)
    step = EplbStep(c.L, c.T, c.K, c.E, c.P, c.G, c.N, c.gpus, window=W_, device=DEV, fused=True,
                    token_offset=1000, single_launch=single)
    assert step.launches_per_step == (1 if single else 2)
    step.fill_history(hist)
    ring = np.concatenate([_np(hist), np.zeros((1, c.L, c.E), np.int64)], axis=0)
    plan_ref = _oracle_plan_from_ring(ring, c, step.X)
    _assert_plan_equal(step.plan, plan_ref)
    batches = [dsv3_idx, W.routed_indices("dsv3_prefill", device=DEV, shard=1), dsv3_idx.flip(1).contiguous()]
    for s_i, idx in enumerate(batches):
        used, out = step(idx)
        torch.cuda.synchronize()
        assert int(step.status.item()) == 0
        idx_h = _np(idx)
        red, _ = oracle.redirect(idx_h, plan_ref[3], plan_ref[2], 1000)
        assert np.array_equal(_np(out), red), f"step {s_i}: redirect"
        counts, _ = oracle.count_loads(idx_h, c.E)
        ring[(W_ - 1 + s_i) % W_] = counts
        plan_ref = _oracle_plan_from_ring(ring, c, step.X)
        _assert_plan_equal(step.plan, plan_ref)
        assert int(step.layer_done.cpu().numpy().astype("int64").sum()) == 0


@pytest.mark.parametrize("single", [True, False])
@pytest.mark.parametrize("steps_done", [2, 7, 13])
def test_pipeline_history_with_a_step_count(tiny_idx, single, steps_done):
    """A step primed with history at any step count keeps the right steps in
    its window: the plan fill_history builds covers the history rows kept
    (at most W - 1), and the plan each step builds covers the last W steps,
    that step included.  The oracle, given the same per-step counts in step
    order, sums the same window before and after each new step."""
    from moe_expert_load_eplb_b200.pipeline import EplbStep
    c = W.TINY
    W_ = 4
    hist = W.histogram_steps(2, c.L, c.E, c.T * c.K, c.stream, device=DEV)
    step = EplbStep(c.L, c.T, c.K, c.E, c.P, c.G, c.N, c.gpus, window=W_, device=DEV, fused=True,
                    single_launch=single)
    step.fill_history(hist, steps_done=steps_done)
    steps = [_np(hist[0]), _np(hist[1])]  # per-step counts in step order

    def ref_plan():
        win = np.stack(steps[-W_:], axis=0)
        return _oracle_plan_from_ring(win, c, step.X)

    plan_ref = ref_plan()
    _assert_plan_equal(step.plan, plan_ref)
    for s_i, idx in enumerate([tiny_idx, tiny_idx.flip(1).contiguous(), tiny_idx,
                               tiny_idx.flip(2).contiguous()]):
        used, out = step(idx)
        torch.cuda.synchronize()
        assert int(step.status.item()) == 0
        red, _ = oracle.redirect(_np(idx), plan_ref[3], plan_ref[2])
        assert np.array_equal(_np(out), red), f"step {s_i}: redirect"
        steps.append(oracle.count_loads(_np(idx), c.E)[0])
        plan_ref = ref_plan()
        _assert_plan_equal(step.plan, plan_ref)
    assert step.steps_done == steps_done + 4


def test_pipeline_serving_with_an_nccl_group_of_one(tiny_idx):
    """The multi-rank serving step (count+redirect, NCCL all-reduce of the
    counts, window + rebalance) on a one-rank NCCL group: same plans and
    redirects as the oracle."""
    import socket
    import torch.distributed as dist
    from moe_expert_load_eplb_b200.pipeline import EplbStep
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device(DEV))
    try:
        group = dist.new_group([0])
        c = W.TINY
        W_ = 3
        hist = W.histogram_steps(W_ - 1, c.L, c.E, c.T * c.K, c.stream, device=DEV)
        step = EplbStep(c.L, c.T, c.K, c.E, c.P, c.G, c.N, c.gpus, window=W_, device=DEV,
                        group=group, token_offset=77)
        assert step.launches_per_step == 2 and not step.single
        step.fill_history(hist)
        ring = np.concatenate([_np(hist), np.zeros((1, c.L, c.E), np.int64)], axis=0)
        plan_ref = _oracle_plan_from_ring(ring, c, step.X)
        for s_i, idx in enumerate([tiny_idx, tiny_idx.flip(1).contiguous()]):
            used, out = step(idx)
            torch.cuda.synchronize()
            assert int(step.status.item()) == 0
            red, _ = oracle.redirect(_np(idx), plan_ref[3], plan_ref[2], 77)
            assert np.array_equal(_np(out), red)
            ring[(W_ - 1 + s_i) % W_] = oracle.count_loads(_np(idx), c.E)[0]
            plan_ref = _oracle_plan_from_ring(ring, c, step.X)
            _assert_plan_equal(step.plan, plan_ref)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("fused,single", [(True, False), (True, True), (False, False)])
def test_step_graphs_replay_matches_eager(tiny_idx, fused, single):
    """CUDA-graph replay of the step (one graph per phase of the ring slot and
    plan buffer) gives exactly the eager steps' outputs, plans and ring."""
    from moe_expert_load_eplb_b200.pipeline import EplbStep, StepGraphs
    c = W.TINY
    hist = W.histogram_steps(2, c.L, c.E, c.T * c.K, c.stream, device=DEV)
    mk = lambda: EplbStep(c.L, c.T, c.K, c.E, c.P, c.G, c.N, c.gpus, window=3, device=DEV,
                          fused=fused, single_launch=single, token_offset=5)
    eager, graphed = mk(), mk()
    eager.fill_history(hist)
    graphed.fill_history(hist)
    buf = torch.empty_like(tiny_idx)
    sg = StepGraphs(graphed, buf)
    assert sg.period == 6
    batches = [tiny_idx, tiny_idx.flip(1), tiny_idx.roll(7, dims=1), (tiny_idx + 3) % c.E]
    for k in range(9):
        b = batches[k % len(batches)].contiguous()
        buf.copy_(b)
        used_g, out_g = sg()
        used_e, out_e = eager(b)
        torch.cuda.synchronize()
        assert torch.equal(out_g, out_e), f"step {k}: redirected indices"
        for a_, b_ in zip(used_g, used_e):
            assert torch.equal(a_, b_), f"step {k}: plan used"
        for a_, b_ in zip(graphed.plan, eager.plan):
            assert torch.equal(a_, b_), f"step {k}: new plan"
        assert torch.equal(graphed.ring, eager.ring), f"step {k}: ring"
    assert int(graphed.status.item()) == 0


@pytest.mark.parametrize("single", [False, True])
def test_pipeline_checkpoint_resume(tiny_idx, single):
    """A step restored mid-sweep from state_dict (through torch.save) continues
    exactly as the step it was taken from: outputs, plans and ring."""
    import io
    from moe_expert_load_eplb_b200.pipeline import EplbStep
    c = W.TINY
    W_ = 3
    hist = W.histogram_steps(W_ - 1, c.L, c.E, c.T * c.K, c.stream, device=DEV)
    mk = lambda: EplbStep(c.L, c.T, c.K, c.E, c.P, c.G, c.N, c.gpus, window=W_, device=DEV,
                          fused=True, single_launch=single)
    batches = [tiny_idx, tiny_idx.flip(1).contiguous(), tiny_idx.roll(1, 2).contiguous(),
               tiny_idx.flip(2).contiguous(), tiny_idx.roll(7, 1).contiguous()]
    a = mk()
    a.fill_history(hist)
    for b in batches[:2]:
        a(b)
    buf = io.BytesIO()
    torch.save(a.state_dict(), buf)
    buf.seek(0)
    ref = []
    for b in batches[2:]:
        _, out = a(b)
        ref.append((out.clone(), [t.clone() for t in a.plan]))
    r = mk()
    r.load_state_dict(torch.load(buf))
    for b, (out_ref, plan_ref) in zip(batches[2:], ref):
        _, out = r(b)
        assert torch.equal(out, out_ref)
        for x, y in zip(r.plan, plan_ref):
            assert torch.equal(x, y)
    assert torch.equal(r.ring, a.ring)
    assert int(a.status.item()) == 0 and int(r.status.item()) == 0


# ---------------------------------------------------------- guard bands --

_GUARD = 64  # elements on each side (256 B for int32: keeps 16-byte alignment)


def _guarded(shape, dtype, fill=-7):
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * _GUARD,), fill, dtype=dtype, device=DEV)
    return buf, buf[_GUARD:_GUARD + n].view(shape)


def _intact(buf, fill=-7):
    return bool((buf[:_GUARD] == fill).all()) and bool((buf[-_GUARD:] == fill).all())


@pytest.mark.parametrize("shape", [(3, 1001, 3, 12, 16, 4, 2, 8), (2, 70001, 5, 256, 288, 8, 4, 32),
                                   (1, 1, 1, 12, 16, 4, 2, 8), (5, 3, 7, 24, 40, 6, 2, 4)])
def test_outputs_stay_inside_their_buffers(shape):
    """Every entry point writing caller-owned memory, on ragged shapes, leaves
    guard bands around each output untouched."""
    L, T, K, E, P, G, N, gpus = shape
    X = P - E + 1
    rng = np.random.default_rng(T + E)
    idx = _dev(rng.integers(-1, E + 1, (L, T, K)).astype(np.int32))
    bufs = []

    def g(shape_, dtype):
        b, t = _guarded(shape_, dtype)
        bufs.append(b)
        return t

    def gplan():
        return eplb.Plan(g((L, P), torch.int32), g((L, P), torch.int32), g((L, E), torch.int32),
                         g((L, E, X), torch.int32))

    st = _status()
    counts = eplb.count_loads(idx, E, counts=g((L, E), torch.int64))
    plan = eplb.rebalance(counts, P, G, N, gpus, slots=X, out=gplan(), status=st)
    eplb.redirect(idx, plan.log2phy, plan.logcnt, 5, out=g((L, T, K), torch.int32), status=st)
    eplb.count_redirect(idx, E, plan.log2phy, plan.logcnt, 5, counts=g((L, E), torch.int64),
                        out=g((L, T, K), torch.int32), status=st)
    steps = _dev(rng.integers(0, 1000, (4, L, E)).astype(np.int64))
    eplb.window_accumulate(steps, 2, out=g((4, L, E), torch.int64))
    ring = g((3, L, E), torch.int64)
    ring.copy_(steps[:3])
    eplb.rebalance_window(ring, P, G, N, gpus, zero_slot=1, slots=X, out=gplan(),
                          loads_out=g((L, E), torch.int64), status=st)
    done = g((L,), torch.int32)
    done.zero_()
    done = done.view(torch.uint32)
    eplb.serve_step(idx, plan, ring, 1, gplan(), done, G, N, gpus, zero_slot=2, token_offset=9,
                    out=g((L, T, K), torch.int32), loads_out=g((L, E), torch.int64), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert all(_intact(b) for b in bufs)


# ------------------------------------------------------- one-launch serve step --

def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


@pytest.mark.parametrize("shape", [
    (2, 4096, 2, 12, 16, 4, 2, 8),      # the worked example's sizes, many tokens
    (3, 70001, 8, 24, 40, 6, 2, 4),     # several chunks per layer, ragged tail
    (5, 3, 7, 24, 40, 6, 2, 4),         # fewer indices than a vector per layer
    (4, 0, 4, 24, 40, 6, 2, 4),         # no tokens: the plan from the ring alone
    (2, 20000, 3, 32, 48, 4, 3, 6),     # global policy (G % N != 0), K not a multiple of 4
    (58, 8192, 8, 256, 288, 8, 4, 32),  # DeepSeek-V3 shape, decode-sized batch
    (3, 5000, 8, 256, 288, 1, 2, 144),  # global policy, two replicas per GPU on 144 GPUs
    (2, 3000, 6, 64, 128, 32, 16, 32),  # two groups per node on 16 nodes
])
@pytest.mark.parametrize("W_,slot,zero_slot", [(3, 1, 2), (1, 0, 0), (4, 3, -1)])
def test_serve_step_matches_oracle(shape, W_, slot, zero_slot):
    L, T, K, E, P, G, N, gpus = shape
    X = P - E + 1
    rng = np.random.default_rng(L * 31 + T + K + W_ * 7 + slot)
    ring = rng.integers(0, 5000, (W_, L, E)).astype(np.int64)
    ring[slot] = rng.integers(0, 3, (L, E))  # counts already in the slot are added to
    plan_in = oracle.rebalance(rng.integers(0, 10000, (L, E)), P, G, N, gpus, slots=X)
    idx = rng.integers(-1, E + 1, (L, T, K)).astype(np.int32)
    t0 = 4321
    ring_d = _dev(ring)
    used = eplb.Plan(*[_dev(a) for a in plan_in])
    nxt = eplb.Plan(*[torch.full(a.shape, 7, dtype=torch.int32, device=DEV) for a in plan_in])
    done = torch.zeros(L, dtype=torch.uint32, device=DEV)
    loads = torch.zeros((L, E), dtype=torch.int64, device=DEV)
    bad = torch.zeros(1, dtype=torch.int64, device=DEV)
    st = _status()
    out = eplb.serve_step(_dev(idx), used, ring_d, slot, nxt, done, G, N, gpus, zero_slot=zero_slot,
                          token_offset=t0, loads_out=loads, bad=bad, status=st)
    torch.cuda.synchronize()
    counts, nbad = oracle.count_loads(idx, E)
    ring_ref = ring.copy()
    ring_ref[slot] += counts
    loads_ref = ring_ref.sum(axis=0)
    next_ref = oracle.rebalance(loads_ref, P, G, N, gpus, slots=X)
    red, _ = oracle.redirect(idx, plan_in[3], plan_in[2], t0)
    if zero_slot >= 0:
        ring_ref[zero_slot] = 0
    assert int(st.item()) == 0
    assert np.array_equal(_np(out), red)
    assert int(bad.item()) == nbad
    assert np.array_equal(_np(loads), loads_ref)
    _assert_plan_equal(nxt, next_ref)
    assert np.array_equal(_np(ring_d), ring_ref)
    assert not done.cpu().numpy().any()


def test_serve_step_reports_range_and_keeps_going():
    """A window sum outside [0, 2^40) marks its row and sets EPLB_ERR_RANGE;
    the counters still end at zero."""
    L, T, K, E, P, G, N, gpus = 3, 1000, 4, 24, 40, 6, 2, 4
    X = P - E + 1
    rng = np.random.default_rng(5)
    ring = rng.integers(0, 100, (2, L, E)).astype(np.int64)
    ring[1, 1, 3] = 1 << 41
    plan_in = oracle.rebalance(rng.integers(0, 100, (L, E)), P, G, N, gpus, slots=X)
    used = eplb.Plan(*[_dev(a) for a in plan_in])
    nxt = eplb.Plan(*[torch.empty(a.shape, dtype=torch.int32, device=DEV) for a in plan_in])
    done = torch.zeros(L, dtype=torch.uint32, device=DEV)
    st = _status()
    idx = _dev(rng.integers(0, E, (L, T, K)).astype(np.int32))
    eplb.serve_step(idx, used, _dev(ring), 0, nxt, done, G, N, gpus, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 4
    assert not done.cpu().numpy().any()
    assert (_np(nxt.phy2log)[1] == -1).all()
    loads = ring.sum(axis=0) + oracle.count_loads(_np(idx), E)[0]  # slot 0 received the counts
    ref = oracle.rebalance(loads[[0, 2]], P, G, N, gpus, slots=X)
    assert np.array_equal(_np(nxt.phy2log)[[0, 2]], ref[0])


def test_serve_step_host_errors():
    L, T, K, E, P, G, N, gpus = 2, 64, 4, 12, 16, 4, 2, 8
    X = P - E + 1
    plan = eplb.Plan(torch.zeros((L, P), dtype=torch.int32, device=DEV),
                     torch.zeros((L, P), dtype=torch.int32, device=DEV),
                     torch.ones((L, E), dtype=torch.int32, device=DEV),
                     torch.zeros((L, E, X), dtype=torch.int32, device=DEV))
    ring = torch.zeros((2, L, E), dtype=torch.int64, device=DEV)
    idx = torch.zeros((L, T, K), dtype=torch.int32, device=DEV)
    done = torch.zeros(L, dtype=torch.uint32, device=DEV)
    with pytest.raises(eplb.EplbError) as ei:  # the next plan is the plan in force
        eplb.serve_step(idx, plan, ring, 0, plan, done, G, N, gpus)
    assert ei.value.code == 2
    nxt = eplb.Plan(*[torch.empty_like(t) for t in plan])
    for slot, zero_slot in ((2, -1), (-1, 0), (0, 2), (0, -2)):
        with pytest.raises(eplb.EplbError) as ei:
            eplb.serve_step(idx, plan, ring, slot, nxt, done, G, N, gpus, zero_slot=zero_slot)
        assert ei.value.code == 2
    with pytest.raises(eplb.EplbError) as ei:  # E % G
        eplb.serve_step(idx, plan, ring, 0, nxt, done, 5, N, gpus)
    assert ei.value.code == 3


def test_binding_rejects_malformed_arguments():
    """The C ABI takes bare pointers; the binding refuses, before any launch,
    tensors whose shape, dtype or device would let a kernel run off a buffer."""
    L, T, K, E, P, G, N, gpus = 2, 64, 4, 12, 16, 4, 2, 8
    X = P - E + 1
    mk = lambda shape, dt=torch.int32: torch.zeros(shape, dtype=dt, device=DEV)
    plan = eplb.Plan(mk((L, P)), mk((L, P)), torch.ones((L, E), dtype=torch.int32, device=DEV),
                     mk((L, E, X)))
    nxt = eplb.Plan(*[torch.empty_like(t) for t in plan])
    ring = mk((2, L, E), torch.int64)
    idx = mk((L, T, K))
    short = eplb.Plan(nxt.phy2log, nxt.phyrank, nxt.logcnt, mk((L, E, X - 1)))
    call = eplb.serve_step_noalloc
    with pytest.raises(ValueError):  # next plan's log2phy narrower than the plan in force
        call(idx, plan, ring, 0, short, G, N, gpus)
    with pytest.raises(ValueError):  # phyrank of the wrong width
        call(idx, plan, ring, 0, eplb.Plan(nxt.phy2log, mk((L, P - 1)), nxt.logcnt, nxt.log2phy),
             G, N, gpus)
    with pytest.raises(TypeError):  # ring of the wrong dtype
        call(idx, plan, ring.to(torch.int32), 0, nxt, G, N, gpus)
    with pytest.raises(ValueError):  # loads_out too small
        call(idx, plan, ring, 0, nxt, G, N, gpus, loads_out=mk((L, E - 1), torch.int64))
    with pytest.raises(ValueError):
        eplb.serve_step(idx, plan, ring, 0, short, mk(L), G, N, gpus)
    with pytest.raises(TypeError):  # bad is a 64-bit word
        eplb.redirect(idx, plan.log2phy, plan.logcnt, bad=mk(1))
    with pytest.raises(TypeError):  # status is an int32 word
        eplb.redirect(idx, plan.log2phy, plan.logcnt, status=mk(1, torch.int64))
    with pytest.raises(ValueError):
        eplb.count_redirect(idx, E, plan.log2phy, plan.logcnt, status=mk(0))
    with pytest.raises(TypeError):  # a table left on the host
        eplb.count_redirect(idx, E, plan.log2phy.cpu(), plan.logcnt)
    with pytest.raises(ValueError):
        eplb.plan_stats(mk((L, E), torch.int64), plan.phy2log, mk((L, E + 1)), gpus)
    with pytest.raises(ValueError):
        eplb.fold_loads(mk((L, P), torch.int64), mk((L, P + 1)), E)
    with pytest.raises(ValueError):
        eplb.plan_diff(plan.phy2log, mk((L, P - 1)), E, gpus)
    torch.cuda.synchronize()


# ------------------------------------------- plan stats, fold, initial map, diff --

def _plans_for(c, loads_np):
    return oracle.rebalance(loads_np, c.P, c.G, c.N, c.gpus)


@pytest.mark.parametrize("cfg", ["tiny", "dsv3_prefill", "global_policy"])
def test_plan_stats_matches_oracle(cfg, request):
    c = W.WORKLOADS[cfg]
    if cfg == "global_policy":
        loads_np = W.global_policy_loads()
    else:
        idx = request.getfixturevalue({"tiny": "tiny_idx", "dsv3_prefill": "dsv3_idx"}[cfg])
        loads_np, _ = oracle.count_loads(_np(idx), c.E)
    p2l, _, cnt, _ = _plans_for(c, loads_np)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    st_word = _status()
    gl, st = eplb.plan_stats(dev(loads_np), dev(p2l), dev(cnt), c.gpus, status=st_word)
    ref_gl, ref_st = oracle.plan_stats(loads_np, p2l, cnt, c.gpus)
    # fp64, same operations in the same order: identical bits
    assert np.array_equal(_np(gl), ref_gl) and np.array_equal(_np(st), ref_st)
    assert int(st_word.item()) == 0


def test_plan_stats_worked_example_gpu():
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "eplb_readme_example.json")) as f:
        ex = json.load(f)
    w = np.array(ex["weight"], dtype=np.int64)
    plan = eplb.rebalance(torch.from_numpy(w).to(DEV), 16, 4, 2, 8)
    _, st = eplb.plan_stats(torch.from_numpy(w).to(DEV), plan.phy2log, plan.logcnt, 8)
    h = ex["layer0_gpu_load_hierarchical"]
    assert _np(st)[0, 0] == h["min"] and _np(st)[0, 1] == h["max"]


def _quality_bufs(R, gpus):
    return (torch.full((R, gpus), -7.0, dtype=torch.float64, device=DEV),
            torch.full((R, 4), -7.0, dtype=torch.float64, device=DEV))


@pytest.mark.parametrize("cfg", ["tiny", "dsv3_prefill", "global_policy"])
def test_rebalance_fused_quality_matches_oracle(cfg, request):
    """The plan quality written by the rebalance launch itself equals the
    oracle's plan_stats of the oracle's plan, bit for bit (fp64, same order)."""
    c = W.WORKLOADS[cfg]
    if cfg == "global_policy":
        loads_np = W.global_policy_loads()
    else:
        idx = request.getfixturevalue({"tiny": "tiny_idx", "dsv3_prefill": "dsv3_idx"}[cfg])
        loads_np, _ = oracle.count_loads(_np(idx), c.E)
    gl, st = _quality_bufs(loads_np.shape[0], c.gpus)
    word = _status()
    plan = eplb.rebalance(torch.from_numpy(loads_np).to(DEV), c.P, c.G, c.N, c.gpus, status=word,
                          gpu_load=gl, stats=st)
    torch.cuda.synchronize()
    assert int(word.item()) == 0
    ref = oracle.rebalance(loads_np, c.P, c.G, c.N, c.gpus, slots=plan.log2phy.shape[2])
    _assert_plan_equal(plan, ref)
    ref_gl, ref_st = oracle.plan_stats(loads_np, ref[0], ref[2], c.gpus)
    assert np.array_equal(_np(gl), ref_gl) and np.array_equal(_np(st), ref_st)
    # either output alone
    gl2, st2 = _quality_bufs(loads_np.shape[0], c.gpus)
    eplb.rebalance(torch.from_numpy(loads_np).to(DEV), c.P, c.G, c.N, c.gpus, stats=st2)
    eplb.rebalance(torch.from_numpy(loads_np).to(DEV), c.P, c.G, c.N, c.gpus, gpu_load=gl2)
    assert np.array_equal(_np(gl2), ref_gl) and np.array_equal(_np(st2), ref_st)


@pytest.mark.parametrize("shape", SHAPES[:12])
def test_rebalance_fused_quality_shapes(shape):
    E, G, P, N, gpus = shape
    rng = np.random.default_rng(E * 7 + P)
    loads_np = rng.integers(0, 1 << 30, (9, E)).astype(np.int64)
    loads_np[3] = 0  # all-zero row: balancedness 1
    gl, st = _quality_bufs(9, gpus)
    plan = eplb.rebalance(torch.from_numpy(loads_np).to(DEV), P, G, N, gpus, gpu_load=gl, stats=st)
    ref = oracle.rebalance(loads_np, P, G, N, gpus, slots=plan.log2phy.shape[2])
    ref_gl, ref_st = oracle.plan_stats(loads_np, ref[0], ref[2], gpus)
    assert np.array_equal(_np(gl), ref_gl) and np.array_equal(_np(st), ref_st)
    assert _np(st)[3, 3] == 1.0


@pytest.mark.parametrize("shape", [(256, 8, 288, 4, 32), (256, 1, 288, 2, 144), (12, 4, 16, 2, 8),
                                   (64, 32, 128, 16, 32), (300, 5, 602, 7, 7),
                                   (96, 3, 2048, 2, 8), (1024, 32, 2048, 8, 64)])
@pytest.mark.parametrize("dist", ["pareto", "huge"])
def test_rebalance_many_rows(shape, dist):
    """More rows than two per SM take the 128-thread many-row kernel and its
    compact shared-memory layout (step 3's outputs in a key area; the
    staging arrays in the table's place): the same plans and plan quality as
    the oracle's, with the bitonic path (1,024 replicas a node), a log2phy
    table outside shared memory and 128-bit keys among the cases."""
    E, G, P, N, gpus = shape
    R = 2 * torch.cuda.get_device_properties(0).multi_processor_count + 11
    rng = np.random.default_rng(E + P + R + len(dist))
    if dist == "pareto":
        loads_np = (rng.pareto(1.3, (R, E)) * 1000).astype(np.int64)
    else:
        loads_np = rng.integers((1 << 40) - 100000, 1 << 40, (R, E)).astype(np.int64)
    loads_np[5] = 0
    gl, st = _quality_bufs(R, gpus)
    status = _status()
    plan = eplb.rebalance(torch.from_numpy(loads_np).to(DEV), P, G, N, gpus, gpu_load=gl, stats=st,
                          status=status)
    torch.cuda.synchronize()
    ref, ref_status = _oracle_rows(loads_np, P, G, N, gpus, plan.log2phy.shape[2])
    assert int(status.item()) == ref_status
    _assert_plan_equal(plan, ref)
    if ref_status == 0:
        ref_gl, ref_st = oracle.plan_stats(loads_np, ref[0], ref[2], gpus)
        assert np.array_equal(_np(gl), ref_gl) and np.array_equal(_np(st), ref_st)


def test_rebalance_fused_quality_worked_example():
    # the per-GPU load range the page prints for layer 0 of its example
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "eplb_readme_example.json")) as f:
        ex = json.load(f)
    w = torch.from_numpy(np.array(ex["weight"], dtype=np.int64)).to(DEV)
    for G, key in ((4, "layer0_gpu_load_hierarchical"), (3, "layer0_gpu_load_global_groups3")):
        gl, st = _quality_bufs(2, 8)
        eplb.rebalance(w, 16, G, 2, 8, gpu_load=gl, stats=st)
        assert _np(st)[0, 0] == ex[key]["min"] and _np(st)[0, 1] == ex[key]["max"]


def test_rebalance_fused_quality_error_rows_are_nan():
    loads_np = np.full((3, 12), 5, dtype=np.int64)
    loads_np[1, 4] = 1 << 41  # outside [0, 2^40): the row is rejected
    gl, st = _quality_bufs(3, 8)
    word = _status()
    eplb.rebalance(torch.from_numpy(loads_np).to(DEV), 16, 4, 2, 8, status=word, gpu_load=gl,
                   stats=st)
    torch.cuda.synchronize()
    assert int(word.item()) == oracle.ERR_RANGE
    assert np.isnan(_np(gl)[1]).all() and np.isnan(_np(st)[1]).all()
    ref = oracle.rebalance(loads_np[[0, 2]], 16, 4, 2, 8)
    ref_gl, ref_st = oracle.plan_stats(loads_np[[0, 2]], ref[0], ref[2], 8)
    assert np.array_equal(_np(gl)[[0, 2]], ref_gl) and np.array_equal(_np(st)[[0, 2]], ref_st)


@pytest.mark.parametrize("single", [True, False])
def test_serving_step_reports_the_next_plans_quality(dsv3_idx, single):
    """The serving step (one launch or two) writes the quality of the plan it
    builds: the oracle's plan_stats on the window sums and the oracle's plan."""
    from moe_expert_load_eplb_b200.pipeline import EplbStep
    c = W.DSV3_PREFILL
    W_ = 4
    hist = W.histogram_steps(W_ - 1, c.L, c.E, c.T * c.K, c.stream, device=DEV)
    step = EplbStep(c.L, c.T, c.K, c.E, c.P, c.G, c.N, c.gpus, window=W_, device=DEV,
                    single_launch=single)
    step.fill_history(hist)
    ring = np.concatenate([_np(hist), np.zeros((1, c.L, c.E), np.int64)], axis=0)

    def check():
        loads = oracle.window(ring, W_, W_ - 1)[0]
        ref = oracle.rebalance(loads, c.P, c.G, c.N, c.gpus, slots=step.X)
        ref_gl, ref_st = oracle.plan_stats(loads, ref[0], ref[2], c.gpus)
        assert np.array_equal(_np(step.gpu_load), ref_gl)
        assert np.array_equal(_np(step.stats), ref_st)

    check()  # the plan fill_history built
    for s_i, idx in enumerate([dsv3_idx, dsv3_idx.flip(1).contiguous()]):
        step(idx)
        torch.cuda.synchronize()
        assert int(step.status.item()) == 0
        ring[(W_ - 1 + s_i) % W_] = oracle.count_loads(_np(idx), c.E)[0]
        check()


@pytest.mark.parametrize("shape", [(58, 256, 288), (3, 12, 16), (1000, 64, 96), (2, 1, 1)])
def test_fold_loads_matches_oracle(shape):
    R, E, P = shape
    rng = np.random.default_rng(R + E + P)
    p2l = rng.integers(0, E, (R, P)).astype(np.int32)
    phys = rng.integers(0, 1 << 40, (R, P))
    got = eplb.fold_loads(torch.from_numpy(phys).to(DEV), torch.from_numpy(p2l).to(DEV), E)
    assert np.array_equal(_np(got), oracle.fold_loads(phys, p2l, E))


def test_fold_of_physical_counts_after_redirect(dsv3_idx):
    c = W.DSV3_PREFILL
    counts = eplb.count_loads(dsv3_idx, c.E)
    plan = eplb.rebalance(counts, c.P, c.G, c.N, c.gpus)
    out = eplb.redirect(dsv3_idx, plan.log2phy, plan.logcnt)
    phys = eplb.count_loads(out, c.P)
    assert torch.equal(eplb.fold_loads(phys, plan.phy2log, c.E), counts)


def test_initial_map_matches_oracle():
    p2l, prk = eplb.initial_map(58, 256, 288, device=DEV)
    ref_p, ref_r = oracle.initial_map(58, 256, 288)
    assert np.array_equal(_np(p2l), ref_p) and np.array_equal(_np(prk), ref_r)


@pytest.mark.parametrize("cfg", ["dsv3_prefill", "global_policy"])
def test_plan_diff_matches_oracle(cfg, sweep_steps):
    c = W.WORKLOADS[cfg]
    if cfg == "global_policy":
        old_l = W.global_policy_loads()
        new_l = np.roll(old_l, 1, axis=1)
    else:
        snaps = _np(sweep_steps)
        old_l, new_l = snaps[10], snaps[900]
    old = _plans_for(c, old_l)[0]
    new = _plans_for(c, new_l)[0]
    src, moves = eplb.plan_diff(torch.from_numpy(old).to(DEV), torch.from_numpy(new).to(DEV),
                                c.E, c.gpus)
    ref_src, ref_moves = oracle.plan_diff(old, new, c.E, c.gpus)
    assert np.array_equal(_np(src), ref_src) and np.array_equal(_np(moves), ref_moves)


def test_plan_diff_initial_to_first_plan(dsv3_idx):
    c = W.DSV3_PREFILL
    init, _ = eplb.initial_map(c.L, c.E, c.P, device=DEV)
    plan = eplb.rebalance(eplb.count_loads(dsv3_idx, c.E), c.P, c.G, c.N, c.gpus)
    src, moves = eplb.plan_diff(init, plan.phy2log, c.E, c.gpus)
    ref_src, ref_moves = oracle.plan_diff(_np(init), _np(plan.phy2log), c.E, c.gpus)
    assert np.array_equal(_np(src), ref_src) and np.array_equal(_np(moves), ref_moves)


# ------------------------------------------------------- rebalance_window --

@pytest.mark.parametrize("W_,zero", [(16, 3), (1, -1), (4, 0), (7, -1)])
def test_rebalance_window_matches_window_then_rebalance(W_, zero):
    c = W.DSV3_PREFILL
    ring = W.histogram_steps(W_, c.L, c.E, c.T * c.K, 7, device=DEV).contiguous()
    ring_h = _np(ring).copy()
    loads_out = torch.empty((c.L, c.E), dtype=torch.int64, device=DEV)
    st = _status()
    plan = eplb.rebalance_window(ring, c.P, c.G, c.N, c.gpus, zero_slot=zero, loads_out=loads_out,
                                 status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    sums = oracle.window(ring_h, W_, W_ - 1)[0]
    assert np.array_equal(_np(loads_out), sums)
    ref = oracle.rebalance(sums, c.P, c.G, c.N, c.gpus, slots=plan.log2phy.shape[2])
    _assert_plan_equal(plan, ref)
    after = _np(ring)
    for k in range(W_):
        if k == zero:
            assert (after[k] == 0).all()
        else:
            assert np.array_equal(after[k], ring_h[k])


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("dist", ["uniform", "huge"])
def test_rebalance_window_rotating_ring_shapes(shape, dist):
    """A rotating ring (zero_slot >= 0: the serving step's call, which runs
    the instruction warm-up on shapes with room for its scratch) and a fixed
    one give the same plan, the oracle's for the summed rows; the cleared
    slot is all zero afterwards."""
    E, G, P, N, gpus = shape
    rng = np.random.default_rng(abs(hash((E, G, P, N, gpus, dist))) % (1 << 31))
    R = 5
    if dist == "uniform":
        w = rng.integers(0, 5000, (R, E))
    else:
        w = rng.integers((1 << 40) - 100000, 1 << 40, (R, E))
    w = w.astype(np.int64)
    ring_h = np.stack([w // 3, w // 3, w - 2 * (w // 3)])
    plans, statuses = [], []
    for zero in (-1, 1):
        ring = torch.from_numpy(ring_h.copy()).to(DEV)
        st = _status()
        plans.append(eplb.rebalance_window(ring, P, G, N, gpus, zero_slot=zero, status=st))
        torch.cuda.synchronize()
        after = _np(ring)
        assert np.array_equal(after[0], ring_h[0]) and np.array_equal(after[2], ring_h[2])
        assert np.array_equal(after[1], ring_h[1] if zero < 0 else np.zeros_like(ring_h[1]))
        statuses.append(int(st.item()))
    ref, ref_status = _oracle_rows(w, P, G, N, gpus, plans[0].log2phy.shape[2])
    assert statuses == [ref_status, ref_status]
    for plan in plans:
        _assert_plan_equal(plan, ref)


def test_rebalance_window_range_error():
    ring = torch.full((2, 3, 12), 1 << 39, dtype=torch.int64, device=DEV)  # sums reach 2^40
    ring[:, 1] = 5
    st = _status()
    plan = eplb.rebalance_window(ring, 16, 4, 2, 8, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 4
    assert (_np(plan.phy2log[0]) == -1).all() and (_np(plan.phy2log[2]) == -1).all()
    ref = oracle.rebalance(np.full((1, 12), 10, np.int64), 16, 4, 2, 8, slots=plan.log2phy.shape[2])
    for got, want in zip(plan, ref):
        assert np.array_equal(_np(got)[1:2], want)
