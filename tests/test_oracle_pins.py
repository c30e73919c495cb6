"""Pins of the CPU oracle to facts outside itself (CPU only).

Each test names what fixes the expected value: the pages' worked example and
exercises (values in tests/golden/eplb_readme_example.json), textbook
routines (D'Hondt apportionment, numpy bincount / cumsum / fancy indexing),
closed forms of the packing greedy on special inputs, brute force over all
plans on tiny inputs, and invariants the pages' assertions state.
"""
from __future__ import annotations

import itertools
import json
import os
import zlib
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests._invariants import check_plan, gpu_loads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "eplb_readme_example.json")


@pytest.fixture(scope="module")
def ex():
    with open(GOLDEN) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# The pages' worked example (section "Интерфейс и пример" and the boxes)
# --------------------------------------------------------------------------

def _example_plan(ex, num_groups=None):
    w = np.array(ex["weight"], dtype=np.int64)
    return w, oracle.rebalance(w, ex["num_replicas"], num_groups or ex["num_groups"],
                               ex["num_nodes"], ex["num_gpus"])


def test_example_phy2log(ex):
    _, (p2l, _, _, _) = _example_plan(ex)
    assert p2l.tolist() == ex["phy2log"]["value"]


def test_example_layer0_derivation(ex):
    w, (p2l, prk, cnt, l2p) = _example_plan(ex)
    w0 = w[0]
    assert [int(w0[3 * g:3 * g + 3].sum()) for g in range(4)] == ex["layer0_group_loads"]["value"]
    ppn = ex["num_replicas"] // ex["num_nodes"]
    for n, groups in enumerate(ex["layer0_node_groups"]["value"]):
        experts = set(p2l[0, n * ppn:(n + 1) * ppn].tolist())
        assert experts == {3 * g + i for g in groups for i in range(3)}
        assert int(sum(w0[e] for e in experts)) == ex["layer0_node_groups"]["node_loads"][n]
        assert sorted(e for e in experts if cnt[0, e] > 1) == sorted(ex["layer0_replicated"]["value"][n])
    assert cnt[0].tolist() == ex["layer0_logcnt"]["value"]


def test_example_gpu_load_ranges(ex):
    w, (p2l, _, cnt, _) = _example_plan(ex)
    loads = gpu_loads(w[0], p2l[0], cnt[0], ex["num_gpus"])
    h = ex["layer0_gpu_load_hierarchical"]
    assert min(loads) == Fraction(h["min"]) and max(loads) == Fraction(h["max"])
    assert round(float(sum(loads) / len(loads))) == h["mean_rounded"]
    g = ex["layer0_gpu_load_global_groups3"]
    w, (p2l, _, cnt, _) = _example_plan(ex, num_groups=g["num_groups"])
    loads = gpu_loads(w[0], p2l[0], cnt[0], ex["num_gpus"])
    assert min(loads) == Fraction(g["min"]) and max(loads) == Fraction(g["max"])


def test_example_log2phy(ex):
    _, (_, _, _, l2p) = _example_plan(ex)
    d = ex["layer0_log2phy"]
    assert l2p[0, 1, :2].tolist() == d["expert1"]
    assert l2p[0, 0, :2].tolist() == d["expert0"]


def test_example_invariants(ex):
    w, plan = _example_plan(ex)
    check_plan(w, *plan, ex["num_replicas"], ex["num_groups"], ex["num_nodes"], ex["num_gpus"])
    w, plan = _example_plan(ex, num_groups=3)
    check_plan(w, *plan, ex["num_replicas"], 3, ex["num_nodes"], ex["num_gpus"])


# --------------------------------------------------------------------------
# replicate_experts == D'Hondt (Jefferson) highest averages, a textbook routine
# --------------------------------------------------------------------------

def _dhondt(votes, seats):
    """Textbook D'Hondt: award ``seats`` to the largest quotients v_i/d, d = 1, 2, ...

    Ties go to the lower party index, then to the smaller divisor.  Returns
    the awarded (party, divisor) pairs in award order.
    """
    quot = [(Fraction(int(v), d), i, d) for i, v in enumerate(votes) for d in range(1, seats + 1)]
    quot.sort(key=lambda q: (-q[0], q[1], q[2]))
    return [(i, d) for _, i, d in quot[:seats]]


@pytest.mark.parametrize("seed", range(40))
def test_replicate_is_dhondt(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 12))
    extra = int(rng.integers(0, 14))
    kind = seed % 4
    if kind == 0:
        w = rng.integers(0, 1000, n)
    elif kind == 1:
        w = rng.integers(0, 4, n) * 6          # many exact ties
    elif kind == 2:
        w = np.zeros(n, dtype=np.int64)        # all zero: expert 0 takes every extra
    else:
        w = rng.integers(0, 1 << 39, n)
    p2l, rank, cnt = oracle.replicate_experts(w, n + extra)
    assert p2l[:n].tolist() == list(range(n)) and (rank[:n] == 0).all()
    awards = _dhondt(w, extra)
    assert [(int(a), int(b)) for a, b in zip(p2l[n:], rank[n:])] == awards
    seats = np.bincount([i for i, _ in awards], minlength=n) if awards else np.zeros(n, int)
    assert (cnt == 1 + seats).all()


@pytest.mark.parametrize("seed", range(30))
def test_replicate_minimises_max_load_per_replica(seed):
    """Brute force: no count vector with the same total has a smaller max w/c."""
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(1, 5))
    extra = int(rng.integers(0, 6))
    w = rng.integers(0, 50, n)
    _, _, cnt = oracle.replicate_experts(w, n + extra)
    got = max(Fraction(int(w[i]), int(cnt[i])) for i in range(n))
    best = None
    for c in itertools.product(range(1, extra + 2), repeat=n):
        if sum(c) != n + extra:
            continue
        m = max(Fraction(int(w[i]), c[i]) for i in range(n))
        best = m if best is None or m < best else best
    assert got == best


# --------------------------------------------------------------------------
# balanced_packing: closed forms on special inputs, brute-force lower bound
# --------------------------------------------------------------------------

def test_pack_one_per_pack_is_identity():
    # the pages' short-cut: n/m == 1 maps item i -> pack i regardless of weight
    pi, ri = oracle.balanced_packing([5, 1, 9, 3], 4)
    assert pi.tolist() == [0, 1, 2, 3] and ri.tolist() == [0, 0, 0, 0]


def test_pack_single_pack_ranks_in_sorted_order():
    w = [4, 9, 4, 1, 9, 0]
    pi, ri = oracle.balanced_packing(w, 1)
    assert (pi == 0).all()
    order = sorted(range(len(w)), key=lambda i: (-w[i], i))  # stable descending
    assert [order.index(i) for i in range(len(w))] == ri.tolist()


@pytest.mark.parametrize("m,cap", [(2, 3), (3, 4), (4, 2), (8, 9), (5, 5)])
def test_pack_equal_weights_round_robin(m, cap):
    # equal positive weights: stable order is by index, every pack ties in turn
    n = m * cap
    pi, ri = oracle.balanced_packing([7] * n, m)
    assert pi.tolist() == [i % m for i in range(n)]
    assert ri.tolist() == [i // m for i in range(n)]


@pytest.mark.parametrize("m", [2, 3, 7, 144])
def test_pack_cap2_strictly_decreasing_is_snake(m):
    # cap 2, distinct positive weights: the m heaviest open the packs in order,
    # then the next ones fill the packs from the lightest (last) backwards
    rng = np.random.default_rng(m)
    w = rng.permutation(np.arange(1, 2 * m + 1) * 3 + 1)
    pi, ri = oracle.balanced_packing(w, m)
    order = np.argsort(-w, kind="stable")
    for pos, i in enumerate(order):
        if pos < m:
            assert (pi[i], ri[i]) == (pos, 0)
        else:
            assert (pi[i], ri[i]) == (2 * m - 1 - pos, 1)


def test_pack_zero_weights_fill_lowest_pack_first():
    # all zero: every pack ties at weight 0, the lowest non-full pack wins
    pi, ri = oracle.balanced_packing([0] * 6, 3)
    assert pi.tolist() == [0, 0, 1, 1, 2, 2] and ri.tolist() == [0, 1, 0, 1, 0, 1]


def test_pack_fraction_weights_are_exact():
    # exact ties between sums of fractions (1 + 1/3 == 1 + 1/3) go to the lower pack
    num = [1, 1, 1, 1, 1, 0]
    den = [3, 3, 3, 1, 1, 1]
    pi, ri = oracle.balanced_packing_frac(num, den, 2)
    # sorted: items 3, 4 (load 1), 0, 1, 2 (1/3), 5 (0)
    # 3 -> pack 0; 4 -> pack 1; 0 -> 0 (tie 1 vs 1, lowest); 1 -> 1; 2 -> 0 (4/3 vs 4/3); 5 -> 1
    assert pi.tolist() == [0, 1, 0, 0, 1, 1]
    assert ri.tolist() == [1, 1, 2, 0, 0, 2]


def _pack_opt(w, m):
    n = len(w)
    cap = n // m
    best = None
    for labels in itertools.product(range(m), repeat=n):
        if any(labels.count(p) != cap for p in range(m)):
            continue
        mx = max(sum(w[i] for i in range(n) if labels[i] == p) for p in range(m))
        best = mx if best is None or mx < best else best
    return best


@pytest.mark.parametrize("seed", range(25))
def test_pack_invariants_and_brute_force_bound(seed):
    rng = np.random.default_rng(200 + seed)
    m = int(rng.integers(1, 4))
    cap = int(rng.integers(1, 4))
    n = m * cap
    w = rng.integers(0, 30, n)
    pi, ri = oracle.balanced_packing(w, m)
    for p in range(m):
        members = np.flatnonzero(pi == p)
        assert len(members) == cap and sorted(ri[members].tolist()) == list(range(cap))
    greedy = max(int(w[pi == p].sum()) for p in range(m))
    assert greedy >= _pack_opt(w.tolist(), m)
    assert sum(int(w[pi == p].sum()) for p in range(m)) == int(w.sum())


# --------------------------------------------------------------------------
# Whole plan: invariants on random rows; brute-force optimum on tiny inputs
# --------------------------------------------------------------------------

SHAPES = [
    # E, G, P, N, gpus
    (12, 4, 16, 2, 8),
    (12, 3, 16, 2, 8),      # global (3 % 2 != 0)
    (16, 4, 16, 2, 4),      # no redundancy
    (16, 4, 32, 4, 8),      # groups_per_node == 1 short-cut
    (8, 2, 16, 2, 16),      # one replica per GPU short-cut
    (24, 6, 36, 3, 6),
    (256, 8, 288, 4, 32),   # DeepSeek-V3 prefill shape
    (256, 1, 288, 2, 144),  # global, 2 per GPU
    (64, 8, 96, 8, 16),
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("dist", ["uniform", "ties", "zeros", "huge"])
def test_plan_invariants(shape, dist):
    E, G, P, N, gpus = shape
    rng = np.random.default_rng(zlib.crc32(repr((shape, dist)).encode()))
    R = 3
    if dist == "uniform":
        w = rng.integers(0, 5000, (R, E))
    elif dist == "ties":
        w = rng.integers(0, 3, (R, E)) * 12
    elif dist == "zeros":
        w = np.zeros((R, E), dtype=np.int64)
    else:
        w = rng.integers((1 << 40) - 1000, 1 << 40, (R, E))
    plan = oracle.rebalance(w, P, G, N, gpus)
    check_plan(w, *plan, P, G, N, gpus)


def test_plan_scale_invariance():
    # only ratios of loads enter the comparisons: k * w gives the same plan
    rng = np.random.default_rng(7)
    for shape in SHAPES:
        E, G, P, N, gpus = shape
        w = rng.integers(0, 3000, (2, E))
        base = oracle.rebalance(w, P, G, N, gpus)
        for k in (2, 3, 1000):
            scaled = oracle.rebalance(w * k, P, G, N, gpus)
            for a, b in zip(base, scaled):
                assert (a == b).all()


def test_global_policy_dispatch():
    # num_groups % num_nodes != 0 runs the same procedure with 1 group on 1 node
    rng = np.random.default_rng(8)
    w = rng.integers(0, 999, (4, 12))
    a = oracle.rebalance(w, 16, 3, 2, 8)
    b = oracle.rebalance(w, 16, 1, 1, 8)
    for x, y in zip(a, b):
        assert (x == y).all()


@pytest.mark.parametrize("seed", range(12))
def test_global_plan_vs_brute_force_optimum(seed):
    """Tiny global case: greedy max GPU load >= the optimum over all plans."""
    rng = np.random.default_rng(300 + seed)
    E, P, gpus = 4, 6, 3
    w = rng.integers(1, 40, (1, E))
    p2l, _, cnt, _ = oracle.rebalance(w, P, 1, 1, gpus)
    greedy = max(gpu_loads(w[0], p2l[0], cnt[0], gpus))
    best = None
    for c in itertools.product(range(1, P - E + 2), repeat=E):
        if sum(c) != P:
            continue
        items = [Fraction(int(w[0, e]), c[e]) for e in range(E) for _ in range(c[e])]
        for labels in itertools.product(range(gpus), repeat=P):
            if any(labels.count(g) != P // gpus for g in range(gpus)):
                continue
            mx = max(sum((items[i] for i in range(P) if labels[i] == g), Fraction(0)) for g in range(gpus))
            best = mx if best is None or mx < best else best
    assert greedy >= best
    assert greedy <= 2 * best  # the greedy gap on these inputs is small; a gross error is not


def test_rebalance_errors():
    w = np.ones((1, 12), dtype=np.int64)
    with pytest.raises(oracle.OracleError) as e:
        oracle.rebalance(w, 16, 5, 2, 8)            # 12 % 5 != 0
    assert e.value.code == oracle.ERR_DIVISIBILITY
    with pytest.raises(oracle.OracleError) as e:
        oracle.rebalance(w, 18, 4, 2, 8)            # 18 % 8 != 0
    assert e.value.code == oracle.ERR_DIVISIBILITY
    with pytest.raises(oracle.OracleError) as e:
        oracle.rebalance(w, 18, 4, 4, 6)            # hierarchical needs gpus % nodes == 0
    assert e.value.code == oracle.ERR_DIVISIBILITY
    oracle.rebalance(w, 18, 3, 2, 3)                # global: 3 % 2 != 0 is fine
    with pytest.raises(oracle.OracleError) as e:
        oracle.rebalance(w, 8, 4, 2, 8)             # fewer replicas than experts
    assert e.value.code == oracle.ERR_SHAPE
    with pytest.raises(oracle.OracleError) as e:
        oracle.rebalance(w * (1 << 40), 16, 4, 2, 8)
    assert e.value.code == oracle.ERR_RANGE
    w2 = np.array([[1000, 1, 1, 1]], dtype=np.int64)
    with pytest.raises(oracle.OracleError) as e:
        oracle.rebalance(w2, 8, 1, 1, 4, slots=2)   # expert 0 gets 5 replicas
    assert e.value.code == oracle.ERR_SLOTS


# --------------------------------------------------------------------------
# S1 count, S2 window, S5 redirect: closed forms via numpy routines
# --------------------------------------------------------------------------

@pytest.mark.parametrize("shape", [(1, 0, 8), (2, 4096, 2), (3, 1001, 8), (5, 7, 3)])
def test_count_is_bincount(shape):
    L, T, K = shape
    E = 40
    rng = np.random.default_rng(L * 1000 + T)
    idx = rng.integers(-3, E + 3, (L, T, K)).astype(np.int32)
    counts, bad = oracle.count_loads(idx, E)
    ref = np.stack([np.bincount(idx[l][(idx[l] >= 0) & (idx[l] < E)], minlength=E) for l in range(L)]) \
        if T else np.zeros((L, E), np.int64)
    assert (counts == ref).all()
    assert bad == int(((idx < 0) | (idx >= E)).sum())
    again, _ = oracle.count_loads(idx, E, counts=counts.copy())
    assert (again == 2 * ref).all()


@pytest.mark.parametrize("S,W,s_first", [(1, 1, 0), (10, 3, 0), (10, 10, 0), (10, 100, 0),
                                          (17, 4, 5), (9, 9, 8), (6, 1, 0)])
def test_window_is_direct_sum(S, W, s_first):
    rng = np.random.default_rng(S * 100 + W)
    steps = rng.integers(0, 1 << 30, (S, 3, 5))
    snaps = oracle.window(steps, W, s_first)
    direct = np.stack([steps[max(0, s - W + 1):s + 1].sum(0) for s in range(s_first, S)])
    assert (snaps == direct).all()
    c = np.cumsum(steps, axis=0)
    via_cumsum = np.stack([c[s] - (c[s - W] if s - W >= 0 else 0) for s in range(s_first, S)])
    assert (snaps == via_cumsum).all()


@pytest.mark.parametrize("t0", [0, 5, 123456789])
def test_redirect_closed_form_and_round_trip(t0):
    rng = np.random.default_rng(t0 % 1000)
    L, T, K, E, P = 3, 257, 3, 12, 16
    w = rng.integers(0, 500, (L, E))
    p2l, prk, cnt, l2p = oracle.rebalance(w, P, 4, 2, 8)
    idx = rng.integers(-1, E + 1, (L, T, K)).astype(np.int32)
    out, bad = oracle.redirect(idx, l2p, cnt, t0)
    valid = (idx >= 0) & (idx < E)
    assert bad == int((~valid).sum())
    assert (out[~valid] == -1).all()
    ll, tt, kk = np.nonzero(valid)
    e = idx[ll, tt, kk]
    slot = (t0 + tt) % cnt[ll, e]
    assert (out[ll, tt, kk] == l2p[ll, e, slot]).all()
    # round trip: the physical replica serves the same logical expert, with rank (t0+t) mod cnt
    assert (p2l[ll, out[ll, tt, kk]] == e).all()
    assert (prk[ll, out[ll, tt, kk]] == slot).all()


def test_redirect_shards_concatenate():
    rng = np.random.default_rng(11)
    L, T, K, E = 2, 100, 4, 12
    w = rng.integers(0, 500, (L, E))
    _, _, cnt, l2p = oracle.rebalance(w, 16, 4, 2, 8)
    idx = rng.integers(0, E, (L, T, K)).astype(np.int32)
    whole, _ = oracle.redirect(idx, l2p, cnt, 0)
    a, _ = oracle.redirect(idx[:, :37], l2p, cnt, 0)
    b, _ = oracle.redirect(idx[:, 37:], l2p, cnt, 37)
    assert (np.concatenate([a, b], axis=1) == whole).all()


# --------------------------------------------------------------------------
# Plan quality, physical-load fold, initial map, plan diff
# --------------------------------------------------------------------------

def test_plan_stats_worked_example(ex):
    # the per-GPU loads the page prints for layer 0, both policies
    w = np.array(ex["weight"], dtype=np.int64)
    for G, key in ((4, "layer0_gpu_load_hierarchical"), (3, "layer0_gpu_load_global_groups3")):
        p2l, _, cnt, _ = oracle.rebalance(w, 16, G, 2, 8)
        gl, st = oracle.plan_stats(w, p2l, cnt, 8)
        exact = gpu_loads(w[0], p2l[0], cnt[0], 8)
        assert [float(x) for x in exact] == gl[0].tolist()
        assert st[0, 0] == ex[key]["min"] and st[0, 1] == ex[key]["max"]
        assert st[0, 2] == float(sum(exact) / 8) and st[0, 3] == st[0, 2] / st[0, 1]
        assert round(st[0, 2]) == ex["layer0_gpu_load_hierarchical"]["mean_rounded"]


def test_plan_stats_zero_loads_are_balanced():
    w = np.zeros((2, 12), dtype=np.int64)
    p2l, _, cnt, _ = oracle.rebalance(w, 16, 4, 2, 8)
    gl, st = oracle.plan_stats(w, p2l, cnt, 8)
    assert (gl == 0).all() and (st[:, 3] == 1.0).all()


def test_fold_is_weighted_bincount():
    rng = np.random.default_rng(5)
    R, E, P = 4, 12, 20
    p2l = rng.integers(0, E, (R, P)).astype(np.int32)
    phys = rng.integers(0, 1 << 40, (R, P))
    got = oracle.fold_loads(phys, p2l, E)
    for r in range(R):
        want = np.zeros(E, dtype=np.int64)
        np.add.at(want, p2l[r], phys[r])
        assert (got[r] == want).all()


def test_fold_of_redirected_counts_is_the_logical_count():
    # counting redirected (physical) indices and folding gives the logical counts
    rng = np.random.default_rng(6)
    L, T, K, E, P = 2, 300, 4, 12, 16
    p2l, prk, cnt, l2p = oracle.rebalance(rng.integers(0, 99, (L, E)), P, 4, 2, 8)
    idx = rng.integers(0, E, (L, T, K)).astype(np.int32)
    out, _ = oracle.redirect(idx, l2p, cnt)
    phys, _ = oracle.count_loads(out, P)
    logical, _ = oracle.count_loads(idx, E)
    assert (oracle.fold_loads(phys, p2l, E) == logical).all()


@pytest.mark.parametrize("E,P", [(256, 288), (12, 16), (4, 13), (1, 5), (7, 7), (32, 100)])
def test_initial_map_routed_experts_first(E, P):
    # vLLM eplb_state glossary prose: the physical experts are the routed
    # (logical) experts followed by the redundant ones (256 routed + 32
    # redundant = 288 on DeepSeek-V3), so slot p < E holds expert p, rank 0
    p2l, prk = oracle.initial_map(2, E, P)
    assert (p2l[:, :E] == np.arange(E)).all() and (prk[:, :E] == 0).all()


@pytest.mark.parametrize("E,P", [(256, 288), (12, 16), (4, 13), (1, 5), (7, 7), (32, 100)])
def test_initial_map_is_a_valid_plan(E, P):
    # every slot names an expert, every expert has a replica, and a slot's
    # rank counts the earlier slots of its expert (ranks 0 .. cnt-1 in slot
    # order), so logcnt = bincount(phy2log) sums to P
    p2l, prk = oracle.initial_map(3, E, P)
    for r in range(3):
        assert ((p2l[r] >= 0) & (p2l[r] < E)).all()
        cnt = np.bincount(p2l[r], minlength=E)
        assert cnt.sum() == P and (cnt >= 1).all()
        seen = np.zeros(E, dtype=np.int64)
        for p in range(P):
            e = p2l[r, p]
            assert prk[r, p] == seen[e]
            seen[e] += 1


@pytest.mark.parametrize("E,P", [(256, 288), (12, 16), (4, 13), (1, 5), (7, 7), (32, 100), (5, 23)])
def test_initial_map_is_replicate_experts_on_equal_loads(E, P):
    # Before any load is measured every expert is taken as equally loaded.
    # The appendix's replicate_experts (pinned to textbook D'Hondt above)
    # then hands each redundant slot to the lowest-index expert among those
    # with the fewest replicas: the initial map's cycle from expert 0.  A
    # different cycle (another start, a reversed order, two redundant slots
    # for one expert before another gets its first) fails here.
    p2l, prk = oracle.initial_map(1, E, P)
    want_p2l, want_rank, want_cnt = oracle.replicate_experts(np.full(E, 1000, np.int64), P)
    assert (p2l[0] == want_p2l).all() and (prk[0] == want_rank).all()
    assert (np.bincount(p2l[0], minlength=E) == want_cnt).all()
    assert want_cnt.max() - want_cnt.min() <= 1  # the redundant slots are spread evenly


def test_plan_diff_identity_and_swap():
    rng = np.random.default_rng(9)
    w = rng.integers(0, 500, (3, 24))
    p2l, _, _, _ = oracle.rebalance(w, 32, 6, 2, 8)
    src, moves = oracle.plan_diff(p2l, p2l, 24, 8)
    assert (src == -1).all() and (moves == 0).all()
    # swapping the contents of GPUs 0 and 1 (4 slots each) moves every slot of
    # both GPUs whose expert the other GPU did not hold
    swapped = p2l.copy()
    swapped[:, 0:4], swapped[:, 4:8] = p2l[:, 4:8], p2l[:, 0:4]
    src, moves = oracle.plan_diff(p2l, swapped, 24, 8)
    assert (src[:, 8:] == -1).all()
    for r in range(3):
        for g, other in ((0, 1), (1, 0)):
            for k in range(4):
                p = g * 4 + k
                e = swapped[r, p]
                if e in p2l[r, g * 4:(g + 1) * 4]:
                    continue
                assert src[r, p] == int(np.flatnonzero(p2l[r] == e)[0])


@pytest.mark.parametrize("seed", range(20))
def test_plan_diff_invariants(seed):
    rng = np.random.default_rng(400 + seed)
    E, P, gpus = 16, 32, 8
    a, _, _, _ = oracle.rebalance(rng.integers(0, 300, (2, E)), P, 4, 2, gpus)
    b, _, _, _ = oracle.rebalance(rng.integers(0, 300, (2, E)), P, 4, 2, gpus)
    src, moves = oracle.plan_diff(a, b, E, gpus)
    ppg = P // gpus
    for r in range(2):
        assert moves[r] == int((src[r] != -1).sum())
        for g in range(gpus):
            old = list(a[r, g * ppg:(g + 1) * ppg])
            new = list(b[r, g * ppg:(g + 1) * ppg])
            kept = [int(b[r, g * ppg + k]) for k in range(ppg) if src[r, g * ppg + k] == -1]
            for e in set(new):
                assert kept.count(e) == min(old.count(e), new.count(e))
            for k in range(ppg):
                s = src[r, g * ppg + k]
                if s != -1:
                    assert a[r, s] == b[r, g * ppg + k]   # the copy source holds the expert
