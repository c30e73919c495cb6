"""Plan invariants that the EPLB pages fix, written independently of any implementation.

Used by the oracle pin tests and by the GPU parity tests.  Sources: page
"DualPipe и EPLB: конвейер в обе стороны и балансировщик экспертов", Part 2,
appendix eplb.py (assertions and docstrings of balanced_packing,
replicate_experts, rebalance_experts_hierarchical, rebalance_experts) and the
section "Иерархическая балансировка" (groups stay on one node).
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np


def check_plan(loads, phy2log, phyrank, logcnt, log2phy, P, G, N, gpus):
    """Assert every invariant of one rebalance result (all rows)."""
    loads = np.asarray(loads)
    R, E = loads.shape
    assert phy2log.shape == (R, P) and phyrank.shape == (R, P) and logcnt.shape == (R, E)
    X = log2phy.shape[2]
    hier = G % N == 0
    for r in range(R):
        p2l, prk, cnt, l2p = phy2log[r], phyrank[r], logcnt[r], log2phy[r]
        # every logical expert keeps at least one replica; replicas add up to P
        assert (cnt >= 1).all()
        assert int(cnt.sum()) == P
        assert ((p2l >= 0) & (p2l < E)).all()
        # replica ranks of expert e are exactly 0 .. logcnt[e]-1
        occ = np.bincount(p2l, minlength=E)
        assert (occ == cnt).all()
        for e in range(E):
            ranks = sorted(prk[p2l == e].tolist())
            assert ranks == list(range(int(cnt[e])))
        # log2phy inverts phy2log, -1 beyond logcnt
        for e in range(E):
            c = int(cnt[e])
            assert c <= X
            for k in range(X):
                if k < c:
                    p = int(l2p[e, k])
                    assert 0 <= p < P and p2l[p] == e and prk[p] == k
                else:
                    assert l2p[e, k] == -1
        if hier and N > 1:
            # each node holds whole groups, and the node's replicas are those of its groups
            gs, lpn, ppn = E // G, E // N, P // N
            for n in range(N):
                experts = set(p2l[n * ppn:(n + 1) * ppn].tolist())
                groups = {e // gs for e in experts}
                assert len(groups) == G // N
                assert experts == {g * gs + i for g in groups for i in range(gs)}
                assert int(cnt[sorted(experts)].sum()) == ppn
                assert len(experts) == lpn


def gpu_loads(w_row, p2l_row, cnt_row, gpus):
    """Exact per-GPU load: sum of w[e]/logcnt[e] over the GPU's replicas."""
    P = len(p2l_row)
    ppg = P // gpus
    return [sum((Fraction(int(w_row[e]), int(cnt_row[e])) for e in p2l_row[g * ppg:(g + 1) * ppg]),
                Fraction(0)) for g in range(gpus)]
