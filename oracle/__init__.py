"""CPU oracle of the EPLB hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product (``moe_expert_load_eplb_b200``) never imports, loads or calls it, and
the two share no code: the arithmetic lives in ``eplb_oracle.c`` (plain C,
exact integers, single thread) and this module only marshals numpy arrays
through ctypes.

Every function cites the passage it follows in ``eplb_oracle.c``; the pages
are the EPLB README translation with its ``eplb.py`` appendix (page
"DualPipe и EPLB: конвейер в обе стороны и балансировщик экспертов") and the
LPLB usage example (page "DeepSeek开源LPLB：基于线性规划的MoE负载均衡器").
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "eplb_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_eplb.so")

OK, ERR_SHAPE, ERR_DIVISIBILITY, ERR_RANGE, ERR_SLOTS, ERR_ALLOC = 0, 2, 3, 4, 5, 9


def build(force: bool = False) -> str:
    """Compile eplb_oracle.c into liboracle_eplb.so beside it (gcc, -O2)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=gnu11", "-shared", "-fPIC", "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        p = ctypes.c_void_p
        i64, i32 = ctypes.c_int64, ctypes.c_int32
        lib.oracle_count_loads.argtypes = [p, i64, i64, i32, i32, p, ctypes.c_int, p]
        lib.oracle_count_loads.restype = None
        lib.oracle_window.argtypes = [p, i64, i64, i32, i64, i64, p]
        lib.oracle_window.restype = None
        lib.oracle_rebalance.argtypes = [p, i64, i32, i32, i32, i32, i32, i32, p, p, p, p]
        lib.oracle_rebalance.restype = ctypes.c_int
        lib.oracle_redirect.argtypes = [p, i64, i64, i32, i32, p, i32, p, i64, p, p]
        lib.oracle_redirect.restype = None
        lib.oracle_balanced_packing.argtypes = [p, i32, i32, p, p]
        lib.oracle_balanced_packing.restype = ctypes.c_int
        lib.oracle_balanced_packing_frac.argtypes = [p, p, i32, i32, p, p]
        lib.oracle_balanced_packing_frac.restype = ctypes.c_int
        lib.oracle_replicate_experts.argtypes = [p, i32, i32, p, p, p]
        lib.oracle_replicate_experts.restype = None
        lib.oracle_plan_stats.argtypes = [p, p, p, i64, i32, i32, i32, p, p]
        lib.oracle_plan_stats.restype = None
        lib.oracle_fold_loads.argtypes = [p, p, i64, i32, i32, p]
        lib.oracle_fold_loads.restype = None
        lib.oracle_initial_map.argtypes = [i64, i32, i32, p, p]
        lib.oracle_initial_map.restype = None
        lib.oracle_plan_diff.argtypes = [p, p, i64, i32, i32, i32, p, p]
        lib.oracle_plan_diff.restype = ctypes.c_int
        _lib = lib
    return _lib


class OracleError(RuntimeError):
    def __init__(self, code: int):
        super().__init__(f"oracle status {code}")
        self.code = code


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def count_loads(idx: np.ndarray, E: int, counts: np.ndarray | None = None):
    """S1: counts[l, e] = number of (t, k) with idx[l, t, k] == e.

    ``idx`` is int32 [L, T, K].  Returns (counts int64 [L, E], bad) where bad
    is the number of indices outside [0, E).  If ``counts`` is given the
    result is added to it in place.
    """
    idx = _c(idx, np.int32)
    L, T, K = idx.shape
    acc = counts is not None
    if counts is None:
        counts = np.zeros((L, E), dtype=np.int64)
    assert counts.dtype == np.int64 and counts.flags.c_contiguous and counts.shape == (L, E)
    bad = ctypes.c_uint64(0)
    _load().oracle_count_loads(_ptr(idx), L, T, K, E, _ptr(counts), int(acc), ctypes.addressof(bad))
    return counts, int(bad.value)


def window(steps: np.ndarray, W: int, s_first: int = 0) -> np.ndarray:
    """S2: snaps[s - s_first] = sum of steps[max(0, s-W+1) .. s], s >= s_first."""
    steps = _c(steps, np.int64)
    S, L, E = steps.shape
    out = np.zeros((max(S - s_first, 0), L, E), dtype=np.int64)
    _load().oracle_window(_ptr(steps), S, L, E, W, s_first, _ptr(out))
    return out


def rebalance(loads: np.ndarray, num_replicas: int, num_groups: int, num_nodes: int,
              num_gpus: int, slots: int | None = None):
    """S3/S4: rebalance_experts over every row of ``loads`` (int64 [R, E]).

    Returns (phy2log [R, P], phyrank [R, P], logcnt [R, E], log2phy [R, E, X])
    as int32, X = ``slots`` (default P - E + 1, always enough).
    """
    loads = _c(loads, np.int64)
    R, E = loads.shape
    P = num_replicas
    X = P - E + 1 if slots is None else slots
    phy2log = np.empty((R, P), dtype=np.int32)
    phyrank = np.empty((R, P), dtype=np.int32)
    logcnt = np.empty((R, E), dtype=np.int32)
    log2phy = np.empty((R, E, max(X, 1)), dtype=np.int32)
    rc = _load().oracle_rebalance(_ptr(loads), R, E, P, num_groups, num_nodes, num_gpus, X,
                                  _ptr(phy2log), _ptr(phyrank), _ptr(logcnt), _ptr(log2phy))
    if rc != OK:
        raise OracleError(rc)
    return phy2log, phyrank, logcnt, log2phy


def redirect(idx: np.ndarray, log2phy: np.ndarray, logcnt: np.ndarray, t0: int = 0):
    """S5: out[l, t, k] = log2phy[l, e, (t0 + t) mod logcnt[l, e]], e = idx[l, t, k].

    Returns (out int32 [L, T, K], bad); out-of-range indices give -1.
    """
    idx = _c(idx, np.int32)
    log2phy = _c(log2phy, np.int32)
    logcnt = _c(logcnt, np.int32)
    L, T, K = idx.shape
    _, E, X = log2phy.shape
    out = np.empty_like(idx)
    bad = ctypes.c_uint64(0)
    _load().oracle_redirect(_ptr(idx), L, T, K, E, _ptr(log2phy), X, _ptr(logcnt), t0,
                            _ptr(out), ctypes.addressof(bad))
    return out, int(bad.value)


def balanced_packing(weight, num_packs: int):
    """One row of balanced_packing on integer weights -> (pack_index, rank_in_pack)."""
    w = _c(weight, np.int64)
    n = w.shape[0]
    pi = np.empty(n, dtype=np.int32)
    ri = np.empty(n, dtype=np.int32)
    rc = _load().oracle_balanced_packing(_ptr(w), n, num_packs, _ptr(pi), _ptr(ri))
    if rc != OK:
        raise OracleError(rc)
    return pi, ri


def balanced_packing_frac(num, den, num_packs: int):
    """One row of balanced_packing on exact fractions num/den."""
    num = _c(num, np.int64)
    den = _c(den, np.int32)
    n = num.shape[0]
    pi = np.empty(n, dtype=np.int32)
    ri = np.empty(n, dtype=np.int32)
    rc = _load().oracle_balanced_packing_frac(_ptr(num), _ptr(den), n, num_packs, _ptr(pi), _ptr(ri))
    if rc != OK:
        raise OracleError(rc)
    return pi, ri


def replicate_experts(weight, num_phy: int):
    """One row of replicate_experts -> (phy2log [num_phy], rank [num_phy], logcnt [num_log])."""
    w = _c(weight, np.int64)
    n = w.shape[0]
    p = np.empty(num_phy, dtype=np.int32)
    r = np.empty(num_phy, dtype=np.int32)
    c = np.empty(n, dtype=np.int32)
    _load().oracle_replicate_experts(_ptr(w), n, num_phy, _ptr(p), _ptr(r), _ptr(c))
    return p, r, c


def plan_stats(loads, phy2log, logcnt, num_gpus: int):
    """Per-GPU load (sum of w/logcnt over the GPU's replicas, fp64, slot order)
    and per-row {min, max, mean, mean/max}."""
    loads = _c(loads, np.int64)
    phy2log = _c(phy2log, np.int32)
    logcnt = _c(logcnt, np.int32)
    R, E = loads.shape
    P = phy2log.shape[1]
    gl = np.empty((R, num_gpus), dtype=np.float64)
    st = np.empty((R, 4), dtype=np.float64)
    _load().oracle_plan_stats(_ptr(loads), _ptr(phy2log), _ptr(logcnt), R, E, P, num_gpus,
                              _ptr(gl), _ptr(st))
    return gl, st


def fold_loads(phys, phy2log, num_logical: int):
    """logical[r, e] = sum of phys[r, p] over slots p with phy2log[r, p] == e."""
    phys = _c(phys, np.int64)
    phy2log = _c(phy2log, np.int32)
    R, P = phys.shape
    out = np.empty((R, num_logical), dtype=np.int64)
    _load().oracle_fold_loads(_ptr(phys), _ptr(phy2log), R, num_logical, P, _ptr(out))
    return out


def initial_map(R: int, num_logical: int, num_replicas: int):
    """phy2log[p] = p mod E (routed experts first, then redundant), phyrank = p div E."""
    p2l = np.empty((R, num_replicas), dtype=np.int32)
    prk = np.empty((R, num_replicas), dtype=np.int32)
    _load().oracle_initial_map(R, num_logical, num_replicas, _ptr(p2l), _ptr(prk))
    return p2l, prk


def plan_diff(old_phy2log, new_phy2log, num_logical: int, num_gpus: int):
    """src[r, p]: -1 if new slot p's expert stays on its GPU, else the old slot to copy
    from; moves[r]: number of copies."""
    old = _c(old_phy2log, np.int32)
    new = _c(new_phy2log, np.int32)
    R, P = new.shape
    src = np.empty((R, P), dtype=np.int32)
    moves = np.empty(R, dtype=np.int32)
    rc = _load().oracle_plan_diff(_ptr(old), _ptr(new), R, num_logical, P, num_gpus, _ptr(src),
                                  _ptr(moves))
    if rc != OK:
        raise OracleError(rc)
    return src, moves
