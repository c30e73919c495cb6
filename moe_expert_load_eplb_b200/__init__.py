"""B200-native EPLB hot path: Python binding of libeplb.so.

The four stages of the Expert-Parallelism Load Balancer's data path run in
hand-written sm_100a kernels behind a C ABI (``include/eplb.h``); this module
only marshals torch CUDA tensors (pointers, sizes, the current stream) into
those calls.  There is no fallback: if ``libeplb.so`` is missing or no CUDA
device is present, every call raises.

    counts  = count_loads(idx, E)                        # S1  int64 [L, E]
    snaps   = window_accumulate(steps, W)                # S2  int64 [S, L, E]
    plan    = rebalance(loads, P, G, N, gpus)            # S3/S4 Plan(phy2log, phyrank, logcnt, log2phy)
    phys    = redirect(idx, plan.log2phy, plan.logcnt)   # S5  int32 [L, T, K]

Sources: page "DualPipe и EPLB: конвейер в обе стороны и балансировщик
экспертов" (EPLB README translation with the eplb.py appendix) and the LPLB
usage example (page "DeepSeek开源LPLB：基于线性规划的MoE负载均衡器").
"""
from __future__ import annotations

import ctypes
import os
from typing import NamedTuple, Optional

import torch

__all__ = [
    "EplbError", "Plan", "count_loads", "window_accumulate", "rebalance", "redirect", "count_redirect",
    "plan_stats", "fold_loads", "initial_map", "plan_diff", "rebalance_window", "serve_step",
    "serve_step_noalloc",
    "default_slots", "lib_path", "load_library", "STATUS",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
# EPLB_LIBRARY=checks selects the checking build (internal index checks that
# report EPLB_ERR_INTERNAL; same ABI and results), built with
# `python -m moe_expert_load_eplb_b200.build --checks`
_LIB_PATH = os.path.join(_PKG, "libeplb_checks.so" if os.environ.get("EPLB_LIBRARY") == "checks"
                         else "libeplb.so")

STATUS = {
    0: "EPLB_OK", 1: "EPLB_ERR_NULL", 2: "EPLB_ERR_SHAPE", 3: "EPLB_ERR_DIVISIBILITY",
    4: "EPLB_ERR_RANGE", 5: "EPLB_ERR_SLOTS", 6: "EPLB_ERR_CUDA", 7: "EPLB_ERR_TIMEOUT",
    8: "EPLB_ERR_ALIGN", 9: "EPLB_ERR_LIMIT", 10: "EPLB_ERR_INTERNAL",
}


class EplbError(RuntimeError):
    """A non-zero eplb_status returned by the C ABI (or read from a status word)."""

    def __init__(self, code: int, where: str, detail: str = ""):
        self.code = int(code)
        msg = f"{where}: {STATUS.get(self.code, self.code)}"
        super().__init__(msg + (f" ({detail})" if detail else ""))


class Plan(NamedTuple):
    phy2log: torch.Tensor   # int32 [R, P]
    phyrank: torch.Tensor   # int32 [R, P]
    logcnt: torch.Tensor    # int32 [R, E]
    log2phy: torch.Tensor   # int32 [R, E, X]


_lib = None


def lib_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libeplb.so (built by ``python -m moe_expert_load_eplb_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing: build it with "
                          "`python -m moe_expert_load_eplb_b200.build` (nvcc, sm_100a; "
                          "--checks for the checking build)")
    lib = ctypes.CDLL(_LIB_PATH)
    p, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    sig = {
        "eplb_status_string": ([i32], ctypes.c_char_p),
        "eplb_last_cuda_error": ([], ctypes.c_char_p),
        "eplb_abi_version": ([], i32),
        "eplb_checking_build": ([], i32),
        "eplb_count_loads": ([p, i64, i64, i32, i32, p, i32, p, p], i32),
        "eplb_window_accumulate": ([p, i64, i64, i32, i64, i64, p, i64, p], i32),
        "eplb_rebalance": ([p, i64, i32, i32, i32, i32, i32, i32, p, p, p, p, p, p, p, p], i32),
        "eplb_redirect": ([p, i64, i64, i32, i32, p, i32, p, i64, p, p, p, p], i32),
        "eplb_count_redirect": ([p, i64, i64, i32, i32, p, i32, p, i32, p, i64, p, p, p, p], i32),
        "eplb_plan_stats": ([p, p, p, i64, i32, i32, i32, p, p, p, p], i32),
        "eplb_rebalance_window": ([p, i64, i64, i64, i32, i32, i32, i32, i32, i32, p, p, p, p, p, p,
                                   p, p, p], i32),
        "eplb_fold_loads": ([p, p, i64, i32, i32, p, p, p], i32),
        "eplb_initial_map": ([i64, i32, i32, p, p, p], i32),
        "eplb_plan_diff": ([p, p, i64, i32, i32, i32, p, p, p, p], i32),
        "eplb_serve_step": ([p, i64, i64, i32, i32, p, i32, p, i64, p, p, p, i64, i64, i64,
                             i32, i32, i32, i32, p, p, p, p, p, p, p, p, p, p], i32),
        "eplb_serve_step_noalloc": ([p, i64, i64, i32, i32, p, i32, p, i64, p, p, p, i64, i64,
                                     i64, i32, i32, i32, i32, p, p, p, p, p, p, p, p, p], i32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def _check(code: int, where: str):
    if code != 0:
        detail = load_library().eplb_last_cuda_error().decode() if code == 6 else ""
        raise EplbError(code, where, detail)


def _cuda(t: torch.Tensor, dtype: torch.dtype, name: str,
          device: Optional[torch.device] = None) -> torch.Tensor:
    """t must be a contiguous CUDA tensor of dtype (on ``device`` if given):
    the C ABI takes bare pointers and cannot check any of it."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}; the call runs on {device}")
    return t


_BAD_DTYPES = (torch.int64, torch.uint64)


def _word(t: Optional[torch.Tensor], dtypes, name: str, device: torch.device):
    """An optional device word: the bad-index tally (64-bit) or the status
    word (int32).  None passes a null pointer (the word is not written)."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} must be one of {dtypes}, got {t.dtype}")
    if t.numel() < 1:
        raise ValueError(f"{name} must hold at least one element")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}; the call runs on {device}")
    return t


def _words(device: torch.device, bad=None, status=None):
    _word(bad, _BAD_DTYPES, "bad", device)
    _word(status, (torch.int32,), "status", device)


def _check_quality(gpu_load: Optional[torch.Tensor], stats: Optional[torch.Tensor], R: int,
                   gpus: int, device: torch.device):
    """The optional plan-quality outputs: float64 gpu_load [R, gpus] and
    stats [R, 4] (min, max, mean, mean / max of the GPU loads)."""
    if gpu_load is not None:
        _cuda(gpu_load, torch.float64, "gpu_load", device)
        if tuple(gpu_load.shape) != (R, gpus):
            raise ValueError(f"gpu_load must be {(R, gpus)}")
    if stats is not None:
        _cuda(stats, torch.float64, "stats", device)
        if tuple(stats.shape) != (R, 4):
            raise ValueError(f"stats must be {(R, 4)}")


def _check_plan(plan, name: str, R: int, E: int, X: int, P: Optional[int],
                device: torch.device):
    """The four plan tensors: log2phy [R, E, X], logcnt [R, E] and, if P is
    given, phy2log / phyrank [R, P]; all int32 on ``device``."""
    _cuda(plan.log2phy, torch.int32, f"{name}.log2phy", device)
    _cuda(plan.logcnt, torch.int32, f"{name}.logcnt", device)
    if tuple(plan.log2phy.shape) != (R, E, X) or tuple(plan.logcnt.shape) != (R, E):
        raise ValueError(f"{name}: log2phy must be {(R, E, X)} and logcnt {(R, E)}")
    if P is not None:
        _cuda(plan.phy2log, torch.int32, f"{name}.phy2log", device)
        _cuda(plan.phyrank, torch.int32, f"{name}.phyrank", device)
        if tuple(plan.phy2log.shape) != (R, P) or tuple(plan.phyrank.shape) != (R, P):
            raise ValueError(f"{name}: phy2log and phyrank must be {(R, P)}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(device: torch.device):
    """The current stream of ``device`` as a raw handle."""
    if _raw_stream is not None:
        return ctypes.c_void_p(_raw_stream(device.index if device.index is not None
                                           else torch.cuda.current_device()))
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


class _on_device:
    """Makes ``device`` current for the call; free when it already is."""

    __slots__ = ("index", "prev")

    def __init__(self, device: torch.device):
        self.index = device.index
        self.prev = None

    def __enter__(self):
        if self.index is not None:
            cur = torch.cuda.current_device()
            if cur != self.index:
                self.prev = cur
                torch.cuda.set_device(self.index)
        return self

    def __exit__(self, *exc):
        if self.prev is not None:
            torch.cuda.set_device(self.prev)
        return False


def count_loads(idx: torch.Tensor, num_experts: int, counts: Optional[torch.Tensor] = None,
                accumulate: bool = False, bad: Optional[torch.Tensor] = None) -> torch.Tensor:
    """S1: counts[l, e] (+)= #{(t, k): idx[l, t, k] == e} for int32 idx [L, T, K]."""
    _cuda(idx, torch.int32, "idx")
    if idx.dim() != 3:
        raise ValueError("idx must be [L, T, K]")
    L, T, K = idx.shape
    if counts is None:
        counts = torch.empty((L, num_experts), dtype=torch.int64, device=idx.device)
        accumulate = False
    _cuda(counts, torch.int64, "counts", idx.device)
    if tuple(counts.shape) != (L, num_experts):
        raise ValueError("counts must be [L, E]")
    _words(idx.device, bad)
    with _on_device(idx.device):
        _check(load_library().eplb_count_loads(
            _ptr(idx), L, T, K, num_experts, _ptr(counts), int(bool(accumulate)),
            _ptr(bad), _stream(idx.device)), "eplb_count_loads")
    return counts


def window_accumulate(steps: torch.Tensor, window: int, s_first: int = 0,
                      out: Optional[torch.Tensor] = None, zero_row: int = -1) -> torch.Tensor:
    """S2: out[s - s_first] = sum of steps[max(0, s-window+1) .. s] (int64 [S, L, E]);
    zero_row >= 0 clears that row of ``steps`` after it has been read."""
    _cuda(steps, torch.int64, "steps")
    if steps.dim() != 3:
        raise ValueError("steps must be [S, L, E]")
    S, L, E = steps.shape
    if out is None:
        out = torch.empty((max(S - s_first, 0), L, E), dtype=torch.int64, device=steps.device)
    _cuda(out, torch.int64, "out", steps.device)
    if tuple(out.shape) != (S - s_first, L, E):
        raise ValueError("out must be [S - s_first, L, E]")
    with _on_device(steps.device):
        _check(load_library().eplb_window_accumulate(
            _ptr(steps), S, L, E, window, s_first, _ptr(out), int(zero_row), _stream(steps.device)),
            "eplb_window_accumulate")
    return out


def default_slots(num_logical: int, num_replicas: int, num_groups: int, num_nodes: int) -> int:
    """log2phy width that always suffices: the most replicas one expert can get."""
    nodes = num_nodes if num_nodes > 0 and num_groups % num_nodes == 0 else 1
    return max(1, (num_replicas - num_logical) // nodes + 1)


def rebalance(loads: torch.Tensor, num_replicas: int, num_groups: int, num_nodes: int,
              num_gpus: int, slots: Optional[int] = None, out: Optional[Plan] = None,
              status: Optional[torch.Tensor] = None, gpu_load: Optional[torch.Tensor] = None,
              stats: Optional[torch.Tensor] = None) -> Plan:
    """S3/S4: rebalance_experts for every row of int64 loads [R, E] (hierarchical
    policy when num_groups % num_nodes == 0, else global).  ``gpu_load``
    (float64 [R, gpus]) and ``stats`` (float64 [R, 4]), if given, receive the
    new plans' quality in the same launch (the figures of ``plan_stats``)."""
    _cuda(loads, torch.int64, "loads")
    if loads.dim() != 2:
        raise ValueError("loads must be [R, E]")
    R, E = loads.shape
    P = num_replicas
    X = default_slots(E, P, num_groups, num_nodes) if slots is None else slots
    dev = loads.device
    if out is None:
        out = Plan(torch.empty((R, P), dtype=torch.int32, device=dev),
                   torch.empty((R, P), dtype=torch.int32, device=dev),
                   torch.empty((R, E), dtype=torch.int32, device=dev),
                   torch.empty((R, E, X), dtype=torch.int32, device=dev))
    for name, t, shape in (("phy2log", out.phy2log, (R, P)), ("phyrank", out.phyrank, (R, P)),
                           ("logcnt", out.logcnt, (R, E)), ("log2phy", out.log2phy, (R, E, X))):
        _cuda(t, torch.int32, name, dev)
        if tuple(t.shape) != shape:
            raise ValueError(f"{name} must be {shape}")
    _words(dev, status=status)
    _check_quality(gpu_load, stats, R, num_gpus, dev)
    with _on_device(dev):
        _check(load_library().eplb_rebalance(
            _ptr(loads), R, E, P, num_groups, num_nodes, num_gpus, X,
            _ptr(out.phy2log), _ptr(out.phyrank), _ptr(out.logcnt), _ptr(out.log2phy),
            _ptr(gpu_load), _ptr(stats), _ptr(status), _stream(dev)), "eplb_rebalance")
    return out


def rebalance_window(ring: torch.Tensor, num_replicas: int, num_groups: int, num_nodes: int,
                     num_gpus: int, zero_slot: int = -1, slots: Optional[int] = None,
                     out: Optional[Plan] = None, loads_out: Optional[torch.Tensor] = None,
                     status: Optional[torch.Tensor] = None, gpu_load: Optional[torch.Tensor] = None,
                     stats: Optional[torch.Tensor] = None) -> Plan:
    """S2 + S3/S4 in one launch: rebalance_experts on the window sum of a ring of
    per-step counts (int64 [W, R, E]); zero_slot >= 0 clears that ring row after
    reading it (the next step's counting slot).  ``gpu_load`` / ``stats`` as
    for ``rebalance``."""
    _cuda(ring, torch.int64, "ring")
    if ring.dim() != 3:
        raise ValueError("ring must be [W, R, E]")
    Wr, R, E = ring.shape
    P = num_replicas
    X = default_slots(E, P, num_groups, num_nodes) if slots is None else slots
    dev = ring.device
    if out is None:
        out = Plan(torch.empty((R, P), dtype=torch.int32, device=dev),
                   torch.empty((R, P), dtype=torch.int32, device=dev),
                   torch.empty((R, E), dtype=torch.int32, device=dev),
                   torch.empty((R, E, X), dtype=torch.int32, device=dev))
    for name, t, shape in (("phy2log", out.phy2log, (R, P)), ("phyrank", out.phyrank, (R, P)),
                           ("logcnt", out.logcnt, (R, E)), ("log2phy", out.log2phy, (R, E, X))):
        _cuda(t, torch.int32, name, dev)
        if tuple(t.shape) != shape:
            raise ValueError(f"{name} must be {shape}")
    _words(dev, status=status)
    if loads_out is not None:
        _cuda(loads_out, torch.int64, "loads_out", dev)
        if tuple(loads_out.shape) not in ((R, E), (1, R, E)):
            raise ValueError("loads_out must be [R, E]")
    _check_quality(gpu_load, stats, R, num_gpus, dev)
    with _on_device(dev):
        _check(load_library().eplb_rebalance_window(
            _ptr(ring), Wr, zero_slot, R, E, P, num_groups, num_nodes, num_gpus, X, _ptr(loads_out),
            _ptr(out.phy2log), _ptr(out.phyrank), _ptr(out.logcnt), _ptr(out.log2phy),
            _ptr(gpu_load), _ptr(stats), _ptr(status), _stream(dev)), "eplb_rebalance_window")
    return out


def redirect(idx: torch.Tensor, log2phy: torch.Tensor, logcnt: torch.Tensor, token_offset: int = 0,
             out: Optional[torch.Tensor] = None, bad: Optional[torch.Tensor] = None,
             status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """S5: out[l, t, k] = log2phy[l, e, (token_offset + t) mod logcnt[l, e]], e = idx[l, t, k]."""
    _cuda(idx, torch.int32, "idx")
    _cuda(log2phy, torch.int32, "log2phy", idx.device)
    _cuda(logcnt, torch.int32, "logcnt", idx.device)
    if idx.dim() != 3 or log2phy.dim() != 3 or logcnt.dim() != 2:
        raise ValueError("idx [L, T, K], log2phy [L, E, X], logcnt [L, E] expected")
    L, T, K = idx.shape
    _, E, X = log2phy.shape
    if log2phy.shape[0] != L or tuple(logcnt.shape) != (L, E):
        raise ValueError("table shapes do not match idx")
    if out is None:
        out = torch.empty_like(idx)
    _cuda(out, torch.int32, "out", idx.device)
    if out.shape != idx.shape:
        raise ValueError("out must match idx")
    _words(idx.device, bad, status)
    with _on_device(idx.device):
        _check(load_library().eplb_redirect(
            _ptr(idx), L, T, K, E, _ptr(log2phy), X, _ptr(logcnt), int(token_offset),
            _ptr(out), _ptr(bad), _ptr(status), _stream(idx.device)), "eplb_redirect")
    return out


def count_redirect(idx: torch.Tensor, num_experts: int, log2phy: torch.Tensor, logcnt: torch.Tensor,
                   token_offset: int = 0, counts: Optional[torch.Tensor] = None,
                   accumulate: bool = False, out: Optional[torch.Tensor] = None,
                   bad: Optional[torch.Tensor] = None,
                   status: Optional[torch.Tensor] = None):
    """S1 + S5 in one pass over idx: counts (+)= histogram of idx and
    out = redirect(idx, log2phy, logcnt, token_offset).  Returns (counts, out)."""
    _cuda(idx, torch.int32, "idx")
    _cuda(log2phy, torch.int32, "log2phy", idx.device)
    _cuda(logcnt, torch.int32, "logcnt", idx.device)
    if idx.dim() != 3 or log2phy.dim() != 3 or logcnt.dim() != 2:
        raise ValueError("idx [L, T, K], log2phy [L, E, X], logcnt [L, E] expected")
    L, T, K = idx.shape
    _, E, X = log2phy.shape
    if E != num_experts or log2phy.shape[0] != L or tuple(logcnt.shape) != (L, E):
        raise ValueError("table shapes do not match idx / num_experts")
    if counts is None:
        counts = torch.empty((L, E), dtype=torch.int64, device=idx.device)
        accumulate = False
    _cuda(counts, torch.int64, "counts", idx.device)
    if tuple(counts.shape) != (L, E):
        raise ValueError("counts must be [L, E]")
    if out is None:
        out = torch.empty_like(idx)
    _cuda(out, torch.int32, "out", idx.device)
    if out.shape != idx.shape:
        raise ValueError("out must match idx")
    _words(idx.device, bad, status)
    with _on_device(idx.device):
        _check(load_library().eplb_count_redirect(
            _ptr(idx), L, T, K, E, _ptr(counts), int(bool(accumulate)), _ptr(log2phy), X,
            _ptr(logcnt), int(token_offset), _ptr(out), _ptr(bad), _ptr(status),
            _stream(idx.device)), "eplb_count_redirect")
    return counts, out


def _serve_args(idx, plan, ring, next_plan, out, loads_out, bad, status):
    """Checks shared by both one-launch entry points; returns (L, T, K, W, E,
    P, X, out)."""
    _cuda(idx, torch.int32, "idx")
    dev = idx.device
    _cuda(ring, torch.int64, "ring", dev)
    if idx.dim() != 3 or ring.dim() != 3:
        raise ValueError("idx [L, T, K] and ring [W, L, E] expected")
    L, T, K = idx.shape
    Wr, Lr, E = ring.shape
    if Lr != L:
        raise ValueError("ring and idx disagree on L")
    if next_plan.phy2log.dim() != 2 or plan.log2phy.dim() != 3:
        raise ValueError("plan.log2phy [L, E, X] and next_plan.phy2log [L, P] expected")
    P = next_plan.phy2log.shape[1]
    X = plan.log2phy.shape[2]
    _check_plan(plan, "plan", L, E, X, None, dev)
    _check_plan(next_plan, "next_plan", L, E, X, P, dev)
    if out is None:
        out = torch.empty_like(idx)
    _cuda(out, torch.int32, "out", dev)
    if out.shape != idx.shape:
        raise ValueError("out must match idx")
    if loads_out is not None:
        _cuda(loads_out, torch.int64, "loads_out", dev)
        if loads_out.numel() != L * E:
            raise ValueError("loads_out must be [L, E]")
    _words(dev, bad, status)
    return L, T, K, Wr, E, P, X, out


def serve_step(idx: torch.Tensor, plan: Plan, ring: torch.Tensor, slot: int, next_plan: Plan,
               layer_done: torch.Tensor, num_groups: int, num_nodes: int, num_gpus: int,
               zero_slot: int = -1, token_offset: int = 0, out: Optional[torch.Tensor] = None,
               loads_out: Optional[torch.Tensor] = None, bad: Optional[torch.Tensor] = None,
               status: Optional[torch.Tensor] = None, gpu_load: Optional[torch.Tensor] = None,
               stats: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The serving step in one launch: count idx into ring[slot] and redirect it
    with ``plan`` (the plan in force), then rebuild every layer's plan from the
    window sum over the ring into ``next_plan`` (clearing ring[zero_slot]).
    ``layer_done``: uint32 [L] work array, zero before and after;
    ``gpu_load`` / ``stats``: the next plan's quality, as for ``rebalance``.
    Returns out."""
    L, T, K, Wr, E, P, X, out = _serve_args(idx, plan, ring, next_plan, out, loads_out, bad,
                                            status)
    if not isinstance(layer_done, torch.Tensor) or not layer_done.is_cuda or \
            layer_done.dtype != torch.uint32 or layer_done.numel() != L:
        raise TypeError("layer_done must be a CUDA uint32 tensor of L elements")
    if not layer_done.is_contiguous() or layer_done.device != idx.device:
        raise ValueError("layer_done must be contiguous and on the device of idx")
    _check_quality(gpu_load, stats, L, num_gpus, idx.device)
    with _on_device(idx.device):
        _check(load_library().eplb_serve_step(
            _ptr(idx), L, T, K, E, _ptr(plan.log2phy), X, _ptr(plan.logcnt), int(token_offset),
            _ptr(out), _ptr(bad), _ptr(ring), Wr, slot, zero_slot, P, num_groups, num_nodes,
            num_gpus, _ptr(loads_out), _ptr(next_plan.phy2log), _ptr(next_plan.phyrank),
            _ptr(next_plan.logcnt), _ptr(next_plan.log2phy), _ptr(gpu_load), _ptr(stats),
            _ptr(layer_done), _ptr(status), _stream(idx.device)), "eplb_serve_step")
    return out


def serve_step_noalloc(idx: torch.Tensor, plan: Plan, ring: torch.Tensor, slot: int,
                       next_plan: Plan, num_groups: int, num_nodes: int, num_gpus: int,
                       zero_slot: int = -1, token_offset: int = 0,
                       out: Optional[torch.Tensor] = None,
                       loads_out: Optional[torch.Tensor] = None,
                       bad: Optional[torch.Tensor] = None,
                       status: Optional[torch.Tensor] = None,
                       gpu_load: Optional[torch.Tensor] = None,
                       stats: Optional[torch.Tensor] = None) -> torch.Tensor:
    """serve_step with the library's own per-layer counters (no work array;
    calls must not overlap on one device).  ``out`` must be given or is
    allocated here by torch, outside the call."""
    L, T, K, Wr, E, P, X, out = _serve_args(idx, plan, ring, next_plan, out, loads_out, bad,
                                            status)
    _check_quality(gpu_load, stats, L, num_gpus, idx.device)
    with _on_device(idx.device):
        _check(load_library().eplb_serve_step_noalloc(
            _ptr(idx), L, T, K, E, _ptr(plan.log2phy), X, _ptr(plan.logcnt), int(token_offset),
            _ptr(out), _ptr(bad), _ptr(ring), Wr, slot, zero_slot, P, num_groups, num_nodes,
            num_gpus, _ptr(loads_out), _ptr(next_plan.phy2log), _ptr(next_plan.phyrank),
            _ptr(next_plan.logcnt), _ptr(next_plan.log2phy), _ptr(gpu_load), _ptr(stats),
            _ptr(status), _stream(idx.device)), "eplb_serve_step_noalloc")
    return out


def plan_stats(loads: torch.Tensor, phy2log: torch.Tensor, logcnt: torch.Tensor, num_gpus: int,
               status: Optional[torch.Tensor] = None):
    """Per-GPU load (fp64, sum of w/logcnt over the GPU's slots in order) and
    per-row stats {min, max, mean, mean/max}.  Returns (gpu_load [R, gpus], stats [R, 4])."""
    _cuda(loads, torch.int64, "loads")
    _cuda(phy2log, torch.int32, "phy2log", loads.device)
    _cuda(logcnt, torch.int32, "logcnt", loads.device)
    if loads.dim() != 2 or phy2log.dim() != 2:
        raise ValueError("loads [R, E] and phy2log [R, P] expected")
    R, E = loads.shape
    P = phy2log.shape[1]
    if phy2log.shape[0] != R or tuple(logcnt.shape) != (R, E):
        raise ValueError("phy2log must be [R, P] and logcnt [R, E]")
    _words(loads.device, status=status)
    gl = torch.empty((R, num_gpus), dtype=torch.float64, device=loads.device)
    st = torch.empty((R, 4), dtype=torch.float64, device=loads.device)
    with _on_device(loads.device):
        _check(load_library().eplb_plan_stats(
            _ptr(loads), _ptr(phy2log), _ptr(logcnt), R, E, P, num_gpus, _ptr(gl), _ptr(st),
            _ptr(status), _stream(loads.device)), "eplb_plan_stats")
    return gl, st


def fold_loads(phys: torch.Tensor, phy2log: torch.Tensor, num_logical: int,
               status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """logical[r, e] = sum of phys[r, p] over slots with phy2log[r, p] == e."""
    _cuda(phys, torch.int64, "phys")
    _cuda(phy2log, torch.int32, "phy2log", phys.device)
    if phys.dim() != 2 or phy2log.shape != phys.shape:
        raise ValueError("phys and phy2log must both be [R, P]")
    R, P = phys.shape
    _words(phys.device, status=status)
    out = torch.empty((R, num_logical), dtype=torch.int64, device=phys.device)
    with _on_device(phys.device):
        _check(load_library().eplb_fold_loads(
            _ptr(phys), _ptr(phy2log), R, num_logical, P, _ptr(out), _ptr(status),
            _stream(phys.device)), "eplb_fold_loads")
    return out


def initial_map(rows: int, num_logical: int, num_replicas: int, device="cuda"):
    """phy2log[r, p] = p mod E, phyrank[r, p] = p div E (routed first, then redundant)."""
    p2l = torch.empty((rows, num_replicas), dtype=torch.int32, device=device)
    prk = torch.empty((rows, num_replicas), dtype=torch.int32, device=device)
    dev = p2l.device
    with _on_device(dev):
        _check(load_library().eplb_initial_map(rows, num_logical, num_replicas, _ptr(p2l), _ptr(prk),
                                               _stream(dev)), "eplb_initial_map")
    return p2l, prk


def plan_diff(old_phy2log: torch.Tensor, new_phy2log: torch.Tensor, num_logical: int, num_gpus: int,
              status: Optional[torch.Tensor] = None):
    """src[r, p] = -1 where the new slot keeps its expert on its GPU, else the old slot
    to copy from; moves[r] = number of copies.  Returns (src, moves)."""
    _cuda(new_phy2log, torch.int32, "new_phy2log")
    _cuda(old_phy2log, torch.int32, "old_phy2log", new_phy2log.device)
    if new_phy2log.dim() != 2 or old_phy2log.shape != new_phy2log.shape:
        raise ValueError("plans must both be [R, P]")
    R, P = new_phy2log.shape
    _words(new_phy2log.device, status=status)
    src = torch.empty((R, P), dtype=torch.int32, device=new_phy2log.device)
    moves = torch.empty((R,), dtype=torch.int32, device=new_phy2log.device)
    with _on_device(new_phy2log.device):
        _check(load_library().eplb_plan_diff(
            _ptr(old_phy2log), _ptr(new_phy2log), R, num_logical, P, num_gpus, _ptr(src),
            _ptr(moves), _ptr(status), _stream(new_phy2log.device)), "eplb_plan_diff")
    return src, moves
