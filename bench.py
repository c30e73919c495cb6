"""Benchmark of the EPLB hot path on B200: one step = count -> window ->
rebalance -> redirect over the DeepSeek-V3-shaped prefill workload.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload (per rank): 58 MoE layers x 65,536 tokens x top-8 group-limited
routed int32 indices over 256 experts in 8 groups (popularity log-normal,
seeded, synthetic), a 16-step load window, plans of 288 physical experts
over 4 nodes x 8 GPUs.  Metric: layer-rebalances per second of the whole
step; the load-count and redirect kernels are reported against the measured
HBM bandwidth.  Rank 0 prints one JSON line.

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and a
device synchronisation; each step is timed on its stream with CUDA events
(one between every two stages); L2 is flushed (a 512 MB write) between steps,
outside the events.  With N > 1 (torchrun) every rank counts and redirects
its own 65,536 tokens per layer and the per-step counts are summed with one
NCCL all-reduce; every rank then computes the same plan.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

CFG = W.DSV3_PREFILL
WINDOW = 16
METRIC = "EPLB layer-rebalances/sec on 1 B200 + load-count GB/s vs HBM peak"
UNIT = "layer-rebalances/s"
FLUSH_BYTES = 512 << 20


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--clock-ms", type=float, default=400.0,
                    help="repeat the timed region until the clock record spans about this long")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer e2e measurement")
    ap.add_argument("--no-fresh", action="store_true", help="skip the fresh-plan-order comparison")
    ap.add_argument("--fresh-only", action="store_true",
                    help="time only the fresh-plan order (for profiling its kernels)")
    ap.add_argument("--legs", default="hbm_stream,global_policy,window_sweep",
                    help="single-GPU legs on the other workloads, comma-separated ('' for none)")
    ap.add_argument("--legs-only", action="store_true",
                    help="run only the legs (no serving step): for profiling their kernels")
    a = ap.parse_args()
    a.legs = [x for x in a.legs.split(",") if x]
    return a


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def _config(world: int) -> dict:
    return {"workload": CFG.name, "layers": CFG.L, "experts": CFG.E, "groups": CFG.G,
            "replicas": CFG.P, "nodes": CFG.N, "plan_gpus": CFG.gpus,
            "tokens_per_layer_per_rank": CFG.T, "top_k": CFG.K, "window": WINDOW,
            "l2": "flushed between steps (512 MB write)", "parallelism": f"dp{world}"}


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML while running."""

    NAMES = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
             0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks",
             0x10: "sync_boost", 0x100: "display_clock"}

    def __init__(self, device: int, period: float = 0.002):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period, self._stop, self.ok = period, threading.Event(), False
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device)
            uuid = getattr(props, "uuid", None)
            h = None
            if uuid is not None:
                try:
                    h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + str(uuid)).encode())
                except Exception:
                    h = None
            if h is None:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES")
                phys = int(vis.split(",")[device]) if vis and vis.split(",")[device].isdigit() else device
                h = pynvml.nvmlDeviceGetHandleByIndex(phys)
            self.h, self.nv = h, pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        nv = self.nv
        get_r = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        self.t_first = self.t_last = None
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.t_last = time.perf_counter()
                if self.t_first is None:
                    self.t_first = self.t_last
                r = get_r(self.h)
                for bit, name in self.NAMES.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return None
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "sm_mhz_min": min(self.samples), "reasons": sorted(self.reasons),
                "samples": len(self.samples),
                "span_ms": round(1e3 * (self.t_last - self.t_first), 1) if self.t_first else 0.0}


# --------------------------------------------------------------- profiles --

def _kernel_sha(name: str) -> str:
    """sha256 (first 16 hex digits) of a kernel's source; several files
    separated by '+' are hashed in that order."""
    h = hashlib.sha256()
    for part in name.split("+"):
        with open(os.path.join(ROOT, "moe_expert_load_eplb_b200", "csrc", part), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


# B200 HBM3e datasheet bandwidth (about 8 TB/s), reported beside the measured peak
DATASHEET_HBM_GBS = 8000.0

# the serving-step kernel's code: its file and the two headers it inlines
SERVE_SOURCES = "serve.cu+redirect_chunk.cuh+rebalance_row.cuh"


def _traffic(kernel_file: str, profile: str, scale: float):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", profile)
    try:
        text = open(path).read()
    except OSError:
        return None
    m_sha = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", text)
    m_b = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not m_sha or not m_b or m_sha.group(1) != _kernel_sha(kernel_file):
        return None
    return float(m_b.group(1)) * scale


# --------------------------------------------------------------------- ours --

STAGES = ("count", "allreduce", "window", "rebalance", "redirect")


def _timed_steps(step, idx, flush, K, group, dev, staged=False, scrub=None, clock_ms=0.0):
    """Runs K steps, each between a start and an end event (the L2 flush
    before each step stays outside them); returns (total ms of the K steps,
    max over ranks; per-stage mean ms or None; clock summary; ms per step of
    every repeat).  With ``staged`` the step also records events between its
    stages for the per-stage breakdown -- those extra records cost time of
    their own, so the headline is taken without them.  ``scrub`` (a buffer
    larger than L2): read after the flush write, so that L2 holds clean
    lines and none of the flush's dirty lines is written back inside the
    timed step.  ``clock_ms``: the K-step region is then repeated (same
    count on every rank) until the clock sampler, running throughout, has
    seen about that many milliseconds; the first region is the one
    returned as the total, the repeats only widen the clock record."""
    n_ev = 6 if staged else 2

    def region():
        marks = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(K)]
        if group is not None:
            torch.distributed.barrier(group=group)
        torch.cuda.synchronize()
        for i in range(K):
            flush.fill_(i & 0xff)
            if scrub is not None:
                scrub.max()
            if staged:
                step(idx, marks[i])
            else:
                marks[i][0].record()
                step(idx)
                marks[i][1].record()
        torch.cuda.synchronize()
        if group is not None:
            torch.distributed.barrier(group=group)
        tot = torch.tensor([sum(m[0].elapsed_time(m[-1]) for m in marks)], dtype=torch.float64,
                           device=dev)
        if group is not None:
            torch.distributed.all_reduce(tot, op=torch.distributed.ReduceOp.MAX, group=group)
        return float(tot.item()), marks

    with ClockSampler(dev.index) as clocks:
        t_wall = time.perf_counter()
        total, marks = region()
        wall_ms = (time.perf_counter() - t_wall) * 1e3
        # a repeat count every rank derives from the same all-reduced figure
        reps = 0 if clock_ms <= 0 else min(2000, int(clock_ms / max(wall_ms, 1e-3)))
        if group is not None and reps:
            r = torch.tensor([reps], dtype=torch.int64, device=dev)
            torch.distributed.all_reduce(r, op=torch.distributed.ReduceOp.MIN, group=group)
            reps = int(r.item())
        repeats = [total / K]
        for _ in range(reps):
            repeats.append(region()[0] / K)
    per_stage = None
    if staged:
        per_stage = {n: statistics.mean(m[k].elapsed_time(m[k + 1]) for m in marks)
                     for k, n in enumerate(STAGES)}
    return total, per_stage, clocks.summary(), repeats


def _stage_report(per_stage, fused, X, world, hbm_peak):
    c = CFG
    n_idx = c.L * c.T * c.K
    algo = {"window": 8.0 * WINDOW * c.L * c.E + 8.0 * c.L * c.E,
            "rebalance": 8.0 * c.L * c.E + 4.0 * c.L * (2 * c.P + c.E + c.E * X)}
    if fused:
        algo["count"] = 8.0 * n_idx + 8.0 * c.L * c.E  # indices in, physical indices + counts out
        algo["rebalance"] += 8.0 * (WINDOW - 1) * c.L * c.E  # the ring rows it sums
    else:
        algo["count"] = 4.0 * n_idx
        algo["redirect"] = 8.0 * n_idx
    stages = {}
    names = (["count", "rebalance"] if fused else ["count", "window", "rebalance", "redirect"])
    names += ["allreduce"] if world > 1 else []
    for n in names:
        ms = per_stage[n]
        d = {"ms": round(ms, 5)}
        if n in algo and ms > 0:
            gbs = algo[n] / (ms / 1e3) / 1e9
            d.update(algo_bytes=algo[n], gbs=round(gbs, 1))
            if n != "rebalance":
                d["frac_hbm"] = round(gbs / hbm_peak, 4)
        stages[n] = d
    if fused:
        stages["count"]["kernel"] = "count_redirect (S1+S5 fused)"
        stages["rebalance"]["kernel"] = "rebalance_window (S2 ring sum + S3/S4 fused)"
    stages["rebalance"]["us_per_call"] = round(per_stage["rebalance"] * 1e3, 2)
    stages["rebalance"]["rows_per_s"] = round(c.L / (per_stage["rebalance"] / 1e3), 1)
    return stages


# ------------------------------------------------- the other configurations --
# Single-GPU legs on the pages' other workloads: the 16x larger routed batch
# (HBM streaming), the global policy over 144 GPUs and the 1000-step window
# sweep.  Each call is timed alone between CUDA events on the launching
# stream, with the clock sampler running; median over the calls.

def _time_calls(fn, n, dev, flush=None):
    """Times n calls of fn (after 3 untimed ones), each between two events on
    the current stream; ``flush`` is written before every call, outside the
    events.  Returns (median ms, mean ms, clock summary)."""
    for i in range(3):
        if flush is not None:
            flush.fill_(i & 0xff)
        fn()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(n)]
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clocks:
        for i in range(n):
            if flush is not None:
                flush.fill_(i & 0xff)
            ev[i][0].record()
            fn()
            ev[i][1].record()
        torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in ev]
    return statistics.median(ms), statistics.mean(ms), clocks.summary()


def _hbm_entry(algo_bytes, med, mean, clocks, hbm_peak, extra=None):
    gbs = algo_bytes / (med / 1e3) / 1e9
    d = {"ms": round(med, 5), "ms_mean": round(mean, 5), "algo_bytes": algo_bytes,
         "gbs": round(gbs, 1), "frac_hbm": round(gbs / hbm_peak, 4),
         "frac_of_datasheet": round(gbs / DATASHEET_HBM_GBS, 4), "clocks": clocks}
    if extra:
        d.update(extra)
    return d


def leg_hbm_stream(n, dev, hbm_peak):
    """hbm_stream: 58 layers x 1,048,576 tokens x top-8 (486.5 M int32
    indices, 1.95 GB).  count_loads, redirect and the fused count_redirect,
    each on the whole batch, against the plan rebuilt from the batch's own
    counts.  Inputs and outputs are 16x the L2, so no flush is needed."""
    import moe_expert_load_eplb_b200 as eplb
    c = W.HBM_STREAM
    torch.cuda.empty_cache()
    idx = W.routed_indices("hbm_stream", device=dev)
    n_idx = idx.numel()
    counts = eplb.count_loads(idx, c.E)
    plan = eplb.rebalance(counts, c.P, c.G, c.N, c.gpus)
    out = torch.empty_like(idx)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    res = {"workload": c.name, "layers": c.L, "tokens_per_layer": c.T, "top_k": c.K,
           "indices": n_idx, "calls": n, "l2": "not flushed: 1.95 GB in (+1.95 GB out) per call"}
    m = _time_calls(lambda: eplb.count_loads(idx, c.E, counts=counts), n, dev)
    res["count"] = _hbm_entry(4.0 * n_idx, *m, hbm_peak,
                              {"target_ms": round(4.0 * n_idx / (0.7 * hbm_peak * 1e9) * 1e3, 4)})
    m = _time_calls(lambda: eplb.redirect(idx, plan.log2phy, plan.logcnt, out=out, status=st), n, dev)
    res["redirect"] = _hbm_entry(8.0 * n_idx, *m, hbm_peak,
                                 {"target_ms": round(8.0 * n_idx / (0.7 * hbm_peak * 1e9) * 1e3, 4)})
    m = _time_calls(lambda: eplb.count_redirect(idx, c.E, plan.log2phy, plan.logcnt, counts=counts,
                                                out=out, status=st), n, dev)
    res["count_redirect"] = _hbm_entry(8.0 * n_idx + 8.0 * c.L * c.E, *m, hbm_peak)
    torch.cuda.synchronize()
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())} in the hbm_stream leg")
    del idx, out
    torch.cuda.empty_cache()
    return res


def leg_global_policy(n, dev, flush):
    """global_policy: rebalance_experts on 58 rows of 256 Pareto loads, 288
    replicas, one group over 2 nodes (global policy), 144 GPUs (two replicas
    each).  L2 flushed before every call."""
    import moe_expert_load_eplb_b200 as eplb
    c = W.GLOBAL_POLICY
    loads = torch.from_numpy(W.global_policy_loads()).to(dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    plan = eplb.rebalance(loads, c.P, c.G, c.N, c.gpus, status=st)
    med, mean, clocks = _time_calls(
        lambda: eplb.rebalance(loads, c.P, c.G, c.N, c.gpus, out=plan, status=st), n, dev, flush)
    torch.cuda.synchronize()
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())} in the global_policy leg")
    return {"workload": c.name, "rows": c.L, "experts": c.E, "replicas": c.P, "plan_gpus": c.gpus,
            "policy": "global", "calls": n, "l2": "flushed before every call (512 MB write)",
            "rebalance": {"us_per_call": round(med * 1e3, 2), "us_mean": round(mean * 1e3, 2),
                          "rows_per_s": round(c.L / (med / 1e3), 1), "clocks": clocks}}


def leg_window_sweep(n, dev, flush, hbm_peak):
    """window_sweep: 1000 steps x 58 layers x 256 experts of per-step counts
    (8,192 tokens x top-8 each); the W = 1000 window sum of every step
    (running totals, int64 [1000, 58, 256] in and out), then rebalance_experts
    on all 58,000 windowed rows.  L2 flushed before every call."""
    import moe_expert_load_eplb_b200 as eplb
    c = W.WINDOW_SWEEP
    steps = W.window_sweep_steps(device=dev)
    snaps = eplb.window_accumulate(steps, c.W)
    loads = snaps.view(-1, c.E)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    plan = eplb.rebalance(loads, c.P, c.G, c.N, c.gpus, status=st)
    elems = steps.numel()
    res = {"workload": c.name, "steps": c.S, "layers": c.L, "experts": c.E, "window": c.W,
           "calls": n, "l2": "flushed before every call (512 MB write)"}
    m = _time_calls(lambda: eplb.window_accumulate(steps, c.W, out=snaps), n, dev, flush)
    res["window"] = _hbm_entry(16.0 * elems, *m, hbm_peak,
                               {"kernel": "window_kernel",
                                "traffic": _traffic("window.cu", "window_window_sweep.md", 1.0)})
    med, mean, clocks = _time_calls(
        lambda: eplb.rebalance(loads, c.P, c.G, c.N, c.gpus, out=plan, status=st), n, dev, flush)
    res["rebalance"] = {"rows": loads.shape[0], "ms": round(med, 4), "ms_mean": round(mean, 4),
                        "rows_per_s": round(loads.shape[0] / (med / 1e3), 1), "clocks": clocks}
    torch.cuda.synchronize()
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())} in the window_sweep leg")
    del steps, snaps, plan
    torch.cuda.empty_cache()
    return res


def run_legs(args, dev, legs):
    """The single-GPU legs named in ``legs`` (one GPU only)."""
    hbm_peak, _ = _peaks()
    n = max(20, min(args.steps, 200))
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    out = {}
    if "hbm_stream" in legs:
        out["hbm_stream"] = leg_hbm_stream(n, dev, hbm_peak)
    if "global_policy" in legs:
        out["global_policy"] = leg_global_policy(n, dev, flush)
    if "window_sweep" in legs:
        out["window_sweep"] = leg_window_sweep(n, dev, flush, hbm_peak)
    del flush
    return out


def run_ours(args, rank: int, world: int, group):
    import moe_expert_load_eplb_b200 as eplb
    from moe_expert_load_eplb_b200.pipeline import EplbStep

    dev = torch.device("cuda", torch.cuda.current_device())
    c = CFG
    idx = W.routed_indices("dsv3_prefill", device=dev, shard=rank)
    hist = W.histogram_steps(WINDOW - 1, c.L, c.E, c.T * c.K * world, c.stream, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    hbm_peak, peak_kind = _peaks()

    def make(fused, single=False):
        st = EplbStep(c.L, c.T, c.K, c.E, c.P, c.G, c.N, c.gpus, window=WINDOW, device=dev,
                      token_offset=rank * c.T, group=group, fused=fused, single_launch=single)
        st.fill_history(hist)
        return st

    def check(st, where):
        torch.cuda.synchronize()
        code = int(st.status.item())
        if code != 0:
            raise RuntimeError(f"device status {eplb.STATUS.get(code)} in {where}")

    if args.fresh_only:
        fresh = make(False)
        for i in range(args.warmup):
            flush.fill_(i & 0xff)
            fresh(idx)
        check(fresh, "fresh-order warm-up")
        f_total, _, clocks, _ = _timed_steps(fresh, idx, flush, args.steps, group, dev)
        _, f_stage, _, _ = _timed_steps(fresh, idx, flush, min(args.steps, 500), group, dev, staged=True)
        check(fresh, "fresh-order steps")
        return {"fresh_only": True, "steps": args.steps, "ms_per_step": round(f_total / args.steps, 5),
                "stages": _stage_report(f_stage, False, fresh.X, world, hbm_peak), "clocks": clocks}

    # ---- the timed step: serving order (count+redirect, [all-reduce], plan) --
    step = make(True)
    for i in range(args.warmup):
        flush.fill_(i & 0xff)
        step(idx)
    check(step, "warm-up")
    K = args.steps
    total_ms, _, clocks, repeats = _timed_steps(step, idx, flush, K, group, dev,
                                                clock_ms=args.clock_ms)
    check(step, "timed steps")
    ms_per_step = total_ms / K
    if clocks is not None:
        clocks["region"] = (f"the {K} timed steps, then {len(repeats) - 1} repeats of them "
                            f"(sampled every 2 ms throughout)")
        clocks["step_kcycles"] = round(ms_per_step * clocks["sm_mhz"], 2)
    value = c.L * K / (total_ms / 1e3)
    # per-stage breakdown: a separate pass with events between the stages
    _, per_stage, _, _ = _timed_steps(step, idx, flush, max(3, min(K, 500)), group, dev, staged=True)
    check(step, "staged steps")
    stages = _stage_report(per_stage, True, step.X, world, hbm_peak)
    stages["count"]["traffic"] = _traffic("redirect.cu+redirect_chunk.cuh",
                                          "count_redirect_dsv3_prefill.md", 1.0)
    roof = {"kernel": "count_redirect", "bound": "hbm", "achieved": stages["count"]["gbs"],
            "peak": hbm_peak, "peak_kind": peak_kind, "unit": "GB/s",
            "frac": stages["count"]["frac_hbm"], "traffic": stages["count"]["traffic"],
            "frac_of_datasheet": round(stages["count"]["gbs"] / DATASHEET_HBM_GBS, 4)}
    order = ("serving: count+redirect with the plan in force (fused, one pass over the indices) "
             + ("-> all-reduce of the counts " if world > 1 else "")
             + "-> window sum + rebalance (fused) -> next plan")

    out = {"metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
           "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64",
           "data": "synthetic (seeded group-limited routing, log-normal popularity)",
           "config": dict(_config(world), step_order=order),
           "gpu_launches": step.launches_per_step * K,
           "tokens_per_s": round(world * c.T * K / (total_ms / 1e3), 1),
           "stages": stages, "roofline": roof, "clocks": clocks,
           "repeats_ms_per_step": {"n": len(repeats), "median": round(statistics.median(repeats), 5),
                                   "min": round(min(repeats), 5), "max": round(max(repeats), 5)}}

    # ---- the same step after a clean flush, one GPU only --------------------
    # The headline's flush (a 512 MB write) leaves L2 full of dirty lines that
    # are written back while the timed step runs.  Here a 256 MB read follows
    # the write, so L2 starts the step holding clean lines of another buffer,
    # as ncu's cold-cache replays do (they write back and invalidate L2).
    if world == 1 and not args.no_fresh:
        scrub = torch.zeros(FLUSH_BYTES // 2, dtype=torch.uint8, device=dev)
        Kc = max(3, min(K, 500))
        c_total, _, _, _ = _timed_steps(step, idx, flush, Kc, group, dev, scrub=scrub)
        _, c_stage, _, _ = _timed_steps(step, idx, flush, Kc, group, dev, staged=True, scrub=scrub)
        check(step, "clean-flush steps")
        cst = _stage_report(c_stage, True, step.X, world, hbm_peak)
        out["clean_l2"] = {
            "steps": Kc, "ms_per_step": round(c_total / Kc, 5),
            "value": round(c.L * Kc / (c_total / 1e3), 1),
            "l2": "512 MB write, then a 256 MB read (clean lines), between steps",
            "count_redirect": {k: cst["count"][k] for k in ("ms", "gbs", "frac_hbm")},
            "rebalance_ms": cst["rebalance"]["ms"]}
        del scrub

    # ---- the same step in one launch (serve_step), one GPU only -------------
    if world == 1 and not args.no_fresh:
        one = make(True, single=True)
        for i in range(max(3, args.warmup // 4)):
            flush.fill_(i & 0xff)
            one(idx)
        check(one, "one-launch warm-up")
        Ko = max(3, min(K, 500))
        o_total, _, _, _ = _timed_steps(one, idx, flush, Ko, group, dev)
        check(one, "one-launch steps")
        n_idx = c.L * c.T * c.K
        # indices in and out, count atomics, ring rows summed, cleared slot,
        # window sums and the next plan written
        algo = (8.0 * n_idx + 8.0 * c.L * c.E + 8.0 * WINDOW * c.L * c.E + 16.0 * c.L * c.E
                + 4.0 * c.L * (2 * c.P + c.E + c.E * one.X))
        o_ms = o_total / Ko
        out["one_launch_order"] = {
            "steps": Ko, "ms_per_step": round(o_ms, 5), "value": round(c.L * Ko / (o_total / 1e3), 1),
            "kernel": "serve_kernel (S1+S5 per chunk, then S2+S3/S4 per layer once counted)",
            "algo_bytes": algo, "gbs": round(algo / (o_ms / 1e3) / 1e9, 1),
            "traffic": _traffic(SERVE_SOURCES, "serve_step_dsv3_prefill.md", 1.0)}
        del one

    # ---- decode-sized step: eager calls vs CUDA-graph replay -----------------
    # At 8,192 tokens per layer the GPU step is short, so the host's enqueue
    # time per step matters; a captured step is one graph launch.
    if world == 1 and not args.no_fresh:
        from moe_expert_load_eplb_b200.pipeline import EplbStep, StepGraphs
        Td = 8192
        idx_d = W.routed_indices("dsv3_prefill", device=dev, T=Td)
        hist_d = W.histogram_steps(WINDOW - 1, c.L, c.E, Td * c.K, c.stream, device=dev)

        def make_d():
            st = EplbStep(c.L, Td, c.K, c.E, c.P, c.G, c.N, c.gpus, window=WINDOW, device=dev)
            st.fill_history(hist_d)
            return st

        eager_d = make_d()
        graphed_d = make_d()
        buf_d = idx_d.clone()
        sg = StepGraphs(graphed_d, buf_d)

        def run_d(fn, n):
            for i in range(3):
                flush.fill_(i & 0xff)
                fn()
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(n)]
            host = 0.0
            torch.cuda.synchronize()
            for i in range(n):
                flush.fill_(i & 0xff)  # keeps the GPU busy while the host enqueues
                ev[i][0].record()
                h0 = time.perf_counter()
                fn()
                host += time.perf_counter() - h0
                ev[i][1].record()
            torch.cuda.synchronize()
            return (sum(a.elapsed_time(b) for a, b in ev) / n, host / n * 1e6)

        Kd = max(3, min(K, 500))
        e_ms, e_host = run_d(lambda: eager_d(idx_d), Kd)
        g_ms, g_host = run_d(sg, Kd)
        check(eager_d, "decode eager steps")
        check(graphed_d, "decode graph steps")
        out["decode_8192_tokens"] = {
            "steps": Kd, "l2": "flushed between steps (512 MB write)",
            "eager": {"ms_per_step": round(e_ms, 5), "host_us_per_step": round(e_host, 1),
                      "value": round(c.L / (e_ms / 1e3), 1)},
            "graph_replay": {"ms_per_step": round(g_ms, 5), "host_us_per_step": round(g_host, 1),
                             "value": round(c.L / (g_ms / 1e3), 1)}}
        del eager_d, graphed_d, sg

    # ---- the same four stages in the fresh-plan order, for comparison -----
    if args.no_fresh:
        return _finish(out, args, step, idx, hist, flush, group, dev, rank, world)
    fresh = make(False)
    for i in range(max(3, args.warmup // 4)):
        flush.fill_(i & 0xff)
        fresh(idx)
    check(fresh, "fresh-order warm-up")
    Kf = max(3, min(K, 500))
    f_total, _, _, _ = _timed_steps(fresh, idx, flush, Kf, group, dev)
    _, f_stage, _, _ = _timed_steps(fresh, idx, flush, Kf, group, dev, staged=True)
    check(fresh, "fresh-order steps")
    fstages = _stage_report(f_stage, False, fresh.X, world, hbm_peak)
    out["fresh_order"] = {"steps": Kf, "ms_per_step": round(f_total / Kf, 5),
                          "value": round(c.L * Kf / (f_total / 1e3), 1), "stages": fstages}
    out["load_count_c2"] = {"gbs": fstages["count"]["gbs"], "frac_hbm": fstages["count"]["frac_hbm"],
                            "stage": "fresh-order count stage on the 121.6 MB batch"}
    del fresh
    return _finish(out, args, step, idx, hist, flush, group, dev, rank, world)


def _finish(out, args, step, idx, hist, flush, group, dev, rank, world):
    c = CFG
    K = args.steps
    if world == 1 and args.legs:
        out.update(run_legs(args, dev, args.legs))
    # load-count GB/s: on the 1.95 GB stream (the workload the HBM target is
    # set on) when that leg ran, else on the timed batch
    if "hbm_stream" in out:
        out["load_count_gbs"] = out["hbm_stream"]["count"]["gbs"]
        out["load_count_frac_hbm"] = out["hbm_stream"]["count"]["frac_hbm"]
        out["load_count_workload"] = "hbm_stream"
    elif "load_count_c2" in out:
        out["load_count_gbs"] = out["load_count_c2"]["gbs"]
        out["load_count_frac_hbm"] = out["load_count_c2"]["frac_hbm"]
        out["load_count_workload"] = "dsv3_prefill"

    def check(st, where):
        torch.cuda.synchronize()
        code = int(st.status.item())
        if code != 0:
            raise RuntimeError(f"device status {code} in {where}")

    # ---- e2e: the serving step through the public API with host buffers --
    # Every step copies its indices from pinned host memory and reads back
    # the redirected indices and the new plan.  Copies run on their own
    # streams, double-buffered, so step i's upload, step i-1's compute and
    # step i-2's download overlap (the two copy directions use separate copy
    # engines); the timed region runs from the first upload to the last
    # download.  No L2 flush: each step's fresh 243 MB of indices in and out
    # exceed the L2.  At least 50 steps whatever K, so that filling and
    # draining the three-stage pipeline (one upload and one download, about
    # 4.4 ms) is a small part of the timed region.
    if not args.no_e2e:
        Ke = max(50, min(K, 200))
        idx_host = idx.cpu().pin_memory()
        out_host = [torch.empty(step.out.shape, dtype=torch.int32).pin_memory() for _ in range(2)]
        plan_host = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in step.plan]
                     for _ in range(2)]
        idx_dev = [torch.empty_like(idx) for _ in range(2)]
        out_dev = [step.out, torch.empty_like(step.out)]
        compute = torch.cuda.current_stream(dev)
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()
        uploaded = [ev() for _ in range(Ke)]
        computed = [ev() for _ in range(Ke)]
        downloaded = [ev() for _ in range(Ke)]
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        if group is not None:
            torch.distributed.barrier(group=group)
        torch.cuda.synchronize()
        t_start.record(up)
        for i in range(Ke):
            b_ = i % 2
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(computed[i - 2])  # idx_dev[b_] no longer read
                idx_dev[b_].copy_(idx_host, non_blocking=True)
                uploaded[i].record(up)
            compute.wait_event(uploaded[i])
            if i >= 2:
                compute.wait_event(downloaded[i - 2])  # out_dev[b_] and the plan buffer read back
            step.out = out_dev[b_]
            step(idx_dev[b_])
            computed[i].record(compute)
            with torch.cuda.stream(down):
                down.wait_event(computed[i])
                out_host[b_].copy_(out_dev[b_], non_blocking=True)
                for h, d in zip(plan_host[b_], step.plan):
                    h.copy_(d, non_blocking=True)
                downloaded[i].record(down)
        t_end.record(down)
        torch.cuda.synchronize()
        step.out = out_dev[0]
        check(step, "e2e steps")
        e2e_ms = torch.tensor([t_start.elapsed_time(t_end)], dtype=torch.float64, device=dev)
        if group is not None:
            torch.distributed.all_reduce(e2e_ms, op=torch.distributed.ReduceOp.MAX, group=group)
        e2e_ms = float(e2e_ms.item())
        out["e2e"] = {"value": round(c.L * Ke / (e2e_ms / 1e3), 1), "unit": UNIT,
                      "h2d_bytes_per_step": idx.numel() * 4,
                      "d2h_bytes_per_step": out_host[0].numel() * 4 + sum(t.numel() * 4 for t in plan_host[0]),
                      "steps": Ke, "ms_per_step": round(e2e_ms / Ke, 4),
                      "copies": "pinned host buffers, upload / compute / download on three streams, "
                                "double-buffered"}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        idx_h, hist_h = idx.cpu().numpy(), hist.cpu().numpy()
        out["cpu_baseline"] = cpu_baseline(idx_h, hist_h, args.cpu_seconds)
        out["cpu_baseline_parallel"] = cpu_baseline_parallel(idx_h, hist_h, args.cpu_seconds)
    return out


# ------------------------------------------------------------ the oracle --

def _oracle_plan(hist_h, layers):
    import numpy as np
    import oracle
    c = CFG
    ring = np.concatenate([hist_h[:, :layers], np.zeros((1, layers, c.E), np.int64)], axis=0)
    loads = oracle.window(ring, WINDOW, WINDOW - 1)[0]
    return oracle.rebalance(loads, c.P, c.G, c.N, c.gpus, slots=(c.P - c.E) // c.N + 1)


def _oracle_step(idx_h, hist_h, layers, plan):
    """One serving step of the oracle on the first `layers` layers: count and
    redirect with the plan in force, window, rebalance (the GPU step's work)."""
    import numpy as np
    import oracle
    c = CFG
    sub = idx_h[:layers]
    counts, _ = oracle.count_loads(sub, c.E)
    oracle.redirect(sub, plan[3], plan[2])
    ring = np.concatenate([hist_h[:, :layers], counts[None]], axis=0)
    loads = oracle.window(ring, WINDOW, WINDOW - 1)[0]
    return oracle.rebalance(loads, c.P, c.G, c.N, c.gpus, slots=(c.P - c.E) // c.N + 1)


def cpu_baseline(idx_h, hist_h, seconds: float):
    plan = _oracle_plan(hist_h, CFG.L)  # also loads the oracle library, outside the timing
    n, t0 = 0, time.perf_counter()
    while True:
        _oracle_step(idx_h, hist_h, CFG.L, plan)
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return {"value": round(CFG.L * n / el, 2), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{n} full serving steps (58 layers x 65,536 tokens x top-8: count and "
                      f"redirect, 16-step window, rebalance), single-thread plain C, {el:.1f} s"}


def _oracle_pool(idx_h, hist_h, timing: dict):
    """Runs ``python -m oracle.pool`` (worker processes that import only numpy
    and the oracle) on inputs handed over in shared memory; ``timing`` holds
    ``seconds`` or ``steps`` and ``warmup``.  Returns (result dict, cores)."""
    import subprocess
    from multiprocessing import shared_memory

    import numpy as np
    c = CFG
    cores = min(len(os.sched_getaffinity(0)), c.L)
    shm_i = shared_memory.SharedMemory(create=True, size=idx_h.nbytes)
    shm_h = shared_memory.SharedMemory(create=True, size=hist_h.nbytes)
    try:
        np.ndarray(idx_h.shape, np.int32, buffer=shm_i.buf)[:] = idx_h
        np.ndarray(hist_h.shape, np.int64, buffer=shm_h.buf)[:] = hist_h
        spec = dict(timing, idx_name=shm_i.name, idx_shape=list(idx_h.shape), hist_name=shm_h.name,
                    hist_shape=list(hist_h.shape), P=c.P, G=c.G, N=c.N, gpus=c.gpus,
                    X=(c.P - c.E) // c.N + 1, cores=cores)
        res = subprocess.run([sys.executable, "-m", "oracle.pool", json.dumps(spec)], cwd=ROOT,
                             capture_output=True, text=True, timeout=600)
        if res.returncode != 0:
            raise RuntimeError(f"oracle pool failed: {res.stderr.strip()[-200:]}")
        return json.loads(res.stdout.strip().splitlines()[-1]), cores
    finally:
        shm_i.close()
        shm_i.unlink()
        shm_h.close()
        shm_h.unlink()


def cpu_baseline_parallel(idx_h, hist_h, seconds: float):
    """The same oracle step with its layers spread over the host cores."""
    try:
        r, cores = _oracle_pool(idx_h, hist_h, {"seconds": seconds})
    except Exception as e:  # a host without process pools still gets its GPU line
        return {"unavailable": str(e)[:200]}
    return {"value": round(r["layers_per_s"], 2), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{r['steps']} full serving steps, the 58 layers spread over {cores} worker "
                      f"processes (plain C oracle per layer), {r['seconds']:.1f} s"}


def run_reference(args):
    """The CPU oracle timed as the reference arm on this host's cores: the
    full serving step, its 58 layers spread over worker processes (one per
    core, up to 58); one core if no process pool can be had."""
    c = CFG
    idx_h = W.routed_indices("dsv3_prefill", device="cpu", T=c.T).numpy()
    hist_h = W.histogram_steps(WINDOW - 1, c.L, c.E, c.T * c.K, c.stream).numpy()
    try:
        r, cores = _oracle_pool(idx_h, hist_h, {"steps": args.steps, "warmup": args.warmup})
        layers, el = c.L, r["seconds"]
        sample = (f"58 of 58 layers per step (count and redirect 65,536 tokens x top-8, 16-step "
                  f"window, rebalance), plain C oracle per layer over {cores} worker processes")
    except Exception:
        cores = 1
        plan1 = _oracle_plan(hist_h, 1)
        t0 = time.perf_counter()
        _oracle_step(idx_h, hist_h, 1, plan1)
        t_layer = max(time.perf_counter() - t0, 1e-4)
        layers = int(max(1, min(c.L, 60.0 / ((args.steps + args.warmup) * t_layer))))
        plan = _oracle_plan(hist_h, layers)
        for _ in range(args.warmup):
            _oracle_step(idx_h, hist_h, layers, plan)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            _oracle_step(idx_h, hist_h, layers, plan)
        el = time.perf_counter() - t0
        sample = (f"{layers} of 58 layers per step (count and redirect 65,536 tokens x top-8, "
                  f"16-step window, rebalance), single-thread plain C oracle")
    value = layers * args.steps / el
    return {"metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(el / args.steps * 1e3, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int64", "data": "synthetic",
            "config": _config(1), "impl": "reference",
            "cpu_baseline": {"value": round(value, 2), "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    args = _args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    from moe_expert_load_eplb_b200.distributed import init_from_env
    rank, world, local, group = init_from_env("nccl" if world > 1 else None)
    torch.cuda.set_device(local)
    if args.legs_only:
        if world == 1:
            print(json.dumps(run_legs(args, torch.device("cuda", local), args.legs)), flush=True)
        return
    try:
        res = run_ours(args, rank, world, group)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if group is not None:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
