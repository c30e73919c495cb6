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
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer e2e measurement")
    ap.add_argument("--no-fresh", action="store_true", help="skip the fresh-plan-order comparison")
    ap.add_argument("--fresh-only", action="store_true",
                    help="time only the fresh-plan order (for profiling its kernels)")
    return ap.parse_args()


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

    def __init__(self, device: int, period: float = 0.02):
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
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
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
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


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


def _timed_steps(step, idx, flush, K, group, dev, staged=False, scrub=None):
    """Runs K steps, each between a start and an end event (the L2 flush
    before each step stays outside them); returns (total ms, max over ranks,
    per-stage mean ms or None, clock summary).  With ``staged`` the step also
    records events between its stages for the per-stage breakdown -- those
    extra records cost time of their own, so the headline is taken without
    them.  ``scrub`` (a buffer larger than L2): read after the flush write,
    so that L2 holds clean lines and none of the flush's dirty lines is
    written back inside the timed step."""
    n_ev = 6 if staged else 2
    marks = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(K)]
    if group is not None:
        torch.distributed.barrier(group=group)
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clocks:
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
    per_stage = None
    if staged:
        per_stage = {n: statistics.mean(m[k].elapsed_time(m[k + 1]) for m in marks)
                     for k, n in enumerate(STAGES)}
    total = torch.tensor([sum(m[0].elapsed_time(m[-1]) for m in marks)], dtype=torch.float64,
                         device=dev)
    if group is not None:
        torch.distributed.all_reduce(total, op=torch.distributed.ReduceOp.MAX, group=group)
    return float(total.item()), per_stage, clocks.summary()


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
        f_total, _, clocks = _timed_steps(fresh, idx, flush, args.steps, group, dev)
        _, f_stage, _ = _timed_steps(fresh, idx, flush, min(args.steps, 500), group, dev, staged=True)
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
    total_ms, _, clocks = _timed_steps(step, idx, flush, K, group, dev)
    check(step, "timed steps")
    ms_per_step = total_ms / K
    value = c.L * K / (total_ms / 1e3)
    # per-stage breakdown: a separate pass with events between the stages
    _, per_stage, _ = _timed_steps(step, idx, flush, max(3, min(K, 500)), group, dev, staged=True)
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
           "stages": stages, "roofline": roof, "clocks": clocks}

    # ---- the same step after a clean flush, one GPU only --------------------
    # The headline's flush (a 512 MB write) leaves L2 full of dirty lines that
    # are written back while the timed step runs.  Here a 256 MB read follows
    # the write, so L2 starts the step holding clean lines of another buffer,
    # as ncu's cold-cache replays do (they write back and invalidate L2).
    if world == 1 and not args.no_fresh:
        scrub = torch.zeros(FLUSH_BYTES // 2, dtype=torch.uint8, device=dev)
        Kc = max(3, min(K, 500))
        c_total, _, _ = _timed_steps(step, idx, flush, Kc, group, dev, scrub=scrub)
        _, c_stage, _ = _timed_steps(step, idx, flush, Kc, group, dev, staged=True, scrub=scrub)
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
        o_total, _, _ = _timed_steps(one, idx, flush, Ko, group, dev)
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
    f_total, _, _ = _timed_steps(fresh, idx, flush, Kf, group, dev)
    _, f_stage, _ = _timed_steps(fresh, idx, flush, Kf, group, dev, staged=True)
    check(fresh, "fresh-order steps")
    fstages = _stage_report(f_stage, False, fresh.X, world, hbm_peak)
    out["fresh_order"] = {"steps": Kf, "ms_per_step": round(f_total / Kf, 5),
                          "value": round(c.L * Kf / (f_total / 1e3), 1), "stages": fstages}
    out["load_count_gbs"] = fstages["count"]["gbs"]
    out["load_count_frac_hbm"] = fstages["count"]["frac_hbm"]
    del fresh
    return _finish(out, args, step, idx, hist, flush, group, dev, rank, world)


def _finish(out, args, step, idx, hist, flush, group, dev, rank, world):
    c = CFG
    K = args.steps

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
    # exceed the L2.
    if not args.no_e2e:
        Ke = max(5, min(K, 50))
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
    try:
        res = run_ours(args, rank, world, group)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if group is not None:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
