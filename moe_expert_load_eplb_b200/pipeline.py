"""One step of the EPLB hot path on one GPU, with preallocated buffers.

Two orders of the same four stages, both stream-ordered with no host
round-trip:

serving (default): the plan in force (built from earlier steps' loads, the
  moving-average estimate of page "DualPipe и EPLB", Part 2, section
  "Алгоритм") redirects this step's indices in the same pass that counts
  them, so the indices cross HBM once; two launches per step (with
  single_launch=True and no process group, one: serve_step builds each
  layer's next plan as soon as that layer's indices are all counted -- on the
  DeepSeek-V3 prefill step this measured slower, the early layers' plans
  holding SM slots the later layers' chunks wait for):
    1. count_redirect: indices -> ring row (step % W, cleared beforehand) and
       physical indices;
    2. rebalance_window: the window sum over the ring and the next plan of
       every layer, clearing the ring row the next step counts into.
fresh: the plan is rebuilt from this step's counts before redirecting:
    count_loads -> window_accumulate -> rebalance -> redirect.

With ``group`` set (torch.distributed, NCCL), every rank counts its own
token shard and the ring row is summed over ranks with one all-reduce before
the window; every rank then computes the identical plan locally (the plan is
an exact, deterministic function of the summed loads) and redirects its own
tokens with its global token offset.
"""
from __future__ import annotations

from typing import Optional, Sequence

import torch

from . import (Plan, count_loads, count_redirect, default_slots, rebalance, rebalance_window,
               redirect, serve_step, window_accumulate)
from .distributed import allreduce_loads


def _plan(L, E, P, X, dev) -> Plan:
    return Plan(torch.empty((L, P), dtype=torch.int32, device=dev),
                torch.empty((L, P), dtype=torch.int32, device=dev),
                torch.empty((L, E), dtype=torch.int32, device=dev),
                torch.empty((L, E, X), dtype=torch.int32, device=dev))


class EplbStep:
    STAGES = ("count", "allreduce", "window", "rebalance", "redirect")

    def __init__(self, L: int, T: int, K: int, E: int, P: int, G: int, N: int, gpus: int,
                 window: int = 1, device="cuda", slots: Optional[int] = None,
                 token_offset: int = 0, group=None, fused: bool = True,
                 single_launch: bool = False, quality: bool = True):
        self.L, self.T, self.K, self.E = L, T, K, E
        self.P, self.G, self.N, self.gpus = P, G, N, gpus
        self.W = window
        self.device = torch.device(device)
        self.X = default_slots(E, P, G, N) if slots is None else slots
        self.token_offset = token_offset
        self.group = group
        self.fused = fused
        # one launch per step needs every rank's counts before a layer's plan:
        # only without a process group
        self.single = fused and single_launch and group is None
        dev = self.device
        self.ring = torch.zeros((window, L, E), dtype=torch.int64, device=dev)
        self.loads = torch.zeros((1, L, E), dtype=torch.int64, device=dev)
        self.plans = [_plan(L, E, P, self.X, dev), _plan(L, E, P, self.X, dev)]
        self.cur = 0  # index of the plan in force
        self.out = torch.empty((L, T, K), dtype=torch.int32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.bad = torch.zeros(1, dtype=torch.int64, device=dev)
        self.layer_done = torch.zeros(L, dtype=torch.uint32, device=dev)
        # quality of the newest plan, computed by the launch that builds it:
        # per-GPU load [L, gpus] and {min, max, mean, mean / max} [L, 4]
        self.gpu_load = torch.zeros((L, gpus), dtype=torch.float64, device=dev) if quality else None
        self.stats = torch.zeros((L, 4), dtype=torch.float64, device=dev) if quality else None
        self.steps_done = 0
        self.primed = False

    @property
    def launches_per_step(self) -> int:
        """Kernels of this library launched per step."""
        return 1 if self.single else (2 if self.fused else 4)

    @property
    def plan(self) -> Plan:
        """The plan in force (the newest one built)."""
        return self.plans[self.cur]

    def load_history(self, history: torch.Tensor, steps_done: Optional[int] = None):
        """Put earlier per-step counts (int64 [S, L, E], oldest first; the last
        W - 1 rows are kept) into the ring where the steps that made them
        would have left them: with s = steps_done (default: the rows kept),
        row i of the n kept rows is step s - n + i and sits in slot
        (s - n + i) mod W; slot s mod W, which the next step counts into, is
        cleared.  Host-side bookkeeping only: no kernel runs."""
        n = min(history.shape[0], self.W - 1)
        s = n if steps_done is None else int(steps_done)
        if s < n:
            raise ValueError(f"steps_done={s} is less than the {n} history rows kept")
        self.ring.zero_()
        for i in range(n):
            self.ring[(s - n + i) % self.W].copy_(history[history.shape[0] - n + i])
        self.steps_done = s

    def fill_history(self, history: torch.Tensor, steps_done: Optional[int] = None):
        """load_history, then build the plan in force from the ring."""
        self.load_history(history, steps_done)
        self._plan_from_ring(self.plans[self.cur])
        self.primed = True

    def state_dict(self) -> dict:
        """The step's state, copied to the host: the ring of per-step counts,
        the plan in force, the number of steps done.  A step restored from it
        (``load_state_dict``, on any device) continues bit for bit as this one
        would: the plan is an exact function of the ring, and the ring and the
        step count are all the window keeps."""
        return {"shape": self._shape(), "steps_done": self.steps_done, "primed": self.primed,
                "cur": self.cur, "token_offset": self.token_offset,
                "ring": self.ring.cpu(), "plan": [t.cpu() for t in self.plans[self.cur]]}

    def load_state_dict(self, state: dict):
        """Restore a state taken by ``state_dict`` from a step of the same shape."""
        if tuple(state["shape"]) != self._shape():
            raise ValueError(f"state of shape {tuple(state['shape'])}, step of shape {self._shape()}")
        self.ring.copy_(state["ring"])
        self.cur = int(state["cur"])
        for dst, src in zip(self.plans[self.cur], state["plan"]):
            dst.copy_(src)
        self.steps_done = int(state["steps_done"])
        self.primed = bool(state["primed"])
        self.token_offset = int(state["token_offset"])

    def _shape(self):
        return (self.L, self.T, self.K, self.E, self.P, self.G, self.N, self.gpus, self.W, self.X)

    def _plan_from_ring(self, plan: Plan):
        window_accumulate(self.ring, self.W, s_first=self.W - 1, out=self.loads)
        rebalance(self.loads[0], self.P, self.G, self.N, self.gpus, slots=self.X, out=plan,
                  status=self.status, gpu_load=self.gpu_load, stats=self.stats)

    def __call__(self, idx: torch.Tensor, marks: Optional[Sequence] = None):
        """Run one step on idx (int32 [L, T, K]).

        Returns (plan used for this step's redirect, redirected indices); the
        serving order's new plan is ``self.plan`` afterwards.  ``marks``: six
        CUDA events recorded on the current stream around the stages
        count | allreduce | window | rebalance | redirect (the two-launch
        serving order records its fused count+redirect under count, its fused
        window+rebalance under rebalance, and empty window / redirect stages;
        the one-launch serving step records the whole step under count).
        """
        if self.fused and not self.primed:
            raise RuntimeError("serving order needs a plan in force: call fill_history() first")
        rec = (lambda k: marks[k].record()) if marks else (lambda k: None)
        row = self.ring[self.steps_done % self.W]
        used = self.plans[self.cur]
        rec(0)
        if self.single:
            nxt = self.plans[1 - self.cur]
            serve_step(idx, used, self.ring, self.steps_done % self.W, nxt, self.layer_done, self.G,
                       self.N, self.gpus, zero_slot=(self.steps_done + 1) % self.W,
                       token_offset=self.token_offset, out=self.out, loads_out=self.loads,
                       bad=self.bad, status=self.status, gpu_load=self.gpu_load, stats=self.stats)
            for k in range(1, 6):
                rec(k)
            self.steps_done += 1
            self.cur = 1 - self.cur
            return used, self.out
        if self.fused:
            # the ring row was cleared by the previous step's rebalance_window
            count_redirect(idx, self.E, used.log2phy, used.logcnt, self.token_offset, counts=row,
                           accumulate=True, out=self.out, bad=self.bad, status=self.status)
        else:
            # the ring row was cleared by the previous step's window launch
            # (fill_history clears it for the first step)
            count_loads(idx, self.E, counts=row, accumulate=True, bad=self.bad)
        rec(1)
        if self.group is not None:
            allreduce_loads(row, self.group)
        rec(2)
        if self.fused:
            rec(3)
            nxt = self.plans[1 - self.cur]
            rebalance_window(self.ring, self.P, self.G, self.N, self.gpus,
                             zero_slot=(self.steps_done + 1) % self.W, slots=self.X, out=nxt,
                             loads_out=self.loads, status=self.status, gpu_load=self.gpu_load,
                             stats=self.stats)
        else:
            window_accumulate(self.ring, self.W, s_first=self.W - 1, out=self.loads,
                              zero_row=(self.steps_done + 1) % self.W)
            rec(3)
            nxt = used
            rebalance(self.loads[0], self.P, self.G, self.N, self.gpus, slots=self.X, out=nxt,
                      status=self.status, gpu_load=self.gpu_load, stats=self.stats)
        rec(4)
        if not self.fused:
            redirect(idx, nxt.log2phy, nxt.logcnt, self.token_offset, out=self.out, bad=self.bad,
                     status=self.status)
        rec(5)
        self.steps_done += 1
        if self.fused:
            self.cur = 1 - self.cur
            return used, self.out
        return nxt, self.out


class StepGraphs:
    """Replays an EplbStep's steps as CUDA graphs.

    A step's launches depend on its phase only: the ring slot it counts into
    (step mod W) and which of the two plan buffers is in force (step mod 2).
    ``lcm(W, 2)`` consecutive steps are captured once, each as one graph that
    reads its indices from the fixed buffer ``idx``; ``step_graphs()`` then
    replays the graph of the current phase, so a step costs one graph launch
    on the host instead of one call per kernel.  The captured steps are not
    executed by the capture; the EplbStep's bookkeeping advances only on
    replay.  One GPU (no process group), as the one-process serving step.
    """

    def __init__(self, step: "EplbStep", idx: torch.Tensor):
        if not step.primed or step.group is not None:
            raise ValueError("capture needs a primed EplbStep without a process group")
        if tuple(idx.shape) != (step.L, step.T, step.K) or idx.dtype != torch.int32:
            raise ValueError("idx must be the step's int32 [L, T, K] input buffer")
        import math
        self.step = step
        self.idx = idx
        self.period = math.lcm(step.W, 2)
        self.first = step.steps_done
        dev = step.device
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        saved = (step.steps_done, step.cur)
        self.graphs = []
        with torch.cuda.stream(side):
            for _ in range(self.period):
                g = torch.cuda.CUDAGraph()
                # relaxed: the library's launch set-up (function attributes,
                # occupancy queries) is not stream work but is still allowed
                with torch.cuda.graph(g, stream=side, capture_error_mode="relaxed"):
                    step(idx)
                self.graphs.append(g)
        torch.cuda.current_stream(dev).wait_stream(side)
        step.steps_done, step.cur = saved  # capturing ran nothing

    def __call__(self):
        """Runs one step on the current contents of ``idx``; returns (plan used,
        redirected indices) like EplbStep.__call__."""
        st = self.step
        k = (st.steps_done - self.first) % self.period
        used = st.plans[st.cur]
        self.graphs[k].replay()
        st.steps_done += 1
        if st.fused:
            st.cur = 1 - st.cur
        return used, st.out
