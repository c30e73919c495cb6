"""One serving step of the EPLB hot path on one GPU, with preallocated buffers.

Per step (all stream-ordered, no host round-trip):
  1. count_loads: this step's routed indices -> its row of the load window
     ring (int64 [W, L, E], row step % W);
  2. window_accumulate over the ring (s_first = W - 1): the window sum, which
     is the moving-average load estimate times W (page "DualPipe и EPLB",
     Part 2, section "Алгоритм");
  3. rebalance: the replica/placement plan of every layer;
  4. redirect: this step's indices to physical replicas.

With ``group`` set (torch.distributed, NCCL), every rank counts its own
token shard and the ring row is summed over ranks with one all-reduce before
the window; every rank then computes the identical plan locally (the plan is
an exact, deterministic function of the summed loads) and redirects its own
tokens with its global token offset.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import Plan, count_loads, default_slots, rebalance, redirect, window_accumulate


class EplbStep:
    def __init__(self, L: int, T: int, K: int, E: int, P: int, G: int, N: int, gpus: int,
                 window: int = 1, device="cuda", slots: Optional[int] = None,
                 token_offset: int = 0, group=None):
        self.L, self.T, self.K, self.E = L, T, K, E
        self.P, self.G, self.N, self.gpus = P, G, N, gpus
        self.W = window
        self.device = torch.device(device)
        self.X = default_slots(E, P, G, N) if slots is None else slots
        self.token_offset = token_offset
        self.group = group
        dev = self.device
        self.ring = torch.zeros((window, L, E), dtype=torch.int64, device=dev)
        self.loads = torch.zeros((1, L, E), dtype=torch.int64, device=dev)
        self.plan = Plan(torch.empty((L, P), dtype=torch.int32, device=dev),
                         torch.empty((L, P), dtype=torch.int32, device=dev),
                         torch.empty((L, E), dtype=torch.int32, device=dev),
                         torch.empty((L, E, self.X), dtype=torch.int32, device=dev))
        self.out = torch.empty((L, T, K), dtype=torch.int32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.bad = torch.zeros(1, dtype=torch.int64, device=dev)
        self.steps_done = 0

    def fill_history(self, history: torch.Tensor):
        """Set the ring to earlier per-step counts (int64 [W, L, E])."""
        self.ring.copy_(history)

    def __call__(self, idx: torch.Tensor):
        """Run one step on idx (int32 [L, T, K]); returns (plan, redirected indices)."""
        slot = self.steps_done % self.W
        row = self.ring[slot]
        count_loads(idx, self.E, counts=row, bad=self.bad, status=self.status)
        if self.group is not None:
            torch.distributed.all_reduce(row, group=self.group)
        window_accumulate(self.ring, self.W, s_first=self.W - 1, out=self.loads, status=self.status)
        rebalance(self.loads[0], self.P, self.G, self.N, self.gpus, slots=self.X, out=self.plan,
                  status=self.status)
        redirect(idx, self.plan.log2phy, self.plan.logcnt, self.token_offset, out=self.out,
                 bad=self.bad, status=self.status)
        self.steps_done += 1
        return self.plan, self.out

    launches_per_step = 4  # count, window, rebalance, redirect kernels
