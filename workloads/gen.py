"""Seeded synthetic inputs for the EPLB hot path.

The pages give no dataset or routing trace; these generators stand in for the
DeepSeek-V3 setting they describe (256 logical experts in 8 groups, 32
redundant replicas, group-limited top-8 routing, page "DualPipe и EPLB",
Part 2, boxes "От переводчика: термины" and "что сделать руками").  The
recipes (distributions, seeds) are stated per function; nothing here performs
any step of the balancing method.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

BASE_SEED = 20250227


def seed_for(stream: int, sub: int = 0) -> int:
    """Seed of sub-stream ``sub`` (layer, step, ...) of seed stream ``stream``
    (each workload draws from its own stream, ``Workload.stream``)."""
    return BASE_SEED + 1000 * stream + sub


@dataclass(frozen=True)
class Workload:
    stream: int     # seed stream (seed_for)
    name: str
    L: int          # MoE layers (rows of one rebalance call)
    E: int          # logical experts per layer
    G: int          # expert groups
    P: int          # physical experts (replicas) per layer
    N: int          # nodes
    gpus: int       # GPUs
    T: int = 0      # tokens per layer (per step for the window sweep)
    K: int = 0      # top-k
    S: int = 0      # steps of the window sweep
    W: int = 0      # window length
    extra: dict = field(default_factory=dict)

    @property
    def hierarchical(self) -> bool:
        return self.G % self.N == 0

    @property
    def slots(self) -> int:
        """A log2phy width that always suffices: most replicas one expert can get."""
        n = self.N if self.hierarchical else 1
        return (self.P - self.E) // n + 1


# The workloads by name: the pages' worked-example sizes, DeepSeek-V3-shaped
# prefill, the global policy over 144 GPUs, a 1000-step window sweep, and a
# 16x larger routed batch that streams ~2 GB of indices.
TINY = Workload(1, "tiny", L=2, E=12, G=4, P=16, N=2, gpus=8, T=4096, K=2)
DSV3_PREFILL = Workload(2, "dsv3_prefill", L=58, E=256, G=8, P=288, N=4, gpus=32, T=65536, K=8)
GLOBAL_POLICY = Workload(3, "global_policy", L=58, E=256, G=1, P=288, N=2, gpus=144)
WINDOW_SWEEP = Workload(4, "window_sweep", L=58, E=256, G=8, P=288, N=4, gpus=32, T=8192, K=8,
                        S=1000, W=1000)
HBM_STREAM = Workload(5, "hbm_stream", L=58, E=256, G=8, P=288, N=4, gpus=32, T=1048576, K=8)
WORKLOADS = {w.name: w for w in (TINY, DSV3_PREFILL, GLOBAL_POLICY, WINDOW_SWEEP, HBM_STREAM)}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def zipf_indices(L: int, T: int, K: int, E: int, s: float, stream: int, device="cpu") -> torch.Tensor:
    """int32 [L, T, K]: per layer, expert popularity p_r ∝ r^-s over ranks r = 1..E
    mapped to experts through a seeded permutation; each token draws K distinct
    experts (sampling without replacement, as a router's top-k is distinct)."""
    out = torch.empty((L, T, K), dtype=torch.int32, device=device)
    ranks = torch.arange(1, E + 1, dtype=torch.float64)
    base = ranks.pow(-s)
    for l in range(L):
        g = _gen(seed_for(stream, l), "cpu")
        perm = torch.randperm(E, generator=g)
        p = torch.empty(E, dtype=torch.float64)
        p[perm] = base / base.sum()
        if T:
            draws = torch.multinomial(p.float().expand(T, E), K, replacement=False, generator=g)
            out[l] = draws.to(device=device, dtype=torch.int32)
    return out


def tiny_indices(device="cpu") -> torch.Tensor:
    """Tiny workload: 2 layers x 4096 tokens x top-2 over 12 experts, Zipf(s=1.2)."""
    c = TINY
    return zipf_indices(c.L, c.T, c.K, c.E, 1.2, c.stream, device)


def group_limited_indices(popularity: torch.Tensor, T: int, K: int, G: int, groups_per_token: int,
                          seed: int, device="cpu", t_chunk: int = 1 << 17) -> torch.Tensor:
    """int32 [L, T, K] group-limited routing for popularity [L, E] (> 0).

    Token score of expert e: s = p_e / X with X ~ Exp(1) (so the top-1 choice
    has probability ∝ p_e); a group's score is the sum of its experts' scores;
    the token keeps the ``groups_per_token`` best groups and takes its top-K
    experts inside them (descending score).
    """
    L, E = popularity.shape
    gs = E // G
    out = torch.empty((L, T, K), dtype=torch.int32, device=device)
    pop = popularity.to(device=device, dtype=torch.float32)
    for l in range(L):
        g = _gen(seed + l, device)
        for t0 in range(0, T, t_chunk):
            n = min(t_chunk, T - t0)
            x = torch.empty((n, E), dtype=torch.float32, device=device).exponential_(generator=g)
            score = pop[l] / x
            gscore = score.view(n, G, gs).sum(-1)
            keep = torch.zeros((n, G), dtype=torch.bool, device=device)
            keep.scatter_(1, gscore.topk(groups_per_token, dim=1).indices, True)
            score = score.masked_fill(~keep.repeat_interleave(gs, dim=1), -1.0)
            out[l, t0:t0 + n] = score.topk(K, dim=1).indices.to(torch.int32)
            del x, score, gscore, keep
    return out


def routed_indices(workload: str, device="cpu", T: int | None = None, L: int | None = None,
                   shard: int = 0) -> torch.Tensor:
    """Routed indices of the dsv3_prefill and hbm_stream workloads (optionally
    with fewer tokens / layers).

    dsv3_prefill: popularity LogNormal(mu=0, sigma=1) per expert per layer.
    hbm_stream: popularity ∝ rank^-1.0 (Zipf s=1.0) through a seeded permutation.
    Both: 8 groups of 32, 4 groups per token, top-8.  ``shard`` selects an
    independent token stream with the same popularity (one per data-parallel
    rank).
    """
    c = WORKLOADS[workload]
    L = c.L if L is None else L
    T = c.T if T is None else T
    g = _gen(seed_for(c.stream, 999), "cpu")
    if c is DSV3_PREFILL:
        pop = torch.empty((L, c.E), dtype=torch.float64).log_normal_(0.0, 1.0, generator=g)
    elif c is HBM_STREAM:
        base = torch.arange(1, c.E + 1, dtype=torch.float64).pow(-1.0)
        pop = torch.stack([base[torch.randperm(c.E, generator=g)] for _ in range(L)])
    else:
        raise ValueError("routed indices exist for dsv3_prefill and hbm_stream")
    return group_limited_indices(pop.float(), T, c.K, c.G, 4,
                                 seed_for(c.stream, 0) + 100000 * shard, device)


def global_policy_loads(L: int = 58, E: int = 256) -> np.ndarray:
    """global_policy workload: loads int64 [L, E] = round(1e4 * Pareto(alpha=1.5)), x_m = 1."""
    rng = np.random.default_rng(seed_for(GLOBAL_POLICY.stream))
    return np.round(1e4 * (rng.pareto(1.5, size=(L, E)) + 1.0)).astype(np.int64)


def histogram_steps(S: int, L: int, E: int, draws: int, stream: int, sigma: float = 0.05,
                    device="cpu") -> torch.Tensor:
    """int64 [S, L, E]: per step, the histogram of ``draws`` expert choices.

    Log-popularity starts N(0, 1) and takes a Gaussian random walk of step
    ``sigma`` per step; each step's counts are a multinomial draw of
    ``draws`` choices from softmax(log-popularity), sampled exactly as a
    chain of conditional binomials (counts add up to ``draws``).
    """
    g = _gen(seed_for(stream, 0), device)
    theta = torch.randn((1, L, E), generator=g, device=device, dtype=torch.float64)
    walk = torch.randn((S, L, E), generator=g, device=device, dtype=torch.float64) * sigma
    walk[0] = 0
    theta = theta + walk.cumsum(0)
    p = torch.softmax(theta, dim=-1).reshape(S * L, E)
    counts = torch.empty((S * L, E), dtype=torch.int64, device=device)
    n_rem = torch.full((S * L,), float(draws), dtype=torch.float64, device=device)
    mass = torch.ones((S * L,), dtype=torch.float64, device=device)
    for e in range(E - 1):
        q = (p[:, e] / mass.clamp_min(1e-300)).clamp(0.0, 1.0)
        c = torch.binomial(n_rem, q, generator=g)
        counts[:, e] = c.to(torch.int64)
        n_rem = n_rem - c
        mass = mass - p[:, e]
    counts[:, E - 1] = n_rem.to(torch.int64)
    return counts.view(S, L, E)


def window_sweep_steps(device="cpu", S: int | None = None) -> torch.Tensor:
    """window_sweep workload: 1000 steps x 58 layers x 256 experts, 8192 tokens
    x top-8 per step."""
    c = WINDOW_SWEEP
    return histogram_steps(c.S if S is None else S, c.L, c.E, c.T * c.K, c.stream, device=device)
