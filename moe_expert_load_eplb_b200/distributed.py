"""Host-side logic of the multi-GPU EPLB step (one process per GPU).

Load counting and redirection shard over tokens: every rank counts and
redirects its own contiguous token range.  The only exchange is one
all-reduce (sum) of the per-step counts [L, E]; every rank then computes the
same plan locally, because the plan is an exact, deterministic function of
the summed loads (integer arithmetic, fixed tie rules) -- no broadcast is
needed.  The redirect rule uses the global token index, so each rank passes
its range's first token as ``token_offset``.

The functions work with any torch.distributed backend: NCCL for the CUDA
tensors of the GPU step, gloo for host tensors in tests.
"""
from __future__ import annotations

import datetime
import os
from typing import Optional, Tuple

import torch


def token_shard(total_tokens: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous token range [t0, t1) of ``rank``; sizes differ by at most one."""
    if world < 1 or not 0 <= rank < world or total_tokens < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(total_tokens, world)
    t0 = rank * base + min(rank, extra)
    return t0, t0 + base + (1 if rank < extra else 0)


def allreduce_loads(counts: torch.Tensor, group=None) -> torch.Tensor:
    """Sums an int64 load tensor over all ranks of ``group`` in place."""
    if counts.dtype != torch.int64:
        raise TypeError("loads must be int64")
    torch.distributed.all_reduce(counts, op=torch.distributed.ReduceOp.SUM, group=group)
    return counts


def init_from_env(backend: Optional[str] = None, timeout_s: float = 120.0):
    """Joins the process group described by RANK / WORLD_SIZE / MASTER_* (as
    torchrun sets them).  Returns (rank, world, local_rank, group); group is
    None for a single process.  A short timeout makes ranks waiting on a rank
    that died end with an error instead of hanging."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world == 1:
        return rank, world, local, None
    if backend is None:
        backend = "nccl" if torch.cuda.is_available() else "gloo"
    kwargs = {}
    if backend == "nccl":
        torch.cuda.set_device(local)
        kwargs["device_id"] = torch.device("cuda", local)
    torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s),
                                         **kwargs)
    return rank, world, local, torch.distributed.group.WORLD
