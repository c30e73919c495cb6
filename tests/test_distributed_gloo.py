"""Multi-rank logic of the EPLB step on CPU: world size 2, gloo backend.

Each rank takes its token shard, counts it (oracle on the host standing in
for the GPU kernel), all-reduces the counts with the package's
``allreduce_loads``, plans locally and redirects its shard with its global
token offset.  Checked: the summed counts equal the single-process counts,
every rank computes the same plan, and the concatenated redirected shards
equal the single-process redirect.  A rank that raises must not hang the
other: the short process-group timeout turns the wait into an error.
"""
from __future__ import annotations

import os
import socket
import traceback

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, L, T, K, E, P, G, N, gpus, results, fail_rank):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    try:
        import oracle
        from moe_expert_load_eplb_b200.distributed import allreduce_loads, init_from_env, token_shard
        r, w, _, group = init_from_env("gloo", timeout_s=20)
        assert (r, w) == (rank, world)
        rng = np.random.default_rng(123)
        idx = rng.integers(0, E, (L, T, K)).astype(np.int32)   # same batch on every rank
        t0, t1 = token_shard(T, rank, world)
        if rank == fail_rank:
            raise RuntimeError("injected failure before the exchange")
        counts, _ = oracle.count_loads(idx[:, t0:t1], E)
        loads = torch.from_numpy(counts.copy())
        allreduce_loads(loads, group)
        plan = oracle.rebalance(loads.numpy(), P, G, N, gpus)
        out, _ = oracle.redirect(idx[:, t0:t1], plan[3], plan[2], t0)
        results[rank] = ("ok", loads.numpy().tolist(), [p.tolist() for p in plan], out.tolist(), t0, t1)
        torch.distributed.barrier(group)
        torch.distributed.destroy_process_group()
    except Exception as e:  # report to the parent instead of hanging
        results[rank] = ("error", f"{type(e).__name__}: {e}", traceback.format_exc())
        try:
            torch.distributed.destroy_process_group()
        except Exception:
            pass


def _run(world, fail_rank=-1):
    L, T, K, E, P, G, N, gpus = 3, 1001, 4, 24, 32, 6, 2, 8
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, L, T, K, E, P, G, N, gpus, results,
                                                fail_rank)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a rank hung")
    return dict(results), (L, T, K, E, P, G, N, gpus)


def test_token_shards_cover_and_balance():
    from moe_expert_load_eplb_b200.distributed import token_shard
    for total in (0, 1, 7, 65536, 1001):
        for world in (1, 2, 3, 8):
            spans = [token_shard(total, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == total
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1


@pytest.mark.parametrize("world", [2, 3])
def test_ranks_sum_loads_and_agree_on_the_plan(world):
    """World 3 splits the 1001 tokens unevenly (334, 334, 333)."""
    import oracle
    results, (L, T, K, E, P, G, N, gpus) = _run(world)
    ranks = tuple(range(world))
    assert set(results) == set(ranks), results
    for r in ranks:
        assert results[r][0] == "ok", results[r]
    rng = np.random.default_rng(123)
    idx = rng.integers(0, E, (L, T, K)).astype(np.int32)
    counts, _ = oracle.count_loads(idx, E)
    plan = oracle.rebalance(counts, P, G, N, gpus)
    full, _ = oracle.redirect(idx, plan[3], plan[2], 0)
    for r in ranks:
        assert np.array_equal(np.array(results[r][1]), counts)
        for got, want in zip(results[r][2], plan):
            assert np.array_equal(np.array(got), want)
    shards = sorted((results[r][4], np.array(results[r][3])) for r in ranks)
    assert np.array_equal(np.concatenate([s for _, s in shards], axis=1), full)


def test_failed_rank_does_not_hang_the_other():
    results, _ = _run(2, fail_rank=1)
    assert results[1][0] == "error" and "injected failure" in results[1][1]
    # rank 0 waits in the all-reduce until the process-group timeout ends it
    assert results[0][0] == "error"
